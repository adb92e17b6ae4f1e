"""The decode entry point that allocates nothing (atflash_decode_noalloc).

It exists for callers that cannot allocate device memory when they call the
library (for instance a serving loop that must stay out of the CUDA allocator
once running, or a plugin whose host framework owns all device memory).  Its
split-state scratch is a fixed device array inside the library instead of a
caller workspace.  These tests call it through the C ABI twice in a row, with
different problem sizes so the second call runs over the first call's leftover
scratch contents, for fp32 and bf16 inputs and outputs and every contiguous
cache layout, and check each output against atflash_decode's on the same
inputs.  It also checks that a problem too large for the fixed array is
rejected before anything runs.  The file name makes pytest collect it last.
"""
import ctypes

import pytest

import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_attention_pair_b200 as atf  # noqa: E402

LIMIT = 32 * 1024 * 1024  # ATFLASH_NOALLOC_SCRATCH_BYTES


def _fn():
    f = atf.lib().atflash_decode_noalloc
    vp, i, i64, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    f.argtypes = [vp, vp, vp, vp, vp, i, i, i, i64, i, d, d, i, i, i, i, vp]
    f.restype = i
    return f


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


LAYOUTS = {"HND": atf.KV_HND, "NHD": atf.KV_NHD, "PACKED": atf.KV_PACKED}
DTYPES = {"f32": (atf.F32, torch.float32), "bf16": (atf.BF16, torch.bfloat16)}


def _caches(seed, B, Hkv, Nmax, D, dtype, layout, base):
    """(k, v) device caches in one layout (PACKED: K rotated by the RoPE pre-pass, V as HND)."""
    kc = P.gen(seed, "k_cache", (B, Hkv, Nmax, D), dtype)
    vc = P.gen(seed, "v_cache", (B, Hkv, Nmax, D), dtype)
    if layout == "NHD":
        return kc.permute(0, 2, 1, 3).contiguous(), vc.permute(0, 2, 1, 3).contiguous()
    if layout == "PACKED":
        return atf.rope_pack(kc.permute(0, 2, 1, 3).contiguous(), base), vc
    return kc, vc


def _call_noalloc(q, kin, vin, sl, out, Hkv, Nmax, base, kwin, layout, in_dtype, out_dtype):
    B, Hq, D = q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    krot = 1 if layout == "PACKED" else 0
    return _fn()(_ptr(q), _ptr(kin), _ptr(vin), _ptr(sl), _ptr(out), B, Hq, Hkv, Nmax, D, base, kwin, krot,
                 LAYOUTS[layout], in_dtype, out_dtype, stream)


# Two calls in a row per case (the second runs over the first call's leftover
# scratch contents), across input dtypes, cache layouts and output dtypes.
CASES = [
    ("bf16", "HND", "f32", [(4, 28, 4, 20000, 128, 1e7, 16.0), (2, 14, 2, 5000, 64, 1e6, 8.0)]),
    ("f32", "HND", "f32", [(2, 8, 2, 3000, 128, 5e5, 16.0), (3, 4, 4, 1000, 64, 1e4, 1.0)]),
    ("bf16", "NHD", "bf16", [(2, 7, 1, 4097, 64, 1e6, 8.0), (1, 24, 2, 2100, 128, 5e5, 16.0)]),
    ("f32", "NHD", "bf16", [(2, 6, 2, 2500, 64, 1e4, 2.0), (1, 8, 1, 700, 128, 1e7, 64.0)]),
    ("bf16", "PACKED", "f32", [(2, 28, 4, 6000, 128, 1e7, 16.0), (3, 8, 2, 1200, 64, 1e6, 8.0)]),
]


@pytest.mark.parametrize("in_name,layout,out_name,shapes", CASES)
def test_noalloc_decode_matches_workspace_decode_twice(in_name, layout, out_name, shapes):
    in_dtype, tdt = DTYPES[in_name]
    out_dtype, odt = DTYPES[out_name]
    for call, (B, Hq, Hkv, Nmax, D, base, kwin) in enumerate(shapes):
        assert atf.decode_workspace_bytes(B, Hq, Hkv, Nmax, D) <= LIMIT
        q = P.gen(40 + call, "q_dec", (B, Hq, D), in_name)
        kin, vin = _caches(40 + call, B, Hkv, Nmax, D, in_name, layout, base)
        # the last sequence is short (<= 128 tokens) so the fp32 short-row step runs too
        sl = torch.tensor([Nmax - 37 * b for b in range(B - 1)] + [min(Nmax, 100)], dtype=torch.int32,
                          device="cuda")
        out = torch.empty((B, Hq, D), dtype=odt, device="cuda")
        assert _call_noalloc(q, kin, vin, sl, out, Hkv, Nmax, base, kwin, layout, in_dtype, out_dtype) == 0
        ref = atf.decode(q, kin, vin, sl, base, kwin, kcache_rotated=layout == "PACKED", kv_layout=layout,
                         out_dtype=odt)
        torch.cuda.synchronize()
        assert atf.device_status() == 0
        P.check(P.host(out), P.host(ref), "f32" if in_name == "f32" else "bf16",
                f"noalloc {in_name}/{layout}/{out_name} call {call + 1}")


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    B, Hq, Hkv, D = 16, 64, 4, 128
    Nmax = 1 << 20  # 16*64*256*(128+2)*4 bytes of split states: far above the limit
    assert atf.decode_workspace_bytes(B, Hq, Hkv, Nmax, D) > LIMIT
    fake = torch.empty(64, dtype=torch.uint8, device="cuda")  # never touched: rejected first
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _fn()(_ptr(fake), _ptr(fake), _ptr(fake), _ptr(fake), _ptr(fake), B, Hq, Hkv, Nmax, D, 1e7, 16.0, 0,
               atf.KV_HND, atf.BF16, atf.F32, stream)
    assert rc == -3  # ATFLASH_ERR_WORKSPACE
