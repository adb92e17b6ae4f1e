"""The decode entry point that allocates nothing (atflash_decode_noalloc).

It exists for callers that cannot allocate device memory when they call the
library (for instance a serving loop that must stay out of the CUDA allocator
once running, or a plugin whose host framework owns all device memory).  Its
split-state scratch is a fixed device array inside the library instead of a
caller workspace.  This test calls it through the C ABI twice in a row, with
different problem sizes so the second call runs over the first call's leftover
scratch contents, and checks each output against atflash_decode's on the same
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


def _call_noalloc(q, kc, vc, sl, out, base, kwin):
    B, Hq, D = q.shape
    _, Hkv, Nmax, _ = kc.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return _fn()(_ptr(q), _ptr(kc), _ptr(vc), _ptr(sl), _ptr(out), B, Hq, Hkv, Nmax, D, base, kwin, 0,
                 atf.KV_HND, atf.BF16, atf.F32, stream)


@pytest.mark.parametrize("shapes", [[(4, 28, 4, 20000, 128, 1e7, 16.0), (2, 14, 2, 5000, 64, 1e6, 8.0)]])
def test_noalloc_decode_matches_workspace_decode_twice(shapes):
    for call, (B, Hq, Hkv, Nmax, D, base, kwin) in enumerate(shapes):
        assert atf.decode_workspace_bytes(B, Hq, Hkv, Nmax, D) <= LIMIT
        q = P.gen(40 + call, "q_dec", (B, Hq, D), "bf16")
        kc = P.gen(40 + call, "k_cache", (B, Hkv, Nmax, D), "bf16")
        vc = P.gen(40 + call, "v_cache", (B, Hkv, Nmax, D), "bf16")
        sl = torch.tensor([Nmax - 37 * b for b in range(B)], dtype=torch.int32, device="cuda")
        out = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
        assert _call_noalloc(q, kc, vc, sl, out, base, kwin) == 0
        ref = atf.decode(q, kc, vc, sl, base, kwin, out_dtype=torch.float32)
        torch.cuda.synchronize()
        P.check(P.host(out), P.host(ref), "bf16", f"noalloc call {call + 1}")


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    B, Hq, Hkv, D = 16, 64, 4, 128
    Nmax = 1 << 20  # 16*64*512*(128+2)*4 bytes of split states: far above the limit
    assert atf.decode_workspace_bytes(B, Hq, Hkv, Nmax, D) > LIMIT
    fake = torch.empty(64, dtype=torch.uint8, device="cuda")  # never touched: rejected first
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = _fn()(_ptr(fake), _ptr(fake), _ptr(fake), _ptr(fake), _ptr(fake), B, Hq, Hkv, Nmax, D, 1e7, 16.0, 0,
               atf.KV_HND, atf.BF16, atf.F32, stream)
    assert rc == -3  # ATFLASH_ERR_WORKSPACE
