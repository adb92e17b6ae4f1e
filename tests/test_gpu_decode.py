"""GPU parity of the split-KV decode path (C ABI via the binding) against the fp64 oracle."""
import math

import numpy as np
import pytest

import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_attention_pair_b200 as atf  # noqa: E402


def rope_rotate_cache(oracle, kc, base):
    """Pre-rotated cache for the kcache_rotated=1 path (oracle's fp64 RoPE, rounded to the cache dtype)."""
    B, Hkv, Nmax, D = kc.shape
    kh = P.host(kc)
    out = np.empty_like(kh)
    pos = np.arange(Nmax)
    for b in range(B):
        for g in range(Hkv):
            out[b, g] = oracle.rope_rows(kh[b, g], pos, base).astype(np.float32)
    return torch.from_numpy(out).to(kc.dtype).to(kc.device)


def test_tiny_fp32_decode_of_last_row(oracle):
    # Tiny exactness case: decode of row N-1 against the oracle (and against prefill row N-1).
    N, D = 256, 64
    q = P.gen(0, "q", (1, N, 1, D), "f32")
    k = P.gen(0, "k", (1, N, 1, D), "f32")
    v = P.gen(0, "v", (1, N, 1, D), "f32")
    kc = k.permute(0, 2, 1, 3).contiguous()
    vc = v.permute(0, 2, 1, 3).contiguous()
    seqlens = torch.tensor([N], dtype=torch.int32, device="cuda")
    for kwin in (1.0, math.inf):
        out = atf.decode(q[:, N - 1].contiguous(), kc, vc, seqlens, 1e4, kwin)
        pre = atf.prefill(q, k, v, 1e4, kwin)
        torch.cuda.synchronize()
        ref = oracle.decode(P.host(q[:, N - 1]), P.host(kc), P.host(vc), [N], 1e4, kwin)
        P.check(P.host(out), ref, "f32", f"decode k={kwin}")
        P.check(P.host(out), P.host(pre[:, N - 1]), "f32", "decode vs prefill row")


SMALL = [
    # B, Hq, Hkv, Nmax, D, seqlens, base, kwin, krot, dtype
    (3, 8, 2, 5000, 128, [5000, 1, 2049], 1e4, 1.0, 0, "bf16"),
    (2, 7, 1, 4097, 64, [4097, 300], 1e6, 8.0, 0, "bf16"),
    (2, 28, 4, 3000, 128, [3000, 2048], 1e7, 16.0, 0, "bf16"),
    (2, 28, 4, 3000, 128, [3000, 2048], 1e7, math.inf, 0, "bf16"),
    (2, 4, 4, 2500, 128, [2500, 1700], 1e4, 2.0, 1, "bf16"),
    (1, 16, 1, 900, 64, [900], 10.0, 0.25, 0, "bf16"),
    (2, 6, 2, 3000, 128, [3000, 17], 5e5, 16.0, 0, "f32"),
    (1, 4, 2, 1500, 64, [1500], 1e4, 1.0, 1, "f32"),
    # groups of 9..16 heads take two 8-head tiles of the MMA's N
    (2, 24, 2, 2100, 128, [2100, 1500], 5e5, 16.0, 0, "bf16"),
    (1, 10, 1, 1300, 64, [1300], 1e4, 2.0, 1, "bf16"),
    # k = 0: only the query's own position keeps its pairs
    (2, 8, 2, 900, 128, [900, 333], 1e4, 0.0, 0, "bf16"),
]


@pytest.mark.parametrize("B,Hq,Hkv,Nmax,D,seqlens,base,kwin,krot,dtype", SMALL)
def test_decode_matches_oracle(oracle, B, Hq, Hkv, Nmax, D, seqlens, base, kwin, krot, dtype):
    q = P.gen(21, "q_dec", (B, Hq, D), dtype)
    kc = P.gen(21, "k_cache", (B, Hkv, Nmax, D), dtype)
    vc = P.gen(21, "v_cache", (B, Hkv, Nmax, D), dtype)
    if krot:
        kc = rope_rotate_cache(oracle, kc, base)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    out = atf.decode(q, kc, vc, sl, base, kwin, kcache_rotated=bool(krot), out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.decode(P.host(q), P.host(kc), P.host(vc), seqlens, base, kwin, kcache_rotated=bool(krot))
    P.check(P.host(out), ref, dtype, f"decode D={D} k={kwin} krot={krot}")


@pytest.mark.parametrize("B,Hq,Hkv,Nmax,D,seqlens,base,kwin", [
    (3, 8, 2, 5000, 128, [5000, 1, 2049], 1e4, 1.0),
    (2, 28, 4, 3000, 128, [3000, 2048], 1e7, 16.0),
    (2, 7, 1, 4097, 64, [4097, 300], 1e6, 8.0),
    (1, 16, 1, 900, 64, [900], 10.0, 0.25),
    # two head tiles at D = 128; a cache length that is not a multiple of 4
    (2, 24, 2, 2102, 128, [2102, 999], 5e5, 16.0),
    (1, 12, 1, 2048, 128, [2048], 1e4, 4.0),
    (2, 8, 2, 1000, 64, [1000, 65], 1e4, 0.0),
])
def test_packed_rotated_cache_matches_oracle(oracle, B, Hq, Hkv, Nmax, D, seqlens, base, kwin):
    # The RoPE pre-pass writes the packed cache from the un-rotated keys; the oracle
    # rotates the same un-rotated keys itself.
    q = P.gen(23, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(23, "k_cache", (B, Hkv, Nmax, D), "bf16")
    vc = P.gen(23, "v_cache", (B, Hkv, Nmax, D), "bf16")
    kpack = atf.rope_pack(kc.permute(0, 2, 1, 3).contiguous(), base)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    out = atf.decode(q, kpack, vc, sl, base, kwin, kcache_rotated=True, kv_layout="PACKED",
                     out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.decode(P.host(q), P.host(kc), P.host(vc), seqlens, base, kwin)
    P.check(P.host(out), ref, "bf16", f"packed decode D={D} k={kwin}")


def test_decode_window_covering_everything_is_bit_identical_to_off():
    B, Hq, Hkv, Nmax, D, base = 2, 8, 2, 3000, 128, 1e4
    q = P.gen(22, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(22, "k_cache", (B, Hkv, Nmax, D), "bf16")
    vc = P.gen(22, "v_cache", (B, Hkv, Nmax, D), "bf16")
    sl = torch.tensor([3000, 1234], dtype=torch.int32, device="cuda")
    kwin = 2.0 * Nmax / (2 * math.pi)
    a = atf.decode(q, kc, vc, sl, base, kwin)
    b = atf.decode(q, kc, vc, sl, base, math.inf)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def decode_full_size(oracle, B, L, kwin, seed):
    Hq, Hkv, D, base = 28, 4, 128, 1e7
    q = P.gen(seed, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(seed, "k_cache", (B, Hkv, L, D), "bf16")
    vc = P.gen(seed, "v_cache", (B, Hkv, L, D), "bf16")
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    out = atf.decode(q, kc, vc, sl, base, kwin, out_dtype=torch.float32)
    torch.cuda.synchronize()
    got = P.host(out)
    for b in range(B):  # one sequence at a time keeps the host copy small
        ref = oracle.decode(P.host(q[b:b + 1]), P.host(kc[b:b + 1]), P.host(vc[b:b + 1]), [L], base, kwin)
        P.check(got[b:b + 1], ref, "bf16", f"decode L={L} k={kwin} b={b}")


@pytest.mark.slow
@pytest.mark.parametrize("kwin", [16.0, 64.0])
def test_decode_qwen7b_1m_shape(oracle, kwin):
    decode_full_size(oracle, 4, 1 << 20, kwin, seed=31)


@pytest.mark.slow
@pytest.mark.parametrize("kwin", [16.0, 64.0])
def test_decode_qwen7b_128k_16_seqs(oracle, kwin):
    decode_full_size(oracle, 16, 1 << 17, kwin, seed=32)


@pytest.mark.slow
def test_decode_qwen7b_128k_window_off(oracle):
    decode_full_size(oracle, 16, 1 << 17, math.inf, seed=34)


@pytest.mark.slow
def test_decode_qwen7b_1m_packed_cache(oracle):
    B, L, Hq, Hkv, D, base, kwin = 4, 1 << 20, 28, 4, 128, 1e7, 16.0
    q = P.gen(33, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(33, "k_cache", (B, Hkv, L, D), "bf16")
    vc = P.gen(33, "v_cache", (B, Hkv, L, D), "bf16")
    kpack = atf.rope_pack(kc.permute(0, 2, 1, 3).contiguous(), base)
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    out = atf.decode(q, kpack, vc, sl, base, kwin, kcache_rotated=True, kv_layout="PACKED",
                     out_dtype=torch.float32)
    torch.cuda.synchronize()
    got = P.host(out)
    del kpack
    for b in range(B):
        ref = oracle.decode(P.host(q[b:b + 1]), P.host(kc[b:b + 1]), P.host(vc[b:b + 1]), [L], base, kwin)
        P.check(got[b:b + 1], ref, "bf16", f"packed decode 1M b={b}")
