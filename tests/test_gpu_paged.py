"""GPU parity of the paged-cache decode.

A paged cache is the contiguous cache cut into pages and scattered through a
pool by a block table; decoding it must give exactly what decoding the
contiguous cache gives (same splits, same stages), and the oracle's decode of
the gathered cache.
"""
import math

import numpy as np
import pytest

import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_attention_pair_b200 as atf  # noqa: E402


def scatter_pages(B, Hkv, L, P_, seed):
    """Random block table: page ids 0..B*L/P-1 shuffled, plus 3 unused pool pages."""
    mp = L // P_
    rng = np.random.default_rng(seed)
    ids = rng.permutation(B * mp + 3)[: B * mp].astype(np.int32).reshape(B, mp)
    return ids, B * mp + 3


def nhd_pool(cache, ids, n_pool, P_):
    """cache [B, Hkv, L, D] -> pool [n_pool, P, Hkv, D] (unused pages random)."""
    B, Hkv, L, D = cache.shape
    pool = torch.randn((n_pool, P_, Hkv, D), device=cache.device).to(cache.dtype)
    for b in range(B):
        for i in range(L // P_):
            pool[int(ids[b, i])] = cache[b, :, i * P_:(i + 1) * P_, :].permute(1, 0, 2)
    return pool


def packed_pool(kpack, ids, n_pool, P_, Hkv):
    """kpack [B*Hkv, D/16, L, 16] -> pool [n_pool, Hkv, D/16, P, 16]."""
    BH, C, L, _ = kpack.shape
    B = BH // Hkv
    pool = torch.zeros((n_pool, Hkv, C, P_, 16), dtype=kpack.dtype, device=kpack.device)
    for b in range(B):
        for i in range(L // P_):
            pool[int(ids[b, i])] = kpack[b * Hkv:(b + 1) * Hkv, :, i * P_:(i + 1) * P_, :]
    return pool


CASES = [
    # B, Hq, Hkv, L, D, page, seqlens, base, kwin, krot
    (3, 8, 2, 4096, 128, 64, [4096, 1, 2000], 1e7, 16.0, 0),
    (2, 7, 1, 2048, 64, 256, [2048, 777], 1e6, 8.0, 0),
    (2, 28, 4, 3072, 128, 128, [3072, 3000], 1e7, math.inf, 0),
    (2, 4, 4, 1024, 128, 64, [1024, 65], 1e4, 2.0, 1),
    (1, 16, 1, 1024, 128, 64, [1000], 1e4, 4.0, 0),
]


@pytest.mark.parametrize("B,Hq,Hkv,L,D,P_,seqlens,base,kwin,krot", CASES)
def test_paged_nhd_equals_contiguous_and_oracle(oracle, B, Hq, Hkv, L, D, P_, seqlens, base, kwin, krot):
    q = P.gen(71, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(71, "k_cache", (B, Hkv, L, D), "bf16")
    vc = P.gen(71, "v_cache", (B, Hkv, L, D), "bf16")
    if krot:
        kh = P.host(kc)
        rot = np.empty_like(kh)
        for b in range(B):
            for g in range(Hkv):
                rot[b, g] = oracle.rope_rows(kh[b, g], np.arange(L), base).astype(np.float32)
        kc = torch.from_numpy(rot).to(kc.dtype).to(kc.device)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    ids, n_pool = scatter_pages(B, Hkv, L, P_, 72)
    kp, vp = nhd_pool(kc, ids, n_pool, P_), nhd_pool(vc, ids, n_pool, P_)
    bt = torch.as_tensor(ids, device="cuda")
    out = atf.decode_paged(q, kp, vp, bt, sl, P_, base, kwin, kcache_rotated=bool(krot), out_dtype=torch.float32)
    ref = atf.decode(q, kc, vc, sl, base, kwin, kcache_rotated=bool(krot), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    oref = oracle.decode(P.host(q), P.host(kc), P.host(vc), seqlens, base, kwin, kcache_rotated=bool(krot))
    P.check(P.host(out), oref, "bf16", f"paged D={D} page={P_} k={kwin}")


@pytest.mark.parametrize("B,Hq,Hkv,L,D,P_,seqlens,base,kwin", [
    (3, 8, 2, 4096, 128, 64, [4096, 1, 2000], 1e7, 16.0),
    (2, 7, 1, 2048, 64, 128, [2048, 777], 1e6, 8.0),
])
def test_paged_packed_equals_contiguous_packed(oracle, B, Hq, Hkv, L, D, P_, seqlens, base, kwin):
    q = P.gen(73, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(73, "k_cache", (B, Hkv, L, D), "bf16")
    vc = P.gen(73, "v_cache", (B, Hkv, L, D), "bf16")
    kpack = atf.rope_pack(kc.permute(0, 2, 1, 3).contiguous(), base)
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    ids, n_pool = scatter_pages(B, Hkv, L, P_, 74)
    kp = packed_pool(kpack, ids, n_pool, P_, Hkv)
    vp = nhd_pool(vc, ids, n_pool, P_)
    bt = torch.as_tensor(ids, device="cuda")
    out = atf.decode_paged(q, kp, vp, bt, sl, P_, base, kwin, kcache_rotated=True, kv_layout="PACKED",
                           out_dtype=torch.float32)
    ref = atf.decode(q, kpack, vc, sl, base, kwin, kcache_rotated=True, kv_layout="PACKED", out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    oref = oracle.decode(P.host(q), P.host(kc), P.host(vc), seqlens, base, kwin)
    P.check(P.host(out), oref, "bf16", f"paged packed D={D}")


@pytest.mark.parametrize("L,bad_index", [(512, 3), (512, 5), (100, 1)])
def test_paged_bad_page_ids_are_reported(L, bad_index):
    # A page id outside the pool or a negative one is an error the kernels find on
    # the device: the status word reads ATFLASH_ERR_BAD_PAGE (no fault, no hang),
    # and the next call with a valid table reads OK again.  L = 100 takes the
    # short-sequence fp32 path too.
    B, Hq, Hkv, D, P_ = 1, 4, 2, 128, 64
    q = P.gen(75, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(75, "k_cache", (B, Hkv, 512, D), "bf16")
    vc = P.gen(75, "v_cache", (B, Hkv, 512, D), "bf16")
    ids, n_pool = scatter_pages(B, Hkv, 512, P_, 76)
    kp, vp = nhd_pool(kc, ids, n_pool, P_), nhd_pool(vc, ids, n_pool, P_)
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    assert atf.device_status() == 0
    bad = ids.copy()
    bad[0, bad_index] = 10 ** 7 if bad_index != 5 else -4
    atf.decode_paged(q, kp, vp, torch.as_tensor(bad, device="cuda"), sl, P_, 1e7, 16.0, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert atf.device_status() == atf.ERR_BAD_PAGE
    atf.decode_paged(q, kp, vp, torch.as_tensor(ids, device="cuda"), sl, P_, 1e7, 16.0, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert atf.device_status() == 0


@pytest.mark.slow
@pytest.mark.parametrize("packed", [True, False])
def test_paged_bench_size_equals_contiguous(packed):
    # The benchmark's paged workload (4 x 1M keys of the Qwen2.5-7B-1M shape in
    # shuffled 256-token pages): bit-identical to the contiguous cache, whose
    # full-size parity against the oracle the decode tests check.
    B, Hq, Hkv, L, D, P_, base, kwin = 4, 28, 4, 1 << 20, 128, 256, 1e7, 16.0
    q = P.gen(77, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(77, "k_cache", (B, Hkv, L, D), "bf16")
    vc = P.gen(77, "v_cache", (B, Hkv, L, D), "bf16")
    sl = torch.full((B,), L, dtype=torch.int32, device="cuda")
    mp = L // P_
    ids, n_pool = scatter_pages(B, Hkv, L, P_, 78)
    idx = torch.as_tensor(ids.reshape(-1).astype(np.int64), device="cuda")
    C = D // 16
    vp = torch.zeros((n_pool, P_, Hkv, D), dtype=vc.dtype, device="cuda")
    vp[idx] = vc.view(B, Hkv, mp, P_, D).permute(0, 2, 3, 1, 4).reshape(B * mp, P_, Hkv, D)
    if packed:
        kcont = atf.rope_pack(kc.permute(0, 2, 1, 3).contiguous(), base)
        kp = torch.zeros((n_pool, Hkv, C, P_, 16), dtype=kc.dtype, device="cuda")
        kp[idx] = kcont.view(B, Hkv, C, mp, P_, 16).permute(0, 3, 1, 2, 4, 5).reshape(B * mp, Hkv, C, P_, 16)
        kw = dict(kcache_rotated=True, kv_layout="PACKED")
    else:
        kcont = kc
        kp = torch.zeros((n_pool, P_, Hkv, D), dtype=kc.dtype, device="cuda")
        kp[idx] = kc.view(B, Hkv, mp, P_, D).permute(0, 2, 3, 1, 4).reshape(B * mp, P_, Hkv, D)
        kw = {}
    bt = torch.as_tensor(ids, device="cuda")
    out = atf.decode_paged(q, kp, vp, bt, sl, P_, base, kwin, kv_layout=kw.get("kv_layout", "NHD"),
                           kcache_rotated=kw.get("kcache_rotated", False))
    ref = atf.decode(q, kcont, vc, sl, base, kwin, **kw)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    assert torch.equal(out, ref)
