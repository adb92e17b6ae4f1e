"""Rows that see at most 128 keys, computed in fp32 (include/atflash.h, "Accuracy
of short rows").

The tensor-core path rounds the rotated Q~/K~ and P to bf16; on a row with a
handful of keys that rounding does not average out, so every such row is
recomputed in fp32 from the un-rotated inputs.  These tests check, against the
fp64 oracle on the same bytes:
  - the rows of the first 128-row tile at the fp32 bar (1e-4), every row of a
    16-seed sweep at the bf16 bar, for D 64 / 128 with the window on and off;
  - rope_pack + prefill_packed + prefill_short_rows gives the bits of prefill;
  - decode of sequences of at most 128 tokens at the fp32 bar in every cache
    layout (HND, NHD, pre-rotated, packed, paged), and the 129-token boundary.
"""
import math

import numpy as np
import pytest

import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_attention_pair_b200 as atf  # noqa: E402


def inputs(seed, B, N, Hq, Hkv, D):
    return (P.gen(seed, "q", (B, N, Hq, D), "bf16"), P.gen(seed, "k", (B, N, Hkv, D), "bf16"),
            P.gen(seed, "v", (B, N, Hkv, D), "bf16"))


@pytest.mark.parametrize("D,base,kwin", [(64, 1e6, 8.0), (64, 1e6, math.inf), (128, 5e5, 16.0),
                                         (128, 1e7, math.inf)])
def test_seed_sweep_short_rows_exact_and_every_row_in_bound(oracle, D, base, kwin):
    N, Hq, Hkv = 320, 4, 2
    worst_long = 0.0
    for seed in range(16):
        q, k, v = inputs(100 + seed, 1, N, Hq, Hkv, D)
        out, lse = atf.prefill(q, k, v, base, kwin, out_dtype=torch.float32, return_lse=True)
        torch.cuda.synchronize()
        assert atf.device_status() == 0
        ref, rlse = oracle.prefill(P.host(q), P.host(k), P.host(v), base, kwin, want_lse=True)
        got = P.host(out)
        P.check(got[:, :128], ref[:, :128], "f32", f"rows 0-127 seed {seed}")
        P.check(P.host(lse)[:, :, :128], rlse.transpose(0, 2, 1)[:, :, :128], "f32", f"lse rows 0-127 seed {seed}")
        P.check(got, ref, "bf16", f"all rows seed {seed}")
        worst_long = max(worst_long, float(np.abs(got[:, 128:] - ref[:, 128:]).max()))
    # Rows of more than 128 keys keep the tensor-core rounding: measured below 5e-3.
    assert worst_long <= 5e-3, worst_long


@pytest.mark.parametrize("B,N,Hq,Hkv,D,base,kwin", [
    (2, 200, 6, 2, 64, 1e6, 8.0), (1, 1, 2, 1, 128, 1e4, 1.0), (1, 77, 7, 1, 128, 10.0, 0.25),
    (1, 1000, 3, 3, 64, 1e4, math.inf)])
def test_packed_stages_plus_short_rows_equal_fused_call(B, N, Hq, Hkv, D, base, kwin):
    q, k, v = inputs(7, B, N, Hq, Hkv, D)
    a, la = atf.prefill(q, k, v, base, kwin, out_dtype=torch.float32, return_lse=True)
    b = torch.empty_like(a)
    lb = torch.empty_like(la)
    atf.prefill_packed(atf.rope_pack(q, base), atf.rope_pack(k, base), v, base, kwin, out=b, lse=lb)
    atf.prefill_short_rows(q, k, v, b, base, kwin, lse=lb)
    torch.cuda.synchronize()
    assert torch.equal(a, b) and torch.equal(la, lb)


def test_short_rows_bf16_output(oracle):
    q, k, v = inputs(9, 1, 150, 4, 2, 128)
    out = atf.prefill(q, k, v, 5e5, 16.0)
    torch.cuda.synchronize()
    ref = oracle.prefill(P.host(q), P.host(k), P.host(v), 5e5, 16.0)
    err = np.abs(P.host(out)[:, :128] - ref[:, :128])
    half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref[:, :128]), 1e-30))) - 8)
    assert np.all(err <= 1e-4 + half_ulp)


def unpack_rotated(kpack, B, Hkv, Nmax, D):
    """The packed rotated cache [B*Hkv][D/16][Nmax][16] back to [B][Hkv][Nmax][D] (host)."""
    H = D // 2
    x = P.host(kpack).reshape(B, Hkv, D // 16, Nmax, 8, 2)
    out = np.empty((B, Hkv, Nmax, D), np.float32)
    out[..., :H] = x[..., 0].transpose(0, 1, 3, 2, 4).reshape(B, Hkv, Nmax, H)
    out[..., H:] = x[..., 1].transpose(0, 1, 3, 2, 4).reshape(B, Hkv, Nmax, H)
    return out


SEQLENS = [1, 5, 16, 77, 128, 129, 300]


@pytest.mark.parametrize("D,layout,krot", [(128, "HND", 0), (64, "NHD", 0), (128, "HND", 1), (64, "PACKED", 1),
                                           (128, "PACKED", 1)])
def test_short_decode_sequences_exact(oracle, D, layout, krot):
    B, Hq, Hkv, Nmax, base, kwin = len(SEQLENS), 8, 2, 320, 1e6, 8.0
    q = P.gen(81, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(81, "k_cache", (B, Hkv, Nmax, D), "bf16")
    vc = P.gen(81, "v_cache", (B, Hkv, Nmax, D), "bf16")
    sl = torch.tensor(SEQLENS, dtype=torch.int32, device="cuda")
    ref_rot = False
    if layout == "PACKED":
        kin = atf.rope_pack(kc.permute(0, 2, 1, 3).contiguous(), base)
        kref, ref_rot = unpack_rotated(kin, B, Hkv, Nmax, D), True
    elif krot:
        pos = np.arange(Nmax)
        kh = P.host(kc)
        rot = np.stack([np.stack([oracle.rope_rows(kh[b, g], pos, base) for g in range(Hkv)]) for b in range(B)])
        kin = torch.from_numpy(rot.astype(np.float32)).to(torch.bfloat16).cuda()
        kref, ref_rot = P.host(kin), True
    else:
        kin = kc if layout == "HND" else kc.permute(0, 2, 1, 3).contiguous()
        kref = P.host(kc)
    vin = vc if layout != "NHD" else vc.permute(0, 2, 1, 3).contiguous()
    out = atf.decode(q, kin, vin, sl, base, kwin, kcache_rotated=bool(krot), kv_layout=layout,
                     out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    ref = oracle.decode(P.host(q), kref, P.host(vc), SEQLENS, base, kwin, kcache_rotated=ref_rot)
    got = P.host(out)
    short = [i for i, L in enumerate(SEQLENS) if L <= 128]
    longer = [i for i, L in enumerate(SEQLENS) if L > 128]
    P.check(got[short], ref[short], "f32", f"decode L<=128 {layout} krot={krot}")
    P.check(got[longer], ref[longer], "bf16", f"decode L>128 {layout} krot={krot}")


@pytest.mark.parametrize("packed", [False, True])
def test_short_paged_decode_exact(oracle, packed):
    from test_gpu_paged import nhd_pool, packed_pool, scatter_pages
    B, Hq, Hkv, L, D, P_, base, kwin = 3, 8, 2, 256, 128, 64, 1e7, 16.0
    q = P.gen(82, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(82, "k_cache", (B, Hkv, L, D), "bf16")
    vc = P.gen(82, "v_cache", (B, Hkv, L, D), "bf16")
    ids, n_pool = scatter_pages(B, Hkv, L, P_, 83)
    vp = nhd_pool(vc, ids, n_pool, P_)
    seqlens = [3, 128, 100]
    if packed:
        kpack = atf.rope_pack(kc.permute(0, 2, 1, 3).contiguous(), base)
        kp = packed_pool(kpack, ids, n_pool, P_, Hkv)
        kref, ref_rot = unpack_rotated(kpack, B, Hkv, L, D), True
    else:
        kp = nhd_pool(kc, ids, n_pool, P_)
        kref, ref_rot = P.host(kc), False
    out = atf.decode_paged(q, kp, vp, torch.as_tensor(ids, device="cuda"),
                           torch.tensor(seqlens, dtype=torch.int32, device="cuda"), P_, base, kwin,
                           kcache_rotated=packed, kv_layout="PACKED" if packed else "NHD", out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    ref = oracle.decode(P.host(q), kref, P.host(vc), seqlens, base, kwin, kcache_rotated=ref_rot)
    P.check(P.host(out), ref, "f32", f"paged short decode packed={packed}")
