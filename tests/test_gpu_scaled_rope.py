"""GPU parity of the scaled-RoPE calls (caller's frequency table instead of a base).

The oracle runs with the same table installed (``oracle.scaled_rope``), which
replaces base^(-2r/D) in its windows and rotations.  A table equal to the
library's own base table must give bit-identical results to the base-taking
calls.
"""
import math

import numpy as np
import pytest

import parity as P
from scaled import llama3_scaled_theta

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_attention_pair_b200 as atf  # noqa: E402


@pytest.mark.parametrize("B,N,Hq,Hkv,D,base,kwin,dtype", [
    (1, 3000, 4, 2, 128, 5e5, 16.0, "bf16"),     # Llama-3.2-3B heads and base, scaled
    (2, 1500, 7, 1, 64, 1e6, 2.0, "bf16"),
    (1, 1200, 3, 3, 128, 5e5, math.inf, "bf16"),
    (1, 300, 2, 1, 64, 1e4, 0.5, "f32"),
])
def test_scaled_prefill_matches_oracle(oracle, B, N, Hq, Hkv, D, base, kwin, dtype):
    th = llama3_scaled_theta(D, base, factor=32.0, orig_ctx=min(8192.0, N / 2))
    q = P.gen(71, "q", (B, N, Hq, D), dtype)
    k = P.gen(71, "k", (B, N, Hkv, D), dtype)
    v = P.gen(71, "v", (B, N, Hkv, D), dtype)
    out = atf.prefill(q, k, v, 0.0, kwin, theta=th, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    with oracle.scaled_rope(th):
        ref = oracle.prefill(P.host(q), P.host(k), P.host(v), base, kwin)
    P.check(P.host(out), ref, dtype, f"scaled prefill D={D} k={kwin}")


@pytest.mark.parametrize("D,base,kwin", [(64, 1e6, 8.0), (128, 5e5, 16.0)])
def test_scaled_packed_prefill_equals_scaled_prefill(D, base, kwin):
    # rope_pack + prefill_packed + prefill_short_rows with a scaled table is the
    # same computation as the one-call prefill with that table (which carves the
    # same packed scratch and runs the same three steps).
    th = llama3_scaled_theta(D, base, factor=32.0, orig_ctx=512.0)
    q = P.gen(74, "q", (1, 2000, 6, D), "bf16")
    k = P.gen(74, "k", (1, 2000, 2, D), "bf16")
    v = P.gen(74, "v", (1, 2000, 2, D), "bf16")
    qp = atf.rope_pack(q, 0.0, theta=th)
    kp = atf.rope_pack(k, 0.0, theta=th)
    a = atf.prefill_packed(qp, kp, v, 0.0, kwin, theta=th)
    atf.prefill_short_rows(q, k, v, a, 0.0, kwin, theta=th)
    b = atf.prefill(q, k, v, 0.0, kwin, theta=th)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    assert torch.equal(a, b)
    # and not what the unscaled base table gives
    c = atf.prefill_packed(atf.rope_pack(q, base), atf.rope_pack(k, base), v, base, kwin)
    atf.prefill_short_rows(q, k, v, c, base, kwin)
    torch.cuda.synchronize()
    assert not torch.equal(a, c)


@pytest.mark.parametrize("D,base,kwin", [(64, 1e6, 8.0), (128, 5e5, 16.0), (128, 1e7, math.inf)])
def test_base_table_prefill_is_bit_identical(D, base, kwin):
    q = P.gen(72, "q", (1, 1000, 4, D), "bf16")
    k = P.gen(72, "k", (1, 1000, 2, D), "bf16")
    v = P.gen(72, "v", (1, 1000, 2, D), "bf16")
    a = atf.prefill(q, k, v, base, kwin)
    b = atf.prefill(q, k, v, 0.0, kwin, theta=atf.theta_table(D, base))
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("B,Hq,Hkv,Nmax,D,seqlens,base,kwin,layout", [
    (2, 8, 2, 5000, 128, [5000, 1777], 5e5, 16.0, "HND"),
    (1, 7, 1, 4097, 64, [4097], 1e6, 4.0, "NHD"),
    (2, 28, 4, 3000, 128, [3000, 2048], 5e5, 16.0, "PACKED"),
])
def test_scaled_decode_matches_oracle(oracle, B, Hq, Hkv, Nmax, D, seqlens, base, kwin, layout):
    th = llama3_scaled_theta(D, base, factor=32.0, orig_ctx=1024.0)
    q = P.gen(73, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(73, "k_cache", (B, Hkv, Nmax, D), "bf16")
    vc = P.gen(73, "v_cache", (B, Hkv, Nmax, D), "bf16")
    sl = torch.tensor(seqlens, dtype=torch.int32, device="cuda")
    if layout == "PACKED":
        kp = atf.rope_pack(kc.permute(0, 2, 1, 3).contiguous(), 0.0, theta=th)
        out = atf.decode(q, kp, vc, sl, 0.0, kwin, kcache_rotated=True, kv_layout="PACKED",
                         out_dtype=torch.float32, theta=th)
    elif layout == "NHD":
        out = atf.decode(q, kc.permute(0, 2, 1, 3).contiguous(), vc.permute(0, 2, 1, 3).contiguous(), sl, 0.0,
                         kwin, kv_layout="NHD", out_dtype=torch.float32, theta=th)
    else:
        out = atf.decode(q, kc, vc, sl, 0.0, kwin, out_dtype=torch.float32, theta=th)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    with oracle.scaled_rope(th):
        ref = oracle.decode(P.host(q), P.host(kc), P.host(vc), seqlens, base, kwin)
    P.check(P.host(out), ref, "bf16", f"scaled decode {layout} D={D}")


def test_base_table_decode_is_bit_identical():
    B, Hq, Hkv, Nmax, D, base, kwin = 2, 8, 2, 3000, 128, 1e7, 16.0
    q = P.gen(74, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(74, "k_cache", (B, Hkv, Nmax, D), "bf16")
    vc = P.gen(74, "v_cache", (B, Hkv, Nmax, D), "bf16")
    sl = torch.tensor([3000, 1234], dtype=torch.int32, device="cuda")
    a = atf.decode(q, kc, vc, sl, base, kwin)
    b = atf.decode(q, kc, vc, sl, 0.0, kwin, theta=atf.theta_table(D, base))
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_scaled_varlen_prefill_matches_oracle(oracle):
    import test_gpu_varlen as VL
    lens, Hq, Hkv, D, base, kwin = [700, 1, 1300], 4, 2, 128, 5e5, 2.0
    th = llama3_scaled_theta(D, base, factor=32.0, orig_ctx=512.0)
    q, k, v, cu = VL.packed_batch(75, lens, Hq, Hkv, D)
    cu_d = torch.as_tensor(cu, device="cuda")
    out = atf.prefill_varlen(q, k, v, cu_d, max(lens), 0.0, kwin, out_dtype=torch.float32, theta=th)
    base_out = atf.prefill_varlen(q, k, v, cu_d, max(lens), base, kwin, out_dtype=torch.float32)
    same = atf.prefill_varlen(q, k, v, cu_d, max(lens), 0.0, kwin, out_dtype=torch.float32,
                              theta=atf.theta_table(D, base))
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    assert torch.equal(same, base_out)
    with oracle.scaled_rope(th):
        VL.check_against_oracle(oracle, q, k, v, cu, out, base, kwin)


def test_scaled_paged_decode_equals_contiguous_scaled_decode():
    import test_gpu_paged as PG
    B, Hq, Hkv, L, D, P_, base, kwin = 2, 8, 2, 2048, 128, 64, 5e5, 4.0
    th = llama3_scaled_theta(D, base, factor=32.0, orig_ctx=1024.0)
    q = P.gen(76, "q_dec", (B, Hq, D), "bf16")
    kc = P.gen(76, "k_cache", (B, Hkv, L, D), "bf16")
    vc = P.gen(76, "v_cache", (B, Hkv, L, D), "bf16")
    sl = torch.tensor([2048, 999], dtype=torch.int32, device="cuda")
    ids, n_pool = PG.scatter_pages(B, Hkv, L, P_, 77)
    bt = torch.as_tensor(ids, device="cuda")
    kpool, vpool = PG.nhd_pool(kc, ids, n_pool, P_), PG.nhd_pool(vc, ids, n_pool, P_)
    ref = atf.decode(q, kc, vc, sl, 0.0, kwin, out_dtype=torch.float32, theta=th)
    out = atf.decode_paged(q, kpool, vpool, bt, sl, P_, 0.0, kwin, out_dtype=torch.float32, theta=th)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    assert torch.equal(out, ref)


@pytest.mark.slow
def test_scaled_prefill_llama3b_128k_sampled(oracle):
    # The benchmark's scaled-RoPE workload (Llama-3.2-3B shape with its llama3
    # rope_scaling table at 128K), sampled query rows of every head.
    import bench
    wl = bench.WORKLOADS["llama3b_128k_scaled"]
    th = bench.rope_theta(wl)
    N, Hq, Hkv, D, kwin = wl["N"], wl["Hq"], wl["Hkv"], wl["D"], wl["k_window"]
    q = P.gen(76, "q", (1, N, Hq, D), "bf16")
    k = P.gen(76, "k", (1, N, Hkv, D), "bf16")
    v = P.gen(76, "v", (1, N, Hkv, D), "bf16")
    out = atf.prefill(q, k, v, 0.0, kwin, theta=th)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    rows = P.sample_rows(N, 24, 76)
    idx = torch.as_tensor(rows, device=q.device)
    with oracle.scaled_rope(th):
        ref = oracle.prefill_rows(P.host(q[0, idx]), rows, P.host(k[0]), P.host(v[0]), wl["rope_base"], kwin)
    P.check(P.host(out[0, idx]), ref, "bf16", "scaled 128K")
