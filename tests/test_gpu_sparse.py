"""GPU parity of the windowed prefill under a token-level block selection.

The oracle's ``prefill_rows_sparse`` is the definition: key m is visible to
query n iff m <= n and (same 128-position tile, or the block mask entry of the
tiles is set for n's KV group); the window prunes pair terms of the visible
cells and invisible keys take no part in the softmax.
"""
import math

import numpy as np
import pytest

import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_attention_pair_b200 as atf  # noqa: E402


def random_mask(B, Hkv, T, density, seed):
    """Independent random tiles, nothing forced: many query tiles keep no earlier
    key tile, so their rows see only their own tile's causal prefix."""
    rng = np.random.default_rng(seed)
    return (rng.random((B, Hkv, T, T)) < density).astype(np.uint8)


def own_tile_only(mask_bg, T):
    """Query tiles whose mask row keeps no earlier key tile (rows of at most 128 keys)."""
    return [i for i in range(T) if not np.any(mask_bg[i, :i])]


def run(oracle, B, N, Hq, Hkv, D, base, kwin, density, seed, rows=None):
    T = (N + 127) // 128
    q = P.gen(seed, "q", (B, N, Hq, D), "bf16")
    k = P.gen(seed, "k", (B, N, Hkv, D), "bf16")
    v = P.gen(seed, "v", (B, N, Hkv, D), "bf16")
    mask = random_mask(B, Hkv, T, density, seed + 1)
    out, lse = atf.prefill_sparse(q, k, v, torch.as_tensor(mask, device="cuda"), base, kwin,
                                  out_dtype=torch.float32, return_lse=True)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    sel = np.arange(N) if rows is None else rows
    G = Hq // Hkv
    for b in range(B):
        idx = torch.as_tensor(sel, device="cuda")
        ref, rlse = oracle.prefill_rows_sparse(P.host(q[b, idx]), sel, P.host(k[b]), P.host(v[b]), base, kwin,
                                               mask[b], 128, want_lse=True)
        got = P.host(out[b, idx])
        P.check(got, ref, "bf16", f"sparse b={b} D={D} k={kwin} density={density}")
        got_lse = P.host(lse[b][:, idx]).T
        assert np.max(np.abs(got_lse - rlse)) < 1e-2, "lse"
        # Rows of the query tiles that keep no earlier key tile are computed in fp32.
        for g in range(Hkv):
            for i in own_tile_only(mask[b, g], T):
                r = (sel >= 128 * i) & (sel < 128 * (i + 1))
                hs = slice(g * G, (g + 1) * G)
                P.check(got[r][:, hs], ref[r][:, hs], "f32", f"own-tile rows b={b} g={g} tile={i}")
    return q, k, v, mask, out


@pytest.mark.parametrize("B,N,Hq,Hkv,D,base,kwin,density", [
    (1, 2000, 4, 2, 64, 1e6, 8.0, 0.4),       # two heads per CTA, ragged last tile
    (2, 1100, 7, 1, 64, 1e4, 2.0, 0.25),      # odd group: a one-head CTA per group too
    (1, 1500, 3, 3, 64, 1e6, math.inf, 0.5),  # nothing pruned: one head per CTA, two CTAs per SM
    (1, 2049, 6, 2, 128, 5e5, 16.0, 0.3),
    (1, 900, 4, 4, 128, 10.0, 0.25, 0.6),     # many boundary pairs per tile
])
def test_sparse_matches_oracle(oracle, B, N, Hq, Hkv, D, base, kwin, density):
    run(oracle, B, N, Hq, Hkv, D, base, kwin, density, seed=91)


@pytest.mark.parametrize("D,kwin", [(64, 8.0), (64, math.inf), (128, 16.0)])
def test_all_visible_mask_is_bit_identical_to_dense(D, kwin):
    B, N, Hq, Hkv, base = 1, 1300, 4, 2, 1e6
    T = (N + 127) // 128
    q = P.gen(92, "q", (B, N, Hq, D), "bf16")
    k = P.gen(92, "k", (B, N, Hkv, D), "bf16")
    v = P.gen(92, "v", (B, N, Hkv, D), "bf16")
    ones = torch.ones((B, Hkv, T, T), dtype=torch.uint8, device="cuda")
    a = atf.prefill_sparse(q, k, v, ones, base, kwin)
    b = atf.prefill(q, k, v, base, kwin)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_diagonal_and_future_entries_are_ignored():
    B, N, Hq, Hkv, D, base, kwin = 1, 1700, 4, 2, 64, 1e6, 8.0
    T = (N + 127) // 128
    q = P.gen(93, "q", (B, N, Hq, D), "bf16")
    k = P.gen(93, "k", (B, N, Hkv, D), "bf16")
    v = P.gen(93, "v", (B, N, Hkv, D), "bf16")
    m = random_mask(B, Hkv, T, 0.4, 94)
    lower = np.tril(np.ones((T, T), np.uint8), -1)
    a_mask = m * lower                                          # diagonal and above cleared
    b_mask = a_mask + (1 - lower)                               # diagonal and above set
    a = atf.prefill_sparse(q, k, v, torch.as_tensor(a_mask, device="cuda"), base, kwin)
    b = atf.prefill_sparse(q, k, v, torch.as_tensor(b_mask, device="cuda"), base, kwin)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_diagonal_only_mask_matches_oracle(oracle):
    # Every row sees only its own tile's causal prefix (each tile a short sequence).
    B, N, Hq, Hkv, D, base, kwin = 1, 640, 1, 1, 128, 5e5, 16.0
    T = (N + 127) // 128
    q = P.gen(95, "q", (B, N, Hq, D), "bf16")
    k = P.gen(95, "k", (B, N, Hkv, D), "bf16")
    v = P.gen(95, "v", (B, N, Hkv, D), "bf16")
    zeros = np.zeros((B, Hkv, T, T), np.uint8)
    out = atf.prefill_sparse(q, k, v, torch.as_tensor(zeros, device="cuda"), base, kwin, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.prefill_rows_sparse(P.host(q[0]), np.arange(N), P.host(k[0]), P.host(v[0]), base, kwin, zeros[0],
                                     128)
    P.check(P.host(out[0]), ref, "f32", "diagonal only (every row computed in fp32)")


def test_bool_mask_and_shape_checks():
    B, N, Hq, Hkv, D = 1, 300, 2, 1, 64
    q = P.gen(96, "q", (B, N, Hq, D), "bf16")
    k = P.gen(96, "k", (B, N, Hkv, D), "bf16")
    v = P.gen(96, "v", (B, N, Hkv, D), "bf16")
    m = torch.ones((B, Hkv, 3, 3), dtype=torch.bool, device="cuda")
    a = atf.prefill_sparse(q, k, v, m, 1e4, 1.0)
    b = atf.prefill(q, k, v, 1e4, 1.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    with pytest.raises(ValueError):
        atf.prefill_sparse(q, k, v, torch.ones((B, Hkv, 2, 2), dtype=torch.uint8, device="cuda"), 1e4, 1.0)


@pytest.mark.slow
@pytest.mark.parametrize("name,rows", [("qwen05b_32k_sparse", 48), ("llama3b_128k_sparse", 16)])
def test_sparse_bench_workload_sampled(oracle, name, rows):
    # The benchmark's block-selected workloads (bf16 out, its mask recipe):
    # sampled query rows of every head against the oracle.
    import bench
    wl = bench.SPARSE_WORKLOADS[name]
    B, N, Hq, Hkv, D = wl["B"], wl["N"], wl["Hq"], wl["Hkv"], wl["D"]
    T = (N + 127) // 128
    mask = bench.block_mask_recipe(wl, T)
    q = P.gen(97, "q", (B, N, Hq, D), "bf16")
    k = P.gen(97, "k", (B, N, Hkv, D), "bf16")
    v = P.gen(97, "v", (B, N, Hkv, D), "bf16")
    out = atf.prefill_sparse(q, k, v, torch.as_tensor(mask, device="cuda"), wl["rope_base"], wl["k_window"])
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    sel = P.sample_rows(N, rows, 98)
    idx = torch.as_tensor(sel, device="cuda")
    ref = oracle.prefill_rows_sparse(P.host(q[0, idx]), sel, P.host(k[0]), P.host(v[0]), wl["rope_base"],
                                     wl["k_window"], mask[0], 128)
    P.check(P.host(out[0, idx]), ref, "bf16", name)


def test_theta_table_variant(oracle):
    # The base table through the _theta call is bit-identical to the base-taking
    # call; a scaled table matches the oracle with the same table installed.
    from scaled import llama3_scaled_theta
    B, N, Hq, Hkv, D, base, kwin = 1, 1500, 4, 2, 128, 5e5, 16.0
    T = (N + 127) // 128
    q = P.gen(99, "q", (B, N, Hq, D), "bf16")
    k = P.gen(99, "k", (B, N, Hkv, D), "bf16")
    v = P.gen(99, "v", (B, N, Hkv, D), "bf16")
    mask = random_mask(B, Hkv, T, 0.4, 100)
    m = torch.as_tensor(mask, device="cuda")
    a = atf.prefill_sparse(q, k, v, m, base, kwin)
    b = atf.prefill_sparse(q, k, v, m, 0.0, kwin, theta=atf.theta_table(D, base))
    th = llama3_scaled_theta(D, base, factor=32.0, orig_ctx=256.0)
    c = atf.prefill_sparse(q, k, v, m, 0.0, kwin, theta=th, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    with oracle.scaled_rope(th):
        ref = oracle.prefill_rows_sparse(P.host(q[0]), np.arange(N), P.host(k[0]), P.host(v[0]), base, kwin, mask[0],
                                         128)
    P.check(P.host(c[0]), ref, "bf16", "scaled sparse")
