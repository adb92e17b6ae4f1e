"""Pins of the fp64 CPU oracle against facts fixed by the pages and by mathematics.

Each test pins the oracle to something other than itself:
  * textbook causal RoPE attention (k = inf), written in matrix form with numpy;
  * brute-force enumeration of the term count against the closed form;
  * hand-derived window values (lambda_0 = 2*pi exactly, the middle pair's
    lambda = 2*pi*sqrt(base));
  * the relative-angle property of RoPE (scores invariant under a common shift
    of both positions) and the per-pair decomposition of the full dot product;
  * the k = 0 closed form (only the diagonal keeps its pairs, every other cell
    is the empty sum 0);
  * the pages' printed pruning percentages;
  * reachability of every key through the lowest-frequency pair.
"""
import json
import math
import os

import numpy as np
import pytest

from long_context_attention_pair_b200 import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rope_textbook(x, pos, base):
    """Rotate-half RoPE in the usual matrix form x*cos + rotate_half(x)*sin."""
    D = x.shape[-1]
    H = D // 2
    inv_freq = 1.0 / (base ** (np.arange(0, D, 2, dtype=np.float64) / D))
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv_freq[None, :]
    cos = np.concatenate([np.cos(ang), np.cos(ang)], axis=-1)
    sin = np.concatenate([np.sin(ang), np.sin(ang)], axis=-1)
    x = np.asarray(x, dtype=np.float64)
    rot = np.concatenate([-x[:, H:], x[:, :H]], axis=-1)
    return x * cos + rot * sin


def attention_textbook(q, k, v, base):
    """softmax(RoPE(Q) RoPE(K)^T / sqrt(D) + causal mask) V for one head, fp64."""
    N, D = q.shape
    pos = np.arange(N)
    qt, kt = rope_textbook(q, pos, base), rope_textbook(k, pos, base)
    s = qt @ kt.T / math.sqrt(D)
    s = np.where(np.tril(np.ones((N, N), dtype=bool)), s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ np.asarray(v, dtype=np.float64)


def rand(shape, seed, name="q", dtype="f32"):
    return synthetic.tensor(seed, name, shape, dtype)


# --------------------------------------------------------------------------- window
def test_window_lowest_index_pair_is_two_pi_k(oracle):
    # theta_0 = base^0 = 1, so lambda_0 = 2*pi for every base and head dim.
    for D, base in [(64, 1e4), (128, 5e5), (8, 10.0)]:
        for k, w0 in [(1, 6), (8, 50), (16, 100), (64, 402), (0.25, 1), (0, 0)]:
            assert oracle.window_limits(D, base, k)[0] == w0


def test_window_middle_pair_is_two_pi_sqrt_base(oracle):
    # r = D/4 gives theta = base^(-1/2): lambda = 2*pi*sqrt(base).
    # base 1e4: 2*pi*100 = 628.318...; base 1e6: 2*pi*1000 = 6283.18...
    assert oracle.window_limits(64, 1e4, 1)[16] == 628
    assert oracle.window_limits(128, 1e6, 1)[32] == 6283
    assert oracle.window_limits(128, 1e6, 2)[32] == 12566


def test_window_monotone_and_infinite(oracle):
    for D, base, k in [(64, 1e4, 1), (64, 1e6, 8), (128, 5e5, 16), (128, 1e7, 64)]:
        w = oracle.window_limits(D, base, k)
        assert np.all(np.diff(w) >= 0)
    assert np.all(np.isinf(oracle.window_limits(64, 1e4, math.inf)))


# --------------------------------------------------------------------------- counts
COUNT_CASES = [
    (1, 8, 10.0, 1.0), (7, 8, 10.0, 0.25), (64, 8, 10.0, 0.0), (256, 64, 1e4, 1.0),
    (256, 64, 1e4, math.inf), (300, 64, 1e6, 8.0), (513, 128, 5e5, 16.0), (1000, 128, 1e7, 4.0),
    (2048, 64, 1e6, 8.0), (129, 128, 1e7, 0.01), (2, 2, 1e4, 1.0), (777, 16, 100.0, 3.5),
]


@pytest.mark.parametrize("N,D,base,k", COUNT_CASES)
def test_count_closed_equals_bruteforce(oracle, N, D, base, k):
    assert oracle.count_closed(N, D, base, k) == oracle.count_bruteforce(N, D, base, k)
    kept, total = oracle.count_closed(N, D, base, k)
    assert total == (D // 2) * N * (N + 1) // 2


def test_count_tiny_config_regression(oracle):
    # Tiny exactness case (N=256, D=64, base 1e4, k=1): pinned by brute force above;
    # recorded here so a change shows up as a diff.
    assert oracle.count_closed(256, 64, 1e4, 1.0) == (780051, 1052672)
    assert oracle.count_closed(256, 64, 1e4, math.inf) == (1052672, 1052672)


def test_count_monotone_in_k_and_deepens_with_n(oracle):
    prev = -1
    for k in [0, 0.5, 1, 2, 4, 8, 16, 64, math.inf]:
        kept, _ = oracle.count_closed(4096, 64, 1e6, k)
        assert kept >= prev
        prev = kept
    # The pruned share grows with N at fixed k ("deepening with N").
    fr = [1 - np.divide(*oracle.count_closed(n, 128, 1e7, 16)) for n in (8192, 65536, 524288)]
    assert fr[0] < fr[1] < fr[2]


def test_pages_printed_pruning_percentages(oracle):
    cases = json.load(open(os.path.join(GOLDEN, "pages_pruning.json")))["cases"]
    for c in cases:
        kept, total = oracle.count_closed(c["N"], c["D"], c["base"], c["k"])
        frac = 1.0 - kept / total
        if "printed_lo" in c:
            assert c["printed_lo"] <= frac <= c["printed_hi"], (c["model"], frac)
        else:
            assert round(100 * frac) == c["printed_round_percent"], (c["model"], frac)


# ------------------------------------------------------------------- reachability (check d)
CONFIGS_REACH = [  # (N, D, base, k) of every workload shape
    (256, 64, 1e4, 1.0), (32768, 64, 1e6, 8.0), (131072, 128, 5e5, 16.0),
    (524288, 128, 1e7, 16.0), (524288, 128, 1e7, 64.0), (1048576, 128, 1e7, 16.0),
    (1048576, 128, 1e7, 64.0),
]


@pytest.mark.parametrize("N,D,base,k", CONFIGS_REACH)
def test_every_key_reachable(oracle, N, D, base, k):
    w = oracle.window_limits(D, base, k)
    assert w[-1] >= N - 1  # lowest-frequency pair covers the whole context
    if N <= 32768:
        assert oracle.min_kept_pairs(N, D, base, k) >= 1


# ------------------------------------------------------------------------ RoPE (check c)
def test_rope_rows_matches_textbook(oracle):
    x = rand((40, 64), 11)
    pos = np.arange(0, 4000, 100)
    np.testing.assert_allclose(oracle.rope_rows(x, pos, 1e4), rope_textbook(x, pos, 1e4),
                               rtol=0, atol=1e-12)


def test_scores_shift_invariant(oracle):
    # RoPE scores depend on n - m only: shifting q and k rows together changes nothing.
    q, k = rand((1, 32), 3), rand((1, 32), 4, "k")
    base = 1e4
    qs = np.repeat(q, 64, axis=0)
    ks = np.repeat(k, 64, axis=0)
    s = oracle.scores(qs, ks, base, math.inf)  # s[n, m] of identical vectors
    for d in range(0, 20):
        diag = np.array([s[n, n - d] for n in range(d, 64)])
        np.testing.assert_allclose(diag, diag[0], rtol=0, atol=1e-12)


def test_pair_decomposition_equals_full_dot(oracle):
    q, k = rand((48, 64), 5), rand((48, 64), 6, "k")
    base = 1e4
    s = oracle.scores(q, k, base, math.inf)
    pos = np.arange(48)
    full = rope_textbook(q, pos, base) @ rope_textbook(k, pos, base).T / 8.0
    np.testing.assert_allclose(np.tril(s), np.tril(full), rtol=0, atol=1e-12)


# ------------------------------------------------------------------ attention (check a)
@pytest.mark.parametrize("N,D,base,Hq,Hkv", [(64, 16, 1e4, 2, 1), (200, 64, 1e4, 3, 3), (97, 128, 5e5, 4, 2)])
def test_k_inf_is_textbook_causal_attention(oracle, N, D, base, Hq, Hkv):
    q = rand((1, N, Hq, D), 21)
    k = rand((1, N, Hkv, D), 22, "k")
    v = rand((1, N, Hkv, D), 23, "v")
    out = oracle.prefill(q, k, v, base, math.inf)
    G = Hq // Hkv
    for h in range(Hq):
        ref = attention_textbook(q[0, :, h], k[0, :, h // G], v[0, :, h // G], base)
        np.testing.assert_allclose(out[0, :, h], ref, rtol=0, atol=1e-12)


def test_k_zero_closed_form(oracle):
    # k = 0: w_r = 0 for all r, so only the diagonal cell keeps pairs; every other
    # causal cell is the empty sum 0:  o_n = (e^{s_nn} v_n + sum_{m<n} v_m) / (e^{s_nn} + n).
    N, D, base = 50, 16, 1e4
    q, k, v = rand((1, N, 1, D), 31), rand((1, N, 1, D), 32, "k"), rand((1, N, 1, D), 33, "v")
    out = oracle.prefill(q, k, v, base, 0.0)[0, :, 0]
    pos = np.arange(N)
    snn = np.sum(rope_textbook(q[0, :, 0], pos, base) * rope_textbook(k[0, :, 0], pos, base), -1) / 4.0
    vv = v[0, :, 0].astype(np.float64)
    csum = np.cumsum(vv, axis=0) - vv  # sum_{m<n} v_m
    ref = (np.exp(snn)[:, None] * vv + csum) / (np.exp(snn) + pos)[:, None]
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)


def test_single_pair_window_bruteforce(oracle):
    # D = 2: one pair with theta = 1, w_0 = floor(2*pi*k).  k = 1 keeps distances 0..6.
    N, base = 20, 1e4
    q, k, v = rand((1, N, 1, 2), 41), rand((1, N, 1, 2), 42, "k"), rand((1, N, 1, 2), 43, "v")
    out = oracle.prefill(q, k, v, base, 1.0)[0, :, 0]
    for n in range(N):
        sc = []
        for m in range(n + 1):
            a = (n - m) * 1.0  # relative angle of the single pair
            qa, qb = float(q[0, n, 0, 0]), float(q[0, n, 0, 1])
            ka, kb = float(k[0, m, 0, 0]), float(k[0, m, 0, 1])
            # q . R(-(n-m)) k  (rotation of k by the relative angle)
            t = qa * (ka * math.cos(a) + kb * math.sin(a)) + qb * (kb * math.cos(a) - ka * math.sin(a))
            sc.append(t / math.sqrt(2.0) if n - m <= 6 else 0.0)
        mx = max(sc)
        p = [math.exp(s - mx) for s in sc]
        ref = [sum(p[m] * float(v[0, m, 0, i]) for m in range(n + 1)) / sum(p) for i in range(2)]
        np.testing.assert_allclose(out[n], ref, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------- decode
def test_decode_equals_prefill_last_row(oracle):
    N, D, Hq, Hkv, base = 77, 64, 4, 2, 1e4
    for kwin in (1.0, math.inf):
        q, k, v = rand((1, N, Hq, D), 51), rand((1, N, Hkv, D), 52, "k"), rand((1, N, Hkv, D), 53, "v")
        ref = oracle.prefill_rows(q[0, N - 1:N], [N - 1], k[0], v[0], base, kwin)[0]
        kc = np.ascontiguousarray(k.transpose(0, 2, 1, 3))
        vc = np.ascontiguousarray(v.transpose(0, 2, 1, 3))
        out = oracle.decode(q[:, N - 1], kc, vc, [N], base, kwin)[0]
        np.testing.assert_allclose(out, ref, rtol=0, atol=1e-13)


def test_decode_rotated_cache_equals_unrotated(oracle):
    B, Hq, Hkv, Nmax, D, base = 2, 4, 2, 90, 32, 1e4
    q = rand((B, Hq, D), 61)
    kc = rand((B, Hkv, Nmax, D), 62, "k")
    vc = rand((B, Hkv, Nmax, D), 63, "v")
    seqlens = [90, 41]
    out0 = oracle.decode(q, kc, vc, seqlens, base, 2.0, kcache_rotated=False)
    kr = np.stack([np.stack([rope_textbook(kc[b, g], np.arange(Nmax), base) for g in range(Hkv)])
                   for b in range(B)])
    out1 = oracle.decode(q, kr.astype(np.float32), vc, seqlens, base, 2.0, kcache_rotated=True)
    # rotated keys were rounded to float32 on the way in: fp32-level agreement
    np.testing.assert_allclose(out1, out0, rtol=0, atol=2e-5)


def test_prefill_rows_subset_equals_full(oracle):
    N, D, Hq, Hkv, base = 150, 64, 2, 1, 1e6
    q, k, v = rand((1, N, Hq, D), 71), rand((1, N, Hkv, D), 72, "k"), rand((1, N, Hkv, D), 73, "v")
    full = oracle.prefill(q, k, v, base, 8.0)[0]
    rows = np.array([0, 1, 63, 64, 149])
    sub = oracle.prefill_rows(q[0, rows], rows, k[0], v[0], base, 8.0)
    np.testing.assert_array_equal(sub, full[rows])


def test_synthetic_rows_match_tensor():
    t = synthetic.tensor(5, "q", (3, 40, 2, 8), "bf16")
    r = synthetic.rows(5, "q", (3, 40, 2, 8), 1, [0, 7, 39], "bf16")
    np.testing.assert_array_equal(r, t[:, [0, 7, 39]])
    # bf16 values: low 16 bits of the float32 pattern are zero
    assert np.all((t.view(np.uint32) & 0xFFFF) == 0)
    assert abs(float(t.mean())) < 0.1 and 0.9 < float(t.std()) < 1.1


# ------------------------------------------------------------------ scaled RoPE tables
from scaled import base_theta, llama3_scaled_theta  # noqa: E402


def rope_textbook_theta(x, pos, theta):
    """Rotate-half RoPE with an explicit frequency table, matrix form."""
    H = x.shape[-1] // 2
    ang = np.asarray(pos, dtype=np.float64)[:, None] * np.asarray(theta, dtype=np.float64)[None, :]
    cos = np.concatenate([np.cos(ang), np.cos(ang)], axis=-1)
    sin = np.concatenate([np.sin(ang), np.sin(ang)], axis=-1)
    x = np.asarray(x, dtype=np.float64)
    rot = np.concatenate([-x[:, H:], x[:, :H]], axis=-1)
    return x * cos + rot * sin


def test_scaled_table_is_a_valid_rope_table():
    th = llama3_scaled_theta(128, 5e5)
    assert np.all(np.diff(th) <= 0) and th[0] == 1.0 and np.all(th > 0)
    # long wavelengths are scaled by the factor, short ones untouched
    b = base_theta(128, 5e5)
    assert th[-1] == b[-1] / 32.0 and th[1] == b[1]


def test_scaled_windows_follow_the_table(oracle):
    th = llama3_scaled_theta(128, 5e5)
    with oracle.scaled_rope(th):
        lim = oracle.window_limits(128, 5e5, 16.0)
    np.testing.assert_array_equal(lim, np.floor(16.0 * 2.0 * np.pi / th))
    # outside the block the base table is back
    np.testing.assert_array_equal(oracle.window_limits(128, 5e5, 16.0),
                                  np.floor(16.0 * 2.0 * np.pi / base_theta(128, 5e5)))


@pytest.mark.parametrize("N,D,base,k", [(700, 64, 1e4, 0.5), (300, 128, 5e5, 0.02)])
def test_scaled_count_closed_equals_bruteforce(oracle, N, D, base, k):
    with oracle.scaled_rope(llama3_scaled_theta(D, base, factor=8.0, orig_ctx=512.0)):
        assert oracle.count_closed(N, D, base, k) == oracle.count_bruteforce(N, D, base, k)


def test_scaled_k_inf_is_textbook_causal_attention(oracle):
    N, D, base = 150, 64, 1e4
    th = llama3_scaled_theta(D, base, factor=8.0, orig_ctx=256.0)
    q, k, v = rand((1, N, 1, D), 31), rand((1, N, 1, D), 32, "k"), rand((1, N, 1, D), 33, "v")
    with oracle.scaled_rope(th):
        out = oracle.prefill(q, k, v, base, math.inf)
    pos = np.arange(N)
    qt, kt = rope_textbook_theta(q[0, :, 0], pos, th), rope_textbook_theta(k[0, :, 0], pos, th)
    s = qt @ kt.T / math.sqrt(D)
    s = np.where(np.tril(np.ones((N, N), dtype=bool)), s, -np.inf)
    p = np.exp(s - s.max(axis=1, keepdims=True))
    ref = (p / p.sum(axis=1, keepdims=True)) @ np.asarray(v[0, :, 0], dtype=np.float64)
    np.testing.assert_allclose(out[0, :, 0], ref, rtol=0, atol=1e-12)


def test_base_table_installed_changes_nothing(oracle):
    N, D, base = 120, 64, 1e4
    q, k, v = rand((1, N, 2, D), 34), rand((1, N, 1, D), 35, "k"), rand((1, N, 1, D), 36, "v")
    plain = oracle.prefill(q, k, v, base, 1.0)
    with oracle.scaled_rope(base_theta(D, base)):
        tab = oracle.prefill(q, k, v, base, 1.0)
    np.testing.assert_allclose(tab, plain, rtol=0, atol=1e-12)


def test_scaled_decode_equals_prefill_last_row(oracle):
    N, D, base = 200, 128, 5e5
    th = llama3_scaled_theta(D, base, factor=8.0, orig_ctx=256.0)
    q, k, v = rand((1, N, 4, D), 37), rand((1, N, 2, D), 38, "k"), rand((1, N, 2, D), 39, "v")
    with oracle.scaled_rope(th):
        pre = oracle.prefill(q, k, v, base, 0.5)
        dec = oracle.decode(q[:, N - 1], k.transpose(0, 2, 1, 3), v.transpose(0, 2, 1, 3), [N], base, 0.5)
    np.testing.assert_allclose(dec, pre[:, N - 1], rtol=0, atol=1e-12)


# ------------------------------------------------- token-level block selection under the window
def visible_textbook(N, tile, mask_g):
    """Boolean [N, N]: key m visible to query n (causal, same tile, or mask entry set)."""
    n = np.arange(N)[:, None]
    m = np.arange(N)[None, :]
    return (m <= n) & ((m // tile == n // tile) | (mask_g[n // tile, m // tile] != 0))


def masked_attention_textbook(s, vis, v):
    s = np.where(vis, s, -np.inf)
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ np.asarray(v, dtype=np.float64)


def random_block_mask(Hkv, T, seed, density=0.4):
    rng = np.random.default_rng(seed)
    return (rng.random((Hkv, T, T)) < density).astype(np.uint8)


@pytest.mark.parametrize("kwin", [math.inf, 1.0])
def test_sparse_equals_textbook_masked_softmax(oracle, kwin):
    # Softmax over the visible keys only, written out with numpy from the score
    # matrix: RoPE in matrix form for k = inf, the oracle's windowed scores
    # (pinned above) otherwise.  Two KV groups with different masks.
    N, D, Hq, Hkv, tile, base = 70, 16, 4, 2, 16, 1e4
    T = (N + tile - 1) // tile
    q, k, v = rand((N, Hq, D), 81), rand((N, Hkv, D), 82, "k"), rand((N, Hkv, D), 83, "v")
    mask = random_block_mask(Hkv, T, 84)
    out = oracle.prefill_rows_sparse(q, np.arange(N), k, v, base, kwin, mask, tile)
    G = Hq // Hkv
    for h in range(Hq):
        g = h // G
        if math.isinf(kwin):
            pos = np.arange(N)
            s = rope_textbook(q[:, h], pos, base) @ rope_textbook(k[:, g], pos, base).T / math.sqrt(D)
        else:
            s = oracle.scores(q[:, h], k[:, g], base, kwin)
        ref = masked_attention_textbook(s, visible_textbook(N, tile, mask[g]), v[:, g])
        np.testing.assert_allclose(out[:, h], ref, rtol=0, atol=1e-12)


def test_sparse_all_visible_equals_dense(oracle):
    N, D, Hq, Hkv, tile, base = 90, 32, 2, 1, 16, 1e4
    T = (N + tile - 1) // tile
    q, k, v = rand((N, Hq, D), 85), rand((N, Hkv, D), 86, "k"), rand((N, Hkv, D), 87, "v")
    rows = np.arange(N)
    dense = oracle.prefill_rows(q, rows, k, v, base, 2.0)
    sparse = oracle.prefill_rows_sparse(q, rows, k, v, base, 2.0, np.ones((Hkv, T, T), np.uint8), tile)
    assert np.array_equal(dense, sparse)


def test_sparse_diagonal_and_future_entries_are_ignored(oracle):
    # The diagonal tile is always visible and entries above it cover only future
    # keys: zeroing the diagonal and setting every entry above it changes nothing.
    N, D, Hq, Hkv, tile, base = 64, 16, 2, 2, 8, 1e4
    T = N // tile
    q, k, v = rand((N, Hq, D), 88), rand((N, Hkv, D), 89, "k"), rand((N, Hkv, D), 90, "v")
    mask = random_block_mask(Hkv, T, 91)
    a_mask = mask.copy()
    for g in range(Hkv):
        a_mask[g] = np.tril(a_mask[g], -1) + np.eye(T, dtype=np.uint8)
    b_mask = mask.copy()
    for g in range(Hkv):
        b_mask[g] = np.tril(b_mask[g], -1) + np.triu(np.ones((T, T), np.uint8), 1)
    rows = np.arange(N)
    a = oracle.prefill_rows_sparse(q, rows, k, v, base, 1.0, a_mask, tile)
    b = oracle.prefill_rows_sparse(q, rows, k, v, base, 1.0, b_mask, tile)
    assert np.array_equal(a, b)
    # a query sees exactly its own tile's causal prefix when only the diagonal is set
    only_diag = oracle.prefill_rows_sparse(q, rows, k, v, base, math.inf, np.zeros((Hkv, T, T), np.uint8), tile)
    n = 21  # tile 2 (positions 16..23): keys 16..21
    ref = attention_textbook(q[16:n + 1, 0], k[16:n + 1, 0], v[16:n + 1, 0], base)[-1]
    # the textbook attention above starts positions at 0; RoPE scores depend on n - m only
    np.testing.assert_allclose(only_diag[n, 0], ref, rtol=0, atol=1e-12)


def test_sparse_under_scaled_table_all_visible_equals_dense(oracle):
    # The block-selected rows take the installed frequency table like the dense ones.
    from scaled import llama3_scaled_theta
    N, D, Hq, Hkv, tile, base = 80, 32, 2, 1, 16, 1e4
    T = (N + tile - 1) // tile
    th = llama3_scaled_theta(D, base, factor=8.0, orig_ctx=64.0)
    q, k, v = rand((N, Hq, D), 101), rand((N, Hkv, D), 102, "k"), rand((N, Hkv, D), 103, "v")
    rows = np.arange(N)
    with oracle.scaled_rope(th):
        dense = oracle.prefill_rows(q, rows, k, v, base, 1.0)
        sparse = oracle.prefill_rows_sparse(q, rows, k, v, base, 1.0, np.ones((Hkv, T, T), np.uint8), tile)
    plain = oracle.prefill_rows(q, rows, k, v, base, 1.0)
    assert np.array_equal(dense, sparse)
    assert not np.allclose(dense, plain)
