"""GPU parity of the prefill path (C ABI via the binding) against the fp64 oracle."""
import math

import numpy as np
import pytest

import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_attention_pair_b200 as atf  # noqa: E402


def inputs(seed, B, N, Hq, Hkv, D, dtype):
    q = P.gen(seed, "q", (B, N, Hq, D), dtype)
    k = P.gen(seed, "k", (B, N, Hkv, D), dtype)
    v = P.gen(seed, "v", (B, N, Hkv, D), dtype)
    return q, k, v


# ------------------------------------------------------------ tiny exactness case
@pytest.mark.parametrize("kwin", [1.0, math.inf])
def test_tiny_fp32_prefill(oracle, kwin):
    q, k, v = inputs(0, 1, 256, 1, 1, 64, "f32")
    out = atf.prefill(q, k, v, 1e4, kwin)
    torch.cuda.synchronize()
    ref = oracle.prefill(P.host(q), P.host(k), P.host(v), 1e4, kwin)
    P.check(P.host(out), ref, "f32", f"tiny k={kwin}")


@pytest.mark.parametrize("N,D,Hq,Hkv,base,kwin", [
    (1, 64, 1, 1, 1e4, 1.0), (129, 128, 4, 2, 5e5, 2.0), (300, 8, 2, 1, 10.0, 0.25), (77, 256, 3, 3, 1e4, 3.0),
    (200, 6, 1, 1, 100.0, 1.5)])
def test_fp32_prefill_shapes(oracle, N, D, Hq, Hkv, base, kwin):
    q, k, v = inputs(1, 2, N, Hq, Hkv, D, "f32")
    out, lse = atf.prefill(q, k, v, base, kwin, return_lse=True)
    torch.cuda.synchronize()
    ref, rlse = oracle.prefill(P.host(q), P.host(k), P.host(v), base, kwin, want_lse=True)
    P.check(P.host(out), ref, "f32", "fp32 prefill")
    P.check(P.host(lse), rlse.transpose(0, 2, 1), "f32", "fp32 lse")


# ----------------------------------------------------------- tensor-core path
SMALL_BF16 = [
    # N spans several tiles with a ragged tail; GQA; window on/off; D 64 and 128
    (1, 1, 64, 1, 1, 1e4, 1.0),
    (1, 127, 64, 2, 1, 1e4, 1.0),
    (1, 128, 128, 2, 2, 1e4, 1.0),
    (1, 129, 128, 2, 1, 1e4, 4.0),
    (2, 700, 64, 4, 2, 1e4, 1.0),
    (1, 700, 128, 3, 1, 5e5, 2.0),
    (1, 1000, 64, 2, 2, 1e6, 8.0),
    (1, 1000, 128, 2, 1, 1e4, math.inf),
    (1, 513, 64, 7, 1, 1e6, math.inf),
    (1, 2048, 128, 2, 1, 1e4, 0.5),
    # k = 0: only distance 0 keeps its pairs, every other cell is the empty sum 0
    (1, 600, 64, 2, 1, 1e4, 0.0),
    (1, 400, 128, 4, 2, 5e5, 0.0),
    # window off at D = 64 with an even GQA group (one head per CTA, two CTAs per SM)
    (2, 640, 64, 4, 2, 1e4, math.inf),
]


@pytest.mark.parametrize("B,N,D,Hq,Hkv,base,kwin", SMALL_BF16)
def test_bf16_prefill_matches_oracle(oracle, B, N, D, Hq, Hkv, base, kwin):
    q, k, v = inputs(2, B, N, Hq, Hkv, D, "bf16")
    out, lse = atf.prefill(q, k, v, base, kwin, out_dtype=torch.float32, return_lse=True)
    torch.cuda.synchronize()
    ref, rlse = oracle.prefill(P.host(q), P.host(k), P.host(v), base, kwin, want_lse=True)
    P.check(P.host(out), ref, "bf16", f"bf16 prefill N={N} D={D} k={kwin}")
    P.check(P.host(lse), rlse.transpose(0, 2, 1), "bf16", "bf16 lse")


# One key whose score exceeds every other score of its rows by >= 15 (natural
# units) sits in a chosen column of its key tile: rows after it see their running
# max jump by > 2^8 at that tile (the O rescale), first in the softmax warp that
# holds that column (with pruning two warps share a row and must adopt the same
# max).  The query and that key share a direction in the pairs that turn less
# than 0.5 rad over the sequence (never pruned at these k); every other key is
# zero there.  The dominant key takes nearly all the weight, so the output does
# not depend on the bf16 rounding of the large score.
@pytest.mark.parametrize("D,base,kwin,m_star", [
    (64, 1e6, 8.0, 128 * 3 + 100),   # column 100: the second half of the tile's row
    (64, 1e6, 8.0, 128 * 3 + 20),    # column 20: the first half
    (128, 5e5, 16.0, 128 * 5 + 90),
    (128, 5e5, 16.0, 128 * 7 + 40),  # the diagonal tile of the last query tile
])
def test_bf16_row_max_jump_in_one_column_half(oracle, D, base, kwin, m_star):
    N, Hq, Hkv = 1024, 2, 1
    q, k, v = inputs(8, 1, N, Hq, Hkv, D, "bf16")
    low = [r for r in range(D // 2) if base ** (-2 * r / D) * N < 0.5]
    assert len(low) >= 14 and min(atf.window_table(D, base, kwin, N)[r] for r in low) == N - 1
    q[..., low] = 2.0
    k[..., low] = 0.0
    k[0, m_star, :, low] = 6.0
    out, lse = atf.prefill(q, k, v, base, kwin, out_dtype=torch.float32, return_lse=True)
    torch.cuda.synchronize()
    ref, rlse = oracle.prefill(P.host(q), P.host(k), P.host(v), base, kwin, want_lse=True)
    # the dominant key carries almost all the weight of every later row
    vh = P.host(v)[0, m_star, 0]
    assert np.abs(ref[0, m_star + 1:, 0] - vh).max() < 0.01
    P.check(P.host(out), ref, "bf16", f"row max jump D={D} m*={m_star}")
    # The log-sum-exp of a later row is about the dominant score itself (15-26 here).
    # Its terms are all positive, so rounding the rotated q~ and k~ to bf16 (relative
    # 2^-9 each) moves it by up to 2^-8 of its size: the bar is relative there.
    got_lse, ref_lse = P.host(lse), rlse.transpose(0, 2, 1)
    assert np.all(np.abs(got_lse - ref_lse) <= 1e-2 + 2.0 ** -8 * np.abs(ref_lse))
    assert atf.device_status() == 0


def test_bf16_output_rounding(oracle):
    # bf16 output: oracle value rounded to bf16, within 1e-2 plus half a bf16 ulp.
    q, k, v = inputs(3, 1, 600, 2, 1, 128, "bf16")
    out = atf.prefill(q, k, v, 1e4, 2.0)
    torch.cuda.synchronize()
    ref = oracle.prefill(P.host(q), P.host(k), P.host(v), 1e4, 2.0)
    err = np.abs(P.host(out) - ref)
    half_ulp = np.exp2(np.floor(np.log2(np.maximum(np.abs(ref), 1e-30))) - 8)
    assert np.all(err <= 1e-2 + half_ulp)


def test_bf16_empty_sum_cells(oracle):
    # base 10, D 64, k 0.25: w_31 = 14, so cells farther than 14 keep no pair and score 0.
    assert atf.window_table(64, 10.0, 0.25, 300)[-1] == 14
    q, k, v = inputs(4, 1, 300, 2, 1, 64, "bf16")
    out = atf.prefill(q, k, v, 10.0, 0.25, out_dtype=torch.float32)
    torch.cuda.synchronize()
    ref = oracle.prefill(P.host(q), P.host(k), P.host(v), 10.0, 0.25)
    P.check(P.host(out), ref, "bf16", "empty-sum cells")


@pytest.mark.parametrize("D,dtype", [(64, "bf16"), (128, "bf16"), (64, "f32")])
def test_window_covering_everything_is_bit_identical_to_off(D, dtype):
    # Every w_r >= N-1 -> the window removes nothing: same bits as k = inf.
    N, base = 777, 1e4
    kwin = 2.0 * N / (2 * math.pi)  # w_0 = floor(2*pi*k) >= N-1
    assert min(atf.window_table(D, base, kwin, N)) == N - 1
    q, k, v = inputs(5, 1, N, 4, 2, D, dtype)
    a = atf.prefill(q, k, v, base, kwin)
    b = atf.prefill(q, k, v, base, math.inf)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_plain_call_equals_ex_call():
    q, k, v = inputs(6, 1, 1000, 4, 2, 128, "bf16")
    a = torch.empty_like(q)
    atf.prefill_bf16(q, k, v, a, 5e5, 16.0)
    b = atf.prefill(q, k, v, 5e5, 16.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_deterministic_repeat():
    q, k, v = inputs(7, 1, 1500, 2, 1, 64, "bf16")
    a = atf.prefill(q, k, v, 1e6, 8.0)
    b = atf.prefill(q, k, v, 1e6, 8.0)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    assert atf.device_status() == 0


# ------------------------------------------------------- workload-size configs
def sampled_parity(oracle, B, N, Hq, Hkv, D, base, kwin, seed, rows_per_head=64):
    q, k, v = inputs(seed, B, N, Hq, Hkv, D, "bf16")
    out = atf.prefill(q, k, v, base, kwin, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rows = P.sample_rows(N, rows_per_head, seed)
    kh, vh = P.host(k[0]), P.host(v[0])
    qh = P.host(q[0, torch.as_tensor(rows, device=q.device)])
    ref = oracle.prefill_rows(qh, rows, kh, vh, base, kwin)
    got = P.host(out[0, torch.as_tensor(rows, device=q.device)])
    P.check(got, ref, "bf16", f"N={N} k={kwin}")
    assert atf.device_status() == 0


def test_qwen05b_shape_32k(oracle):
    sampled_parity(oracle, 1, 32768, 14, 2, 64, 1e6, 8.0, seed=11)


@pytest.mark.slow
@pytest.mark.parametrize("N", [8192, 32768, 131072])
def test_llama3b_shape(oracle, N):
    sampled_parity(oracle, 1, N, 24, 8, 128, 5e5, 16.0, seed=12)


@pytest.mark.slow
@pytest.mark.parametrize("N,kwin", [(262144, 16.0), (262144, 64.0), (524288, 16.0), (524288, 64.0)])
def test_qwen7b_1m_shape(oracle, N, kwin):
    sampled_parity(oracle, 1, N, 28, 4, 128, 1e7, kwin, seed=13)


# Window off (k = inf) at workload size: the one-head D = 64 form (two CTAs per SM)
# and the two-head D = 128 form over every key tile.
@pytest.mark.slow
def test_qwen05b_shape_32k_window_off(oracle):
    sampled_parity(oracle, 1, 32768, 14, 2, 64, 1e6, math.inf, seed=14)


@pytest.mark.slow
def test_llama3b_shape_128k_window_off(oracle):
    sampled_parity(oracle, 1, 131072, 24, 8, 128, 5e5, math.inf, seed=15)
