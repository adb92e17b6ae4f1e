"""GPU parity of the ragged-batch (variable-length) prefill.

A batch packed along the token axis is, by definition, independent causal
windowed attention within each sequence with positions restarting at 0; the
reference is the oracle's prefill of each sequence on its own.
"""
import math

import numpy as np
import pytest

import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_attention_pair_b200 as atf  # noqa: E402


def packed_batch(seed, lens, Hq, Hkv, D):
    total = int(sum(lens))
    q = P.gen(seed, "q", (total, Hq, D), "bf16")
    k = P.gen(seed, "k", (total, Hkv, D), "bf16")
    v = P.gen(seed, "v", (total, Hkv, D), "bf16")
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return q, k, v, cu


def check_against_oracle(oracle, q, k, v, cu, out, base, kwin, max_rows=48, lse=None, seed=0):
    rng = np.random.default_rng(seed)
    for b in range(len(cu) - 1):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        n = t1 - t0
        if n == 0:
            continue
        rows = np.arange(n) if n <= max_rows else np.unique(np.concatenate(
            [[0, n - 1], rng.choice(n, max_rows - 2, replace=False)]))
        idx = torch.as_tensor(t0 + rows, device=q.device)
        ref, rlse = oracle.prefill_rows(P.host(q[idx]), rows, P.host(k[t0:t1]), P.host(v[t0:t1]), base, kwin,
                                        want_lse=True)
        P.check(P.host(out[idx]), ref, "bf16", f"varlen seq {b} (len {n})")
        if lse is not None:
            got = P.host(lse[:, idx]).T
            assert np.max(np.abs(got - rlse)) < 1e-2, f"lse seq {b}"


@pytest.mark.parametrize("lens,Hq,Hkv,D,base,kwin", [
    ([1, 127, 128, 129, 300, 1000], 4, 2, 64, 1e6, 8.0),
    ([700, 1, 0, 257, 2049], 6, 2, 128, 5e5, 16.0),
    ([513, 64, 1500], 7, 1, 128, 1e7, math.inf),
    ([33, 4000], 2, 2, 64, 10.0, 0.25),
    ([300, 1, 0, 700], 7, 1, 64, 1e4, math.inf),
])
def test_varlen_matches_oracle_per_sequence(oracle, lens, Hq, Hkv, D, base, kwin):
    q, k, v, cu = packed_batch(61, lens, Hq, Hkv, D)
    cu_d = torch.as_tensor(cu, device="cuda")
    out, lse = atf.prefill_varlen(q, k, v, cu_d, max(lens), base, kwin, out_dtype=torch.float32,
                                  return_lse=True)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    check_against_oracle(oracle, q, k, v, cu, out, base, kwin, lse=lse)


def test_varlen_sequence_equals_single_sequence_prefill():
    # One sequence of a ragged batch gives the same rows as prefilling it alone.
    lens, Hq, Hkv, D, base, kwin = [300, 1200, 77], 4, 2, 128, 5e5, 16.0
    q, k, v, cu = packed_batch(62, lens, Hq, Hkv, D)
    out = atf.prefill_varlen(q, k, v, torch.as_tensor(cu, device="cuda"), max(lens), base, kwin,
                             out_dtype=torch.float32)
    for b in range(len(lens)):
        t0, t1 = int(cu[b]), int(cu[b + 1])
        alone = atf.prefill(q[None, t0:t1].contiguous(), k[None, t0:t1].contiguous(), v[None, t0:t1].contiguous(),
                            base, kwin, out_dtype=torch.float32)
        torch.cuda.synchronize()
        # Same arithmetic up to the order of fp32 sums (the window table is clamped to
        # the longest sequence, which may start the dense chunks one chunk earlier).
        P.check(P.host(out[t0:t1]), P.host(alone[0]), "bf16", f"seq {b} alone")


def test_varlen_malformed_table_leaves_those_rows_untouched(oracle):
    lens, Hq, Hkv, D, base, kwin = [200, 300], 2, 1, 64, 1e4, 2.0
    q, k, v, cu = packed_batch(63, lens, Hq, Hkv, D)
    bad = cu.copy()
    bad[2] = 10 ** 6  # past the end of the token axis: the second sequence is rejected in the kernel
    out = torch.full(q.shape, 7.0, dtype=torch.float32, device="cuda")
    atf.prefill_varlen(q, k, v, torch.as_tensor(bad, device="cuda"), 300, base, kwin, out=out)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    assert torch.all(out[200:] == 7.0)
    check_against_oracle(oracle, q, k, v, cu[:2], out, base, kwin)


@pytest.mark.slow
@pytest.mark.parametrize("name,rows", [("varlen_qwen05b_256k", 16), ("varlen_qwen7b_1m", 6)])
def test_varlen_bench_mix_sampled(oracle, name, rows):
    # The benchmark's ragged batches, in its launch configuration (bf16 out,
    # caller's workspace): sampled rows of every sequence against the oracle.
    import bench
    wl = bench.VARLEN_WORKLOADS[name]
    lens = bench.ragged_lengths(wl["seed"], wl["total"], wl["len_lo"], wl["len_hi"])
    q, k, v, cu = packed_batch(64, lens, wl["Hq"], wl["Hkv"], wl["D"])
    ws = torch.empty(int(atf.lib().atflash_prefill_varlen_workspace_bytes(wl["Hq"], wl["Hkv"], q.shape[0], wl["D"])),
                     dtype=torch.uint8, device="cuda")
    out = atf.prefill_varlen(q, k, v, torch.as_tensor(cu, device="cuda"), max(lens), wl["rope_base"],
                             wl["k_window"], workspace=ws)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    check_against_oracle(oracle, q, k, v, cu, out, wl["rope_base"], wl["k_window"], max_rows=rows, seed=65)


def test_varlen_first_tile_rows_are_exact(oracle):
    # Rows 0..127 of every sequence see at most 128 keys and are computed in fp32.
    lens, Hq, Hkv, D, base, kwin = [1, 77, 128, 129, 300], 6, 2, 128, 5e5, 16.0
    q, k, v, cu = packed_batch(66, lens, Hq, Hkv, D)
    out, lse = atf.prefill_varlen(q, k, v, torch.as_tensor(cu, device="cuda"), max(lens), base, kwin,
                                  out_dtype=torch.float32, return_lse=True)
    torch.cuda.synchronize()
    assert atf.device_status() == 0
    for b in range(len(lens)):
        t0, n = int(cu[b]), lens[b]
        rows = np.arange(min(n, 128))
        idx = torch.as_tensor(t0 + rows, device="cuda")
        ref, rlse = oracle.prefill_rows(P.host(q[idx]), rows, P.host(k[t0:t0 + n]), P.host(v[t0:t0 + n]), base,
                                        kwin, want_lse=True)
        P.check(P.host(out[idx]), ref, "f32", f"varlen seq {b} first tile")
        P.check(P.host(lse[:, idx]).T, rlse, "f32", f"varlen seq {b} first-tile lse")
