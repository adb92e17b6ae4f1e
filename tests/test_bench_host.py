"""Host-side checks of the benchmark's workload tables (no GPU)."""
import math

import bench


def test_ragged_lengths_fill_the_total_within_bounds():
    for wl in bench.VARLEN_WORKLOADS.values():
        lens = bench.ragged_lengths(wl["seed"], wl["total"], wl["len_lo"], wl["len_hi"])
        assert sum(lens) == wl["total"]
        assert all(1 <= n <= wl["len_hi"] for n in lens)
        # every length but the cut last one lies in [lo, hi]
        assert all(n >= wl["len_lo"] for n in lens[:-1])
        assert len(set(lens)) > 1  # ragged, not uniform
        assert lens == bench.ragged_lengths(wl["seed"], wl["total"], wl["len_lo"], wl["len_hi"])


def test_paged_workloads_split_into_whole_pages():
    for name, wl in bench.DECODE_WORKLOADS.items():
        if "page" in wl:
            assert wl["page"] % 64 == 0 and wl["N"] % wl["page"] == 0, name


def test_workload_names_are_unique_across_tables():
    names = list(bench.WORKLOADS) + list(bench.DECODE_WORKLOADS) + list(bench.VARLEN_WORKLOADS)
    assert len(names) == len(set(names))
    assert all(math.isfinite(w["k_window"]) for w in bench.VARLEN_WORKLOADS.values())


def test_scaled_workload_theta_is_the_llama3_table():
    import numpy as np
    from scaled import llama3_scaled_theta
    for name in ("llama3b_128k_scaled",):
        wl = bench.WORKLOADS[name]
        sc = wl["rope_scaling"]
        th = np.array(bench.rope_theta(wl))
        ref = llama3_scaled_theta(wl["D"], wl["rope_base"], factor=sc["factor"], low=sc["low_freq_factor"],
                                  high=sc["high_freq_factor"], orig_ctx=sc["original_max_position_embeddings"])
        np.testing.assert_allclose(th, ref, rtol=1e-13, atol=0)
        assert np.all(np.diff(th) <= 0) and th[0] <= math.pi and th[-1] > 0
        assert bench.rope_theta(bench.WORKLOADS["llama3b_32k"]) is None


def test_scaled_workload_table_is_accepted_by_the_library():
    import long_context_attention_pair_b200 as atf
    wl = bench.WORKLOADS["llama3b_128k_scaled"]
    th = bench.rope_theta(wl)
    w = atf.window_table(wl["D"], 0.0, wl["k_window"], wl["N"], theta=th)
    w0 = atf.window_table(wl["D"], wl["rope_base"], wl["k_window"], wl["N"])
    # scaling divides the low frequencies: their windows only grow
    assert all(a >= b for a, b in zip(w, w0)) and w != w0


def test_captured_traffic_is_reported_only_for_its_own_workload():
    wl = dict(bench.WORKLOADS["qwen05b_32k"])
    same_source = bench.TRAFFIC["source_sha1"] == bench.kernel_sha1()
    assert (bench.prefill_traffic("qwen05b_32k", wl) is not None) == same_source
    assert bench.prefill_traffic("llama3b_128k", dict(bench.WORKLOADS["llama3b_128k"])) is None
    assert bench.prefill_traffic("qwen05b_32k", dict(wl, N=65536)) is None
    assert bench.prefill_traffic("qwen05b_32k", dict(wl, k_window=float("inf"))) is None
    assert bench.decode_traffic("decode_128k", 1 << 17) is None
    # natural layouts read the whole cache: the capture scales with L; packed does not
    rec = bench.DECODE_TRAFFIC["decode_1m"]
    same = rec["source_sha1"] == bench.kernel_sha1(*bench.DECODE_SOURCES)
    got = bench.decode_traffic("decode_1m", 1 << 20)
    assert (got == round(rec["bytes_per_launch"] * (1 << 20) / rec["captured_L"])) if same else got is None
    assert bench.decode_traffic("decode_1m_packed", 1 << 20) is None
    pk = bench.DECODE_TRAFFIC["decode_1m_packed"]
    assert (bench.decode_traffic("decode_1m_packed", pk["captured_L"]) == pk["bytes_per_launch"]) == same
    # a sweep over the number of sequences: the natural layout scales with B * L, packed is not reported
    got1 = bench.decode_traffic("decode_1m", 1 << 19, B=1)
    assert (got1 == round(rec["bytes_per_launch"] * (1 << 19) / (4 * rec["captured_L"]))) if same else got1 is None
    assert bench.decode_traffic("decode_1m_packed", pk["captured_L"], B=1) is None


def test_tile_flops_sum_to_the_dense_retained_flops():
    # Summed over every causal tile pair, the per-distance tile FLOPs of the
    # block-selected lines equal the closed-form retained FLOPs of one head.
    import long_context_attention_pair_b200 as atf
    for wl in bench.SPARSE_WORKLOADS.values():
        T = wl["N"] // 128
        per_t = bench.tile_retained_flops(atf, wl, T)
        terms = atf.pruned_terms(wl["N"], wl["D"], wl["rope_base"], wl["k_window"])
        dense = 4 * terms["kept"] + wl["D"] * wl["N"] * (wl["N"] + 1)
        assert sum(per_t[t] * (T - t) for t in range(T)) == dense


def test_block_mask_recipe_shape_and_structure():
    import numpy as np
    wl = bench.SPARSE_WORKLOADS["qwen05b_32k_sparse"]
    T = wl["N"] // 128
    m = bench.block_mask_recipe(wl, T)
    assert m.shape == (wl["B"], wl["Hkv"], T, T) and m.dtype == np.uint8
    assert not np.any(np.triu(m[0, 0], 1))                      # causal tiles only
    assert np.all(np.diag(m[0, 0]) == 1)                         # local band includes the diagonal
    assert np.all(m[0, :, wl["sink_tiles"]:, :wl["sink_tiles"]] == 1)
    assert np.array_equal(m, bench.block_mask_recipe(wl, T))    # seeded


def test_default_line_is_the_largest_single_gpu_prefill_config():
    wl = bench.WORKLOADS[bench.DEFAULT_WORKLOAD]
    assert (wl["N"], wl["Hq"], wl["Hkv"], wl["D"], wl["k_window"]) == (524288, 28, 4, 128, 16.0)
    assert max(w["N"] for w in bench.WORKLOADS.values()) == wl["N"]
    for name in bench.SUB_RECORDS:
        assert name in bench.WORKLOADS or name in bench.DECODE_WORKLOADS


def test_both_arms_sample_the_oracle_by_one_rule_and_report_one_config():
    assert bench.oracle_rows_per_step(bench.WORKLOADS["qwen7b_512k"]) == 5
    assert bench.oracle_rows_per_step(bench.WORKLOADS["qwen05b_32k"]) == 293
    for wl in bench.WORKLOADS.values():
        assert bench.oracle_rows_per_step(wl) >= 1
        for world in (1, 2, 8):
            assert bench.line_config(dict(wl), world) == bench.line_config(dict(wl), world)
            assert bench.line_config(dict(wl), world)["parallelism"] == ("replicas" if world > 1 else "single GPU")
