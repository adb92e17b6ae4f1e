#!/usr/bin/env python
"""Benchmark of the windowed-attention hot path; prints ONE JSON line (rank 0).

Workload (default): Qwen2.5-7B-1M-shaped single-layer prefill, B=1, Hq=28,
Hkv=4 (GQA), D=128, RoPE base 1e7, N=524288, k=16, bf16 inputs i.i.d. N(0,1)
from seed 3, plus the decode of the last row against the same K/V.  One step =
RoPE pre-pass (q and k) -> windowed tcgen05 prefill -> fp32 short rows ->
split-KV decode -> merge -> short decode rows: every row of the hot path.
`value` is prefill tokens/s (B*N tokens per step) with inputs resident in HBM
(3.7 GB of queries alone, far larger than the 126 MB L2, which is also flushed
before every step by writing a 256 MiB buffer outside the timed events).  The
default line also carries sub-records measured in the same run: the 4 x 1M
decode over the packed rotated and the natural HND caches, and the
Qwen2.5-0.5B-shaped 32K prefill line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --workload NAME ...

Other workloads (`--workload`): the prefill shapes of the larger models
(WORKLOADS), decode over contiguous or paged caches (DECODE_WORKLOADS), ragged
batches (VARLEN_WORKLOADS) and the window over a block selection
(SPARSE_WORKLOADS); each prints the same kind of line for its own step.

N > 1 (torchrun): every rank runs an independent replica of the workload on
its own GPU (the path has no exchange step); time = max over ranks.
"""
import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "prefill tokens/s + decode µs/token vs N; % of bf16 TC / HBM roofline"


def _pf(name, B, Hq, Hkv, D, N, base, k, seed):
    return {"workload": name, "B": B, "Hq": Hq, "Hkv": Hkv, "D": D, "N": N, "rope_base": base, "k_window": k,
            "seed": seed}


# Prefill workloads: one step = RoPE pre-pass -> windowed prefill -> decode of the last row.
WORKLOADS = {
    "qwen05b_32k": _pf("Qwen2.5-0.5B-shaped single-layer windowed prefill + decode of the last row",
                       1, 14, 2, 64, 32768, 1e6, 8.0, 1),
    "llama3b_8k": _pf("Llama-3.2-3B-shaped single-layer windowed prefill + decode of the last row",
                      1, 24, 8, 128, 8192, 5e5, 16.0, 2),
    "llama3b_32k": _pf("Llama-3.2-3B-shaped single-layer windowed prefill + decode of the last row",
                       1, 24, 8, 128, 32768, 5e5, 16.0, 2),
    "llama3b_128k": _pf("Llama-3.2-3B-shaped single-layer windowed prefill + decode of the last row",
                        1, 24, 8, 128, 131072, 5e5, 16.0, 2),
    "qwen7b_256k": _pf("Qwen2.5-7B-1M-shaped single-layer windowed prefill + decode of the last row",
                       1, 28, 4, 128, 262144, 1e7, 16.0, 3),
    "qwen7b_256k_k64": _pf("Qwen2.5-7B-1M-shaped single-layer windowed prefill + decode of the last row",
                           1, 28, 4, 128, 262144, 1e7, 64.0, 3),
    "qwen7b_512k": _pf("Qwen2.5-7B-1M-shaped single-layer windowed prefill + decode of the last row",
                       1, 28, 4, 128, 524288, 1e7, 16.0, 3),
    "qwen7b_512k_k64": _pf("Qwen2.5-7B-1M-shaped single-layer windowed prefill + decode of the last row",
                           1, 28, 4, 128, 524288, 1e7, 64.0, 3),
    # Llama-3.2-3B as released: its RoPE frequencies rescaled (rope_scaling type llama3,
    # factor 32, low/high frequency factors 1 and 4, original context 8192).  Only pairs
    # with wavelengths above 2048 are rescaled, and at k = 16 their windows exceed
    # 32K already, so the scaled table changes the windows only beyond 32K tokens.
    "llama3b_128k_scaled": dict(_pf("Llama-3.2-3B-shaped single-layer windowed prefill + decode of the last row, "
                                    "llama3 rope_scaling", 1, 24, 8, 128, 131072, 5e5, 16.0, 2),
                                rope_scaling={"factor": 32.0, "low_freq_factor": 1.0, "high_freq_factor": 4.0,
                                              "original_max_position_embeddings": 8192}),
}


def rope_theta(wl):
    """Per-pair frequencies of a workload with rope_scaling (None: base^(-2r/D)).

    The llama3 rule: a pair whose wavelength 2*pi/theta_r is shorter than
    orig/high keeps its frequency, one longer than orig/low has it divided by
    `factor`, and in between the two are blended linearly in orig/wavelength."""
    sc = wl.get("rope_scaling")
    if not sc:
        return None
    D, base = wl["D"], wl["rope_base"]
    f, lo, hi = sc["factor"], sc["low_freq_factor"], sc["high_freq_factor"]
    orig = float(sc["original_max_position_embeddings"])
    out = []
    for r in range(D // 2):
        th = base ** (-2.0 * r / D)
        wavelen = 2.0 * math.pi / th
        if wavelen < orig / hi:
            out.append(th)
        elif wavelen > orig / lo:
            out.append(th / f)
        else:
            a = (orig / wavelen - lo) / (hi - lo)
            out.append((1.0 - a) * th / f + a * th)
    return out
# Decode workloads: one step = one decode call (one token for each of B sequences).
DECODE_WORKLOADS = {
    "decode_1m": {"workload": "Qwen2.5-7B-1M-shaped decode, 4 sequences at 1M tokens", "B": 4, "Hq": 28,
                  "Hkv": 4, "D": 128, "N": 1 << 20, "rope_base": 1e7, "k_window": 16.0, "seed": 4},
    "decode_1m_k64": {"workload": "Qwen2.5-7B-1M-shaped decode, 4 sequences at 1M tokens", "B": 4, "Hq": 28,
                      "Hkv": 4, "D": 128, "N": 1 << 20, "rope_base": 1e7, "k_window": 64.0, "seed": 4},
    "decode_128k": {"workload": "Qwen2.5-7B-1M-shaped decode, 16 sequences at 128K tokens", "B": 16, "Hq": 28,
                    "Hkv": 4, "D": 128, "N": 1 << 17, "rope_base": 1e7, "k_window": 16.0, "seed": 5},
    "decode_1m_packed": {"workload": "Qwen2.5-7B-1M-shaped decode, 4 sequences at 1M tokens, packed rotated K cache",
                         "B": 4, "Hq": 28, "Hkv": 4, "D": 128, "N": 1 << 20, "rope_base": 1e7, "k_window": 16.0,
                         "seed": 4, "packed": True},
    "decode_1m_k64_packed": {"workload": "Qwen2.5-7B-1M-shaped decode, 4 sequences at 1M tokens, packed rotated K "
                             "cache", "B": 4, "Hq": 28, "Hkv": 4, "D": 128, "N": 1 << 20, "rope_base": 1e7,
                             "k_window": 64.0, "seed": 4, "packed": True},
    "decode_128k_packed": {"workload": "Qwen2.5-7B-1M-shaped decode, 16 sequences at 128K tokens, packed rotated K "
                           "cache", "B": 16, "Hq": 28, "Hkv": 4, "D": 128, "N": 1 << 17, "rope_base": 1e7,
                           "k_window": 16.0, "seed": 5, "packed": True},
    "decode_128k_k64": {"workload": "Qwen2.5-7B-1M-shaped decode, 16 sequences at 128K tokens", "B": 16,
                        "Hq": 28, "Hkv": 4, "D": 128, "N": 1 << 17, "rope_base": 1e7, "k_window": 64.0,
                        "seed": 5},
    # Paged caches: the contiguous cache cut into pages of `page` tokens and scattered
    # through one pool in a seeded random order (block table per sequence).
    "decode_1m_paged_packed": {"workload": "Qwen2.5-7B-1M-shaped decode, 4 sequences at 1M tokens, paged packed "
                               "rotated K cache (256-token pages, shuffled pool)", "B": 4, "Hq": 28, "Hkv": 4,
                               "D": 128, "N": 1 << 20, "rope_base": 1e7, "k_window": 16.0, "seed": 4,
                               "packed": True, "page": 256},
    "decode_1m_paged": {"workload": "Qwen2.5-7B-1M-shaped decode, 4 sequences at 1M tokens, paged NHD cache "
                        "(256-token pages, shuffled pool)", "B": 4, "Hq": 28, "Hkv": 4, "D": 128, "N": 1 << 20,
                        "rope_base": 1e7, "k_window": 16.0, "seed": 4, "page": 256},
}
# Block-selected prefill workloads (the window on top of a token-level selection):
# one step = one atflash_prefill_sparse call (RoPE pre-pass of Q and K, then the
# windowed prefill over the selected 128 x 128 tiles).  The mask follows the shape
# of dynamic-sparse selections such as MInference's: the first `sink_tiles` key
# tiles of every query tile, a band of `local_tiles` tiles ending at the diagonal,
# and each remaining causal tile with probability `extra` (seeded), per KV head.
SPARSE_WORKLOADS = {
    "qwen05b_32k_sparse": dict(_pf("Qwen2.5-0.5B-shaped single-layer windowed prefill over a block-sparse selection",
                                   1, 14, 2, 64, 32768, 1e6, 8.0, 1),
                               sink_tiles=2, local_tiles=16, extra=0.05, mask_seed=8),
    "llama3b_128k_sparse": dict(_pf("Llama-3.2-3B-shaped single-layer windowed prefill over a block-sparse selection",
                                    1, 24, 8, 128, 131072, 5e5, 16.0, 2),
                                sink_tiles=2, local_tiles=32, extra=0.02, mask_seed=9),
}


def block_mask_recipe(wl, T):
    """uint8 [B, Hkv, T, T] block selection of a SPARSE_WORKLOADS entry."""
    import numpy as np
    rng = np.random.default_rng(wl["mask_seed"])
    m = rng.random((wl["B"], wl["Hkv"], T, T)) < wl["extra"]
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    m |= (j < wl["sink_tiles"]) | ((i - j >= 0) & (i - j < wl["local_tiles"]))
    m &= j <= i
    return m.astype(np.uint8)


def tile_retained_flops(atf, wl, T):
    """Retained FLOPs of one (query tile, key tile) pair of one query head, by
    tile distance t = i - j: 4 per kept pair-term (QK over the kept pairs of each
    cell) + 2*D per cell (PV).  N must be a multiple of 128."""
    import numpy as np
    D, N = wl["D"], wl["N"]
    w = np.array(atf.window_table(D, wl["rope_base"], wl["k_window"], N), dtype=np.int64)
    ws = np.sort(w)
    kept_at = lambda d: len(ws) - np.searchsorted(ws, d, side="left")  # noqa: E731  pairs with w_r >= d
    out = np.zeros(T, dtype=np.float64)
    delta = np.arange(-127, 128)
    mult = 128 - np.abs(delta)
    for t in range(T):
        if t == 0:
            d = np.arange(128)
            cnt = 128 - d                      # cells (a, b) with a - b = d, a >= b
            kept = float(np.sum(cnt * kept_at(d)))
            cells = 128 * 129 / 2
        else:
            d = 128 * t + delta
            kept = float(np.sum(mult * kept_at(d)))
            cells = 128 * 128
        out[t] = 4 * kept + 2 * D * cells
    return out


def run_sparse(args, wl):
    import numpy as np
    import torch
    import long_context_attention_pair_b200 as atf
    from long_context_attention_pair_b200 import synthetic
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    B, N, Hq, Hkv, D = wl["B"], wl["N"], wl["Hq"], wl["Hkv"], wl["D"]
    base, kwin = wl["rope_base"], wl["k_window"]
    T = (N + 127) // 128
    mask_np = block_mask_recipe(wl, T)
    mask = torch.as_tensor(mask_np, device=dev)
    q = synthetic.tensor_torch(wl["seed"], "q", (B, N, Hq, D), "bf16", device=dev)
    k = synthetic.tensor_torch(wl["seed"], "k", (B, N, Hkv, D), "bf16", device=dev)
    v = synthetic.tensor_torch(wl["seed"], "v", (B, N, Hkv, D), "bf16", device=dev)
    out = torch.empty_like(q)
    ws = torch.empty(atf.prefill_workspace_bytes(B, Hq, Hkv, N, D), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def timed(fn, steps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    sparse_on = lambda: atf.prefill_sparse(q, k, v, mask, base, kwin, out=out, workspace=ws)  # noqa: E731
    sparse_off = lambda: atf.prefill_sparse(q, k, v, mask, base, math.inf, out=out, workspace=ws)  # noqa: E731
    dense_on = lambda: atf.prefill(q, k, v, base, kwin, out=out, workspace=ws)  # noqa: E731
    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ms = reduce_max(timed(sparse_on, args.steps), world, dev)
    clocks = sampler.stop()
    ms_off = reduce_max(timed(sparse_off, args.steps), world, dev)
    ms_dense = reduce_max(timed(dense_on, args.steps), world, dev)
    if atf.device_status() != 0:
        raise RuntimeError("a kernel's bounded wait ran out in the timed region")
    per_t = tile_retained_flops(atf, wl, T)
    i = np.arange(T)[:, None]
    j = np.arange(T)[None, :]
    vis = (mask_np != 0) | (i == j)[None, None]
    vis &= (j <= i)[None, None]
    dist = np.broadcast_to(i - j, vis.shape)
    flops = float(np.sum(per_t[dist[vis]])) * (Hq // Hkv)
    density = float(vis.sum()) / (B * Hkv * T * (T + 1) / 2)
    peaks, src = measured_peaks()
    long_region = ms * args.steps > 2000.0
    peak = peaks["bf16_tflops_sustained" if long_region else "bf16_tflops"]
    achieved = flops / (ms / 1e3) / 1e12
    line = {"metric": METRIC, "value": round(world * B * N / (ms / 1e3), 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(wl, tiles_kept=round(density, 4),
                           l2="flushed before every step (256 MiB write, outside the timed events)"),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4), "traffic": None,
                         "kernel": f"whole call: rope_pack(q), rope_pack(k), prefill_tc_kernel<{D}, block mask>, "
                                   "short rows",
                         "peak_source": f"{src} ({'sustained' if long_region else 'burst'} bf16)",
                         "flops_per_launch": flops},
            "window_off": {"ms_per_step": round(ms_off, 4)},
            "on_off_speedup": round(ms_off / ms, 4),
            "dense_window_on": {"ms_per_step": round(ms_dense, 4), "selection_speedup": round(ms_dense / ms, 4)},
            "gpu_launches": 4 * args.steps, "clocks": clocks}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# Ragged-batch prefill workloads: one step = one varlen prefill call (RoPE pre-pass of
# the packed Q and K, then the windowed prefill) over sequences of mixed lengths.
VARLEN_WORKLOADS = {
    "varlen_qwen05b_256k": {"workload": "Qwen2.5-0.5B-shaped single-layer windowed prefill of a ragged batch, "
                            "lengths log-uniform in [1K, 64K] tokens, 256K tokens in all", "Hq": 14, "Hkv": 2,
                            "D": 64, "total": 1 << 18, "len_lo": 1024, "len_hi": 65536, "rope_base": 1e6,
                            "k_window": 8.0, "seed": 6},
    "varlen_qwen7b_1m": {"workload": "Qwen2.5-7B-1M-shaped single-layer windowed prefill of a ragged batch, "
                         "lengths log-uniform in [4K, 256K] tokens, 1M tokens in all", "Hq": 28, "Hkv": 4,
                         "D": 128, "total": 1 << 20, "len_lo": 4096, "len_hi": 262144, "rope_base": 1e7,
                         "k_window": 16.0, "seed": 7},
}
DEFAULT_WORKLOAD = "qwen7b_512k"
# Lines measured in the same run as the default one and reported inside it.
SUB_RECORDS = ("decode_1m_packed", "decode_1m", "qwen05b_32k")
L2_FLUSH_BYTES = 256 << 20
# rope_pack(q), rope_pack(k), prefill_tc, short rows, decode_split, decode_merge, short decode rows
KERNELS_PER_STEP = 7

# DRAM bytes per launch of the tcgen05 prefill kernel, from one ncu capture per
# workload.  Valid only while the kernel source hashes to `source_sha1`;
# otherwise the line reports null.
TRAFFIC = {"workload": "qwen05b_32k", "bytes_per_launch": 99928064,
           "source_sha1": "9c36dbd1d5526ea2ee85f8ca868407a38a2cf948"}
# DRAM bytes per launch of the decode kernel (split states included, merge not),
# from an ncu capture of the same workload at a shorter cache length
# `captured_L`; valid while decode_tc.cu and decode.cu (the split heuristic)
# hash to `source_sha1`.  The natural
# layouts read the whole cache whatever the window (every 128-byte half-row keeps
# a sector), so their traffic grows in proportion to B * L and is scaled to the
# line's; the packed layout's kept share depends on L, so it is reported only at
# the captured length and the workload's own B.
DECODE_TRAFFIC = {"decode_1m": {"captured_L": 131072, "bytes_per_launch": 1078782976, "proportional_to_L": True,
                                "source_sha1": "f90fa0ad91c3ec30c6ce5b524acae257bf566d1f"},
                  "decode_1m_packed": {"captured_L": 131072, "bytes_per_launch": 897764352,
                                       "proportional_to_L": False,
                                       "source_sha1": "f90fa0ad91c3ec30c6ce5b524acae257bf566d1f"}}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-sub-records", action="store_true")
    p.add_argument("--workload", default=DEFAULT_WORKLOAD,
                   choices=sorted(WORKLOADS) + sorted(DECODE_WORKLOADS) + sorted(VARLEN_WORKLOADS) +
                   sorted(SPARSE_WORKLOADS))
    p.add_argument("--N", type=int, default=None, help="override sequence length (sweeps)")
    p.add_argument("--B", type=int, default=None, help="override the number of sequences (decode sweeps)")
    p.add_argument("--k-window", type=float, default=None, help="override k (inf = window off)")
    return p.parse_args()


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def kernel_sha1(*names):
    """sha1 of the named kernel sources, concatenated (default: the prefill kernel's)."""
    h = hashlib.sha1()
    for name in names or ("prefill_tc.cu",):
        with open(os.path.join(ROOT, "long_context_attention_pair_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


# The decode kernel and the split heuristic that sets its launch (keys per CTA).
DECODE_SOURCES = ("decode_tc.cu", "decode.cu")


# ---------------------------------------------------------------- distributed
def prefill_traffic(workload, wl):
    """Captured DRAM bytes of one prefill launch, for the workload (at its own N
    and k) and kernel source the capture was made on; otherwise None."""
    if workload != TRAFFIC["workload"] or TRAFFIC["source_sha1"] != kernel_sha1():
        return None
    ref = WORKLOADS[workload]
    if wl["N"] != ref["N"] or wl["k_window"] != ref["k_window"]:
        return None
    return TRAFFIC["bytes_per_launch"]


def decode_traffic(workload, L, B=None):
    """Captured DRAM bytes of one decode launch for this workload at cache length L
    (and B sequences, default the workload's), or None."""
    rec = DECODE_TRAFFIC.get(workload)
    if rec is None or rec["source_sha1"] != kernel_sha1(*DECODE_SOURCES):
        return None
    B0 = DECODE_WORKLOADS[workload]["B"]
    B = B0 if B is None else B
    if L == rec["captured_L"] and B == B0:
        return rec["bytes_per_launch"]
    if rec.get("proportional_to_L"):
        return round(rec["bytes_per_launch"] * (B * L) / (B0 * rec["captured_L"]))
    return None


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value, world, device):
    """Max of a float over ranks (host plumbing only)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def throughput(world, tokens_per_step, steps, total_ms_max):
    """Whole-job tokens/s: every rank processed `steps` steps of `tokens_per_step`
    tokens; the job took the slowest rank's time."""
    return world * tokens_per_step * steps / (total_ms_max / 1e3)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# --------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed region."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index):
        self.dev = device_index
        self.proc = None
        self.lines = []
        self.error = None

    def _gpu_id(self):
        import torch
        try:
            u = str(torch.cuda.get_device_properties(self.dev).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:  # noqa: BLE001
            return str(self.dev)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._gpu_id(), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception as e:  # noqa: BLE001
            self.error = str(e)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"error": self.error or "nvidia-smi unavailable"}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:  # noqa: BLE001
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for nm, val in zip(names, parts[3:]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return {"error": "no samples", "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------- CPU oracle
def oracle_rows_per_step(wl):
    """Query rows (all heads) the oracle computes per step, one rule for both arms:
    about 2^33 / (N * Hq * D) rows, so that a step is about a second of host work
    whatever the workload (5 rows at the 512K default, 293 at 32K)."""
    return max(1, round(2 ** 33 / (wl["N"] * wl["Hq"] * wl["D"])))


class OracleSample:
    """The fp64 oracle, as it stands, on seeded uniformly drawn query rows of the
    workload (every head; each row attends its full causal prefix)."""

    def __init__(self, wl, k, v, q_rows):
        import numpy as np
        self.wl, self.k, self.v, self.q_rows = wl, k, v, q_rows
        self.rows = oracle_rows_per_step(wl)
        self.rng = np.random.default_rng(99)
        self.th = rope_theta(wl)

    def step(self):
        import contextlib
        import numpy as np
        import oracle
        rows = np.sort(self.rng.choice(self.wl["N"], size=self.rows, replace=False))
        qr = self.q_rows(rows)
        with (oracle.scaled_rope(self.th) if self.th is not None else contextlib.nullcontext()):
            oracle.prefill_rows(qr, rows, self.k, self.v, self.wl["rope_base"], self.wl["k_window"])

    def describe(self, steps, seconds):
        import oracle
        return {"value": steps * self.rows / seconds, "unit": "tokens/s", "cores": oracle.threads(),
                "kind": "oracle",
                "sample": f"{steps} steps of {self.rows} seeded uniformly drawn query rows x all {self.wl['Hq']} "
                          f"heads (each row attends its full causal prefix), {seconds:.1f} s"}


def cpu_baseline(q, k, v, wl, budget_s=10.0):
    """The oracle timed on the host cores, on the reference arm's sampling rule."""
    kh, vh = k[0].float().cpu().numpy(), v[0].float().cpu().numpy()
    smp = OracleSample(wl, kh, vh, lambda rows: q[0, rows].float().cpu().numpy())
    t0 = time.perf_counter()
    smp.step()  # warm-up, also sizes the run
    t1 = time.perf_counter() - t0
    steps = max(3, min(50, int(budget_s / max(t1, 1e-3))))
    t0 = time.perf_counter()
    for _ in range(steps):
        smp.step()
    return smp.describe(steps, time.perf_counter() - t0)


def line_config(wl, world):
    """The `config` of a prefill line; both arms report the same one."""
    big = 2 * wl["B"] * wl["N"] * wl["Hq"] * wl["D"] > (126 << 20)
    l2 = ("inputs larger than L2, which is also flushed before every step (256 MiB write, outside the timed "
          "events)" if big else "flushed before every step (256 MiB write, outside the timed events)")
    return dict(wl, l2=l2, parallelism="replicas" if world > 1 else "single GPU")


def run_reference(args, wl):
    """Reference arm: the fp64 oracle on the host cores, bounded sample per step."""
    world, rank, _ = dist_setup()
    if rank != 0:
        return
    from long_context_attention_pair_b200 import synthetic
    N = wl["N"]
    shape_kv = (wl["B"], N, wl["Hkv"], wl["D"])
    k = synthetic.tensor(wl["seed"], "k", shape_kv, "bf16")[0]
    v = synthetic.tensor(wl["seed"], "v", shape_kv, "bf16")[0]
    qshape = (wl["B"], N, wl["Hq"], wl["D"])
    smp = OracleSample(wl, k, v, lambda rows: synthetic.rows(wl["seed"], "q", qshape, 1, rows, "bf16")[0])
    for _ in range(args.warmup):
        smp.step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        smp.step()
    t = time.perf_counter() - t0
    cb = smp.describe(args.steps, t)
    value = cb["value"]
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": line_config(wl, args.gpus), "cpu_baseline": cb,
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# -------------------------------------------------------------------- our arm
def init_dist(local):
    import torch
    world = dist_setup()[0]
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    return dev


def finish_dist(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_ours(args, wl):
    world, rank, local = dist_setup()
    dev = init_dist(local)
    line = measure_prefill(args, wl, args.workload, dev, e2e_on=not args.no_e2e,
                           cpu_on=rank == 0 and world == 1 and not args.no_cpu_baseline)
    if args.workload == DEFAULT_WORKLOAD and not args.no_sub_records and args.N is None and args.k_window is None:
        import torch
        subs = {}
        torch.cuda.empty_cache()
        for name in SUB_RECORDS:
            if name in DECODE_WORKLOADS:
                subs[name] = measure_decode(args, dict(DECODE_WORKLOADS[name]), name, dev)
            else:
                subs[name] = measure_prefill(args, dict(WORKLOADS[name]), name, dev, e2e_on=False, cpu_on=False)
            torch.cuda.empty_cache()
        line["sub_records"] = subs
        line["gpu_launches"] += sum(r["gpu_launches"] for r in subs.values())
    if rank == 0:
        print(json.dumps(line), flush=True)
    finish_dist(world)


def measure_prefill(args, wl, name, dev, e2e_on, cpu_on):
    """One prefill workload's line (every rank measures; times are max over ranks)."""
    import torch
    import long_context_attention_pair_b200 as atf
    from long_context_attention_pair_b200 import synthetic

    world, rank, local = dist_setup()
    B, N, Hq, Hkv, D = wl["B"], wl["N"], wl["Hq"], wl["Hkv"], wl["D"]
    base, kwin = wl["rope_base"], wl["k_window"]
    th = rope_theta(wl)
    tk = {} if th is None else {"theta": th}
    q = synthetic.tensor_torch(wl["seed"], "q", (B, N, Hq, D), "bf16", device=dev)
    k = synthetic.tensor_torch(wl["seed"], "k", (B, N, Hkv, D), "bf16", device=dev)
    v = synthetic.tensor_torch(wl["seed"], "v", (B, N, Hkv, D), "bf16", device=dev)
    out = torch.empty_like(q)
    qpack = torch.empty((B * Hq, D // 16, N, 16), dtype=torch.bfloat16, device=dev)
    kpack = torch.empty((B * Hkv, D // 16, N, 16), dtype=torch.bfloat16, device=dev)
    q_last = q[:, N - 1].contiguous()
    seqlens = torch.full((B,), N, dtype=torch.int32, device=dev)
    dws = torch.empty(atf.decode_workspace_bytes(B, Hq, Hkv, N, D), dtype=torch.uint8, device=dev)
    dec_out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(kw, ev=None):
        atf.rope_pack(q, base, out=qpack, **tk)
        atf.rope_pack(k, base, out=kpack, **tk)
        if ev is not None:
            ev[0].record(stream)
        atf.prefill_packed(qpack, kpack, v, base, kw, out=out, **tk)
        if ev is not None:
            ev[1].record(stream)
        atf.prefill_short_rows(q, k, v, out, base, kw, **tk)
        atf.decode(q_last, k, v, seqlens, base, kw, kv_layout="NHD", out=dec_out, workspace=dws, **tk)

    def timed(kw, steps):
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True),
                torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        barrier(world)
        torch.cuda.synchronize()
        for e in evs:
            flush.zero_()
            e[0].record(stream)
            step(kw, (e[1], e[2]))
            e[3].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        step_ms = [a.elapsed_time(d) for a, _, _, d in evs]
        kern_ms = [b.elapsed_time(c) for _, b, c, _ in evs]
        return sum(step_ms), statistics.mean(kern_ms), statistics.median(step_ms)

    for _ in range(args.warmup):
        step(kwin)
        step(math.inf)
    torch.cuda.synchronize()
    if atf.device_status() != 0:
        raise RuntimeError("a kernel's bounded wait ran out during warm-up")

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    total_ms, kern_ms, med_ms = timed(kwin, args.steps)
    clocks = sampler.stop()
    total_ms = reduce_max(total_ms, world, dev)
    off_total_ms, off_kern_ms, _ = timed(math.inf, max(3, args.steps // 4))
    off_total_ms = reduce_max(off_total_ms, world, dev)
    if atf.device_status() != 0:
        raise RuntimeError("a kernel's bounded wait ran out in the timed region")

    # Decode alone (one token per sequence), same step otherwise.
    dec_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(50)]
    for a, b in dec_ev:
        flush.zero_()
        a.record(stream)
        atf.decode(q_last, k, v, seqlens, base, kwin, kv_layout="NHD", out=dec_out, workspace=dws, **tk)
        b.record(stream)
    torch.cuda.synchronize()
    dec_us = 1e3 * statistics.median(a.elapsed_time(b) for a, b in dec_ev)

    tokens_per_step = B * N
    ms_per_step = total_ms / args.steps
    value = throughput(world, tokens_per_step, args.steps, total_ms)
    off_ms_per_step = off_total_ms / max(3, args.steps // 4)

    # Roofline of the dominant kernel (tcgen05 prefill): retained FLOPs only.
    terms = atf.pruned_terms(N, D, base, kwin, **tk)
    flops = B * Hq * (4 * terms["kept"] + D * N * (N + 1))
    peaks, src = measured_peaks()
    long_region = total_ms > 2000.0
    peak = peaks["bf16_tflops_sustained" if long_region else "bf16_tflops"]
    achieved = flops / (kern_ms / 1e3) / 1e12
    traffic = prefill_traffic(name, wl)
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": f"prefill_tc_kernel<{D}>",
                "kernel_ms": round(kern_ms, 4),
                "peak_source": f"{src} ({'sustained' if long_region else 'burst'} bf16)",
                "flops_per_launch": flops}

    line = {
        "metric": METRIC, "value": round(value, 1), "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": line_config(wl, world),
        "roofline": roofline,
        "gpu_launches": KERNELS_PER_STEP * args.steps,
        "clocks": clocks,
        "window_off": {"ms_per_step": round(off_ms_per_step, 4),
                       "value": round(world * tokens_per_step / (off_ms_per_step / 1e3), 1),
                       "prefill_kernel_ms": round(off_kern_ms, 4)},
        "on_off_speedup": round(off_ms_per_step / ms_per_step, 4),
        "prefill_kernel_on_off_speedup": round(off_kern_ms / kern_ms, 4),
        "decode": {"us_per_call": round(dec_us, 2), "us_per_token": round(dec_us / B, 2), "L": N},
        "pruned_fraction": round(terms["pruned"] / terms["total"], 6),
        "median_step_ms": round(med_ms, 4),
    }

    if e2e_on:
        del qpack, kpack, out, dws, flush
        torch.cuda.empty_cache()
        line["e2e"] = e2e(atf, q, k, v, wl, args, dev, world)
    if cpu_on:
        line["cpu_baseline"] = cpu_baseline(q, k, v, wl)
    return line


def decode_retained_bytes(atf, wl):
    """Algorithmic bytes of one decode call: V in full, only the kept K elements,
    the query and the output (bf16).  Kept K pairs over distances 0..L-1 of one
    (sequence, KV head): sum_r (min(w_r, L-1) + 1)."""
    B, Hq, Hkv, D, L = wl["B"], wl["Hq"], wl["Hkv"], wl["D"], wl["N"]
    w = atf.window_table(D, wl["rope_base"], wl["k_window"], L)
    kept_pairs = sum(min(x, L - 1) + 1 for x in w)
    per_head = 2 * (D * L) + 2 * (2 * kept_pairs)
    return B * Hkv * per_head + 2 * B * Hq * D * 2


def run_decode(args, wl):
    world, rank, local = dist_setup()
    dev = init_dist(local)
    line = measure_decode(args, wl, args.workload, dev)
    if rank == 0:
        print(json.dumps(line), flush=True)
    finish_dist(world)


def measure_decode(args, wl, name, dev):
    """One decode workload's line (every rank measures; times are max over ranks)."""
    import torch
    import long_context_attention_pair_b200 as atf
    from long_context_attention_pair_b200 import synthetic
    world, rank, local = dist_setup()
    B, Hq, Hkv, D, L = wl["B"], wl["Hq"], wl["Hkv"], wl["D"], wl["N"]
    base, kwin = wl["rope_base"], wl["k_window"]
    q = synthetic.tensor_torch(wl["seed"], "q_dec", (B, Hq, D), "bf16", device=dev)
    kc = synthetic.tensor_torch(wl["seed"], "k_cache", (B, Hkv, L, D), "bf16", device=dev)
    vc = synthetic.tensor_torch(wl["seed"], "v_cache", (B, Hkv, L, D), "bf16", device=dev)
    sl = torch.full((B,), L, dtype=torch.int32, device=dev)
    out = torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(atf.decode_workspace_bytes(B, Hq, Hkv, L, D), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    packed = bool(wl.get("packed"))
    if packed:
        # The RoPE pre-pass writes the rotated, chunk-major K cache once (not timed).
        kc = atf.rope_pack(kc.permute(0, 2, 1, 3).contiguous(), base)
        torch.cuda.synchronize()
    dkw = dict(kcache_rotated=True, kv_layout="PACKED") if packed else {}
    page = wl.get("page")
    if page:
        # Cut the caches into pages and scatter them through one pool in a seeded
        # random order (3 pool pages stay unused); built once, not timed.
        import numpy as np
        mp = L // page
        n_pool = B * mp + 3
        ids = np.random.default_rng(wl["seed"]).permutation(n_pool)[: B * mp].astype(np.int32)
        bt = torch.as_tensor(ids.reshape(B, mp), device=dev)
        idx = torch.as_tensor(ids.astype(np.int64), device=dev)
        C = D // 16
        if packed:  # [B*Hkv, C, L, 16] -> pool [n_pool, Hkv, C, page, 16]
            kp = torch.zeros((n_pool, Hkv, C, page, 16), dtype=torch.bfloat16, device=dev)
            kp[idx] = kc.view(B, Hkv, C, mp, page, 16).permute(0, 3, 1, 2, 4, 5).reshape(B * mp, Hkv, C, page, 16)
        else:  # [B, Hkv, L, D] -> pool [n_pool, page, Hkv, D]
            kp = torch.zeros((n_pool, page, Hkv, D), dtype=torch.bfloat16, device=dev)
            kp[idx] = kc.view(B, Hkv, mp, page, D).permute(0, 2, 3, 1, 4).reshape(B * mp, page, Hkv, D)
        vp = torch.zeros((n_pool, page, Hkv, D), dtype=torch.bfloat16, device=dev)
        vp[idx] = vc.view(B, Hkv, mp, page, D).permute(0, 2, 3, 1, 4).reshape(B * mp, page, Hkv, D)
        del kc, vc, idx
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        ws = torch.empty(atf.decode_workspace_bytes(B, Hq, Hkv, mp * page, D), dtype=torch.uint8, device=dev)

        def call(kw):
            atf.decode_paged(q, kp, vp, bt, sl, page, base, kw, out=out, workspace=ws, **dkw)
    else:
        def call(kw):
            atf.decode(q, kc, vc, sl, base, kw, out=out, workspace=ws, **dkw)

    cache_bytes = 2 * B * Hkv * L * D * 2
    # A cache that L2 could hold is evicted before every call (a 256 MiB write
    # outside the timed events), so that each call reads it from HBM as a decode
    # step of a many-layer model would; larger caches stream back to back.
    small = cache_bytes < 2 * L2_FLUSH_BYTES
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev) if small else None

    def timed(kw, steps):
        for _ in range(args.warmup):
            call(kw)
        torch.cuda.synchronize()
        if small:
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for a, b in evs:
                flush.zero_()
                a.record(stream)
                call(kw)
                b.record(stream)
            torch.cuda.synchronize()
            return sum(a.elapsed_time(b) for a, b in evs) / steps
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            call(kw)
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / steps

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ms = reduce_max(timed(kwin, args.steps), world, dev)
    clocks = sampler.stop()
    ms_off = reduce_max(timed(math.inf, args.steps), world, dev)
    if atf.device_status() != 0:
        raise RuntimeError("a kernel's bounded wait ran out in the timed region")
    peaks, src = measured_peaks()
    nbytes = decode_retained_bytes(atf, wl)
    if page:
        nbytes += 4 * B * (L // page)  # the block table
    gbs = nbytes / (ms / 1e3) / 1e9
    line = {"metric": METRIC, "value": round(world * B / (ms / 1e3), 2), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(wl, l2=("L2 flushed before every call (256 MiB write, outside the timed events; cache of "
                                   "%.1f MB)" % (cache_bytes / 1e6)) if small else
                           "inputs larger than L2 (cache of %.1f GB)" % (cache_bytes / 1e9)),
            "decode": {"us_per_call": round(1e3 * ms, 2), "us_per_token": round(1e3 * ms / B, 2)},
            "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": decode_traffic(name, L, B),
                         "kernel": f"decode_tc_kernel<{D}{', paged' if page else ''}> + decode_merge_kernel",
                         "bytes_per_call": nbytes, "peak_source": src},
            "window_off": {"ms_per_step": round(ms_off, 4), "us_per_token": round(1e3 * ms_off / B, 2)},
            "on_off_speedup": round(ms_off / ms, 4), "gpu_launches": 3 * args.steps, "clocks": clocks}
    return line


def ragged_lengths(seed, total, lo, hi):
    """Sequence lengths drawn log-uniform in [lo, hi] until they sum to `total` (the
    last one cut to fit, so the batch also holds a short ragged tail)."""
    import numpy as np
    rng = np.random.default_rng(seed)
    out, left = [], total
    while left > 0:
        n = min(left, int(round(math.exp(rng.uniform(math.log(lo), math.log(hi))))))
        out.append(n)
        left -= n
    return out


def run_varlen(args, wl):
    import torch
    import long_context_attention_pair_b200 as atf
    from long_context_attention_pair_b200 import synthetic
    world, rank, local = dist_setup()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)
    Hq, Hkv, D, base, kwin = wl["Hq"], wl["Hkv"], wl["D"], wl["rope_base"], wl["k_window"]
    lens = ragged_lengths(wl["seed"], wl["total"], wl["len_lo"], wl["len_hi"])
    total, max_len = sum(lens), max(lens)
    cu_host = [0]
    for n in lens:
        cu_host.append(cu_host[-1] + n)
    cu = torch.tensor(cu_host, dtype=torch.int32, device=dev)
    q = synthetic.tensor_torch(wl["seed"], "q", (total, Hq, D), "bf16", device=dev)
    k = synthetic.tensor_torch(wl["seed"], "k", (total, Hkv, D), "bf16", device=dev)
    v = synthetic.tensor_torch(wl["seed"], "v", (total, Hkv, D), "bf16", device=dev)
    out = torch.empty_like(q)
    ws = torch.empty(int(atf.lib().atflash_prefill_varlen_workspace_bytes(Hq, Hkv, total, D)), dtype=torch.uint8,
                     device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def call(kw):
        atf.prefill_varlen(q, k, v, cu, max_len, base, kw, out=out, workspace=ws)

    def timed(kw, steps):
        for _ in range(args.warmup):
            call(kw)
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for a, b in evs:
            flush.zero_()
            a.record(stream)
            call(kw)
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    sampler = ClockSampler(local)
    sampler.start()
    time.sleep(0.3)
    ms = timed(kwin, args.steps)
    clocks = sampler.stop()
    ms = reduce_max(ms, world, dev)
    ms_off = reduce_max(timed(math.inf, args.steps), world, dev)
    if atf.device_status() != 0:
        raise RuntimeError("a kernel's bounded wait ran out in the timed region")

    # Retained FLOPs: QK over the kept pair-terms of every sequence plus the causal PV.
    flops = 0
    kept = pruned = all_terms = 0
    for n in lens:
        t = atf.pruned_terms(n, D, base, kwin)
        flops += Hq * (4 * t["kept"] + D * n * (n + 1))
        kept, pruned, all_terms = kept + t["kept"], pruned + t["pruned"], all_terms + t["total"]
    peaks, src = measured_peaks()
    long_region = ms * args.steps > 2000.0
    peak = peaks["bf16_tflops_sustained" if long_region else "bf16_tflops"]
    achieved = flops / (ms / 1e3) / 1e12
    line = {"metric": METRIC, "value": round(world * total / (ms / 1e3), 1), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": dict(wl, B=len(lens), max_seqlen=max_len, seqlens=lens,
                           l2="flushed before every step (256 MiB write, outside the timed events)"),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4), "traffic": None,
                         "kernel": f"whole call: rope_pack(q), rope_pack(k), prefill_tc_kernel<{D}, varlen>, "
                                   "short rows",
                         "peak_source": f"{src} ({'sustained' if long_region else 'burst'} bf16)",
                         "flops_per_launch": flops},
            "window_off": {"ms_per_step": round(ms_off, 4), "value": round(world * total / (ms_off / 1e3), 1)},
            "on_off_speedup": round(ms_off / ms, 4),
            "pruned_fraction": round(pruned / all_terms, 6),
            "gpu_launches": 4 * args.steps, "clocks": clocks}
    if not args.no_e2e:
        line["e2e"] = e2e_varlen(atf, q, k, v, cu, max_len, wl, args, dev, world)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n0 = lens[0]
        line["cpu_baseline"] = cpu_baseline(q[None, :n0], k[None, :n0], v[None, :n0], dict(wl, N=n0))
        line["cpu_baseline"]["sample"] += f" (first sequence of the batch, {n0} tokens)"
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def e2e_varlen(atf, q, k, v, cu, max_len, wl, args, dev, world):
    """The ragged prefill through the public API with host buffers: every step copies
    q/k/v/cu_seqlens from pinned host memory, runs the call and reads the output back,
    all on one stream inside the timed region."""
    import torch
    hq, hk, hv, hcu = (t.cpu().pin_memory() for t in (q, k, v, cu))
    hout = torch.empty(q.shape, dtype=torch.bfloat16).pin_memory()
    dq, dk, dv, dcu, dout = (torch.empty_like(t) for t in (q, k, v, cu, q))
    ws = torch.empty(int(atf.lib().atflash_prefill_varlen_workspace_bytes(wl["Hq"], wl["Hkv"], q.shape[0],
                                                                         wl["D"])), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    total = q.shape[0]

    def step():
        dq.copy_(hq, non_blocking=True)
        dk.copy_(hk, non_blocking=True)
        dv.copy_(hv, non_blocking=True)
        dcu.copy_(hcu, non_blocking=True)
        atf.prefill_varlen(dq, dk, dv, dcu, max_len, wl["rope_base"], wl["k_window"], out=dout, workspace=ws)
        hout.copy_(dout, non_blocking=True)

    step()
    torch.cuda.synchronize()
    steps = max(3, args.steps)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = reduce_max(a.elapsed_time(b) / steps, world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hcu))
    return {"value": round(world * total / (ms / 1e3), 1), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": hout.numel() * hout.element_size(), "ms_per_step": round(ms, 4),
            "api": "prefill_varlen"}


def e2e(atf, q, k, v, wl, args, dev, world):
    """Same metric through the public API with host buffers.  Every step copies
    its inputs from pinned host memory (H2D q/k/v/seqlens), runs the prefill and
    the decode of the last row, and reads its outputs back (D2H out and the
    decoded row), all inside the timed region.  Steps are pipelined over two
    device buffer sets and three streams (copy in, compute, copy out), as a
    serving loop would run them: step i's copies overlap step i-1's compute."""
    import torch
    B, N, Hq, Hkv, D = wl["B"], wl["N"], wl["Hq"], wl["Hkv"], wl["D"]
    base, kwin = wl["rope_base"], wl["k_window"]
    th = rope_theta(wl)
    tk = {} if th is None else {"theta": th}
    hq, hk, hv = (t.cpu().pin_memory() for t in (q, k, v))
    hsl = torch.full((B,), N, dtype=torch.int32).pin_memory()
    nbuf = 2
    hout = [torch.empty((B, N, Hq, D), dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
    hdec = [torch.empty((B, Hq, D), dtype=torch.bfloat16).pin_memory() for _ in range(nbuf)]
    bufs = []
    for _ in range(nbuf):
        bufs.append({
            "q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
            "sl": torch.empty((B,), dtype=torch.int32, device=dev), "out": torch.empty_like(q),
            "qlast": torch.empty((B, Hq, D), dtype=q.dtype, device=dev),
            "dec": torch.empty((B, Hq, D), dtype=torch.bfloat16, device=dev),
            "ws": torch.empty(atf.prefill_workspace_bytes(B, Hq, Hkv, N, D), dtype=torch.uint8, device=dev),
            "dws": torch.empty(atf.decode_workspace_bytes(B, Hq, Hkv, N, D), dtype=torch.uint8, device=dev),
        })
    s_in, s_comp, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_done = [ev() for _ in range(nbuf)]
    comp_done = [ev() for _ in range(nbuf)]
    out_done = [ev() for _ in range(nbuf)]
    used = [False] * nbuf
    steps = max(3, args.steps // 10)

    def step(i):
        bi = i % nbuf
        d = bufs[bi]
        with torch.cuda.stream(s_in):
            if used[bi]:
                s_in.wait_event(comp_done[bi])  # step i-2 is done reading these inputs
            d["q"].copy_(hq, non_blocking=True)
            d["k"].copy_(hk, non_blocking=True)
            d["v"].copy_(hv, non_blocking=True)
            d["sl"].copy_(hsl, non_blocking=True)
            in_done[bi].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(in_done[bi])
            if used[bi]:
                s_comp.wait_event(out_done[bi])  # step i-2's outputs have been read back
            atf.prefill(d["q"], d["k"], d["v"], base, kwin, out=d["out"], workspace=d["ws"], stream=s_comp, **tk)
            d["qlast"].copy_(d["q"][:, N - 1])
            atf.decode(d["qlast"], d["k"], d["v"], d["sl"], base, kwin, kv_layout="NHD", out=d["dec"],
                       workspace=d["dws"], stream=s_comp, **tk)
            comp_done[bi].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[bi])
            hout[bi].copy_(d["out"], non_blocking=True)
            hdec[bi].copy_(d["dec"], non_blocking=True)
            out_done[bi].record(s_out)
        used[bi] = True

    for i in range(2):
        step(i)
    barrier(world)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(steps):
        step(i)
    # The last step's read-back ends the timed region; s_out orders it after every step.
    b.record(s_out)
    torch.cuda.synchronize()
    ms = reduce_max(a.elapsed_time(b), world, dev)
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv, hsl))
    d2h = sum(t.numel() * t.element_size() for t in (hout[0], hdec[0]))
    return {"value": round(world * B * N * steps / (ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(ms / steps, 4),
            "pipelined": "2 buffer sets, H2D / compute / D2H streams"}


def main():
    args = parse()
    if args.steps < 1 or args.warmup < 3:
        raise SystemExit("need --steps >= 1 and --warmup >= 3")
    if args.workload in DECODE_WORKLOADS:
        wl = dict(DECODE_WORKLOADS[args.workload])
        if args.N:
            wl["N"] = args.N
        if args.B:
            wl["B"] = args.B
        if args.k_window is not None:
            wl["k_window"] = args.k_window
        run_decode(args, wl)
        return
    if args.workload in VARLEN_WORKLOADS:
        run_varlen(args, dict(VARLEN_WORKLOADS[args.workload]))
        return
    if args.workload in SPARSE_WORKLOADS:
        run_sparse(args, dict(SPARSE_WORKLOADS[args.workload]))
        return
    wl = dict(WORKLOADS[args.workload])
    if args.N:
        wl["N"] = args.N
    if args.k_window is not None:
        wl["k_window"] = args.k_window
    if args.impl == "reference":
        run_reference(args, wl)
    else:
        run_ours(args, wl)


if __name__ == "__main__":
    main()
