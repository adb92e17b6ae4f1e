"""Seeded synthetic inputs shared by the tests, the benchmark and the oracle runs.

Holds no attention arithmetic: only a counter-based normal generator, so the
value of element i of a tensor depends on (seed, stream, i) alone and any
subset of rows can be regenerated without producing the rest.

Recipe: splitmix64 over the counter gives two 53-bit uniforms per pair of
elements; Box-Muller in fp64 turns them into two N(0, 1) draws (cos branch for
even elements, sin branch for odd ones); the fp64 value is rounded to fp32
(round-to-nearest-even), and for bf16 inputs once more from fp32 to bf16 (RNE).
Values are returned as float32 arrays that hold the rounded values exactly.
"""
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Stream ids: one independent sequence per named tensor.
STREAMS = {"q": 1, "k": 2, "v": 3, "q_dec": 4, "k_cache": 5, "v_cache": 6}


def _mix(z):
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def _key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = np.array([(seed * 0x100000001B3 + stream * 0x632BE59BD9B4E019) & 0xFFFFFFFFFFFFFFFF],
                     dtype=np.uint64)
        return _mix(s + _GOLDEN)[0]


def normal_at(seed: int, stream: int, idx) -> np.ndarray:
    """N(0,1) fp64 draws for the element indices ``idx`` of one stream."""
    idx = np.asarray(idx, dtype=np.uint64)
    key = _key(seed, stream)
    with np.errstate(over="ignore"):
        pair = idx >> np.uint64(1)
        c1 = key + (np.uint64(2) * pair + np.uint64(1)) * _GOLDEN
        c2 = key + (np.uint64(2) * pair + np.uint64(2)) * _GOLDEN
        u1 = ((_mix(c1) >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)
        u2 = (_mix(c2) >> np.uint64(11)).astype(np.float64) * (1.0 / 9007199254740992.0)
    rad = np.sqrt(-2.0 * np.log(u1))
    ang = (2.0 * np.pi) * u2
    odd = (idx & np.uint64(1)).astype(bool)
    return np.where(odd, rad * np.sin(ang), rad * np.cos(ang))


def round_bf16(x32: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even), kept as float32."""
    b = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    lsb = (b >> np.uint32(16)) & np.uint32(1)
    r = ((b + np.uint32(0x7FFF) + lsb) >> np.uint32(16)) << np.uint32(16)
    return r.view(np.float32)


def _round(x64: np.ndarray, dtype: str) -> np.ndarray:
    x32 = x64.astype(np.float32)
    if dtype == "bf16":
        return round_bf16(x32)
    if dtype == "f32":
        return x32
    raise ValueError(f"unknown dtype {dtype}")


def tensor(seed: int, name: str, shape, dtype: str = "bf16", threads: int = 0) -> np.ndarray:
    """Whole tensor of the given shape (row-major element order), float32 holding dtype values."""
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    stream = STREAMS[name]
    chunk = 1 << 22
    starts = list(range(0, n, chunk))

    def work(s):
        e = min(n, s + chunk)
        out[s:e] = _round(normal_at(seed, stream, np.arange(s, e, dtype=np.uint64)), dtype)

    nthreads = threads or min(32, os.cpu_count() or 1)
    if len(starts) == 1 or nthreads == 1:
        for s in starts:
            work(s)
    else:
        with ThreadPoolExecutor(nthreads) as ex:
            list(ex.map(work, starts))
    return out.reshape(shape)


def rows(seed: int, name: str, shape, row_axis: int, row_ids, dtype: str = "bf16") -> np.ndarray:
    """Selected indices along ``row_axis`` of a tensor, identical to slicing ``tensor(...)``."""
    shape = tuple(int(s) for s in shape)
    row_ids = np.asarray(row_ids, dtype=np.int64)
    grids = np.meshgrid(*[row_ids if a == row_axis else np.arange(s) for a, s in enumerate(shape)],
                        indexing="ij")
    strides = np.cumprod((1,) + shape[::-1][:-1])[::-1]
    flat = sum(g.astype(np.uint64) * np.uint64(st) for g, st in zip(grids, strides))
    return _round(normal_at(seed, STREAMS[name], flat.ravel()), dtype).reshape(flat.shape)


# ---------------------------------------------------------------- device twin
def _i64(u: int) -> int:
    """uint64 constant as the int64 with the same bits."""
    return u - (1 << 64) if u >= (1 << 63) else u


def _lsr(z, k: int):
    """Logical right shift of int64 tensors holding uint64 bits."""
    return (z >> k) & ((1 << (64 - k)) - 1)


def _mix_t(z):
    z = (z ^ _lsr(z, 30)) * _i64(0xBF58476D1CE4E5B9)
    z = (z ^ _lsr(z, 27)) * _i64(0x94D049BB133111EB)
    return z ^ _lsr(z, 31)


def tensor_torch(seed: int, name: str, shape, dtype: str = "bf16", device="cuda", chunk: int = 1 << 26):
    """Same draws as ``tensor`` generated with torch ops on ``device`` (int64
    arithmetic wraps like uint64); returns a torch tensor of dtype bf16/f32."""
    import torch
    n = int(np.prod(shape))
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = torch.empty(n, dtype=tdt, device=device)
    key = _i64(int(_key(seed, STREAMS[name])))
    golden = _i64(int(_GOLDEN))
    scale = 1.0 / 9007199254740992.0
    for s in range(0, n, chunk):
        e = min(n, s + chunk)
        idx = torch.arange(s, e, dtype=torch.int64, device=device)
        pair = idx >> 1
        u1 = _lsr(_mix_t(key + (2 * pair + 1) * golden), 11).to(torch.float64)
        u2 = _lsr(_mix_t(key + (2 * pair + 2) * golden), 11).to(torch.float64)
        u1 = (u1 + 1.0) * scale
        u2 = u2 * scale
        rad = torch.sqrt(-2.0 * torch.log(u1))
        ang = (2.0 * np.pi) * u2
        val = torch.where((idx & 1).bool(), rad * torch.sin(ang), rad * torch.cos(ang))
        out[s:e] = val.to(torch.float32).to(tdt)
    return out.reshape(tuple(shape))
