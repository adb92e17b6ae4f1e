"""Plain fp64 CPU oracle for per-RoPE-wavelength windowed causal attention.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, by ``__graft_entry__.smoke()``
and by the CPU-baseline leg of ``bench.py``; never by the product package.
It shares no code with the CUDA path (the C source is ``atflash_oracle.c``).

Method source: "ATFlash — Per-RoPE-Wavelength Attention Windows"
(gh.bsm-lab.com/ATFlash/ATFlash-Kernel), sections "The idea" (pair
decomposition, window w_r = k * lambda_r, pruned terms are zero and the rest is
summed), "Porting to something else" (the pair loop inside the two attention
loops), and the arXiv 2608.02947 abstract (closed form, reachability).

Parity status: pinned.  Every function below is pinned by ``tests/test_oracle.py``
against textbook causal attention (k = inf), a brute-force count, the
relative-angle identity of RoPE, the k = 0 closed form and the pages' printed
pruning percentages.
"""
import ctypes
import math
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        d, i, i64, u64p, dp, fp, i64p, i32p = (ctypes.c_double, ctypes.c_int, ctypes.c_int64,
                                                ctypes.POINTER(ctypes.c_uint64),
                                                ctypes.POINTER(ctypes.c_double),
                                                ctypes.POINTER(ctypes.c_float),
                                                ctypes.POINTER(ctypes.c_int64),
                                                ctypes.POINTER(ctypes.c_int32))
        L.orc_window_limits.argtypes = [i, d, d, dp]
        L.orc_count_bruteforce.argtypes = [i64, i, d, d, u64p, u64p]
        L.orc_count_closed.argtypes = [i64, i, d, d, u64p, u64p]
        L.orc_min_kept_pairs.argtypes = [i64, i, d, d]
        L.orc_min_kept_pairs.restype = i64
        L.orc_prefill_rows.argtypes = [fp, i64p, i64, fp, fp, i, i, i64, i, d, d, dp, dp]
        L.orc_prefill_rows.restype = i
        L.orc_prefill_rows_sparse.argtypes = [fp, i64p, i64, fp, fp, i, i, i64, i, d, d,
                                              ctypes.POINTER(ctypes.c_ubyte), i64, dp, dp]
        L.orc_prefill_rows_sparse.restype = i
        L.orc_decode.argtypes = [fp, fp, fp, i32p, i, i, i, i64, i, d, d, i, dp, dp]
        L.orc_decode.restype = i
        L.orc_rope_rows.argtypes = [fp, i64p, i64, i, d, dp]
        L.orc_scores.argtypes = [fp, fp, i64, i, d, d, dp]
        L.orc_threads.restype = i
        L.orc_set_theta.argtypes = [dp, i]
        L.orc_set_theta.restype = i
        _lib = L
    return _lib


class scaled_rope:
    """Context manager: the oracle uses the frequency table ``theta`` (D/2 values,
    scaled RoPE) instead of base^(-2r/D) for windows and rotations inside the block."""

    def __init__(self, theta):
        self.theta = np.ascontiguousarray(np.asarray(theta, dtype=np.float64))

    def __enter__(self):
        if lib().orc_set_theta(self.theta.ctypes.data_as(ctypes.POINTER(ctypes.c_double)), len(self.theta)) != 0:
            raise ValueError("oracle rejected the frequency table")
        return self

    def __exit__(self, *exc):
        lib().orc_set_theta(None, 0)
        return False


def _f32(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32))


def _ptr(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def threads() -> int:
    """OpenMP threads the oracle uses."""
    return lib().orc_threads()


def window_limits(D: int, base: float, k: float) -> np.ndarray:
    """floor(k * lambda_r) for r < D/2 as float64 (inf when k = inf)."""
    out = np.zeros(D // 2, dtype=np.float64)
    lib().orc_window_limits(D, base, k, _ptr(out, ctypes.c_double))
    return out


def count_bruteforce(N: int, D: int, base: float, k: float):
    """(kept, total) pair-terms of one (sequence, head) by enumeration."""
    kp, tt = ctypes.c_uint64(), ctypes.c_uint64()
    lib().orc_count_bruteforce(N, D, base, k, ctypes.byref(kp), ctypes.byref(tt))
    return kp.value, tt.value


def count_closed(N: int, D: int, base: float, k: float):
    """(kept, total) pair-terms of one (sequence, head) by the closed form."""
    kp, tt = ctypes.c_uint64(), ctypes.c_uint64()
    lib().orc_count_closed(N, D, base, k, ctypes.byref(kp), ctypes.byref(tt))
    return kp.value, tt.value


def min_kept_pairs(N: int, D: int, base: float, k: float) -> int:
    """Fewest kept pairs over all causal distances 0..N-1."""
    return int(lib().orc_min_kept_pairs(N, D, base, k))


def rope_rows(x, pos, base: float) -> np.ndarray:
    """Rotate-half RoPE of rows x[n, D] at positions pos[n], fp64."""
    x = _f32(x)
    pos = np.ascontiguousarray(np.asarray(pos, dtype=np.int64))
    n, D = x.shape
    y = np.zeros((n, D), dtype=np.float64)
    lib().orc_rope_rows(_ptr(x, ctypes.c_float), _ptr(pos, ctypes.c_int64), n, D, base,
                        _ptr(y, ctypes.c_double))
    return y


def scores(q, k, base: float, kwin: float) -> np.ndarray:
    """Windowed scaled score matrix s[n, m] of one head (0 above the diagonal)."""
    q, k = _f32(q), _f32(k)
    N, D = q.shape
    s = np.zeros((N, N), dtype=np.float64)
    lib().orc_scores(_ptr(q, ctypes.c_float), _ptr(k, ctypes.c_float), N, D, base, kwin,
                     _ptr(s, ctypes.c_double))
    return s


def prefill_rows(q_rows, rows, k, v, base: float, kwin: float, want_lse: bool = False):
    """Prefill output rows of ONE sequence.

    q_rows [R, Hq, D] (un-rotated queries of the selected rows), rows [R] their
    positions, k/v [N, Hkv, D].  Returns out [R, Hq, D] float64 (and lse [R, Hq]).
    """
    q_rows, k, v = _f32(q_rows), _f32(k), _f32(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    R, Hq, D = q_rows.shape
    N, Hkv, _ = k.shape
    out = np.zeros((R, Hq, D), dtype=np.float64)
    lse = np.zeros((R, Hq), dtype=np.float64)
    rc = lib().orc_prefill_rows(_ptr(q_rows, ctypes.c_float), _ptr(rows, ctypes.c_int64), R,
                                _ptr(k, ctypes.c_float), _ptr(v, ctypes.c_float), Hq, Hkv, N, D,
                                base, kwin, _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle prefill_rows rejected its arguments")
    return (out, lse) if want_lse else out


def prefill_rows_sparse(q_rows, rows, k, v, base: float, kwin: float, block_mask, tile: int = 128,
                        want_lse: bool = False):
    """prefill_rows under a token-level block selection: block_mask [Hkv, T, T]
    (T = ceil(N / tile)); key m is visible to query n iff m <= n and (same tile,
    or block_mask[g, n // tile, m // tile] != 0) for the query heads of KV head g."""
    q_rows, k, v = _f32(q_rows), _f32(k), _f32(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    R, Hq, D = q_rows.shape
    N, Hkv, _ = k.shape
    T = (N + tile - 1) // tile
    mask = np.ascontiguousarray(np.asarray(block_mask) != 0, dtype=np.uint8)
    if mask.shape != (Hkv, T, T):
        raise ValueError(f"block_mask must be [{Hkv}, {T}, {T}]")
    out = np.zeros((R, Hq, D), dtype=np.float64)
    lse = np.zeros((R, Hq), dtype=np.float64)
    rc = lib().orc_prefill_rows_sparse(_ptr(q_rows, ctypes.c_float), _ptr(rows, ctypes.c_int64), R,
                                       _ptr(k, ctypes.c_float), _ptr(v, ctypes.c_float), Hq, Hkv, N, D,
                                       base, kwin, _ptr(mask, ctypes.c_ubyte), tile,
                                       _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle prefill_rows_sparse rejected its arguments")
    return (out, lse) if want_lse else out


def prefill(q, k, v, base: float, kwin: float, want_lse: bool = False):
    """Full prefill of q/k/v [B, N, H, D]; returns out [B, N, Hq, D] float64."""
    q, k, v = _f32(q), _f32(k), _f32(v)
    B, N, Hq, D = q.shape
    outs, lses = [], []
    rows = np.arange(N, dtype=np.int64)
    for b in range(B):
        o, l = prefill_rows(q[b], rows, k[b], v[b], base, kwin, want_lse=True)
        outs.append(o)
        lses.append(l)
    out, lse = np.stack(outs), np.stack(lses)
    return (out, lse) if want_lse else out


def decode(q, kcache, vcache, seqlens, base: float, kwin: float, kcache_rotated: bool = False,
           want_lse: bool = False):
    """Decode: q [B, Hq, D], caches [B, Hkv, Nmax, D], seqlens [B] -> out [B, Hq, D]."""
    q, kcache, vcache = _f32(q), _f32(kcache), _f32(vcache)
    seqlens = np.ascontiguousarray(np.asarray(seqlens, dtype=np.int32))
    B, Hq, D = q.shape
    _, Hkv, Nmax, _ = kcache.shape
    out = np.zeros((B, Hq, D), dtype=np.float64)
    lse = np.zeros((B, Hq), dtype=np.float64)
    rc = lib().orc_decode(_ptr(q, ctypes.c_float), _ptr(kcache, ctypes.c_float),
                          _ptr(vcache, ctypes.c_float), _ptr(seqlens, ctypes.c_int32),
                          B, Hq, Hkv, Nmax, D, base, kwin, int(bool(kcache_rotated)),
                          _ptr(out, ctypes.c_double), _ptr(lse, ctypes.c_double))
    if rc != 0:
        raise ValueError("oracle decode rejected its arguments")
    return (out, lse) if want_lse else out


INF = math.inf
