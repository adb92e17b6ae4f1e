"""B200-native (sm_100a) per-RoPE-wavelength windowed causal attention.

Python binding of ``libatflash.so`` (C ABI in ``include/atflash.h``).  This
module only marshals arguments: every step of the attention runs in the CUDA
kernels of the library.  PyTorch supplies device memory and streams.  There
is no CPU fallback: if the library is missing, every call raises.

Method: "ATFlash — Per-RoPE-Wavelength Attention Windows"
(gh.bsm-lab.com/ATFlash/ATFlash-Kernel), section "The idea": the term of RoPE
frequency pair r (dims r and r + D/2) enters the query-key score only while
n - m <= floor(k * 2*pi / theta_r), theta_r = base^(-2r/D); k = inf is plain
causal RoPE attention.
"""
import ctypes
import math
import os

__all__ = [
    "lib", "prefill", "decode", "pruned_terms", "window_table", "prefill_workspace_bytes",
    "decode_workspace_bytes", "device_status", "AtflashError", "F32", "BF16", "rope_pack", "prefill_packed",
    "prefill_bf16", "theta_table", "prefill_sparse", "prefill_short_rows",
]

F32 = 0
BF16 = 1
KV_HND = 0
KV_NHD = 1
KV_PACKED = 2
OK = 0
ERR_TIMEOUT = -5
ERR_BAD_PAGE = -7

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libatflash.so")
_lib = None


class AtflashError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


class Terms(ctypes.Structure):
    _fields_ = [("total", ctypes.c_uint64), ("kept", ctypes.c_uint64), ("pruned", ctypes.c_uint64),
                ("total_dims", ctypes.c_uint64), ("kept_dims", ctypes.c_uint64)]


def lib():
    """The loaded C library; raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m long_context_attention_pair_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i, i64, d, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_size_t
        L.atflash_status_string.argtypes = [i]
        L.atflash_status_string.restype = ctypes.c_char_p
        L.atflash_version.restype = i
        L.atflash_window_table.argtypes = [i, d, d, i64, ctypes.POINTER(ctypes.c_int64)]
        L.atflash_pruned_terms.argtypes = [i64, i, d, d, ctypes.POINTER(Terms)]
        L.atflash_prefill.argtypes = [vp, vp, vp, vp, i, i, i, i64, i, d, d, vp]
        L.atflash_prefill_workspace_bytes.argtypes = [i, i, i, i64, i, i]
        L.atflash_prefill_workspace_bytes.restype = sz
        L.atflash_prefill_ex.argtypes = [vp, vp, vp, vp, i, i, i, i64, i, d, d, i, i, vp, vp, sz, vp]
        L.atflash_decode_workspace_bytes.argtypes = [i, i, i, i64, i]
        L.atflash_decode_workspace_bytes.restype = sz
        L.atflash_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i64, i, d, d, i, i, i, i, vp, sz, vp]
        L.atflash_rope_pack.argtypes = [vp, vp, i, i64, i, i, d, i, vp]
        L.atflash_rope_pack_bytes.argtypes = [i, i64, i, i, i]
        L.atflash_rope_pack_bytes.restype = sz
        L.atflash_prefill_packed.argtypes = [vp, vp, vp, vp, i, i, i, i64, i, d, d, i, i, vp, vp]
        L.atflash_device_status.argtypes = [i]
        L.atflash_prefill_varlen.argtypes = [vp, vp, vp, vp, vp, i, i64, i64, i, i, i, d, d, i, vp, vp, sz, vp]
        L.atflash_prefill_varlen_workspace_bytes.argtypes = [i, i, i64, i]
        L.atflash_prefill_varlen_workspace_bytes.restype = sz
        L.atflash_decode_paged.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, d, d, i, i, i, vp, sz, vp]
        dp = ctypes.POINTER(ctypes.c_double)
        L.atflash_theta_table.argtypes = [i, d, dp]
        L.atflash_window_table_theta.argtypes = [i, dp, d, i64, ctypes.POINTER(ctypes.c_int64)]
        L.atflash_pruned_terms_theta.argtypes = [i64, i, dp, d, ctypes.POINTER(Terms)]
        L.atflash_rope_pack_theta.argtypes = [vp, vp, i, i64, i, i, dp, i, vp]
        L.atflash_prefill_theta.argtypes = [vp, vp, vp, vp, i, i, i, i64, i, dp, d, i, i, vp, vp, sz, vp]
        L.atflash_decode_theta.argtypes = [vp, vp, vp, vp, vp, i, i, i, i64, i, dp, d, i, i, i, i, vp, sz, vp]
        L.atflash_prefill_varlen_theta.argtypes = [vp, vp, vp, vp, vp, i, i64, i64, i, i, i, dp, d, i, vp, vp, sz, vp]
        L.atflash_decode_paged_theta.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, dp, d, i, i, i, vp, sz,
                                                 vp]
        L.atflash_prefill_packed_theta.argtypes = [vp, vp, vp, vp, i, i, i, i64, i, dp, d, i, i, vp, vp]
        L.atflash_prefill_sparse.argtypes = [vp, vp, vp, vp, vp, i, i, i, i64, i, d, d, i, vp, vp, sz, vp]
        L.atflash_prefill_sparse_theta.argtypes = [vp, vp, vp, vp, vp, i, i, i, i64, i, dp, d, i, vp, vp, sz, vp]
        L.atflash_prefill_short_rows.argtypes = [vp, vp, vp, vp, i, i, i, i64, i, d, d, i, vp, vp]
        L.atflash_prefill_short_rows_theta.argtypes = [vp, vp, vp, vp, i, i, i, i64, i, dp, d, i, vp, vp]
        for f in ("atflash_window_table", "atflash_pruned_terms", "atflash_prefill", "atflash_prefill_ex",
                  "atflash_decode", "atflash_device_status", "atflash_rope_pack", "atflash_prefill_packed",
                  "atflash_prefill_varlen", "atflash_decode_paged", "atflash_theta_table",
                  "atflash_window_table_theta", "atflash_pruned_terms_theta", "atflash_rope_pack_theta",
                  "atflash_prefill_theta", "atflash_decode_theta", "atflash_prefill_varlen_theta",
                  "atflash_decode_paged_theta", "atflash_prefill_packed_theta", "atflash_prefill_sparse",
                  "atflash_prefill_sparse_theta", "atflash_prefill_short_rows",
                  "atflash_prefill_short_rows_theta"):
            getattr(L, f).restype = i
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().atflash_status_string(int(status)).decode()


def _check(status, what):
    if status != OK:
        raise AtflashError(status, what)


def _theta_arg(theta, D):
    """A caller's RoPE frequency table (scaled RoPE) as a host fp64 array of D/2."""
    vals = [float(x) for x in theta]
    if len(vals) != D // 2:
        raise ValueError(f"theta must hold D/2 = {D // 2} frequencies, got {len(vals)}")
    return (ctypes.c_double * len(vals))(*vals)


def theta_table(D: int, rope_base: float):
    """theta_r = base^(-2r/D), r < D/2: the frequencies the base-taking calls use."""
    arr = (ctypes.c_double * (D // 2))()
    _check(lib().atflash_theta_table(D, float(rope_base), arr), "atflash_theta_table")
    return list(arr)


def window_table(D: int, rope_base: float, k_window: float, N: int, *, theta=None):
    """Per-pair windows min(floor(k * lambda_r), N - 1), r < D/2 (host computation).
    ``theta`` (D/2 frequencies) replaces base^(-2r/D) for scaled RoPE."""
    arr = (ctypes.c_int64 * (D // 2))()
    if theta is None:
        _check(lib().atflash_window_table(D, rope_base, k_window, N, arr), "atflash_window_table")
    else:
        _check(lib().atflash_window_table_theta(D, _theta_arg(theta, D), k_window, N, arr),
               "atflash_window_table_theta")
    return list(arr)


def pruned_terms(N: int, D: int, rope_base: float, k_window: float, *, theta=None) -> dict:
    """Closed-form kept/pruned term counts of one (sequence, head)."""
    t = Terms()
    if theta is None:
        _check(lib().atflash_pruned_terms(N, D, rope_base, k_window, ctypes.byref(t)), "atflash_pruned_terms")
    else:
        _check(lib().atflash_pruned_terms_theta(N, D, _theta_arg(theta, D), k_window, ctypes.byref(t)),
               "atflash_pruned_terms_theta")
    return {"total": t.total, "kept": t.kept, "pruned": t.pruned, "total_dims": t.total_dims,
            "kept_dims": t.kept_dims}


def prefill_workspace_bytes(B, Hq, Hkv, N, D, in_dtype=BF16) -> int:
    return int(lib().atflash_prefill_workspace_bytes(B, Hq, Hkv, N, D, in_dtype))


def decode_workspace_bytes(B, Hq, Hkv, Nmax, D) -> int:
    return int(lib().atflash_decode_workspace_bytes(B, Hq, Hkv, Nmax, D))


def _torch():
    import torch
    return torch


def _dtype_code(t):
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream_ptr(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def prefill(q, k, v, rope_base: float, k_window: float = math.inf, *, out=None, out_dtype=None,
            return_lse: bool = False, workspace=None, stream=None, theta=None):
    """Windowed causal RoPE prefill.

    q [B, N, Hq, D], k/v [B, N, Hkv, D] (un-rotated q/k; bf16 -> tensor-core path,
    fp32 -> exact CUDA-core path).  Returns out [B, N, Hq, D] (dtype ``out_dtype``,
    default q's dtype) and, with ``return_lse``, lse [B, Hq, N] fp32.  ``theta``
    (D/2 frequencies) replaces base^(-2r/D) for scaled RoPE.
    """
    torch = _torch()
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    in_dtype = _dtype_code(q)
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise TypeError("q, k, v must share one dtype")
    if out is None:
        od = out_dtype if out_dtype is not None else q.dtype
        out = torch.empty((B, N, Hq, D), dtype=od, device=q.device)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if return_lse else None
    need = prefill_workspace_bytes(B, Hq, Hkv, N, D, in_dtype)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    fn, name = lib().atflash_prefill_ex, "atflash_prefill_ex"
    rope = float(rope_base)
    if theta is not None:
        fn, name, rope = lib().atflash_prefill_theta, "atflash_prefill_theta", _theta_arg(theta, D)
    st = fn(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), B, Hq, Hkv, N, D, rope, float(k_window),
            in_dtype, _dtype_code(out), _dev(lse, "lse") if lse is not None else None, _dev(workspace, "workspace"),
            need, _stream_ptr(stream))
    _check(st, name)
    return (out, lse) if return_lse else out


def prefill_sparse(q, k, v, block_mask, rope_base: float, k_window: float = math.inf, *, out=None, out_dtype=None,
                   return_lse: bool = False, workspace=None, stream=None, theta=None):
    """Windowed prefill on top of a token-level block selection.

    q [B, N, Hq, D], k/v [B, N, Hkv, D] bf16 (un-rotated q/k); block_mask
    [B, Hkv, T, T] uint8 or bool on the device, T = ceil(N / 128): entry
    (b, g, i, j) keeps key tile j for query tile i of KV head g's query heads
    (the diagonal tile always; entries above it are ignored).  Returns out
    [B, N, Hq, D] and, with ``return_lse``, lse [B, Hq, N] fp32.
    """
    torch = _torch()
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    T = (N + 127) // 128
    if tuple(block_mask.shape) != (B, Hkv, T, T):
        raise ValueError(f"block_mask must be [{B}, {Hkv}, {T}, {T}], got {tuple(block_mask.shape)}")
    if block_mask.dtype == torch.bool:
        block_mask = block_mask.view(torch.uint8)
    if block_mask.dtype != torch.uint8:
        raise TypeError("block_mask must be uint8 or bool")
    if out is None:
        od = out_dtype if out_dtype is not None else q.dtype
        out = torch.empty((B, N, Hq, D), dtype=od, device=q.device)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=q.device) if return_lse else None
    need = prefill_workspace_bytes(B, Hq, Hkv, N, D, BF16)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    fn, name, rope = lib().atflash_prefill_sparse, "atflash_prefill_sparse", float(rope_base)
    if theta is not None:
        fn, name, rope = lib().atflash_prefill_sparse_theta, "atflash_prefill_sparse_theta", _theta_arg(theta, D)
    st = fn(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(block_mask, "block_mask"), _dev(out, "out"), B, Hq, Hkv,
            N, D, rope, float(k_window), _dtype_code(out), _dev(lse, "lse") if lse is not None else None,
            _dev(workspace, "workspace"), need, _stream_ptr(stream))
    _check(st, name)
    return (out, lse) if return_lse else out


def prefill_varlen(q, k, v, cu_seqlens, max_seqlen: int, rope_base: float, k_window: float = math.inf, *,
                   out=None, out_dtype=None, return_lse: bool = False, workspace=None, stream=None, theta=None):
    """Windowed causal RoPE prefill of a ragged batch packed along the token axis.

    q [total, Hq, D], k/v [total, Hkv, D] bf16 (un-rotated); cu_seqlens int32 [B+1]
    on the device (sequence b is tokens cu[b]..cu[b+1]-1, positions restart at 0);
    max_seqlen >= every sequence length.  Returns out [total, Hq, D] and, with
    ``return_lse``, lse [Hq, total] fp32.
    """
    torch = _torch()
    total, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if cu_seqlens.dtype != torch.int32:
        raise TypeError("cu_seqlens must be int32")
    if out is None:
        out = torch.empty((total, Hq, D), dtype=out_dtype if out_dtype is not None else q.dtype, device=q.device)
    lse = torch.empty((Hq, total), dtype=torch.float32, device=q.device) if return_lse else None
    need = int(lib().atflash_prefill_varlen_workspace_bytes(Hq, Hkv, total, D))
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    fn, name = lib().atflash_prefill_varlen, "atflash_prefill_varlen"
    rope = float(rope_base)
    if theta is not None:
        fn, name, rope = lib().atflash_prefill_varlen_theta, "atflash_prefill_varlen_theta", _theta_arg(theta, D)
    st = fn(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), _dev(cu_seqlens, "cu_seqlens"), B,
            int(max_seqlen), total, Hq, Hkv, D, rope, float(k_window), _dtype_code(out),
            _dev(lse, "lse") if lse is not None else None, ws_ptr, ws_bytes if workspace is not None else need,
            _stream_ptr(stream))
    _check(st, name)
    return (out, lse) if return_lse else out


def decode_paged(q, kpages, vpages, block_table, seqlens, page_size: int, rope_base: float,
                 k_window: float = math.inf, *, kcache_rotated: bool = False, kv_layout: str = "NHD", out=None,
                 out_dtype=None, workspace=None, stream=None, theta=None):
    """One decode step over a paged KV cache.

    q [B, Hq, D] bf16; block_table int32 [B, max_pages]; seqlens int32 [B].
    kv_layout "NHD": kpages/vpages [num_pages, page_size, Hkv, D];
    "PACKED": kpages [num_pages, Hkv, D/16, page_size, 16] (rotated), vpages as NHD.
    page_size must be a multiple of 64.  Returns out [B, Hq, D].
    """
    torch = _torch()
    B, Hq, D = q.shape
    num_pages = vpages.shape[0]
    Hkv = vpages.shape[2]
    max_pages = block_table.shape[1]
    lay = {"NHD": KV_NHD, "PACKED": KV_PACKED}[kv_layout]
    if out is None:
        out = torch.empty((B, Hq, D), dtype=out_dtype if out_dtype is not None else q.dtype, device=q.device)
    need = decode_workspace_bytes(B, Hq, Hkv, max_pages * page_size, D)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    fn, name = lib().atflash_decode_paged, "atflash_decode_paged"
    rope = float(rope_base)
    if theta is not None:
        fn, name, rope = lib().atflash_decode_paged_theta, "atflash_decode_paged_theta", _theta_arg(theta, D)
    st = fn(_dev(q, "q"), _dev(kpages, "kpages"), _dev(vpages, "vpages"), _dev(block_table, "block_table"),
            _dev(seqlens, "seqlens"), _dev(out, "out"), B, Hq, Hkv, max_pages, num_pages, int(page_size), D, rope,
            float(k_window), 1 if kcache_rotated else 0, lay, _dtype_code(out), _dev(workspace, "workspace"), need,
            _stream_ptr(stream))
    _check(st, name)
    return out


def rope_pack(x, rope_base: float, *, out=None, stream=None, theta=None):
    """Rotate x [B, N, H, D] once into the packed layout ``prefill_packed`` reads.

    bf16 -> [B*H, D/16, N, 16] bf16 (8 pairs per 32-byte chunk, pair-interleaved);
    fp32 -> [B*H, N, D] fp32 pair-interleaved.
    """
    torch = _torch()
    B, N, H, D = x.shape
    dt = _dtype_code(x)
    need = int(lib().atflash_rope_pack_bytes(B, N, H, D, dt))
    if need == 0:
        raise AtflashError(-2, "atflash_rope_pack_bytes")
    if out is None:
        shape = (B * H, D // 16, N, 16) if dt == BF16 else (B * H, N, D)
        out = torch.empty(shape, dtype=x.dtype, device=x.device)
    if theta is None:
        _check(lib().atflash_rope_pack(_dev(x, "x"), _dev(out, "out"), B, N, H, D, float(rope_base), dt,
                                       _stream_ptr(stream)), "atflash_rope_pack")
    else:
        _check(lib().atflash_rope_pack_theta(_dev(x, "x"), _dev(out, "out"), B, N, H, D, _theta_arg(theta, D), dt,
                                             _stream_ptr(stream)), "atflash_rope_pack_theta")
    return out


def prefill_packed(qpack, kpack, v, rope_base: float, k_window: float = math.inf, *, B=None, Hq=None,
                   out=None, out_dtype=None, lse=None, stream=None, theta=None):
    """Attention over ``rope_pack`` outputs; v [B, N, Hkv, D] un-rotated values.
    With ``theta``, qpack/kpack come from ``rope_pack(..., theta=theta)``."""
    torch = _torch()
    Bv, N, Hkv, D = v.shape
    B = Bv if B is None else B
    Hq = (qpack.shape[0] // B) if Hq is None else Hq
    if out is None:
        od = out_dtype if out_dtype is not None else v.dtype
        out = torch.empty((B, N, Hq, D), dtype=od, device=v.device)
    fn, name, rope = lib().atflash_prefill_packed, "atflash_prefill_packed", float(rope_base)
    if theta is not None:
        fn, name, rope = lib().atflash_prefill_packed_theta, "atflash_prefill_packed_theta", _theta_arg(theta, D)
    st = fn(_dev(qpack, "qpack"), _dev(kpack, "kpack"), _dev(v, "v"), _dev(out, "out"), B, Hq, Hkv, N, D, rope,
            float(k_window), _dtype_code(v), _dtype_code(out), _dev(lse, "lse") if lse is not None else None,
            _stream_ptr(stream))
    _check(st, name)
    return out


def prefill_short_rows(q, k, v, out, rope_base: float, k_window: float = math.inf, *, lse=None, stream=None,
                       theta=None):
    """The short-row step on its own: recompute in fp32 the rows that see at most
    128 keys (the first 128-row tile of every sequence) from the un-rotated bf16
    q [B, N, Hq, D], k/v [B, N, Hkv, D], overwriting them in ``out`` (and ``lse``
    [B, Hq, N]).  Queue it after ``prefill_packed`` on the same stream; the
    three steps then give the bits of ``prefill``."""
    B, N, Hq, D = q.shape
    fn, name, rope = lib().atflash_prefill_short_rows, "atflash_prefill_short_rows", float(rope_base)
    if theta is not None:
        fn, name, rope = (lib().atflash_prefill_short_rows_theta, "atflash_prefill_short_rows_theta",
                          _theta_arg(theta, D))
    st = fn(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), B, Hq, k.shape[2], N, D, rope,
            float(k_window), _dtype_code(out), _dev(lse, "lse") if lse is not None else None, _stream_ptr(stream))
    _check(st, name)
    return out


def prefill_bf16(q, k, v, out, rope_base: float, k_window: float = math.inf, stream=None):
    """The plain bf16 call (library-managed scratch), writing into ``out``."""
    B, N, Hq, D = q.shape
    st = lib().atflash_prefill(_dev(q, "q"), _dev(k, "k"), _dev(v, "v"), _dev(out, "out"), B, Hq, k.shape[2],
                               N, D, float(rope_base), float(k_window), _stream_ptr(stream))
    _check(st, "atflash_prefill")
    return out


def decode(q, k_cache, v_cache, seqlens, rope_base: float, k_window: float = math.inf, *,
           kcache_rotated: bool = False, kv_layout: str = "HND", out=None, out_dtype=None, workspace=None,
           stream=None, theta=None):
    """Windowed decode: q [B, Hq, D], seqlens int32 [B] (device), caches in
    ``kv_layout`` "HND" [B, Hkv, Nmax, D], "NHD" [B, Nmax, Hkv, D], or "PACKED":
    k_cache = ``rope_pack`` output [B*Hkv, D/16, Nmax, 16] (rotated; requires
    ``kcache_rotated=True``) and v_cache [B, Hkv, Nmax, D].

    The query of sequence b sits at position seqlens[b] - 1.  Returns out [B, Hq, D].
    """
    torch = _torch()
    B, Hq, D = q.shape
    if kv_layout == "HND":
        _, Hkv, Nmax, _ = k_cache.shape
        lay = KV_HND
    elif kv_layout == "NHD":
        _, Nmax, Hkv, _ = k_cache.shape
        lay = KV_NHD
    elif kv_layout == "PACKED":
        _, Hkv, Nmax, _ = v_cache.shape
        lay = KV_PACKED
    else:
        raise ValueError("kv_layout must be 'HND', 'NHD' or 'PACKED'")
    in_dtype = _dtype_code(q)
    if seqlens.dtype != torch.int32:
        raise TypeError("seqlens must be int32")
    if out is None:
        od = out_dtype if out_dtype is not None else q.dtype
        out = torch.empty((B, Hq, D), dtype=od, device=q.device)
    need = decode_workspace_bytes(B, Hq, Hkv, Nmax, D)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    fn, name = lib().atflash_decode, "atflash_decode"
    rope = float(rope_base)
    if theta is not None:
        fn, name, rope = lib().atflash_decode_theta, "atflash_decode_theta", _theta_arg(theta, D)
    st = fn(_dev(q, "q"), _dev(k_cache, "k_cache"), _dev(v_cache, "v_cache"), _dev(seqlens, "seqlens"),
            _dev(out, "out"), B, Hq, Hkv, Nmax, D, rope, float(k_window), int(bool(kcache_rotated)), lay, in_dtype,
            _dtype_code(out), _dev(workspace, "workspace"), need, _stream_ptr(stream))
    _check(st, name)
    return out


def device_status(clear: bool = True) -> int:
    """ATFlash device status word: 0, -5 after a kernel's bounded wait ran out, or
    -7 after a paged decode met a bad page index (the first event is kept)."""
    return int(lib().atflash_device_status(1 if clear else 0))


def set_wait_limit_ms(ms: float) -> None:
    """Limit of the kernels' pipeline waits for launches after this call."""
    f = lib().atflash_set_wait_limit_ms
    f.argtypes = [ctypes.c_double]
    f.restype = ctypes.c_int
    _check(f(float(ms)), "atflash_set_wait_limit_ms")


def selftest_wait_timeout(limit_ms: float, stream=None) -> None:
    """Launch the failure-detection self-test (a bounded wait that must run out)."""
    import torch
    f = lib().atflash_selftest_wait_timeout
    f.argtypes = [ctypes.c_double, ctypes.c_void_p]
    f.restype = ctypes.c_int
    st = (stream or torch.cuda.current_stream()).cuda_stream
    _check(f(float(limit_ms), ctypes.c_void_p(st)), "atflash_selftest_wait_timeout")
