"""Host-side checks of the C ABI (no GPU needed, no compute launched).

* libatflash.so loads and exports every function declared in include/atflash.h;
* the window table and the closed-form term counts equal the oracle's,
  bit-exactly, on every workload shape and on edge cases;
* invalid arguments return the documented status before anything is launched.
"""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import long_context_attention_pair_b200 as atf

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "atflash.h")


@pytest.fixture(scope="module")
def L():
    from long_context_attention_pair_b200 import build
    build.build()
    return atf.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(atflash_\w+)\s*\(", text)))


def test_header_declares_the_three_north_star_calls():
    names = declared_functions()
    for f in ("atflash_prefill", "atflash_decode", "atflash_pruned_terms"):
        assert f in names


def test_library_exports_every_declared_symbol(L):
    for name in declared_functions():
        assert hasattr(L, name), name


def test_status_strings(L):
    for s in (0, -1, -2, -3, -4, -5, -6, -7):
        assert atf.status_string(s) != "unknown status"


WINDOW_CASES = [
    (64, 1e4, 1.0, 256), (64, 1e4, math.inf, 256), (64, 1e6, 8.0, 32768), (128, 5e5, 16.0, 131072),
    (128, 1e7, 16.0, 524288), (128, 1e7, 64.0, 1048576), (128, 1e7, 4.0, 1048576), (8, 10.0, 0.25, 300),
    (2, 1e4, 0.0, 10), (256, 1e4, 2.5, 5000),
]


@pytest.mark.parametrize("D,base,k,N", WINDOW_CASES)
def test_window_table_equals_oracle(L, oracle, D, base, k, N):
    got = np.array(atf.window_table(D, base, k, N), dtype=np.float64)
    ref = np.minimum(oracle.window_limits(D, base, k), N - 1)
    np.testing.assert_array_equal(got, ref)


@pytest.mark.parametrize("D,base,k,N", WINDOW_CASES + [(64, 1e4, 1.0, 1), (128, 1e7, 16.0, 1 << 26)])
def test_pruned_terms_equal_oracle_closed_form(L, oracle, D, base, k, N):
    t = atf.pruned_terms(N, D, base, k)
    kept, total = oracle.count_closed(N, D, base, k)
    assert (t["kept"], t["total"]) == (kept, total)
    assert t["pruned"] == total - kept
    assert t["kept_dims"] == 2 * kept and t["total_dims"] == 2 * total


@pytest.mark.parametrize("N,D,base,k", [(256, 64, 1e4, 1.0), (300, 8, 10.0, 0.25), (513, 128, 5e5, 16.0),
                                        (1000, 128, 1e7, 4.0)])
def test_pruned_terms_equal_bruteforce(L, oracle, N, D, base, k):
    t = atf.pruned_terms(N, D, base, k)
    assert (t["kept"], t["total"]) == oracle.count_bruteforce(N, D, base, k)


def test_pruned_terms_rejects_bad_args(L):
    t = atf.Terms()
    for args in [(0, 64, 1e4, 1.0), (256, 63, 1e4, 1.0), (256, 64, 1.0, 1.0), (256, 64, 1e4, -1.0),
                 (256, 64, 1e4, float("nan")), (256, 512, 1e4, 1.0)]:
        assert L.atflash_pruned_terms(*args, ctypes.byref(t)) == -1
    assert L.atflash_pruned_terms(256, 64, 1e4, 1.0, None) == -1


# Fake, aligned, never-dereferenced device addresses: every case below must be
# rejected by the argument checks before any CUDA call.
P = ctypes.c_void_p(1 << 20)


def prefill_ex(L, **kw):
    a = dict(q=P, k=P, v=P, out=P, B=1, Hq=2, Hkv=1, N=256, D=64, base=1e4, kwin=1.0, ind=atf.BF16,
             outd=atf.BF16, lse=None, ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    return L.atflash_prefill_ex(a["q"], a["k"], a["v"], a["out"], a["B"], a["Hq"], a["Hkv"], a["N"], a["D"],
                                a["base"], a["kwin"], a["ind"], a["outd"], a["lse"], a["ws"], a["wsb"],
                                a["stream"])


def test_prefill_argument_errors(L):
    assert prefill_ex(L, q=None) == -1
    assert prefill_ex(L, B=0) == -1
    assert prefill_ex(L, Hq=3, Hkv=2) == -1
    assert prefill_ex(L, N=0) == -1
    assert prefill_ex(L, N=1 << 31) == -1
    assert prefill_ex(L, kwin=-1.0) == -1
    assert prefill_ex(L, kwin=float("nan")) == -1
    assert prefill_ex(L, base=1.0) == -1
    assert prefill_ex(L, D=96) == -2          # no tensor-core kernel for D=96
    assert prefill_ex(L, ind=7) == -2
    assert prefill_ex(L, q=ctypes.c_void_p((1 << 20) + 8)) == -6
    assert prefill_ex(L, ws=None) == -3
    assert prefill_ex(L, wsb=10) == -3
    assert prefill_ex(L, ws=ctypes.c_void_p((1 << 20) + 16)) == -6


def prefill_sparse(L, **kw):
    a = dict(q=P, k=P, v=P, mask=P, out=P, B=1, Hq=2, Hkv=1, N=256, D=64, base=1e4, kwin=1.0, outd=atf.BF16,
             lse=None, ws=P, wsb=1 << 40, stream=None)
    a.update(kw)
    return L.atflash_prefill_sparse(a["q"], a["k"], a["v"], a["mask"], a["out"], a["B"], a["Hq"], a["Hkv"], a["N"],
                                    a["D"], a["base"], a["kwin"], a["outd"], a["lse"], a["ws"], a["wsb"],
                                    a["stream"])


def test_prefill_sparse_argument_errors(L):
    assert prefill_sparse(L, mask=None) == -1
    assert prefill_sparse(L, q=None) == -1
    assert prefill_sparse(L, Hq=3, Hkv=2) == -1
    assert prefill_sparse(L, kwin=float("nan")) == -1
    assert prefill_sparse(L, base=0.5) == -1
    assert prefill_sparse(L, D=96) == -2       # bf16 tensor-core path only
    assert prefill_sparse(L, outd=9) == -2
    assert prefill_sparse(L, out=ctypes.c_void_p((1 << 20) + 8)) == -6
    assert prefill_sparse(L, ws=None) == -3
    assert prefill_sparse(L, wsb=100) == -3
    assert prefill_sparse(L, ws=ctypes.c_void_p((1 << 20) + 16)) == -6


def test_rope_pack_and_packed_prefill_argument_errors(L):
    assert L.atflash_rope_pack(None, P, 1, 256, 2, 64, 1e4, atf.BF16, None) == -1
    assert L.atflash_rope_pack(P, P, 1, 256, 2, 96, 1e4, atf.BF16, None) == -2
    assert L.atflash_rope_pack(P, ctypes.c_void_p((1 << 20) + 32), 1, 256, 2, 64, 1e4, atf.BF16, None) == -6
    assert L.atflash_rope_pack_bytes(1, 256, 2, 64, atf.BF16) == 256 * 2 * 64 * 2
    assert L.atflash_rope_pack_bytes(1, 256, 2, 6, atf.F32) == 256 * 2 * 6 * 4
    assert L.atflash_prefill_packed(P, P, P, None, 1, 2, 1, 256, 64, 1e4, 1.0, atf.BF16, atf.BF16, None,
                                    None) == -1
    assert L.atflash_prefill_packed(P, P, P, P, 1, 2, 1, 256, 128, 1e4, -2.0, atf.BF16, atf.BF16, None,
                                    None) == -1


def test_workspace_sizes(L):
    assert atf.prefill_workspace_bytes(1, 14, 2, 32768, 64) == 14 * 32768 * 64 * 2 + 2 * 32768 * 64 * 2
    assert atf.prefill_workspace_bytes(1, 1, 1, 256, 64, atf.F32) == 2 * 256 * 64 * 4
    assert atf.prefill_workspace_bytes(0, 1, 1, 256, 64) == 0
    assert atf.decode_workspace_bytes(4, 28, 4, 1 << 20, 128) > 0
    assert atf.decode_workspace_bytes(4, 28, 4, 1 << 20, 96) == 0


def test_decode_argument_errors(L):
    def dec(**kw):
        a = dict(q=P, kc=P, vc=P, sl=P, out=P, B=4, Hq=28, Hkv=4, Nmax=4096, D=128, base=1e7, kwin=16.0, krot=0,
                 lay=atf.KV_HND, ind=atf.BF16, outd=atf.F32, ws=P, wsb=1 << 40, stream=None)
        a.update(kw)
        return L.atflash_decode(a["q"], a["kc"], a["vc"], a["sl"], a["out"], a["B"], a["Hq"], a["Hkv"],
                                a["Nmax"], a["D"], a["base"], a["kwin"], a["krot"], a["lay"], a["ind"], a["outd"],
                                a["ws"], a["wsb"], a["stream"])
    assert dec(sl=None) == -1
    assert dec(Hq=30) == -1
    assert dec(krot=2) == -1
    assert dec(lay=5) == -1
    assert dec(lay=atf.KV_PACKED, krot=0) == -1      # packed caches hold rotated keys
    assert dec(lay=atf.KV_PACKED, krot=1, ind=atf.F32) == -2
    assert dec(D=80) == -2
    assert dec(Hq=68, Hkv=4) == -2   # more than 16 query heads per KV head
    assert dec(ws=None) == -3
    assert dec(wsb=100) == -3
    assert dec(vc=ctypes.c_void_p((1 << 20) + 4)) == -6


def test_wait_limit_and_selftest_argument_errors(L):
    import ctypes
    L.atflash_set_wait_limit_ms.argtypes = [ctypes.c_double]
    L.atflash_set_wait_limit_ms.restype = ctypes.c_int
    L.atflash_selftest_wait_timeout.argtypes = [ctypes.c_double, ctypes.c_void_p]
    L.atflash_selftest_wait_timeout.restype = ctypes.c_int
    for bad in (0.0, -1.0, float("nan"), 60001.0):
        assert L.atflash_set_wait_limit_ms(bad) == -1
    for bad in (0.0, -3.0, float("nan"), 10001.0):
        assert L.atflash_selftest_wait_timeout(bad, None) == -1  # rejected before any launch
    assert L.atflash_set_wait_limit_ms(2000.0) == 0


def test_varlen_argument_errors(L):
    import ctypes
    vp = ctypes.c_void_p(4096)

    def call(**kw):
        a = dict(q=vp, k=vp, v=vp, out=vp, cu=vp, B=2, maxs=100, total=150, Hq=4, Hkv=2, D=128, base=1e4,
                 kwin=8.0, outd=atf.BF16, lse=None, ws=vp, wsb=1 << 40)
        a.update(kw)
        return L.atflash_prefill_varlen(a["q"], a["k"], a["v"], a["out"], a["cu"], a["B"], a["maxs"], a["total"],
                                        a["Hq"], a["Hkv"], a["D"], a["base"], a["kwin"], a["outd"], a["lse"],
                                        a["ws"], a["wsb"], None)
    assert call(cu=None) == -1
    assert call(total=50) == -1          # shorter than max_seqlen
    assert call(B=0) == -1
    assert call(Hq=3) == -1
    assert call(D=80) == -2
    assert call(outd=7) == -2
    assert call(q=ctypes.c_void_p(4098)) == -6
    assert call(wsb=10) == -3
    assert atf.lib().atflash_prefill_varlen_workspace_bytes(4, 2, 150, 128) > 0
    assert atf.lib().atflash_prefill_varlen_workspace_bytes(4, 2, 150, 96) == 0


def test_paged_decode_argument_errors(L):
    import ctypes
    vp = ctypes.c_void_p(4096)

    def call(**kw):
        a = dict(q=vp, kp=vp, vpg=vp, bt=vp, sl=vp, out=vp, B=2, Hq=8, Hkv=2, mp=16, npool=40, page=64, D=128,
                 base=1e7, kwin=16.0, krot=0, lay=atf.KV_NHD, outd=atf.F32, ws=vp, wsb=1 << 40)
        a.update(kw)
        return L.atflash_decode_paged(a["q"], a["kp"], a["vpg"], a["bt"], a["sl"], a["out"], a["B"], a["Hq"],
                                      a["Hkv"], a["mp"], a["npool"], a["page"], a["D"], a["base"], a["kwin"],
                                      a["krot"], a["lay"], a["outd"], a["ws"], a["wsb"], None)
    assert call(bt=None) == -1
    assert call(page=48) == -1            # not a multiple of 64
    assert call(page=0) == -1
    assert call(mp=0) == -1
    assert call(npool=0) == -1
    assert call(lay=atf.KV_HND) == -1     # pages are NHD or packed
    assert call(lay=atf.KV_PACKED, krot=0) == -1
    assert call(D=96) == -2
    assert call(Hq=34, Hkv=2) == -2       # more than 16 query heads per KV head
    assert call(ws=None) == -3
    assert call(kp=ctypes.c_void_p(4100)) == -6


# ------------------------------------------------------------------ scaled RoPE tables
from scaled import llama3_scaled_theta  # noqa: E402


@pytest.mark.parametrize("D,base,k,N", [(64, 1e6, 8.0, 32768), (128, 5e5, 16.0, 131072), (128, 1e7, 64.0, 1 << 20),
                                        (64, 1e4, 1.0, 256), (128, 1e7, math.inf, 1000)])
def test_base_table_through_theta_calls_is_bit_identical(L, D, base, k, N):
    th = atf.theta_table(D, base)
    assert atf.window_table(D, base, k, N) == atf.window_table(D, 0.0, k, N, theta=th)
    assert atf.pruned_terms(N, D, base, k) == atf.pruned_terms(N, D, 0.0, k, theta=th)


@pytest.mark.parametrize("D,base,k,N", [(128, 5e5, 16.0, 131072), (128, 5e5, 2.0, 3000), (64, 1e4, 0.5, 4096)])
def test_scaled_window_table_equals_oracle(L, oracle, D, base, k, N):
    th = llama3_scaled_theta(D, base)
    with oracle.scaled_rope(th):
        lim = oracle.window_limits(D, base, k)
    ref = [int(min(x, N - 1)) for x in lim]
    assert atf.window_table(D, 0.0, k, N, theta=th) == ref


@pytest.mark.parametrize("N,D,base,k", [(700, 64, 1e4, 0.5), (300, 128, 5e5, 0.02), (2000, 128, 5e5, 1.0)])
def test_scaled_pruned_terms_equal_bruteforce(L, oracle, N, D, base, k):
    th = llama3_scaled_theta(D, base, factor=8.0, orig_ctx=512.0)
    t = atf.pruned_terms(N, D, 0.0, k, theta=th)
    with oracle.scaled_rope(th):
        kept, total = oracle.count_bruteforce(N, D, base, k)
    assert (t["kept"], t["total"]) == (kept, total)


def test_theta_tables_rejected(L):
    good = atf.theta_table(64, 1e4)
    bad = {
        "increasing": good[::-1],
        "zero": [0.0] + good[1:],
        "negative": good[:-1] + [-1e-3],
        "nan": good[:5] + [float("nan")] + good[6:],
        "above pi": [4.0] + good[1:],
    }
    for name, th in bad.items():
        with pytest.raises(atf.AtflashError):
            atf.window_table(64, 0.0, 1.0, 100, theta=th)
        arr = (ctypes.c_double * 32)(*th)
        assert L.atflash_prefill_theta(P, P, P, P, 1, 2, 1, 256, 64, arr, 1.0, atf.BF16, atf.BF16, None, P,
                                       1 << 40, None) == -1, name
        assert L.atflash_decode_theta(P, P, P, P, P, 1, 2, 1, 256, 64, arr, 1.0, 0, atf.KV_HND, atf.BF16,
                                      atf.F32, P, 1 << 40, None) == -1, name
        assert L.atflash_rope_pack_theta(P, P, 1, 256, 2, 64, arr, atf.BF16, None) == -1, name
        assert L.atflash_prefill_varlen_theta(P, P, P, P, P, 1, 256, 256, 2, 1, 64, arr, 1.0, atf.BF16, None, P,
                                              1 << 40, None) == -1, name
        assert L.atflash_decode_paged_theta(P, P, P, P, P, P, 1, 2, 1, 4, 8, 64, 64, arr, 1.0, 0, atf.KV_NHD,
                                            atf.F32, P, 1 << 40, None) == -1, name
        assert L.atflash_prefill_packed_theta(P, P, P, P, 1, 2, 1, 256, 64, arr, 1.0, atf.BF16, atf.BF16, None,
                                              None) == -1, name
        assert L.atflash_prefill_sparse_theta(P, P, P, P, P, 1, 2, 1, 256, 64, arr, 1.0, atf.BF16, None, P,
                                              1 << 40, None) == -1, name
    assert L.atflash_prefill_theta(P, P, P, P, 1, 2, 1, 256, 64, None, 1.0, atf.BF16, atf.BF16, None, P,
                                   1 << 40, None) == -1
    assert L.atflash_prefill_packed_theta(P, P, P, P, 1, 2, 1, 256, 64, None, 1.0, atf.BF16, atf.BF16, None,
                                          None) == -1
    assert L.atflash_theta_table(64, 1.0, (ctypes.c_double * 32)()) == -1
    with pytest.raises(ValueError):
        atf.window_table(64, 0.0, 1.0, 100, theta=good[:-1])


def test_noalloc_decode_rejects_what_atflash_decode_rejects(L):
    # The entry point that allocates nothing shares atflash_decode's argument
    # checks: the same bad argument gives the same status (host only, nothing runs).
    f = L.atflash_decode_noalloc
    vp, i, i64, d = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
    f.argtypes = [vp, vp, vp, vp, vp, i, i, i, i64, i, d, d, i, i, i, i, vp]
    f.restype = i
    A, U = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)  # never dereferenced
    ws = ctypes.c_void_p(1 << 24)
    good = dict(q=A, k=A, v=A, sl=A, out=A, B=2, Hq=8, Hkv=2, N=1000, D=128, base=1e4, kw=1.0, krot=0,
                lay=atf.KV_HND, ind=atf.BF16, outd=atf.F32)
    bad_cases = [dict(q=None), dict(B=0), dict(Hq=7), dict(N=0), dict(D=96), dict(D=65), dict(base=1.0),
                 dict(kw=-1.0), dict(kw=float("nan")), dict(krot=2), dict(lay=7), dict(lay=atf.KV_PACKED),
                 dict(lay=atf.KV_PACKED, krot=1, ind=atf.F32), dict(ind=5), dict(outd=5), dict(Hq=34, Hkv=2),
                 dict(q=U), dict(out=U)]
    for bad in bad_cases:
        a = dict(good, **bad)
        args = [a["q"], a["k"], a["v"], a["sl"], a["out"], a["B"], a["Hq"], a["Hkv"], a["N"], a["D"], a["base"],
                a["kw"], a["krot"], a["lay"], a["ind"], a["outd"]]
        rc_noalloc = f(*args, None)
        rc_decode = L.atflash_decode(*args, ws, 1 << 30, None)
        assert rc_noalloc < 0 and rc_noalloc == rc_decode, (bad, rc_noalloc, rc_decode)


def test_short_rows_step_argument_errors(L):
    # The short-row step on its own rejects what atflash_prefill_ex rejects for bf16 input.
    A, U = ctypes.c_void_p(1 << 20), ctypes.c_void_p((1 << 20) + 8)
    f = L.atflash_prefill_short_rows
    assert f(None, A, A, A, 1, 2, 1, 256, 64, 1e4, 1.0, atf.BF16, None, None) == -1
    assert f(A, A, A, A, 1, 3, 2, 256, 64, 1e4, 1.0, atf.BF16, None, None) == -1      # Hq % Hkv
    assert f(A, A, A, A, 1, 2, 1, 256, 64, 1.0, 1.0, atf.BF16, None, None) == -1      # base <= 1
    assert f(A, A, A, A, 1, 2, 1, 256, 64, 1e4, -1.0, atf.BF16, None, None) == -1     # k < 0
    assert f(A, A, A, A, 1, 2, 1, 256, 96, 1e4, 1.0, atf.BF16, None, None) == -2      # D
    assert f(A, A, A, A, 1, 2, 1, 256, 64, 1e4, 1.0, 7, None, None) == -2             # out dtype
    assert f(U, A, A, A, 1, 2, 1, 256, 64, 1e4, 1.0, atf.BF16, None, None) == -6      # alignment
    g = L.atflash_prefill_short_rows_theta
    assert g(A, A, A, A, 1, 2, 1, 256, 64, None, 1.0, atf.BF16, None, None) == -1     # no table


@pytest.mark.parametrize("B,Hq,Hkv,N", [
    (1, 28, 4, 8192), (1, 28, 4, 1 << 19), (4, 28, 4, 1 << 20), (16, 28, 4, 1 << 17), (1, 14, 2, 32768),
    (1, 24, 8, 131072), (3, 8, 1, 1 << 20), (1, 1, 1, 256), (1, 4, 1, 1000), (64, 32, 8, 4096)])
def test_decode_splits_fill_whole_waves(B, Hq, Hkv, N):
    # The split count behind the workspace size: splits of 256..4096 keys (so at
    # least ceil(N/4096) and at most ceil(N/256) of them), and the B*Hkv*splits
    # CTAs never pass the whole number of 148 x 3 waves that 4096-key splits need.
    D = 128
    ws = atf.decode_workspace_bytes(B, Hq, Hkv, N, D)
    per_split = B * Hq * (D + 2) * 4
    assert ws % per_split == 0
    nsplit = ws // per_split
    assert -(-N // 4096) <= nsplit <= -(-N // 256)
    slots = 148 * 3
    waves = -(-(B * Hkv * -(-N // 64)) // (slots * 64))
    assert B * Hkv * nsplit <= max(waves * slots, B * Hkv * -(-N // 4096))
