"""Failure detection on the GPU without a fault, hang or trap.

Every wait between the warps of a CTA is bounded.  These tests make such
waits run out on purpose and check that the kernels report
ATFLASH_ERR_TIMEOUT through the device status word, exit, and leave the
context usable: the next call with the normal limit is bit-identical to a
call made before the failure.  The prefill is the real kernel used: its warps
wait on one another for several microseconds per key tile, so a 1 us limit
trips reliably.  A decode CTA's waits (one TMA stage) can end inside the
hardware's own try-wait suspension, so the decode is covered by the same
bounded-wait code through the self-test rather than by a timing-dependent run.
"""
import pytest

import parity as P

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

import long_context_attention_pair_b200 as atf  # noqa: E402

TIMEOUT = -5  # ATFLASH_ERR_TIMEOUT


def test_selftest_wait_runs_out_and_is_reported():
    assert atf.device_status(True) == 0
    atf.selftest_wait_timeout(20.0)
    assert atf.device_status(True) == TIMEOUT
    assert atf.device_status(True) == 0  # cleared


def test_short_wait_limit_times_out_prefill_then_recovers():
    q, k, v = P.gen(51, "q", (1, 4096, 4, 128), "bf16"), P.gen(51, "k", (1, 4096, 2, 128), "bf16"), \
        P.gen(51, "v", (1, 4096, 2, 128), "bf16")
    ref = atf.prefill(q, k, v, 5e5, 16.0)
    torch.cuda.synchronize()
    assert atf.device_status(True) == 0
    try:
        atf.set_wait_limit_ms(0.001)  # 1 us: the first TMA wait of every CTA runs out
        atf.prefill(q, k, v, 5e5, 16.0)
        assert atf.device_status(True) == TIMEOUT
    finally:
        atf.set_wait_limit_ms(2000.0)
    again = atf.prefill(q, k, v, 5e5, 16.0)
    torch.cuda.synchronize()
    assert atf.device_status(True) == 0
    assert torch.equal(again, ref)
