"""(Runs last: it is the one test that drives a device error path.)

Failure detection without a GPU fault: a bounded device-side wait that
runs out is reported to the host, and the context stays usable.

la_selftest_wait_timeout enqueues one kernel whose mbarrier wait has nothing
to wait for; the wait gives up after its bound (about a second), records the
timeout in the device error word and returns.  The bound is a deadline
of 1 s on the device's global timer.  No copy or MMA is in flight,
nothing traps, nothing hangs.
"""
import time

import pytest

from causal_kernelized_linear_la_b200 import inputs
from tests import helpers as H

pytestmark = pytest.mark.gpu


def test_bounded_wait_runs_out_and_is_reported():
    import torch
    import causal_kernelized_linear_la_b200 as la
    la.la_prefill_check()   # nothing pending from earlier work
    stream = torch.cuda.current_stream()
    try:
        t0 = time.perf_counter()
        la.la_selftest_wait_timeout()
        with pytest.raises(la.LaError) as ei:
            la.la_prefill_check()
        assert ei.value.code == la.LA_ERR_TIMEOUT
        elapsed = time.perf_counter() - t0
        # the wait gives up at a 1 s deadline of the device's global timer,
        # not after a count of suspended tries whose length is only a hint
        assert 0.5 <= elapsed < 5.0, f"wait gave up after {elapsed:.3f} s"
        la.la_prefill_check()   # reading the error cleared it
    finally:
        # never leave the error word set for later tests
        la.lib().la_prefill_check(None, la._stream_handle(stream))
    # the context is still usable: a prefill afterwards matches the oracle
    p = inputs.make_kernelized(1, 2, 150, 64, 64, dtype="bf16", mode="plain", seed=17)
    H.assert_close(p, H.run_library(p), H.run_oracle(p), [(0, 0), (0, 1)])
