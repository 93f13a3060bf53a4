"""Failure detection of the bounded device-side waits, without a GPU fault.

The chunked forward bounds every mbarrier wait in time; a wait that runs out
stops its CTA cleanly (it lets its copies and products in flight land before it
frees tensor memory) and is counted for m3ssd_device_wait_timeouts.  Here one
completion signal is left out on purpose (a testing hook of the library) under a
20 ms limit: the launch must report the timeout, and the next launch in the same
context must be clean and correct."""
import pytest

import oracle
import selective_state_space_m3ssd_b200 as m3
from selective_state_space_m3ssd_b200.synth import WORKLOADS, make_inputs
from tests.gpu_util import gpu_fwd, rel_max_err, rel_max_err_out

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("L", [40, 130])  # one chunk; several chunks
def test_a_wait_that_runs_out_is_reported_and_the_next_call_is_clean(L):
    inp = make_inputs(WORKLOADS["siso"].with_(batch=1, nheads=2, seqlen=L, seed=8))
    m3.device_wait_timeouts()  # clear the count
    m3.set_wait_limit_for_tests(20_000_000)
    try:
        m3.drop_next_gram_signal_for_tests()
        gpu_fwd(inp)  # outputs undefined
        assert m3.device_wait_timeouts() >= 1
    finally:
        m3.set_wait_limit_for_tests(0)
    ref = oracle.oracle_fwd(**inp)
    got = gpu_fwd(inp)
    assert m3.device_wait_timeouts() == 0
    assert rel_max_err_out(got["Y"], ref["Y"], True) <= 2e-2
    assert rel_max_err(got["hT"], ref["hT"]) <= 2e-2
