"""Failure detection without a GPU fault: the tensor-core kernel's bounded waits and
its range check report through the device status word, and the context stays usable."""
import numpy as np
import pytest

from recurrent_state_memory_b200 import inputs as I

import parity_util as U

pytestmark = pytest.mark.gpu


@pytest.fixture()
def G():
    from recurrent_state_memory_b200 import gdr
    gdr.lib()
    yield gdr
    gdr.debug_set_tc_fault(False, 0)


@pytest.mark.parametrize("algo", ["tcgen05", "tcgen05_split", "tcgen05_chains"])
def test_bounded_wait_gives_up_and_reports(G, algo):
    """A barrier that nothing signals: the wait runs out after 5 ms, the kernel frees
    its tensor memory and returns, the status word says GDR_ERR_TIMEOUT; the next
    normal call on the same context is correct."""
    import torch
    p = I.make_fwd(1, 128, 2, 128, 128, dtype="bf16", seed=7, s0_std=0.2)
    G.debug_set_tc_fault(True, 5_000_000)
    U.run_gpu_fwd(p, algo)
    assert G.query_device_status() == G.GDR_ERR_TIMEOUT
    assert G.query_device_status() == G.GDR_OK            # read-and-clear
    G.debug_set_tc_fault(False, 0)
    o, S = U.run_gpu_fwd(p, algo)
    assert G.query_device_status() == G.GDR_OK
    o_ref, S_ref = U.oracle_fwd(p)
    U.assert_fwd_parity(p, o, S, o_ref, S_ref)


def test_decay_outside_factored_range_is_reported(G):
    """A gate so strong that exp(a) overflows fp32 leaves the factored range of the
    tensor-core kernel: the call reports GDR_ERR_RANGE instead of returning silently."""
    p = I.make_fwd(1, 64, 1, 128, 128, dtype="bf16", seed=8)
    p.g[:, 40] = 200.0
    U.run_gpu_fwd(p, "tcgen05")
    assert G.query_device_status() == G.GDR_ERR_RANGE
    assert G.query_device_status() == G.GDR_OK
