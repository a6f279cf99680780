"""Failure detection: a bounded device wait that runs out is reported, and
nothing faults or hangs.

Every pipelined kernel of the library waits on mbarriers, and the weight
quantizer on a grid barrier, each bounded in time: a wait that gives up sets
the device error word and lets its kernel return, and sbn_get_device_error
reports SBN_ERR_TIMEOUT once. sbn_selftest_wait_timeout runs one such wait on
a condition that never comes, with a 1 ms limit and nothing asynchronous in
flight.
"""

import pytest
import torch

pytestmark = pytest.mark.gpu

SBN_OK, SBN_ERR_TIMEOUT = 0, 7


@pytest.fixture(autouse=True)
def _lib(sbn_lib, cuda_ok):
    return sbn_lib


@pytest.mark.parametrize("which", [0, 1])
def test_bounded_wait_gives_up_and_is_reported(which):
    from sparse_linear_layers_fwd_b200 import sbn
    assert sbn.get_device_error() == SBN_OK           # a clean start
    sbn.selftest_wait_timeout(which, 1_000_000)        # 1 ms
    torch.cuda.synchronize()
    assert sbn.get_device_error() == SBN_ERR_TIMEOUT   # the give-up was recorded
    assert sbn.get_device_error() == SBN_OK            # and cleared by the read


def test_context_stays_usable_after_a_timeout():
    # the kernels after a give-up run and match the oracle as usual
    import numpy as np
    from gpu_util import full_parity
    from sparse_linear_layers_fwd_b200 import sbn, synth
    sbn.selftest_wait_timeout(0, 1_000_000)
    torch.cuda.synchronize()
    assert sbn.get_device_error() == SBN_ERR_TIMEOUT
    d = synth.layer_small()
    full_parity(d["w"], d["x"], d["n"], d["m"])
    assert sbn.get_device_error() == SBN_OK
