"""The tensor-pipe probes behind the prefill roofline (needs a B200).

The sparse MMA of the 2:4 contraction multiplies only the kept half of each
group of four, so on the same tile it retires logical positions at about
twice the rate of the dense MMA; both probes run clean (no device error).
"""

import pytest
import torch

from sparse_linear_layers_fwd_b200 import sbn

pytestmark = pytest.mark.gpu


def _timed(fn):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    fn()                                 # warm-up
    torch.cuda.synchronize()
    e0.record()
    n = fn()
    e1.record()
    torch.cuda.synchronize()
    return n, e0.elapsed_time(e1) * 1e-3


def test_sparse_probe_doubles_the_logical_rate(sbn_lib, cuda_ok):
    iters = 20000
    ctas, t_dense = _timed(lambda: sbn.probe_i8_mma(iters))
    pairs, t_sparse = _timed(lambda: sbn.probe_i8_sparse_mma(iters))
    assert sbn.get_device_error() == 0
    assert ctas > 0 and pairs > 0
    dense = ctas * iters * 2 * 128 * 256 * 32 / t_dense
    sparse_logical = pairs * iters * 2 * 256 * 224 * 64 / t_sparse
    assert sparse_logical > 1.5 * dense, (sparse_logical / 1e12, dense / 1e12)
