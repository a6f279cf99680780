"""N_out-sharded weight quantization on the GPU, through the C ABI.

Every split of a layer's rows into shards, quantized with the summed gamma
bins, must reproduce the unsharded sbn_quantize_weights byte for byte (codes,
meta, gamma); the bins themselves must represent the oracle's exact sum of
|w|.
"""

import numpy as np
import pytest
import torch

import oracle
from gpu_util import packed_to_numpy, run_quantize_weights, to_dev_bf16
from sparse_linear_layers_fwd_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _lib(sbn_lib, cuda_ok):
    return sbn_lib


def _exact_sum_units(bins):
    """sum_e B[e] * 2^(e - 1): the exact sum of |w| in units of 2^-133."""
    return sum(int(b) << (e - 1) for e, b in enumerate(bins) if e >= 1 and int(b))


def _layer(rows, k, seed):
    w = synth.latent_weights(rows, k, seed=seed, tag="shard_gpu")
    w[0, :6] = np.array([0x0001, 0x8003, 0x7F00, 0x4400, 0x0000, 0x8000], dtype=np.uint16)
    return w


@pytest.mark.parametrize("nm", [(6, 8), (2, 4), (8, 16), (12, 16), (4, 4), (1, 4)])
@pytest.mark.parametrize("shape,splits", [((37, 256), [1, 17, 36]), ((130, 1024), [64]),
                                          ((6912, 2560), [3456, 1000])])
def test_sharded_quantization_matches_unsharded(nm, shape, splits):
    from sparse_linear_layers_fwd_b200 import sbn
    n, m = nm
    rows, k = shape
    w = _layer(rows, k, seed=rows + 3 * n)
    ref = packed_to_numpy(run_quantize_weights(w, n, m))
    wd = to_dev_bf16(w)
    for split in splits:
        parts = [wd[:split], wd[split:]]
        bins = [sbn.gamma_bins(p) for p in parts]
        total = bins[0] + bins[1]          # the all-reduce of a two-rank group
        outs = [sbn.quantize_weights_from_bins(p, n, m, total, w.size) for p in parts]
        torch.cuda.synchronize()
        assert sbn.get_device_error() == 0
        got = [packed_to_numpy(o) for o in outs]
        assert got[0][2] == ref[2] and got[1][2] == ref[2], "gamma differs"
        assert np.array_equal(np.concatenate([got[0][0], got[1][0]]), ref[0]), "codes differ"
        if n != m:
            assert np.array_equal(np.concatenate([got[0][1], got[1][1]]), ref[1]), "meta differs"
        # the bins represent the exact sum of |w| of each shard
        for p, b in zip([w[:split], w[split:]], bins):
            assert _exact_sum_units(b.cpu().numpy().astype(np.uint64)) == \
                _exact_sum_units(oracle.gamma_bins(p))


def test_from_bins_equals_quantize_weights_on_whole_tensor():
    from sparse_linear_layers_fwd_b200 import sbn
    w = synth.decode_weights()
    ref = packed_to_numpy(run_quantize_weights(w, 6, 8))
    wd = to_dev_bf16(w)
    out = sbn.quantize_weights_from_bins(wd, 6, 8, sbn.gamma_bins(wd), w.size)
    torch.cuda.synchronize()
    got = packed_to_numpy(out)
    assert got[2] == ref[2]
    assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])
