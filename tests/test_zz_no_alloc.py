"""sbn_quantize_weights_noalloc against sbn_quantize_weights (needs a B200).

The allocation-free entry point serves callers that cannot allocate device
memory (a plugin handed only its buffers, a real-time loop that cannot take
cudaMalloc's synchronization, a process whose pool holds all device memory).
It must give exactly what the workspace entry point gives: gamma, codes and
meta bit for bit, on consecutive calls that reuse the library's one scratch
array. Runs last so a failure here leaves every other test already run.
"""

import ctypes

import numpy as np
import pytest
import torch

from sparse_linear_layers_fwd_b200 import synth

pytestmark = pytest.mark.gpu


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def _outputs(n_out, k, n, m, lib):
    cb = torch.full((lib.sbn_codes_bytes(n_out, k, n, m),), 0x5A, dtype=torch.uint8, device="cuda")
    mb_bytes = lib.sbn_meta_bytes(n_out, k, n, m)
    mb = torch.full((max(mb_bytes, 16),), 0x5A, dtype=torch.uint8, device="cuda")
    g = torch.full((1,), -1.0, dtype=torch.float32, device="cuda")
    return cb, mb, g


def _call_noalloc(lib, w, n_out, k, n, m, cb, mb, g, stream):
    return lib.sbn_quantize_weights_noalloc(w.data_ptr(), n_out, k, n, m, cb.data_ptr(),
                                            mb.data_ptr() if n != m else None, g.data_ptr(),
                                            stream)


def _call_workspace(lib, w, n_out, k, n, m, cb, mb, g, stream):
    ws_bytes = lib.sbn_quantize_weights_workspace_bytes(n_out, k)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    return lib.sbn_quantize_weights(w.data_ptr(), n_out, k, n, m, cb.data_ptr(),
                                    mb.data_ptr() if n != m else None, g.data_ptr(),
                                    ws.data_ptr(), ws_bytes, stream)


@pytest.mark.parametrize("shape_nm", [((6912, 2560), (6, 8)), ((256, 256), (2, 4)),
                                      ((130, 1024), (8, 16)), ((64, 384), (8, 8))])
def test_noalloc_matches_workspace_entry_point_twice(sbn_lib, cuda_ok, shape_nm):
    lib = sbn_lib
    (n_out, k), (n, m) = shape_nm
    stream = torch.cuda.current_stream().cuda_stream
    # two different weight tensors, one after the other: the second call must
    # not see anything the first left in the shared scratch
    for tag in ["first", "second"]:
        w = _dev_bf16(synth.latent_weights(n_out, k, seed=3, tag=f"noalloc_{tag}"))
        a = _outputs(n_out, k, n, m, lib)
        b = _outputs(n_out, k, n, m, lib)
        assert _call_noalloc(lib, w, n_out, k, n, m, *a, stream) == 0
        assert _call_workspace(lib, w, n_out, k, n, m, *b, stream) == 0
        torch.cuda.synchronize()
        assert lib.sbn_get_device_error(stream) == 0
        assert torch.equal(a[2], b[2]), "gamma differs"
        assert torch.equal(a[0], b[0]), "codes differ"
        if n != m:
            assert torch.equal(a[1], b[1]), "meta differs"


def test_noalloc_rejects_before_enqueueing(sbn_lib, cuda_ok):
    lib = sbn_lib
    stream = torch.cuda.current_stream().cuda_stream
    cb, mb, g = _outputs(64, 256, 2, 4, lib)
    w = _dev_bf16(synth.latent_weights(64, 256, seed=4))
    # N_out * K at or above 2^31 is outside the supported sizes
    assert lib.sbn_quantize_weights_noalloc(w.data_ptr(), 1 << 20, 1 << 11, 2, 4, cb.data_ptr(),
                                            mb.data_ptr(), g.data_ptr(), stream) == 2
    assert lib.sbn_quantize_weights_noalloc(None, 64, 256, 2, 4, cb.data_ptr(), mb.data_ptr(),
                                            g.data_ptr(), stream) == 1
    assert lib.sbn_quantize_weights_noalloc(w.data_ptr(), 64, 256, 3, 8, cb.data_ptr(),
                                            mb.data_ptr(), g.data_ptr(), stream) == 3
    torch.cuda.synchronize()
    assert float(g.item()) == -1.0           # nothing was written
