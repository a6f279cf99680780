"""Canary bytes around every output and workspace (needs a B200).

Each buffer a call writes is the middle of a larger allocation whose edges
hold a known byte pattern; after the call the edges must be unchanged. This
catches writes past the end (or before the start) of an output on ragged
shapes, on every route: the decode GEMV, the tensor-core contraction with and
without a workspace, the 2:4 sparse route, the dense pair tiles of both
widths, the weight quantizer, activation quantization, the entropy packer
and decode, the mask flip count and the backward. Values are checked by the
parity tests; here only the edges.
"""

import numpy as np
import pytest
import torch

from gpu_util import to_dev_bf16
from sparse_linear_layers_fwd_b200 import sbn, synth

pytestmark = pytest.mark.gpu

GUARD = 256          # bytes of canary on each side (keeps every view 16-byte aligned)
CANARY = 0xA5


@pytest.fixture(autouse=True)
def _lib(sbn_lib, cuda_ok):
    return sbn_lib


class Guarded:
    """Views into canary-filled allocations; check() verifies the edges."""

    def __init__(self):
        self.bufs = []

    def tensor(self, shape, dtype):
        nbytes = int(np.prod(shape)) * torch.tensor([], dtype=dtype).element_size()
        buf = torch.full((GUARD + nbytes + GUARD,), CANARY, dtype=torch.uint8, device="cuda")
        self.bufs.append((buf, nbytes))
        return buf[GUARD:GUARD + nbytes].view(dtype).view(shape)

    def packed(self, n_out, k, n, m):
        cr, mr = sbn.codes_row_bytes(k, n, m), sbn.meta_row_bytes(k, n, m)
        codes = self.tensor((n_out, cr), torch.uint8)
        meta = self.tensor((n_out, mr), torch.uint8) if mr else None
        gamma = self.tensor((1,), torch.float32)
        return sbn.PackedWeights(codes, meta, gamma, n_out, k, n, m)

    def check(self):
        torch.cuda.synchronize()
        assert sbn.get_device_error() == 0
        for i, (buf, nbytes) in enumerate(self.bufs):
            b = buf.cpu().numpy()
            assert (b[:GUARD] == CANARY).all(), f"buffer {i}: bytes written before its start"
            assert (b[GUARD + nbytes:] == CANARY).all(), f"buffer {i}: bytes written past its end"


# (T, K, N_out, n, m): decode GEMV (T <= 16), dense pair tiles narrow and
# wide, 2:4 sparse, a dense pattern without keep bits; ragged on every axis
CASES = [
    (5, 384, 257, 6, 8),
    (16, 1024, 130, 8, 16),
    (100, 512, 257, 6, 8),
    (300, 640, 520, 4, 8),
    (1000, 384, 4000, 6, 8),
    (225, 384, 129, 2, 4),
    (33, 256, 64, 8, 8),
]


@pytest.mark.parametrize("case", CASES, ids=[f"t{c[0]}_k{c[1]}_n{c[2]}_{c[3]}of{c[4]}" for c in CASES])
def test_forward_outputs_and_workspaces(case):
    t, k, n_out, n, m = case
    g = Guarded()
    w = to_dev_bf16(synth.latent_weights(n_out, k, seed=31, tag=f"can{case}"))
    x = to_dev_bf16(synth.activations(t, k, seed=31, tag=f"can{case}", outlier_channels=1))
    pw = g.packed(n_out, k, n, m)
    sbn.quantize_weights(w, n, m, out=pw, workspace=g.tensor((sbn.workspace_bytes(n_out, k),), torch.uint8))
    xq, s = g.tensor((t, k), torch.int8), g.tensor((t,), torch.float32)
    sbn.quantize_acts(x, out_q=xq, out_s=s)
    wsb = sbn.bitlinear_workspace_bytes(t, k, n_out)
    ws = g.tensor((wsb,), torch.uint8) if wsb else None
    sbn.bitlinear(xq, s, pw, out=g.tensor((t, n_out), torch.bfloat16), workspace=ws if ws is not None else False)
    sbn.bitlinear(xq, s, pw, out=g.tensor((t, n_out), torch.bfloat16), workspace=False)
    sbn.bitlinear_acc32(xq, pw, out=g.tensor((t, n_out), torch.int32), workspace=ws if ws is not None else False)
    xw = g.tensor((sbn.bitlinear_x_workspace_bytes(t, k, n_out),), torch.uint8)
    sbn.bitlinear_x(x, pw, out=g.tensor((t, n_out), torch.bfloat16), out_q=g.tensor((t, k), torch.int8),
                    out_s=g.tensor((t,), torch.float32), workspace=xw)
    g.check()


# the entropy decode takes m = 4 and m = 8 patterns below n = m; the packer
# and the flip count take every pattern
ENT_DECODABLE = {(1, 4), (2, 4), (3, 4), (2, 8), (4, 8), (6, 8)}


@pytest.mark.parametrize("case", [(5, 384, 257, 6, 8), (16, 1024, 130, 2, 4), (9, 512, 33, 4, 8)])
def test_entropy_and_flips(case):
    t, k, n_out, n, m = case
    g = Guarded()
    w = to_dev_bf16(synth.latent_weights(n_out, k, seed=32, tag=f"cane{case}"))
    x = to_dev_bf16(synth.activations(t, k, seed=32, tag=f"cane{case}"))
    pa = sbn.quantize_weights(w, n, m)
    pb = sbn.quantize_weights((w.float() * 1.01).to(torch.bfloat16), n, m)
    ent = g.tensor((n_out, sbn.entropy_row_bytes(k, n, m)), torch.uint8)
    sbn.pack_entropy(pa, out=ent)
    if (n, m) in ENT_DECODABLE:
        sbn.bitlinear_entropy_x(x, ent, pa, out=g.tensor((t, n_out), torch.bfloat16))
    sbn.mask_flips(pa, pb, out=g.tensor((1,), torch.int64))
    g.check()


@pytest.mark.parametrize("shape", [(100, 384, 257), (64, 256, 136), (40, 1024, 130)])
def test_backward_outputs(shape):
    t, k, n_out = shape
    g = Guarded()
    w = to_dev_bf16(synth.latent_weights(n_out, k, seed=33, tag=f"canb{shape}"))
    x = to_dev_bf16(synth.activations(t, k, seed=33, tag=f"canb{shape}"))
    dy = to_dev_bf16(synth.activations(t, n_out, seed=34, tag=f"canb{shape}"))
    pw = sbn.quantize_weights(w, 2, 4)
    xq, s = sbn.quantize_acts(x)
    sbn.bitlinear_grad_x(dy, pw, out=g.tensor((t, k), torch.bfloat16))
    sbn.bitlinear_grad_w(dy, xq, s, out=g.tensor((n_out, k), torch.bfloat16))
    g.check()
