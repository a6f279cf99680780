"""Helpers of the GPU parity tests: run the CUDA path through the binding on
bf16 bit patterns and compare with the oracle."""

import numpy as np
import torch

import oracle

Y_RTOL = 1e-2   # bf16 output tolerance (relative, elementwise)


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).cuda()


def bf16_tensor_bits(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def run_quantize_weights(w_bits, n, m):
    from sparse_linear_layers_fwd_b200 import sbn
    pw = sbn.quantize_weights(to_dev_bf16(w_bits), n, m)
    torch.cuda.synchronize()
    assert sbn.get_device_error() == 0
    return pw


def packed_to_numpy(pw):
    codes = pw.codes.cpu().numpy()
    meta = pw.meta.cpu().numpy() if pw.meta is not None else np.zeros((pw.n_out, 0), np.uint8)
    gamma = np.float32(pw.gamma.cpu().numpy()[0])
    return codes, meta, gamma


def run_layer(w_bits, x_bits, n, m, want_acc=True, workspace=None):
    """All three calls; returns numpy copies of every intermediate.
    workspace=None: the contraction gets a workspace (for T > 16 the weights
    are expanded into it first); workspace=False: none (expanded in-kernel)."""
    from sparse_linear_layers_fwd_b200 import sbn
    pw = run_quantize_weights(w_bits, n, m)
    xq, s = sbn.quantize_acts(to_dev_bf16(x_bits))
    y = sbn.bitlinear(xq, s, pw, workspace=workspace)
    acc = sbn.bitlinear_acc32(xq, pw, workspace=workspace) if want_acc else None
    torch.cuda.synchronize()
    assert sbn.get_device_error() == 0
    codes, meta, gamma = packed_to_numpy(pw)
    out = dict(codes=codes, meta=meta, gamma=gamma, xq=xq.cpu().numpy(), s=s.cpu().numpy(),
               y=bf16_tensor_bits(y))
    if want_acc:
        out["acc"] = acc.cpu().numpy()
    return out


def assert_y_close(y_bits, ref_bits, rtol=Y_RTOL):
    y = oracle.bf16_bits_to_f32(y_bits).astype(np.float64)
    r = oracle.bf16_bits_to_f32(ref_bits).astype(np.float64)
    bad = np.abs(y - r) > rtol * np.abs(r)
    assert not bad.any(), f"{bad.sum()} of {bad.size} outputs off; first {np.argwhere(bad)[:3]}"


def assert_weights_exact(g, ref_codes, ref_meta, ref_gamma):
    assert g["gamma"] == ref_gamma, (g["gamma"], ref_gamma)
    assert np.array_equal(g["meta"], ref_meta), "meta differs"
    assert np.array_equal(g["codes"], ref_codes), "codes differ"


def full_parity(w_bits, x_bits, n, m, workspace=None):
    g = run_layer(w_bits, x_bits, n, m, workspace=workspace)
    cb, mb, gamma, mask, dense = oracle.quantize_weights(w_bits, n, m)
    assert_weights_exact(g, cb, mb, gamma)
    q, s = oracle.quantize_acts(x_bits)
    assert np.array_equal(g["s"], s), "activation scales differ"
    assert np.array_equal(g["xq"], q), "INT8 activations differ"
    acc = oracle.bitlinear_acc(q, dense)
    assert np.array_equal(g["acc"], acc), "int32 accumulators differ"
    y = oracle.dequant_bf16(acc, s, gamma)
    assert_y_close(g["y"], y)
    return g
