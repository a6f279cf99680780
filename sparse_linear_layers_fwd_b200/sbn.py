"""ctypes binding of libsbn (include/sbn.h): argument marshalling only.

Every step of the BitLinear forward runs in libsbn's CUDA kernels; PyTorch
only supplies device memory and the current stream. There is no CPU
fallback: if ``libsbn.so`` is missing, loading it raises.

    packed = quantize_weights(w_bf16, n=6, m=8)       # dynamic N:M mask + ternary + pack
    xq, s = quantize_acts(x_bf16)                      # per-token absmax INT8
    y = bitlinear(xq, s, packed)                       # INT8 x ternary -> bf16
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsbn.so")

SBN_STATUS = {
    0: "SBN_OK", 1: "SBN_ERR_NULL", 2: "SBN_ERR_SHAPE", 3: "SBN_ERR_PATTERN",
    4: "SBN_ERR_ALIGN", 5: "SBN_ERR_WORKSPACE", 6: "SBN_ERR_CUDA",
    7: "SBN_ERR_TIMEOUT", 8: "SBN_ERR_DEVICE",
}

_c_i32, _c_sz, _c_p = ctypes.c_int32, ctypes.c_size_t, ctypes.c_void_p

# name -> (restype, argtypes), mirroring include/sbn.h
PROTOTYPES = {
    "sbn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "sbn_version": (ctypes.c_int, []),
    "sbn_codes_row_bytes": (_c_sz, [_c_i32, _c_i32, _c_i32]),
    "sbn_codes_bytes": (_c_sz, [_c_i32, _c_i32, _c_i32, _c_i32]),
    "sbn_meta_row_bytes": (_c_sz, [_c_i32, _c_i32, _c_i32]),
    "sbn_meta_bytes": (_c_sz, [_c_i32, _c_i32, _c_i32, _c_i32]),
    "sbn_quantize_weights_workspace_bytes": (_c_sz, [_c_i32, _c_i32]),
    "sbn_quantize_weights": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_p, _c_p,
                                            _c_p, _c_p, _c_sz, _c_p]),
    "sbn_quantize_weights_noalloc": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_p,
                                                    _c_p, _c_p, _c_p]),
    "sbn_gamma_bins": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_p, _c_p]),
    "sbn_quantize_weights_from_bins": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_p,
                                                      ctypes.c_int64, _c_p, _c_p, _c_p, _c_p]),
    "sbn_quantize_acts": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_p, _c_p, _c_p]),
    "sbn_bitlinear": (ctypes.c_int, [_c_p, _c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_p,
                                     _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "sbn_bitlinear_workspace_bytes": (_c_sz, [_c_i32, _c_i32, _c_i32]),
    "sbn_bitlinear_acc32": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_p,
                                           _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "sbn_bitlinear_x": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_p, _c_p,
                                       _c_p, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "sbn_bitlinear_x_workspace_bytes": (_c_sz, [_c_i32, _c_i32, _c_i32]),
    "sbn_mask_flips": (ctypes.c_int, [_c_p, _c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_p, _c_p]),
    "sbn_entropy_row_bytes": (_c_sz, [_c_i32, _c_i32, _c_i32]),
    "sbn_entropy_bytes": (_c_sz, [_c_i32, _c_i32, _c_i32, _c_i32]),
    "sbn_pack_entropy": (ctypes.c_int, [_c_p, _c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_p, _c_p]),
    "sbn_bitlinear_entropy": (ctypes.c_int, [_c_p, _c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32,
                                             _c_p, _c_p, _c_p, _c_p]),
    "sbn_bitlinear_entropy_acc32": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32,
                                                   _c_p, _c_p, _c_p]),
    "sbn_bitlinear_entropy_x": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_p,
                                               _c_p, _c_p, _c_p, _c_p, _c_p, _c_sz, _c_p]),
    "sbn_bitlinear_entropy_x_workspace_bytes": (_c_sz, [_c_i32, _c_i32]),
    "sbn_bitlinear_grad_x": (ctypes.c_int, [_c_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _c_p, _c_p, _c_p,
                                            _c_p, _c_p]),
    "sbn_bitlinear_grad_w": (ctypes.c_int, [_c_p, _c_p, _c_p, _c_i32, _c_i32, _c_i32, _c_p, _c_p]),
    "sbn_probe_i8_mma": (ctypes.c_int, [_c_i32, ctypes.POINTER(ctypes.c_int32), _c_p]),
    "sbn_probe_i8_sparse_mma": (ctypes.c_int, [_c_i32, ctypes.POINTER(ctypes.c_int32), _c_p]),
    "sbn_selftest_wait_timeout": (ctypes.c_int, [_c_i32, ctypes.c_int64, _c_p]),
    "sbn_set_programmatic_launch": (_c_i32, [_c_i32]),
    "sbn_get_device_error": (ctypes.c_int, [_c_p]),
}

_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """Load libsbn.so (once). Raises ImportError if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m sparse_linear_layers_fwd_b200.build` (needs nvcc)")
        cdll = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in PROTOTYPES.items():
            fn = getattr(cdll, name)
            fn.restype = res
            fn.argtypes = args
        _lib = cdll
    return _lib


class SbnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().sbn_status_string(status).decode()
        super().__init__(f"{where}: {msg}")


def _check(status: int, where: str):
    if status != 0:
        raise SbnError(status, where)


def _stream_ptr(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _need(t: torch.Tensor, dtype, what: str):
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")


@dataclass
class Pattern:
    n: int
    m: int


@dataclass
class PackedWeights:
    """Packed ternary weights in the canonical format of include/sbn.h."""
    codes: torch.Tensor            # uint8 [n_out, codes_row_bytes]
    meta: Optional[torch.Tensor]   # uint8 [n_out, meta_row_bytes] or None (n == m)
    gamma: torch.Tensor            # float32 [1]
    n_out: int
    k: int
    n: int
    m: int


def codes_row_bytes(k: int, n: int, m: int) -> int:
    return int(lib().sbn_codes_row_bytes(k, n, m))


def meta_row_bytes(k: int, n: int, m: int) -> int:
    return int(lib().sbn_meta_row_bytes(k, n, m))


def workspace_bytes(n_out: int, k: int) -> int:
    return int(lib().sbn_quantize_weights_workspace_bytes(n_out, k))


def alloc_packed(n_out: int, k: int, n: int, m: int, device) -> PackedWeights:
    cr, mr = codes_row_bytes(k, n, m), meta_row_bytes(k, n, m)
    if cr == 0:
        raise SbnError(3, "alloc_packed")
    codes = torch.empty((n_out, cr), dtype=torch.uint8, device=device)
    meta = torch.empty((n_out, mr), dtype=torch.uint8, device=device) if mr else None
    gamma = torch.empty((1,), dtype=torch.float32, device=device)
    return PackedWeights(codes, meta, gamma, n_out, k, n, m)


def quantize_weights(w: torch.Tensor, n: int, m: int, out: Optional[PackedWeights] = None,
                     workspace: Optional[torch.Tensor] = None, stream=None) -> PackedWeights:
    """sbn_quantize_weights: N:M magnitude mask, absmean ternary codes, packing."""
    _need(w, torch.bfloat16, "w")
    n_out, k = w.shape
    if out is None:
        out = alloc_packed(n_out, k, n, m, w.device)
    if workspace is None:
        workspace = torch.empty(workspace_bytes(n_out, k), dtype=torch.uint8, device=w.device)
    st = lib().sbn_quantize_weights(_ptr(w), n_out, k, n, m, _ptr(out.codes), _ptr(out.meta),
                                    _ptr(out.gamma), _ptr(workspace), workspace.numel(),
                                    _stream_ptr(stream))
    _check(st, "sbn_quantize_weights")
    return out


def quantize_weights_noalloc(w: torch.Tensor, n: int, m: int, out: PackedWeights,
                             stream=None) -> PackedWeights:
    """sbn_quantize_weights_noalloc: like quantize_weights, with the library's
    fixed internal scratch instead of a caller workspace (no allocation)."""
    _need(w, torch.bfloat16, "w")
    n_out, k = w.shape
    st = lib().sbn_quantize_weights_noalloc(_ptr(w), n_out, k, n, m, _ptr(out.codes),
                                            _ptr(out.meta), _ptr(out.gamma), _stream_ptr(stream))
    _check(st, "sbn_quantize_weights_noalloc")
    return out


GAMMA_BINS = 256   # SBN_GAMMA_BINS


def gamma_bins(w: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """sbn_gamma_bins: the exact gamma bins of one shard of rows, as int64 [256]
    (the bit patterns of the library's uint64 bins; every value stays below
    2^63). Bins of several shards add up to the bins of their union, so a
    column-parallel layer sums them with an all-reduce before quantizing."""
    _need(w, torch.bfloat16, "w")
    n_out, k = w.shape
    if out is None:
        out = torch.empty((GAMMA_BINS,), dtype=torch.int64, device=w.device)
    _need(out, torch.int64, "bins")
    st = lib().sbn_gamma_bins(_ptr(w), n_out, k, _ptr(out), _stream_ptr(stream))
    _check(st, "sbn_gamma_bins")
    return out


def quantize_weights_from_bins(w: torch.Tensor, n: int, m: int, bins: torch.Tensor, total_elems: int,
                               out: Optional[PackedWeights] = None, stream=None) -> PackedWeights:
    """sbn_quantize_weights_from_bins: mask, codes and packing of one shard of
    rows with the gamma of the whole tensor (bins summed over all shards,
    total_elems the element count of the whole tensor)."""
    _need(w, torch.bfloat16, "w")
    _need(bins, torch.int64, "bins")
    n_out, k = w.shape
    if out is None:
        out = alloc_packed(n_out, k, n, m, w.device)
    st = lib().sbn_quantize_weights_from_bins(_ptr(w), n_out, k, n, m, _ptr(bins), int(total_elems),
                                              _ptr(out.codes), _ptr(out.meta), _ptr(out.gamma),
                                              _stream_ptr(stream))
    _check(st, "sbn_quantize_weights_from_bins")
    return out


def quantize_acts(x: torch.Tensor, out_q: Optional[torch.Tensor] = None,
                  out_s: Optional[torch.Tensor] = None, stream=None):
    """sbn_quantize_acts: per-token absmax INT8. Returns (xq int8 [T,K], s fp32 [T])."""
    _need(x, torch.bfloat16, "x")
    t, k = x.shape
    if out_q is None:
        out_q = torch.empty((t, k), dtype=torch.int8, device=x.device)
    if out_s is None:
        out_s = torch.empty((t,), dtype=torch.float32, device=x.device)
    st = lib().sbn_quantize_acts(_ptr(x), t, k, _ptr(out_q), _ptr(out_s), _stream_ptr(stream))
    _check(st, "sbn_quantize_acts")
    return out_q, out_s


def bitlinear_workspace_bytes(t: int, k: int, n_out: int) -> int:
    """Bytes of the contraction's optional workspace (0 when T <= 16)."""
    return int(lib().sbn_bitlinear_workspace_bytes(t, k, n_out))


def _bitlinear_ws(workspace, t: int, k: int, n_out: int, device):
    """None: allocate the workspace (expanded-weights route); False: no
    workspace (weights expanded inside the kernel); else the given tensor."""
    if workspace is False:
        return None
    if workspace is None:
        nb = bitlinear_workspace_bytes(t, k, n_out)
        return torch.empty((nb,), dtype=torch.uint8, device=device) if nb else None
    return workspace


def bitlinear(xq: torch.Tensor, s: torch.Tensor, w: PackedWeights,
              out: Optional[torch.Tensor] = None, workspace=None, stream=None) -> torch.Tensor:
    """sbn_bitlinear: y[t, o] = bf16(acc * gamma * s_t / 127)."""
    _need(xq, torch.int8, "xq")
    _need(s, torch.float32, "s")
    t, k = xq.shape
    if k != w.k:
        raise ValueError("K mismatch between activations and weights")
    if out is None:
        out = torch.empty((t, w.n_out), dtype=torch.bfloat16, device=xq.device)
    ws = _bitlinear_ws(workspace, t, k, w.n_out, xq.device)
    st = lib().sbn_bitlinear(_ptr(xq), _ptr(s), t, k, w.n_out, w.n, w.m, _ptr(w.codes),
                             _ptr(w.meta), _ptr(w.gamma), _ptr(out), _ptr(ws),
                             0 if ws is None else ws.numel(), _stream_ptr(stream))
    _check(st, "sbn_bitlinear")
    return out


def bitlinear_acc32(xq: torch.Tensor, w: PackedWeights, out: Optional[torch.Tensor] = None,
                    workspace=None, stream=None) -> torch.Tensor:
    """sbn_bitlinear_acc32: the exact int32 accumulators [T, N_out]."""
    _need(xq, torch.int8, "xq")
    t, k = xq.shape
    if out is None:
        out = torch.empty((t, w.n_out), dtype=torch.int32, device=xq.device)
    ws = _bitlinear_ws(workspace, t, k, w.n_out, xq.device)
    st = lib().sbn_bitlinear_acc32(_ptr(xq), t, k, w.n_out, w.n, w.m, _ptr(w.codes),
                                   _ptr(w.meta), _ptr(out), _ptr(ws),
                                   0 if ws is None else ws.numel(), _stream_ptr(stream))
    _check(st, "sbn_bitlinear_acc32")
    return out


def bitlinear_x_workspace_bytes(t: int, k: int, n_out: int) -> int:
    return int(lib().sbn_bitlinear_x_workspace_bytes(t, k, n_out))


def bitlinear_x(x: torch.Tensor, w: PackedWeights, out: Optional[torch.Tensor] = None,
                out_q: Optional[torch.Tensor] = None, out_s: Optional[torch.Tensor] = None,
                workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """sbn_bitlinear_x: y = bitlinear(quantize_acts(x)) in one call (one kernel
    for T <= 16). out_q / out_s, if given, receive Xq and s."""
    _need(x, torch.bfloat16, "x")
    t, k = x.shape
    if k != w.k:
        raise ValueError("K mismatch between activations and weights")
    if out is None:
        out = torch.empty((t, w.n_out), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty((bitlinear_x_workspace_bytes(t, k, w.n_out),), dtype=torch.uint8,
                                device=x.device)
    st = lib().sbn_bitlinear_x(_ptr(x), t, k, w.n_out, w.n, w.m, _ptr(w.codes), _ptr(w.meta),
                               _ptr(w.gamma), _ptr(out), _ptr(out_q), _ptr(out_s), _ptr(workspace),
                               workspace.numel(), _stream_ptr(stream))
    _check(st, "sbn_bitlinear_x")
    return out


def mask_flips(a: PackedWeights, b: PackedWeights, out: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
    """sbn_mask_flips: positions whose keep bit differs between two packed
    versions of one layer (device int64 scalar); flip rate = count / (N_out*K)."""
    if (a.n_out, a.k, a.n, a.m) != (b.n_out, b.k, b.n, b.m):
        raise ValueError("the two packed weights describe different layers")
    if out is None:
        out = torch.empty((1,), dtype=torch.int64, device=a.codes.device)
    st = lib().sbn_mask_flips(_ptr(a.meta), _ptr(b.meta), a.n_out, a.k, a.n, a.m, _ptr(out),
                              _stream_ptr(stream))
    _check(st, "sbn_mask_flips")
    return out


def entropy_row_bytes(k: int, n: int, m: int) -> int:
    return int(lib().sbn_entropy_row_bytes(k, n, m))


def pack_entropy(w: PackedWeights, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """sbn_pack_entropy: the entropy-tight format [N_out, entropy_row_bytes] (uint8)."""
    if out is None:
        out = torch.empty((w.n_out, entropy_row_bytes(w.k, w.n, w.m)), dtype=torch.uint8,
                          device=w.codes.device)
    st = lib().sbn_pack_entropy(_ptr(w.codes), _ptr(w.meta), w.n_out, w.k, w.n, w.m, _ptr(out),
                                _stream_ptr(stream))
    _check(st, "sbn_pack_entropy")
    return out


def bitlinear_entropy(xq: torch.Tensor, s: torch.Tensor, ent: torch.Tensor, w: PackedWeights,
                      out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """sbn_bitlinear_entropy: decode contraction over entropy-tight weights
    (shape, pattern and gamma from the PackedWeights they were packed from)."""
    _need(xq, torch.int8, "xq")
    _need(s, torch.float32, "s")
    t, k = xq.shape
    if out is None:
        out = torch.empty((t, w.n_out), dtype=torch.bfloat16, device=xq.device)
    st = lib().sbn_bitlinear_entropy(_ptr(xq), _ptr(s), t, k, w.n_out, w.n, w.m, _ptr(ent),
                                     _ptr(w.gamma), _ptr(out), _stream_ptr(stream))
    _check(st, "sbn_bitlinear_entropy")
    return out


def bitlinear_entropy_acc32(xq: torch.Tensor, ent: torch.Tensor, w: PackedWeights,
                            out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    _need(xq, torch.int8, "xq")
    t, k = xq.shape
    if out is None:
        out = torch.empty((t, w.n_out), dtype=torch.int32, device=xq.device)
    st = lib().sbn_bitlinear_entropy_acc32(_ptr(xq), t, k, w.n_out, w.n, w.m, _ptr(ent), _ptr(out),
                                           _stream_ptr(stream))
    _check(st, "sbn_bitlinear_entropy_acc32")
    return out


def bitlinear_entropy_x(x: torch.Tensor, ent: torch.Tensor, w: PackedWeights,
                        out: Optional[torch.Tensor] = None, out_q: Optional[torch.Tensor] = None,
                        out_s: Optional[torch.Tensor] = None, workspace=None, stream=None) -> torch.Tensor:
    """sbn_bitlinear_entropy_x: y = bitlinear_entropy(quantize_acts(x)) in one
    call (one kernel when the bf16 rows fit in shared memory). out_q / out_s,
    if given, receive Xq and s. workspace: None allocates the two-step route's
    scratch, False passes none."""
    _need(x, torch.bfloat16, "x")
    t, k = x.shape
    if k != w.k:
        raise ValueError("K mismatch between activations and weights")
    if out is None:
        out = torch.empty((t, w.n_out), dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty((int(lib().sbn_bitlinear_entropy_x_workspace_bytes(t, k)),),
                                dtype=torch.uint8, device=x.device)
    ws_ptr, ws_n = (None, 0) if workspace is False else (_ptr(workspace), workspace.numel())
    st = lib().sbn_bitlinear_entropy_x(_ptr(x), t, k, w.n_out, w.n, w.m, _ptr(ent), _ptr(w.gamma),
                                       _ptr(out), _ptr(out_q), _ptr(out_s), ws_ptr, ws_n,
                                       _stream_ptr(stream))
    _check(st, "sbn_bitlinear_entropy_x")
    return out


def bitlinear_grad_x(dy: torch.Tensor, w: PackedWeights, out: Optional[torch.Tensor] = None,
                     stream=None) -> torch.Tensor:
    """sbn_bitlinear_grad_x: dX = dY (gamma C) under the straight-through estimator."""
    _need(dy, torch.bfloat16, "dy")
    t, n_out = dy.shape
    if n_out != w.n_out:
        raise ValueError("N_out mismatch between dY and the weights")
    if out is None:
        out = torch.empty((t, w.k), dtype=torch.bfloat16, device=dy.device)
    st = lib().sbn_bitlinear_grad_x(_ptr(dy), t, w.k, w.n_out, w.n, w.m, _ptr(w.codes), _ptr(w.meta),
                                    _ptr(w.gamma), _ptr(out), _stream_ptr(stream))
    _check(st, "sbn_bitlinear_grad_x")
    return out


def bitlinear_grad_w(dy: torch.Tensor, xq: torch.Tensor, s: torch.Tensor,
                     out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """sbn_bitlinear_grad_w: dW = dY^T (Xq s / 127) under the straight-through
    estimator (every latent weight, pruned ones included)."""
    _need(dy, torch.bfloat16, "dy")
    _need(xq, torch.int8, "xq")
    _need(s, torch.float32, "s")
    t, n_out = dy.shape
    if xq.shape[0] != t:
        raise ValueError("T mismatch between dY and Xq")
    k = xq.shape[1]
    if out is None:
        out = torch.empty((n_out, k), dtype=torch.bfloat16, device=dy.device)
    st = lib().sbn_bitlinear_grad_w(_ptr(dy), _ptr(xq), _ptr(s), t, k, n_out, _ptr(out), _stream_ptr(stream))
    _check(st, "sbn_bitlinear_grad_w")
    return out


def set_programmatic_launch(enable: bool) -> bool:
    """sbn_set_programmatic_launch: switch programmatic dependent launch of
    the library's kernels on or off; returns the previous setting."""
    return bool(lib().sbn_set_programmatic_launch(1 if enable else 0))


def get_device_error(stream=None) -> int:
    """sbn_get_device_error: sync the stream, read and clear the device error word."""
    return int(lib().sbn_get_device_error(_stream_ptr(stream)))


class BitLinear(torch.nn.Module):
    """BitLinear layer with a dynamic N:M mask on latent bf16 weights.

    Every forward re-derives the packed ternary weights from the latent
    weights (the mask is dynamic), quantizes the activations per token and
    runs the integer contraction. No bias. Inference only (no autograd).
    """

    def __init__(self, in_features: int, out_features: int, n: int = 6, m: int = 8,
                 device=None, weight: Optional[torch.Tensor] = None):
        super().__init__()
        if weight is None:
            weight = torch.empty((out_features, in_features), dtype=torch.bfloat16, device=device)
            torch.nn.init.normal_(weight, std=0.02)
        self.weight = torch.nn.Parameter(weight, requires_grad=False)
        self.n, self.m = n, m
        self._ws = None
        self._packed = None

    def pack(self) -> PackedWeights:
        w = self.weight.data
        if self._packed is None or self._packed.codes.device != w.device:
            self._packed = alloc_packed(w.shape[0], w.shape[1], self.n, self.m, w.device)
            self._ws = torch.empty(workspace_bytes(*w.shape), dtype=torch.uint8, device=w.device)
        return quantize_weights(w, self.n, self.m, out=self._packed, workspace=self._ws)

    @torch.no_grad()
    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, x.shape[-1]).contiguous()
        packed = self.pack()
        y = bitlinear_x(x2, packed)   # activation quantization fused for T <= 16
        return y.reshape(*lead, packed.n_out)


def probe_i8_mma(iters: int, stream=None) -> int:
    """sbn_probe_i8_mma: launches the tensor-pipe INT8 probe; returns the
    number of CTAs (each issued `iters` MMAs of 2*128*256*32 operations)."""
    ctas = ctypes.c_int32(0)
    _check(lib().sbn_probe_i8_mma(int(iters), ctypes.byref(ctas), _stream_ptr(stream)), "sbn_probe_i8_mma")
    return int(ctas.value)


def probe_i8_sparse_mma(iters: int, stream=None) -> int:
    """sbn_probe_i8_sparse_mma: launches the sparse INT8 probe on CTA pairs;
    returns the number of pairs (each issued `iters` MMAs of 2*256*224*64
    logical operations)."""
    pairs = ctypes.c_int32(0)
    _check(lib().sbn_probe_i8_sparse_mma(int(iters), ctypes.byref(pairs), _stream_ptr(stream)),
           "sbn_probe_i8_sparse_mma")
    return int(pairs.value)


def selftest_wait_timeout(which: int, limit_ns: int, stream=None) -> None:
    """sbn_selftest_wait_timeout: one bounded device wait that runs out (test hook)."""
    _check(lib().sbn_selftest_wait_timeout(int(which), int(limit_ns), _stream_ptr(stream)),
           "sbn_selftest_wait_timeout")
