"""Sparse-BitNet BitLinear forward on B200 (sm_100a).

The compute path lives in ``libsbn.so`` (CUDA kernels behind a C ABI,
``include/sbn.h``); :mod:`sparse_linear_layers_fwd_b200.sbn` is its thin
ctypes binding. Importing this package does not load the library; the first
use of a binding name does, and fails loudly if the library is missing.
"""

__all__ = [
    "quantize_weights", "quantize_acts", "bitlinear", "bitlinear_acc32",
    "Pattern", "PackedWeights", "BitLinear", "SbnError",
]


def __getattr__(name):
    if name in __all__:
        from . import sbn
        return getattr(sbn, name)
    raise AttributeError(name)
