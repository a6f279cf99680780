"""Seeded synthetic inputs for the BitLinear forward.

This module holds no arithmetic of the method: it only draws random numbers
and rounds them to bf16 storage. Both the CUDA path's tests/benchmark and the
CPU oracle take their inputs from here, as raw bf16 bit patterns (uint16).

Workloads (the shapes and value distributions the method is run on):

* ``layer_small``: one BitLinear, T=16 tokens, K=256, N_out=256, 2:4.
* ``decode``: T in {1, 4, 16}, K=2560, N_out=6912 (BitNet-2B FFN up-projection
  shape), 6:8.
* ``prefill``: T=4096 with (K, N_out) = (2560, 6912) and (6912, 2560), 2:4.
* ``qwen05b_stack``: 24 layers of the Qwen2.5-0.5B projections (hidden 896:
  q 896x896, k/v 896x128, o 896x896, gate/up 896x4864, down 4864x896),
  T=2048, 6:8, activations with Student-t (nu=3) heavy-tailed channels.
* ``ffn3b_sweep``: hidden 2048 / intermediate 11008 FFN projections,
  T in {1, 64, 512, 8192}, n:m in {2:4, 4:8, 6:8, 8:16, 8:8}.

Latent weights are N(0, 0.02); activations N(0, 1). Values are drawn in fp32
from numpy's PCG64 generator seeded by (seed, workload, layer, tensor) and
rounded to bf16 with round-to-nearest-even.
"""

from __future__ import annotations

import zlib

import numpy as np

W_STD = 0.02


def _rng(seed: int, *tags) -> np.random.Generator:
    words = [int(seed)]
    for t in tags:
        if isinstance(t, str):
            words.append(zlib.crc32(t.encode()))
        else:
            words.append(int(t))
    return np.random.default_rng(np.random.SeedSequence(words))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Storage rounding of fp32 samples to bf16 (nearest-even), as uint16."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def latent_weights(n_out: int, k: int, seed: int = 0, tag="w", std: float = W_STD) -> np.ndarray:
    """Latent bf16 weights W [n_out, k] ~ N(0, std)."""
    g = _rng(seed, "weights", tag, n_out, k)
    return to_bf16_bits(g.standard_normal((n_out, k), dtype=np.float32) * np.float32(std))


def activations(t: int, k: int, seed: int = 0, tag="x", outlier_channels: int = 0,
                outlier_scale: float = 20.0, heavy_tail_channels: int = 0,
                heavy_tail_nu: float = 3.0) -> np.ndarray:
    """Activations X [t, k] ~ N(0, 1), as bf16 bits.

    ``outlier_channels`` seeded-random channels are multiplied by
    ``outlier_scale``; ``heavy_tail_channels`` seeded-random channels are
    drawn from a Student-t distribution with ``heavy_tail_nu`` degrees of
    freedom instead of the normal.
    """
    g = _rng(seed, "acts", tag, t, k)
    x = g.standard_normal((t, k), dtype=np.float32)
    if outlier_channels:
        ch = g.choice(k, size=outlier_channels, replace=False)
        x[:, ch] *= np.float32(outlier_scale)
    if heavy_tail_channels:
        ch = g.choice(k, size=heavy_tail_channels, replace=False)
        x[:, ch] = g.standard_t(heavy_tail_nu, size=(t, heavy_tail_channels)).astype(np.float32)
    return to_bf16_bits(x)


# --------------------------------------------------------------------------
# workload catalogue
# --------------------------------------------------------------------------

QWEN05B_PROJ = [  # (name, K, N_out)
    ("q", 896, 896), ("k", 896, 128), ("v", 896, 128), ("o", 896, 896),
    ("gate", 896, 4864), ("up", 896, 4864), ("down", 4864, 896),
]

FFN3B_PROJ = [("gate", 2048, 11008), ("up", 2048, 11008), ("down", 11008, 2048)]
FFN3B_PATTERNS = [(2, 4), (4, 8), (6, 8), (8, 16), (8, 8)]
FFN3B_TOKENS = [1, 64, 512, 8192]

DECODE_TOKENS = [1, 4, 16]


def layer_small(seed: int = 0):
    """T=16, K=256, N_out=256, 2:4, two random x20 outlier channels."""
    w = latent_weights(256, 256, seed, tag="layer_small")
    x = activations(16, 256, seed, tag="layer_small", outlier_channels=2)
    return dict(w=w, x=x, n=2, m=4)


def decode(t: int, seed: int = 0):
    """Decode GEMV shape: K=2560, N_out=6912, 6:8."""
    w = latent_weights(6912, 2560, seed, tag="decode")
    x = activations(t, 2560, seed, tag=f"decode_t{t}")
    return dict(w=w, x=x, n=6, m=8)


def decode_weights(seed: int = 0):
    return latent_weights(6912, 2560, seed, tag="decode")


def decode_acts(t: int, seed: int = 0):
    return activations(t, 2560, seed, tag=f"decode_t{t}")


def prefill(which: str = "up", t: int = 4096, seed: int = 0):
    """Prefill GEMM: 'up' is K=2560, N_out=6912; 'down' is K=6912, N_out=2560; 2:4."""
    k, n_out = (2560, 6912) if which == "up" else (6912, 2560)
    w = latent_weights(n_out, k, seed, tag=f"prefill_{which}")
    x = activations(t, k, seed, tag=f"prefill_{which}")
    return dict(w=w, x=x, n=2, m=4)


def qwen_heavy_channels(k: int) -> int:
    return max(2, k // 64)


def qwen05b_layer(layer: int, proj: str, t: int = 2048, seed: int = 0):
    """One projection of the 24-layer Qwen2.5-0.5B-shaped stack (6:8)."""
    k, n_out = {p: (kk, nn) for p, kk, nn in QWEN05B_PROJ}[proj]
    w = latent_weights(n_out, k, seed, tag=f"qwen_l{layer}_{proj}")
    x = activations(t, k, seed, tag=f"qwen_l{layer}_{proj}",
                    heavy_tail_channels=qwen_heavy_channels(k))
    return dict(w=w, x=x, n=6, m=8)


def ffn3b(proj: str, t: int, n: int, m: int, seed: int = 0):
    """One FFN projection of the 3B-scale sweep."""
    k, n_out = {p: (kk, nn) for p, kk, nn in FFN3B_PROJ}[proj]
    w = latent_weights(n_out, k, seed, tag=f"ffn3b_{proj}")
    x = activations(t, k, seed, tag=f"ffn3b_{proj}_t{t}")
    return dict(w=w, x=x, n=n, m=m)
