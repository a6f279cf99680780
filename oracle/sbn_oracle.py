"""Plain, slow CPU oracle of the Sparse-BitNet BitLinear layer: the forward
path and its straight-through backward.

TEST INFRASTRUCTURE. This module is the yardstick the CUDA path is checked
against. It shares no code with ``sparse_linear_layers_fwd_b200`` (no kernels,
headers, helpers, tables or constants) and imports nothing from it. Only
``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline legs use it.

What it computes (the BitLinear forward with a dynamic N:M mask):

1. gamma  -- absmean scale of the latent weight tensor ("BitNet b1.58: How
   Ternary Weights Cut LLM Memory by 82% Without Losing Accuracy", section
   "How ternary quantization works during training": W is divided by its mean
   absolute value, rounded, clamped to [-1, 1]).
2. mask   -- per group of m consecutive weights along K keep the n of largest
   |w| ("Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to
   Semi-Structured Sparsity", Abstract: dynamic N:M sparsification; Figure 6:
   the per-block threshold t = |w|_(N+1), i.e. selection by magnitude).
3. codes  -- ternary values clamp(rint(w / gamma), -1, 1) at kept positions
   (same absmean passage; "Microsoft BitNet 1.58: The Era of 1-Bit Large
   Language Models", section "The BitLinear Layer", third operation).
4. acts   -- per-token absmax INT8 quantization (section "The BitLinear
   Layer", second operation; promptingindex page, same section: INT8 with a
   per-token scale).
5. acc    -- integer contraction of INT8 activations with ternary weights
   ("The BitLinear Layer", fourth operation: addition, subtraction, zero-skips).
6. y      -- dequantization with the preserved scales ("The BitLinear Layer",
   fifth operation).
7. dX, dW -- the backward of the layer under the straight-through estimator
   ("Microsoft BitNet 1.58 ...", section "Training with the Straight-Through
   Estimator": gradients cross the quantizer as the identity, the latent
   weights take the update).

Readings where the pages are silent:
* gamma is taken over the whole dense latent tensor, before masking;
* the exact sum of |w| is rounded once to fp64, divided by N_out*K in fp64,
  rounded to fp32 and floored at 1e-5 (the pages give no precision or epsilon);
* the mask ranks latent |w|; equal magnitudes keep the lower index;
* rint rounds half to even, so |w|/gamma == 0.5 gives code 0;
* activations use the symmetric range +-127; the per-token scale s_t is
  max(max_k |x_tk|, 1e-5), and q = clamp(rint(x * fl32(127 / s_t)), -127, 127);
* every rounding decision that yields an integer (a code, an INT8 value) is
  taken in fp32, the precision of the kernels;
* y = acc * gamma * s_t / 127, evaluated in fp64 and rounded once to bf16.

Packed weight format (shared by every pattern; the pages fix only "four
ternary values per byte, 2 bits each", from the bitnet.cpp section of the
octagono page):
* codes: per row, the kept values in ascending k; value j sits in bits
  2*(j%4)..2*(j%4)+1 of byte j//4; 0 -> 0b00, +1 -> 0b01, -1 -> 0b11;
  the row stride is ceil(K*n/m/4) rounded up to 16 bytes, padding is zero.
* meta: per row, bit k%8 of byte k//8 is set iff position k is kept; the row
  stride is K/8 rounded up to 16 bytes; there is no meta when n == m.

Input arrays carry bf16 values as their raw uint16 bit patterns.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "EPS",
    "Q_ACT",
    "bf16_bits_to_f32",
    "bf16_bits_from_f64_rne",
    "gamma_bins",
    "gamma_from_bins",
    "absmean_gamma",
    "nm_mask",
    "ternary_codes",
    "codes_row_bytes",
    "meta_row_bytes",
    "pack_weights",
    "unpack_weights",
    "quantize_weights",
    "quantize_acts",
    "bitlinear_acc",
    "dequant_bf16",
    "bitlinear",
    "bitlinear_acc_at",
    "bitlinear_at",
    "mask_flips",
    "mask_flip_rate",
    "mask_index_bits",
    "colex_rank",
    "colex_unrank",
    "entropy_group_bits",
    "entropy_row_bytes",
    "entropy_pack",
    "entropy_unpack",
    "ste_grad_x",
    "ste_grad_w",
]

#: floor on gamma and on the per-token activation scale (not on the pages)
EPS = np.float32(1e-5)
#: symmetric INT8 range used for activations
Q_ACT = 127


# --------------------------------------------------------------------------
# bf16 plumbing
# --------------------------------------------------------------------------

def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    b = np.asarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_from_f64_rne(y: np.ndarray) -> np.ndarray:
    """Round float64 values once, to nearest-even, to bf16 bit patterns.

    A bf16 number has an 8-bit significand. With |y| = mant * 2**e and
    0.5 <= mant < 1, the rounded significand is rint(mant * 256) (exact in
    fp64, ties to even), so the result is correctly rounded with no detour
    through fp32. Zeros keep their sign; values must be finite and inside
    the bf16 normal range (or zero).
    """
    y = np.asarray(y, dtype=np.float64)
    if not np.all(np.isfinite(y)):
        raise ValueError("non-finite value in bf16 rounding")
    sign = np.where(np.signbit(y), 0x8000, 0).astype(np.int64)
    a = np.abs(y)
    mant, e = np.frexp(a)
    r = np.rint(mant * 256.0).astype(np.int64)
    carry = r == 256
    r = np.where(carry, 128, r)
    e = np.where(carry, e + 1, e).astype(np.int64)
    biased = e - 1 + 127
    nz = a != 0.0
    if np.any(nz & ((biased < 1) | (biased > 254))):
        raise ValueError("value outside the bf16 normal range")
    bits = np.where(nz, (biased << 7) | (r - 128), 0) | sign
    return bits.astype(np.uint16)


# --------------------------------------------------------------------------
# 1. gamma: absmean scale, exact
# --------------------------------------------------------------------------

def gamma_bins(w_bits: np.ndarray) -> np.ndarray:
    """Exact per-exponent sums of |w| significands.

    A finite bf16 magnitude with biased exponent e and 7-bit fraction f is
    s * 2**(max(e,1) - 134) with s = 128 + f (e >= 1) or s = f (e == 0,
    subnormal). Returns B[e] = sum of s over the elements filed under e
    (index 0 unused, 1..254 used), as exact Python integers.
    """
    mag = np.asarray(w_bits, dtype=np.uint16).reshape(-1) & np.uint16(0x7FFF)
    e = (mag >> np.uint16(7)).astype(np.int64)
    if np.any(e == 255):
        raise ValueError("non-finite latent weight")
    f = (mag & np.uint16(0x7F)).astype(np.int64)
    s = np.where(e >= 1, f + 128, f)
    eb = np.maximum(e, 1)
    # Each bin sums at most 2**32 values below 256, so every partial sum is
    # an integer below 2**53 and the float64 accumulation is exact.
    if mag.size >= 2 ** 32:
        raise ValueError("tensor too large for exact bins")
    sums = np.bincount(eb, weights=s.astype(np.float64), minlength=255)
    bins = [int(v) for v in sums]
    assert all(float(b) == v for b, v in zip(bins, sums))
    return np.array(bins, dtype=object)


def gamma_from_bins(bins, n_elems: int) -> np.float32:
    """gamma = max(fl32(fl64(fl64(S) / n_elems)), 1e-5) with S the exact sum.

    S = sum_e B[e] * 2**(e - 134) is formed as one exact integer times
    2**-133; Python's int -> float conversion rounds it once to the nearest
    double (ties to even). The division is one IEEE fp64 division, and the
    cast to float32 rounds to nearest-even.
    """
    s_int = 0
    for e in range(1, 255):
        b = int(bins[e])
        if b:
            s_int += b << (e - 1)
    d = math.ldexp(float(s_int), -133)   # exact scaling of the rounded double
    q = d / float(n_elems)
    g = np.float32(q)
    return np.float32(max(g, EPS))


def absmean_gamma(w_bits: np.ndarray) -> np.float32:
    """Per-tensor absmean scale gamma of the latent weights W [N_out, K].

    "BitNet b1.58: How Ternary Weights Cut LLM Memory ...", section "How
    ternary quantization works during training": the weight matrix is divided
    by its mean absolute value.
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    return gamma_from_bins(gamma_bins(w_bits), int(w_bits.size))


# --------------------------------------------------------------------------
# 2. N:M magnitude mask
# --------------------------------------------------------------------------

def nm_mask(w_bits: np.ndarray, n: int, m: int) -> np.ndarray:
    """Boolean keep-mask of the dynamic N:M magnitude sparsification.

    For every row and every group of m consecutive positions along K, keep
    the n positions of largest |w|; equal magnitudes keep the lower index
    first. "Sparse-BitNet ...", Abstract (dynamic N:M sparsification) and
    Figure 6 (the per-block threshold t = |w|_(N+1)). For finite bf16 values
    the order of |w| is the integer order of the 15 magnitude bits, and
    -0 ranks equal to +0.
    """
    w_bits = np.asarray(w_bits, dtype=np.uint16)
    rows, k = w_bits.shape
    if k % m != 0 or not (1 <= n <= m):
        raise ValueError("bad N:M pattern for this K")
    mag = (w_bits & np.uint16(0x7FFF)).astype(np.int64).reshape(rows, k // m, m)
    # a stable sort of -|w| lists equal magnitudes in ascending index order
    order = np.argsort(-mag, axis=-1, kind="stable")
    keep = np.zeros(mag.shape, dtype=bool)
    np.put_along_axis(keep, order[..., :n], True, axis=-1)
    return keep.reshape(rows, k)


# --------------------------------------------------------------------------
# 3. ternary codes
# --------------------------------------------------------------------------

def ternary_codes(w_bits: np.ndarray, gamma: np.float32, mask: np.ndarray) -> np.ndarray:
    """code = clamp(rint(fl32(w / gamma)), -1, 1) at kept positions, else 0.

    Division and rint are IEEE fp32 (round to nearest-even). Section "How
    ternary quantization works during training" of the promptingindex page.
    """
    w = bf16_bits_to_f32(w_bits)
    q = np.rint(w / np.float32(gamma)).astype(np.float32)
    c = np.clip(q, -1.0, 1.0).astype(np.int8)
    c[~mask] = 0
    return c


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------

def _round_up(x: int, a: int) -> int:
    return (x + a - 1) // a * a


def codes_row_bytes(k: int, n: int, m: int) -> int:
    """Bytes per row of packed 2-bit codes, padded to 16."""
    kept = k * n // m
    return _round_up((kept + 3) // 4, 16)


def meta_row_bytes(k: int, n: int, m: int) -> int:
    """Bytes per row of the keep bitmask, padded to 16 (0 when n == m)."""
    if n == m:
        return 0
    return _round_up((k + 7) // 8, 16)


def pack_weights(codes: np.ndarray, mask: np.ndarray, n: int, m: int):
    """Pack ternary codes and the keep mask into the canonical byte format.

    Returns (codes_bytes [rows, codes_row_bytes], meta [rows, meta_row_bytes]).
    Every row keeps exactly K*n/m positions, so the kept values of all rows,
    read in row-major order, form a [rows, K*n/m] array in ascending k.
    """
    rows, k = codes.shape
    kept = k * n // m
    if not np.all(mask.sum(axis=1) == kept):
        raise ValueError("mask does not keep K*n/m positions per row")
    vals = codes[mask].reshape(rows, kept).astype(np.int64)
    if np.any(np.abs(vals) > 1):
        raise ValueError("codes must be ternary")
    enc = np.where(vals == 1, 0b01, np.where(vals == -1, 0b11, 0b00))
    pad = (-kept) % 4
    enc = np.concatenate([enc, np.zeros((rows, pad), dtype=np.int64)], axis=1)
    quads = enc.reshape(rows, -1, 4)
    packed = quads[..., 0] | (quads[..., 1] << 2) | (quads[..., 2] << 4) | (quads[..., 3] << 6)
    cb = np.zeros((rows, codes_row_bytes(k, n, m)), dtype=np.uint8)
    cb[:, : packed.shape[1]] = packed.astype(np.uint8)
    mb = np.zeros((rows, meta_row_bytes(k, n, m)), dtype=np.uint8)
    if n != m:
        bits = np.packbits(mask, axis=1, bitorder="little")
        mb[:, : bits.shape[1]] = bits
    return cb, mb


def unpack_weights(codes_bytes: np.ndarray, meta: np.ndarray, k: int, n: int, m: int):
    """Inverse of :func:`pack_weights`: returns (dense codes int8 [rows,K], mask)."""
    rows = codes_bytes.shape[0]
    kept = k * n // m
    if n == m:
        mask = np.ones((rows, k), dtype=bool)
    else:
        mask = np.unpackbits(meta, axis=1, bitorder="little")[:, :k].astype(bool)
        if not np.all(mask.sum(axis=1) == kept):
            raise ValueError("meta does not keep K*n/m positions per row")
    cb = codes_bytes.astype(np.int64)
    fields = np.stack([(cb >> (2 * i)) & 0b11 for i in range(4)], axis=-1)
    fields = fields.reshape(rows, -1)[:, :kept]
    if np.any(fields == 0b10):
        raise ValueError("code 0b10 is never written")
    vals = np.where(fields == 0b01, 1, np.where(fields == 0b11, -1, 0)).astype(np.int8)
    dense = np.zeros((rows, k), dtype=np.int8)
    dense[mask] = vals.reshape(-1)
    return dense, mask


def quantize_weights(w_bits: np.ndarray, n: int, m: int):
    """Steps 1-3 plus packing: returns (codes_bytes, meta, gamma, mask, dense)."""
    gamma = absmean_gamma(w_bits)
    mask = nm_mask(w_bits, n, m)
    dense = ternary_codes(w_bits, gamma, mask)
    cb, mb = pack_weights(dense, mask, n, m)
    return cb, mb, gamma, mask, dense


# --------------------------------------------------------------------------
# 4. per-token absmax INT8 activations
# --------------------------------------------------------------------------

def quantize_acts(x_bits: np.ndarray):
    """Per-token absmax INT8 quantization of X [T, K].

    s_t = max(max_k |x_tk|, 1e-5) (exact in fp32); the multiplier
    fl32(127 / s_t) is one IEEE division; q = clamp(rint(fl32(x * mult)),
    -127, 127). "Microsoft BitNet 1.58 ...", section "The BitLinear Layer",
    second operation (absmax scaling, scale kept for dequantization).
    Returns (Xq int8 [T, K], s float32 [T]).
    """
    x = bf16_bits_to_f32(x_bits)
    s = np.maximum(np.max(np.abs(x), axis=1), EPS).astype(np.float32)
    mult = (np.float32(Q_ACT) / s).astype(np.float32)
    q = np.rint(x * mult[:, None]).astype(np.float32)
    q = np.clip(q, -Q_ACT, Q_ACT).astype(np.int8)
    return q, s


# --------------------------------------------------------------------------
# 5./6. contraction and dequantization
# --------------------------------------------------------------------------

def bitlinear_acc(xq: np.ndarray, dense_codes: np.ndarray) -> np.ndarray:
    """acc[t, n] = sum_k xq[t, k] * code[n, k], exact, returned as int32.

    The product is formed by a float64 matrix product. Every term is an
    integer in [-127, 127] and every partial sum is bounded by 127*K < 2**53,
    so each addition is exact whatever order the library adds in; the result
    is checked to be integral and to fit int32.
    """
    k = xq.shape[1]
    if Q_ACT * k >= 2 ** 53:
        raise ValueError("K too large for an exact fp64 contraction")
    acc = xq.astype(np.float64) @ dense_codes.astype(np.float64).T
    acc_i = acc.astype(np.int64)
    assert np.all(acc_i == acc)
    assert np.all(np.abs(acc_i) < 2 ** 31)
    return acc_i.astype(np.int32)


def dequant_bf16(acc: np.ndarray, s: np.ndarray, gamma: np.float32) -> np.ndarray:
    """y = bf16_rne(acc * gamma * s_t / 127) evaluated in fp64."""
    y = acc.astype(np.float64) * float(gamma) * (s.astype(np.float64)[:, None] / Q_ACT)
    return bf16_bits_from_f64_rne(y)


def bitlinear(xq, s, codes_bytes, meta, gamma, k, n, m):
    """Full contraction from the packed weights: returns (Y bf16 bits, acc)."""
    dense, _ = unpack_weights(codes_bytes, meta, k, n, m)
    acc = bitlinear_acc(xq, dense)
    return dequant_bf16(acc, s, gamma), acc


def bitlinear_acc_at(xq, dense_codes, t_idx, n_idx) -> np.ndarray:
    """acc at sampled (t, n) pairs, one exact integer dot product each."""
    t_idx = np.asarray(t_idx)
    n_idx = np.asarray(n_idx)
    out = np.empty(t_idx.shape, dtype=np.int64)
    for i, (t, nn) in enumerate(zip(t_idx.reshape(-1), n_idx.reshape(-1))):
        out.reshape(-1)[i] = int(np.dot(xq[t].astype(np.int64), dense_codes[nn].astype(np.int64)))
    return out.astype(np.int32)


def bitlinear_at(xq, s, dense_codes, gamma, t_idx, n_idx):
    """y and acc at sampled (t, n) pairs."""
    acc = bitlinear_acc_at(xq, dense_codes, t_idx, n_idx)
    y = acc.astype(np.float64) * float(gamma) * (s.astype(np.float64)[np.asarray(t_idx)] / Q_ACT)
    return bf16_bits_from_f64_rne(y), acc


# --------------------------------------------------------------------------
# mask flip rate between two steps
# --------------------------------------------------------------------------

def mask_flips(mask_a: np.ndarray, mask_b: np.ndarray) -> int:
    """Number of positions whose keep/prune state differs between two masks.

    Sparse-BitNet page, Figure 3(b): the mask flip rate r_t measures how
    stable the dynamic N:M pattern is between training steps; its equation is
    not in the extracted page, so it is read as the fraction of positions
    whose mask entry changed.
    """
    mask_a = np.asarray(mask_a, dtype=bool)
    mask_b = np.asarray(mask_b, dtype=bool)
    if mask_a.shape != mask_b.shape:
        raise ValueError("masks of different shapes")
    return int(np.count_nonzero(mask_a != mask_b))


def mask_flip_rate(mask_a: np.ndarray, mask_b: np.ndarray) -> float:
    """r_t = mask_flips / number of positions."""
    return mask_flips(mask_a, mask_b) / float(np.asarray(mask_a).size)


# --------------------------------------------------------------------------
# entropy-tight packed format
# --------------------------------------------------------------------------
#
# "From 2:4 to 8:16 sparsity patterns in LLMs for Outliers and Weights with
# Variance Correction", Abstract: the mask of 2:4 costs 0.75 and that of 8:16
# 0.875 bits per element. Both equal ceil(log2 C(m, n)) / m, the size of an
# index that numbers every keep pattern of a group. The format below stores,
# per group of m positions, one integer word
#     word = rank(kept positions) * 3**n + sum_i (code_i + 1) * 3**i
# (kept codes in ascending position order, i from 0) in
# ceil(log2(C(m, n) * 3**n)) bits; rank is the combinatorial number system
# (colex) rank: for kept offsets c_1 < ... < c_n within the group,
# rank = sum_i C(c_i, i). The words of a row are concatenated little-endian
# (bit b of the row stream is bit b % 8 of byte b // 8) and the row is padded
# with zero bytes to a multiple of 16.

def mask_index_bits(n: int, m: int) -> int:
    """Bits of an index that numbers the C(m, n) keep patterns of a group."""
    c = math.comb(m, n)
    return 0 if c == 1 else (c - 1).bit_length()


def entropy_group_bits(n: int, m: int) -> int:
    """Bits of one group word: keep pattern and kept ternary values jointly."""
    return (math.comb(m, n) * 3 ** n - 1).bit_length()


def entropy_row_bytes(k: int, n: int, m: int) -> int:
    return _round_up((k // m * entropy_group_bits(n, m) + 7) // 8, 16)


def colex_rank(offsets) -> int:
    return sum(math.comb(c, i + 1) for i, c in enumerate(offsets))


def colex_unrank(rank: int, n: int, m: int):
    """Kept offsets (ascending) of the pattern with the given colex rank."""
    out = []
    for i in range(n, 0, -1):
        c = i - 1
        while math.comb(c + 1, i) <= rank:
            c += 1
        out.append(c)
        rank -= math.comb(c, i)
    return sorted(out)


def entropy_pack(mask: np.ndarray, dense_codes: np.ndarray, n: int, m: int) -> np.ndarray:
    """Rows of group words from the keep mask and the dense codes [rows, K]."""
    rows, k = mask.shape
    bits = entropy_group_bits(n, m)
    out = np.zeros((rows, entropy_row_bytes(k, n, m)), np.uint8)
    for r in range(rows):
        stream = 0
        for g in range(k // m):
            offs = [j for j in range(m) if mask[r, g * m + j]]
            if len(offs) != n:
                raise ValueError("a group does not keep exactly n positions")
            word = colex_rank(offs) * 3 ** n
            for i, j in enumerate(offs):
                word += (int(dense_codes[r, g * m + j]) + 1) * 3 ** i
            stream |= word << (g * bits)
        nbytes = (k // m * bits + 7) // 8
        out[r, :nbytes] = np.frombuffer(stream.to_bytes(nbytes, "little"), np.uint8)
    return out


def entropy_unpack(packed: np.ndarray, k: int, n: int, m: int):
    """Inverse of entropy_pack: (dense codes int8 [rows, K], keep mask)."""
    rows = packed.shape[0]
    bits = entropy_group_bits(n, m)
    dense = np.zeros((rows, k), np.int8)
    mask = np.zeros((rows, k), bool)
    for r in range(rows):
        stream = int.from_bytes(bytes(packed[r]), "little")
        for g in range(k // m):
            word = (stream >> (g * bits)) & ((1 << bits) - 1)
            rank, v = divmod(word, 3 ** n)
            for i, j in enumerate(colex_unrank(rank, n, m)):
                mask[r, g * m + j] = True
                dense[r, g * m + j] = (v // 3 ** i) % 3 - 1
    return dense, mask


# --------------------------------------------------------------------------
# 7. backward through the layer (straight-through estimator)
# --------------------------------------------------------------------------
#
# "Microsoft BitNet 1.58 ...", section "Training with the Straight-Through
# Estimator": in the backward pass the gradients cross the quantizer as if it
# were the identity function, and the full-precision latent weights receive
# them. The forward multiplies Xd = Xq * s_t / 127 (the dequantized
# activations) by Wd = gamma * C (C the dense masked codes): Y = Xd Wd^T.
# With both quantizers (the N:M mask included) passed as the identity, the
# gradients of a loss L with dL/dY = dY are
#     dX = dY Wd      [T, K]     (to the activations X)
#     dW = dY^T Xd    [N_out, K] (to the latent weights W, at every position)
# Both are evaluated in fp64 and rounded once to bf16: gradients are kept in
# bf16 ("BitNet b1.58: How Ternary Weights ...", section "How ternary
# quantization works during training": the optimizer accumulates in FP16 or
# BF16).

def ste_grad_x(dy_bits: np.ndarray, dense_codes: np.ndarray, gamma: np.float32) -> np.ndarray:
    """dX = bf16_rne(dY (gamma C)) for dY bf16 [T, N_out], C int8 [N_out, K]."""
    dy = bf16_bits_to_f32(dy_bits).astype(np.float64)
    wd = float(gamma) * np.asarray(dense_codes).astype(np.float64)
    return bf16_bits_from_f64_rne(dy @ wd)


def ste_grad_w(dy_bits: np.ndarray, xq: np.ndarray, s: np.ndarray) -> np.ndarray:
    """dW = bf16_rne(dY^T (Xq s_t / 127)) for dY bf16 [T, N_out], Xq int8 [T, K]."""
    dy = bf16_bits_to_f32(dy_bits).astype(np.float64)
    xd = np.asarray(xq).astype(np.float64) * (np.asarray(s).astype(np.float64)[:, None] / Q_ACT)
    return bf16_bits_from_f64_rne(dy.T @ xd)
