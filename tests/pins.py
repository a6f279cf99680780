"""Pins of the CPU oracle to facts other than its own formulas.

Each ``check_*`` takes an implementation namespace (the oracle module, or a
copy with one function replaced by a plausible mistake) and raises
AssertionError when the implementation departs from what the pages and the
mathematics fix. The pins use independent machinery: exact rationals
(``fractions.Fraction``), ``math.fsum``, hardware float conversions, brute
force over all subsets, plain per-element loops and hand-worked fixtures.

Pages cited:
* "Sparse-BitNet: 1.58-bit LLMs are Naturally Friendly to Semi-Structured
  Sparsity" -- Abstract (dynamic N:M sparsity), Figure 6 (threshold
  t = |w|_(N+1)), Figure 1 (zeros dominate the ternary states);
* "BitNet b1.58: How Ternary Weights Cut LLM Memory by 82% Without Losing
  Accuracy" -- section "How ternary quantization works during training"
  (divide by mean |W|, round, clamp to [-1, 1]; INT8 per-token activations);
* "Microsoft BitNet 1.58: The Era of 1-Bit Large Language Models" -- section
  "The BitLinear Layer" (five operations), "bitnet.cpp: Matrix-Free
  Inference" (four 2-bit values per byte) and "Training with the
  Straight-Through Estimator" (the quantizer is the identity backward).
"""

from __future__ import annotations

import itertools
import math
from fractions import Fraction
from pathlib import Path

import numpy as np

GOLDEN = Path(__file__).parent / "golden"
EPS32 = np.float32(1e-5)


# --------------------------------------------------------------------------
# independent helpers (hardware conversions and exact rationals)
# --------------------------------------------------------------------------

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact value of bf16 bit patterns via the hardware fp32 widening."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def f64_to_bf16_trunc_bits(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns of values that are already exact bf16 numbers."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32)
    assert np.all((u & np.uint32(0xFFFF)) == 0), "value is not a bf16 number"
    return (u >> np.uint32(16)).astype(np.uint16)


def fraction_to_f32_rne(q: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) fp32 value of a rational."""
    g = np.float32(float(q))
    cands = {np.float32(g), np.nextafter(g, np.float32(-np.inf)), np.nextafter(g, np.float32(np.inf))}
    best = None
    for c in cands:
        d = abs(Fraction(float(c)) - q)
        even = (np.array(c, dtype=np.float32).view(np.uint32) & 1) == 0
        key = (d, 0 if even else 1)
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


def fraction_to_bf16_value(q: Fraction) -> Fraction:
    """Correctly rounded bf16 value of a rational (normal range), by search."""
    if q == 0:
        return Fraction(0)
    sgn = -1 if q < 0 else 1
    a = abs(q)
    e = math.floor(math.log2(float(a)))
    # make sure 2**e <= a < 2**(e+1) exactly
    while Fraction(2) ** e > a:
        e -= 1
    while Fraction(2) ** (e + 1) <= a:
        e += 1
    ulp = Fraction(2) ** (e - 7)
    lo = (a // ulp) * ulp
    hi = lo + ulp
    if a - lo < hi - a:
        r = lo
    elif a - lo > hi - a:
        r = hi
    else:  # tie: pick the even significand
        r = lo if ((lo / ulp) % 2 == 0) else hi
    return sgn * r


def exact_abs_sum_int(w_bits: np.ndarray) -> int:
    """sum |w| * 2**133 as an exact integer (every bf16 |w| * 2**133 is one)."""
    v = np.abs(bf16_to_f64(w_bits)).reshape(-1) * (2.0 ** 133)
    total = 0
    for x in v:
        total += int(x)
    return total


def _impl_quantize_weights(impl, w_bits, n, m):
    g = impl.absmean_gamma(w_bits)
    mask = impl.nm_mask(w_bits, n, m)
    dense = impl.ternary_codes(w_bits, g, mask)
    cb, mb = impl.pack_weights(dense, mask, n, m)
    return cb, mb, g, mask, dense


def read_table(name):
    rows = []
    for line in (GOLDEN / name).read_text().splitlines():
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        rows.append([part.split() for part in line.split("|")])
    return rows


# --------------------------------------------------------------------------
# gamma
# --------------------------------------------------------------------------

def check_gamma_fsum(impl, w_bits):
    """The exact-sum step equals math.fsum (correctly rounded sum of floats)."""
    vals = np.abs(bf16_to_f64(w_bits)).reshape(-1)
    d = math.fsum(vals.tolist())
    expect = np.float32(max(np.float32(d / float(vals.size)), EPS32))
    got = np.float32(impl.absmean_gamma(w_bits))
    assert got == expect, (got, expect)


def check_gamma_bins_exact(impl, w_bits):
    """The per-exponent bins hold the exact sum: sum_e B[e] * 2**(e-1) equals
    sum |w| * 2**133 computed from the hardware-widened values."""
    bins = impl.gamma_bins(w_bits)
    total = sum(int(bins[e]) << (e - 1) for e in range(1, 255))
    assert total == exact_abs_sum_int(w_bits)


def check_gamma_exact_mean(impl, w_bits):
    """gamma is the correctly rounded fp32 mean |w| (floored at 1e-5), up to
    the double rounding fp64 -> fp32, which may only matter when the exact
    mean lies within 2**-50 (relative) of an fp32 rounding midpoint."""
    s = Fraction(exact_abs_sum_int(w_bits), 2 ** 133)
    mean = s / int(np.asarray(w_bits).size)
    ref = fraction_to_f32_rne(mean)
    ref = np.float32(max(ref, EPS32))
    got = np.float32(impl.absmean_gamma(w_bits))
    if got != ref:
        # allowed only at a near-tie of the fp32 rounding
        lo, hi = sorted([Fraction(float(got)), Fraction(float(ref))])
        mid = (lo + hi) / 2
        assert abs(mean - mid) <= mean * Fraction(1, 2 ** 50), (got, ref)


def check_gamma_constant(impl):
    """Closed form: a constant tensor w = c has gamma = |c| (|c| >= 1e-5)."""
    for val in [0.02, -0.02, 1.0, 3.5, -0.0078125, 1e-3, 0.50390625, 255.0, 2.0 ** -20]:
        b = (np.array([val], dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
        c = bf16_to_f64(b)[0]
        for shape in [(1, 8), (3, 16), (7, 64)]:
            w = np.full(shape, b[0], dtype=np.uint16)
            g = np.float32(impl.absmean_gamma(w))
            assert g == np.float32(max(abs(c), 1e-5)), (val, shape, g)


def check_gamma_floor(impl):
    """All-zero and all-tiny tensors hit the 1e-5 floor."""
    assert np.float32(impl.absmean_gamma(np.zeros((4, 16), np.uint16))) == EPS32
    neg0 = np.full((4, 16), 0x8000, np.uint16)
    assert np.float32(impl.absmean_gamma(neg0)) == EPS32
    tiny = np.full((2, 8), 0x0001, np.uint16)          # smallest subnormal, 2**-133
    assert np.float32(impl.absmean_gamma(tiny)) == EPS32


def check_gamma_subnormal_scale(impl):
    """Subnormal bf16 magnitudes are weighted correctly (exact mean)."""
    rng = np.random.default_rng(5)
    w = rng.integers(0, 0x0080, size=(3, 32)).astype(np.uint16)  # subnormals only
    check_gamma_bins_exact(impl, w)
    w[0, 0] = 0x3F80                                             # plus one 1.0
    check_gamma_bins_exact(impl, w)
    check_gamma_exact_mean(impl, w)
    check_gamma_fsum(impl, w)


def check_gamma_gaussian(impl):
    """E|w| = sigma*sqrt(2/pi) for w ~ N(0, sigma^2): within 1% at 1M samples."""
    rng = np.random.default_rng(11)
    x = (rng.standard_normal(1 << 20).astype(np.float32) * np.float32(0.02))
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)   # truncation: no method code
    g = float(impl.absmean_gamma(bits.reshape(1024, 1024)))
    assert abs(g / (0.02 * math.sqrt(2 / math.pi)) - 1) < 0.01, g


# --------------------------------------------------------------------------
# mask
# --------------------------------------------------------------------------

def _bits_of_decimal(tokens):
    vals = np.array([float(t) for t in tokens], dtype=np.float32)
    return (vals.view(np.uint32) >> 16).astype(np.uint16)


def check_mask_hand(impl):
    """Hand-worked groups (tests/golden/mask_hand.txt)."""
    for (nm, ws, kept) in read_table("mask_hand.txt"):
        n, m = int(nm[0]), int(nm[1])
        w = _bits_of_decimal(ws)
        assert np.all(bf16_to_f64(w) == np.array([float(t) for t in ws])), ws
        mask = np.asarray(impl.nm_mask(w.reshape(1, -1), n, m)).reshape(-1)
        assert sorted(np.nonzero(mask)[0].tolist()) == [int(k) for k in kept], (nm, ws, mask)


def bruteforce_mask(vals: np.ndarray, n: int, m: int) -> np.ndarray:
    """Enumerate every n-subset of each group: keep the subset of largest exact
    |w| sum; among equal sums the lexicographically smallest index tuple."""
    rows, k = vals.shape
    keep = np.zeros((rows, k), dtype=bool)
    for r in range(rows):
        for g0 in range(0, k, m):
            mags = [abs(Fraction(float(v))) for v in vals[r, g0:g0 + m]]
            best = None
            for sub in itertools.combinations(range(m), n):
                key = (-sum(mags[i] for i in sub), sub)
                if best is None or key < best:
                    best = key
            for i in best[1]:
                keep[r, g0 + i] = True
    return keep


def check_mask_bruteforce(impl, seed=0):
    """Random tie-heavy groups against brute force over all C(m, n) subsets."""
    rng = np.random.default_rng(seed)
    palette = np.array([0.0, -0.0, 0.25, -0.25, 0.5, -0.5, 0.375, 1.0, -1.0, 2.0 ** -130],
                       dtype=np.float32)
    for (n, m) in [(2, 4), (1, 4), (3, 4), (4, 8), (6, 8), (8, 8), (8, 16), (2, 8)]:
        k = m * 3
        vals = rng.choice(palette, size=(4, k))
        bits = (vals.view(np.uint32) >> 16).astype(np.uint16)
        got = np.asarray(impl.nm_mask(bits, n, m))
        ref = bruteforce_mask(bf16_to_f64(bits), n, m)
        assert np.array_equal(got, ref), (n, m)


def check_mask_invariants(impl, w_bits, n, m):
    """Exactly n kept per group, and every kept |w| >= every pruned |w| in its
    group (the per-block threshold t = |w|_(N+1) of Figure 6)."""
    mask = np.asarray(impl.nm_mask(w_bits, n, m))
    rows, k = w_bits.shape
    mg = mask.reshape(rows, k // m, m)
    assert np.all(mg.sum(-1) == n)
    a = np.abs(bf16_to_f64(w_bits)).reshape(rows, k // m, m)
    kept_min = np.where(mg, a, np.inf).min(-1)
    pruned_max = np.where(mg, -np.inf, a).max(-1)
    assert np.all(kept_min >= pruned_max)


# --------------------------------------------------------------------------
# codes
# --------------------------------------------------------------------------

def check_codes_exact(impl, w_bits, n, m):
    """Codes against the exact ratio |w|/gamma: 0 when |w|/gamma <= 1/2,
    sign(w) when |w|/gamma > 1/2 + 2**-25 (beyond one fp32 rounding of the
    quotient); pruned positions are 0. Half-even rint puts 1/2 itself at 0."""
    g = np.float32(impl.absmean_gamma(w_bits))
    mask = np.asarray(impl.nm_mask(w_bits, n, m))
    c = np.asarray(impl.ternary_codes(w_bits, g, mask)).astype(np.int64)
    w = bf16_to_f64(w_bits)
    a = np.abs(w)
    gg = float(g)
    assert np.all(np.isin(c, [-1, 0, 1]))
    assert np.all(c[~mask] == 0)
    zero_zone = 2.0 * a <= gg                          # exact in fp64
    one_zone = a > gg * (0.5 + 2.0 ** -25)             # exact in fp64 (<= 50-bit product)
    km = mask & zero_zone
    assert np.all(c[km] == 0)
    ko = mask & one_zone
    assert np.all(c[ko] == np.sign(w[ko]).astype(np.int64))


def check_codes_zero_fraction(impl):
    """Dense absmean ternary of N(0, sigma^2): P(code = 0) = P(|z| <= sqrt(2/pi)/2)
    = erf(1/(2 sqrt(pi))) = 0.3101..., within 0.5%."""
    rng = np.random.default_rng(7)
    x = rng.standard_normal((512, 2048)).astype(np.float32) * np.float32(0.02)
    bits = (x.view(np.uint32) >> 16).astype(np.uint16)
    g = impl.absmean_gamma(bits)
    mask = np.ones(bits.shape, dtype=bool)
    c = np.asarray(impl.ternary_codes(bits, g, mask))
    frac = float(np.mean(c == 0))
    expect = math.erf(1.0 / (2.0 * math.sqrt(math.pi)))
    assert abs(frac - expect) < 0.005, (frac, expect)


def check_codes_constant(impl):
    """Closed form: a constant tensor c != 0 quantizes to sign(c) everywhere."""
    for val, code in [(0.02, 1), (-0.5, -1), (3.0, 1)]:
        b = _bits_of_decimal([repr(val)])[0]
        w = np.full((2, 16), b, dtype=np.uint16)
        g = impl.absmean_gamma(w)
        c = np.asarray(impl.ternary_codes(w, g, np.ones(w.shape, bool)))
        assert np.all(c == code)
    # Exact tie: half of the entries 0.25 and half 0.75 gives gamma = 0.5, so
    # 0.25/gamma = 0.5 exactly and rint (ties to even) yields 0; 0.75/gamma =
    # 1.5 rounds to 2 and clamps to 1.
    w = np.array([[0.25, -0.75, 0.75, -0.25] * 4], dtype=np.float32)
    bits = (w.view(np.uint32) >> 16).astype(np.uint16)
    g = impl.absmean_gamma(bits)
    assert np.float32(g) == np.float32(0.5)
    c = np.asarray(impl.ternary_codes(bits, g, np.ones(bits.shape, bool)))
    assert c.tolist() == [[0, -1, 1, 0] * 4]


# --------------------------------------------------------------------------
# packing
# --------------------------------------------------------------------------

def loop_pack(dense, mask, n, m):
    """Plain per-element loops over the canonical layout."""
    rows, k = dense.shape
    kept = k * n // m
    cstride = -(-((kept + 3) // 4) // 16) * 16
    mstride = 0 if n == m else -(-((k + 7) // 8) // 16) * 16
    cb = np.zeros((rows, cstride), np.uint8)
    mb = np.zeros((rows, mstride), np.uint8)
    enc = {0: 0, 1: 1, -1: 3}
    for r in range(rows):
        j = 0
        for kk in range(k):
            if mask[r, kk]:
                cb[r, j // 4] |= enc[int(dense[r, kk])] << (2 * (j % 4))
                j += 1
                if n != m:
                    mb[r, kk // 8] |= 1 << (kk % 8)
    return cb, mb


def check_pack_hand(impl):
    """Hand-worked bytes (tests/golden/pack_hand.txt)."""
    for (hdr, codes, cbytes, mbytes) in read_table("pack_hand.txt"):
        n, m, k = (int(v) for v in hdr)
        mask = np.array([[c != "." for c in codes]])
        dense = np.array([[0 if c == "." else int(c) for c in codes]], dtype=np.int8)
        cb, mb = impl.pack_weights(dense, mask, n, m)
        want_c = [int(h, 16) for h in cbytes]
        assert cb.shape[1] % 16 == 0
        assert cb[0, :len(want_c)].tolist() == want_c, (hdr, cb[0, :4])
        assert np.all(cb[0, len(want_c):] == 0)
        if mbytes == ["-"]:
            assert mb.size == 0
        else:
            want_m = [int(h, 16) for h in mbytes]
            assert mb[0, :len(want_m)].tolist() == want_m
            assert np.all(mb[0, len(want_m):] == 0)
        d2, m2 = impl.unpack_weights(cb, mb, k, n, m)
        assert np.array_equal(d2, dense) and np.array_equal(m2, mask)


def check_pack_random(impl, seed=1):
    """Vectorized packing equals plain loops, and unpack(pack(x)) == x."""
    rng = np.random.default_rng(seed)
    for (n, m) in [(2, 4), (4, 8), (6, 8), (8, 16), (8, 8), (1, 4), (3, 8)]:
        for k in [m * 4, 128, 200 if 200 % m == 0 else 192]:
            rows = 5
            mask = np.zeros((rows, k), bool)
            for r in range(rows):
                for g0 in range(0, k, m):
                    mask[r, g0 + rng.choice(m, n, replace=False)] = True
            dense = rng.integers(-1, 2, size=(rows, k)).astype(np.int8)
            dense[~mask] = 0
            cb, mb = impl.pack_weights(dense, mask, n, m)
            rcb, rmb = loop_pack(dense, mask, n, m)
            assert np.array_equal(cb, rcb) and np.array_equal(mb, rmb), (n, m, k)
            d2, m2 = impl.unpack_weights(cb, mb, k, n, m)
            assert np.array_equal(d2, dense) and np.array_equal(m2, mask)


# --------------------------------------------------------------------------
# activations
# --------------------------------------------------------------------------

def check_acts(impl, x_bits):
    """Per-token absmax INT8: s_t = max|x| (floored), |q| <= 127, the absmax
    element maps to +-127, |x - q s/127| <= s/254 (+1e-6 relative), and q is
    the exact rounding of x*127/s wherever that product is farther than
    2**-15 from a half-integer (beyond the fp32 roundings of the scale)."""
    q, s = impl.quantize_acts(x_bits)
    q = np.asarray(q).astype(np.int64)
    s = np.asarray(s, dtype=np.float32)
    x = bf16_to_f64(x_bits)
    t, k = x.shape
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(s.astype(np.float64), np.maximum(amax, float(EPS32)))
    assert np.all(np.abs(q) <= 127)
    for r in range(t):
        if amax[r] > 0:
            i = int(np.argmax(np.abs(x[r])))
            assert abs(q[r, i]) == 127 and np.sign(q[r, i]) == np.sign(x[r, i])
    sd = s.astype(np.float64)[:, None]
    assert np.all(np.abs(x - q * sd / 127.0) <= sd / 254.0 * (1 + 1e-6) + 1e-30)
    exact = x * 127.0 / sd
    frac = np.abs(exact - np.floor(exact) - 0.5)
    safe = frac > 2.0 ** -15
    ref = np.floor(exact + 0.5)
    assert np.all(q[safe] == ref[safe])


def check_acts_zero_row(impl):
    x = np.zeros((2, 64), np.uint16)
    x[1, 5] = 0x3F80   # 1.0
    q, s = impl.quantize_acts(x)
    assert np.float32(s[0]) == EPS32 and np.all(np.asarray(q)[0] == 0)
    assert np.float32(s[1]) == np.float32(1.0) and int(np.asarray(q)[1, 5]) == 127


# --------------------------------------------------------------------------
# contraction and dequantization
# --------------------------------------------------------------------------

def check_acc_bruteforce(impl, seed=2):
    """acc[t, n] = sum_k xq[t, k] * code[n, k] by plain Python loops."""
    rng = np.random.default_rng(seed)
    for (t, k, nn) in [(1, 8, 3), (3, 16, 5), (4, 32, 7)]:
        xq = rng.integers(-127, 128, size=(t, k)).astype(np.int8)
        codes = rng.integers(-1, 2, size=(nn, k)).astype(np.int8)
        acc = np.asarray(impl.bitlinear_acc(xq, codes))
        assert acc.shape == (t, nn)
        for i in range(t):
            for j in range(nn):
                ref = 0
                for kk in range(k):
                    ref += int(xq[i, kk]) * int(codes[j, kk])
                assert int(acc[i, j]) == ref


def check_acc_extremes(impl):
    """Largest |acc|: all +-127 against all-ones codes gives +-127*K."""
    k = 11008
    xq = np.full((2, k), 127, np.int8)
    xq[1] = -127
    codes = np.ones((3, k), np.int8)
    codes[2] = -1
    acc = np.asarray(impl.bitlinear_acc(xq, codes))
    assert acc[0, 0] == 127 * k and acc[1, 0] == -127 * k and acc[0, 2] == -127 * k


def check_dequant(impl, seed=3):
    """y is the correctly rounded bf16 of acc * gamma * s_t / 127 (exact
    rationals), including a hand-made exact tie."""
    rng = np.random.default_rng(seed)
    acc = rng.integers(-200000, 200000, size=(3, 6)).astype(np.int32)
    acc[0, 0] = 0
    s = np.array([1.0, 3.5, 20.25], dtype=np.float32)
    g = np.float32(0.0159912109375)
    y = np.asarray(impl.dequant_bf16(acc, s, g))
    for i in range(3):
        for j in range(6):
            exact = Fraction(int(acc[i, j])) * Fraction(float(g)) * Fraction(float(s[i])) / 127
            ref = fraction_to_bf16_value(exact)
            got = Fraction(float(bf16_to_f64(np.array([y[i, j]], np.uint16))[0]))
            assert got == ref, (i, j, got, ref)
    # exact ties: 1 + 2**-8 and 1 + 3*2**-8 are midpoints between bf16 neighbours
    t1 = np.asarray(impl.bf16_bits_from_f64_rne(np.array([1 + 2.0 ** -8, 1 + 3 * 2.0 ** -8, -(1 + 2.0 ** -8)])))
    assert t1.tolist() == [0x3F80, 0x3F82, 0xBF80]


def check_layer_vs_float(impl, w_bits, x_bits, n, m):
    """End to end: Y agrees with the fp64 product of the dequantized operands
    (x ~ q s/127, w ~ code gamma) to within bf16 rounding (2**-8 relative),
    and the packed weights survive unpacking."""
    cb, mb, g, mask, dense = _impl_quantize_weights(impl, w_bits, n, m)
    k = w_bits.shape[1]
    d2, m2 = impl.unpack_weights(cb, mb, k, n, m)
    assert np.array_equal(d2, dense) and np.array_equal(m2, mask)
    q, s = impl.quantize_acts(x_bits)
    acc = np.asarray(impl.bitlinear_acc(q, dense)).astype(np.float64)
    y = bf16_to_f64(np.asarray(impl.dequant_bf16(acc.astype(np.int32), s, g)))
    xr = np.asarray(q).astype(np.float64) * (np.asarray(s, np.float64)[:, None] / 127.0)
    wr = dense.astype(np.float64) * float(g)
    ref = xr @ wr.T
    noise = 1e-12 * float(np.abs(ref).max() + 1e-300)   # fp64 rounding of the float product
    assert np.all(np.abs(y - ref) <= np.abs(ref) * 2.0 ** -8 + noise)


# ---- entropy-tight packed format -------------------------------------------

def check_entropy_accounting(impl):
    """'From 2:4 to 8:16 sparsity patterns ...', Abstract: the masks of 2:4 and
    8:16 cost 0.75 and 0.875 bits per element, i.e. ceil(log2 C(m, n)) / m."""
    assert impl.mask_index_bits(2, 4) / 4 == 0.75
    assert impl.mask_index_bits(8, 16) / 16 == 0.875
    for (n, m) in [(1, 4), (2, 4), (6, 8), (8, 16), (8, 8)]:
        # a group word holds every (pattern, values) pair and no more bits than that needs
        total = math.comb(m, n) * 3 ** n
        assert (1 << impl.entropy_group_bits(n, m)) >= total
        assert (1 << (impl.entropy_group_bits(n, m) - 1)) < total


def check_entropy_hand(impl):
    """The worked example of tests/golden/entropy_hand.txt (2:4, K = 8)."""
    text = (Path(__file__).parent / "golden" / "entropy_hand.txt").read_text().splitlines()
    rows = {ln.split(":")[0]: ln.split(":")[1].split() for ln in text if ln and not ln.startswith("#")}
    dense = np.array([[int(v) for v in rows["codes"]]], np.int8)
    mask = np.array([[v == "1" for v in rows["mask"]]])
    want = [int(v, 16) for v in rows["bytes"]]
    packed = impl.entropy_pack(mask, dense, 2, 4)
    assert list(packed[0, :len(want)]) == want and not packed[0, len(want):].any()


def check_entropy_bijection(impl, n=2, m=4):
    """Every (keep pattern, kept values) of a group gets its own word below 2^bits."""
    bits = impl.entropy_group_bits(n, m)
    seen = set()
    for offs in itertools.combinations(range(m), n):
        for digits in itertools.product((-1, 0, 1), repeat=n):
            mask = np.zeros((1, m), bool)
            dense = np.zeros((1, m), np.int8)
            for j, d in zip(offs, digits):
                mask[0, j] = True
                dense[0, j] = d
            word = int.from_bytes(bytes(impl.entropy_pack(mask, dense, n, m)[0]), "little")
            assert word < (1 << bits)
            seen.add(word)
            d2, m2 = impl.entropy_unpack(impl.entropy_pack(mask, dense, n, m), m, n, m)
            assert np.array_equal(d2, dense) and np.array_equal(m2, mask)
    assert len(seen) == math.comb(m, n) * 3 ** n


# ---- backward (straight-through estimator) ----------------------------------
#
# "Microsoft BitNet 1.58 ...", section "Training with the Straight-Through
# Estimator": the quantizer is the identity in the backward pass, so the
# gradients are those of the bilinear map Y = Xd Wd^T of the dequantized
# operands Xd = Xq s_t / 127 and Wd = gamma C that the forward multiplies.

def _random_bf16_bits(rng, shape):
    """Normal bf16 numbers of both signs, magnitudes 2**-7 .. 2**8."""
    e = rng.integers(120, 136, size=shape)
    mant = rng.integers(0, 128, size=shape)
    sign = rng.integers(0, 2, size=shape) << 15
    return (sign | (e << 7) | mant).astype(np.uint16)


def _bf16_value(bits) -> Fraction:
    return Fraction(float(bf16_to_f64(np.array([bits], np.uint16))[0]))


def check_ste_grad_x_exact(impl, seed=41):
    """dX[t, k] = sum_n dY[t, n] gamma C[n, k], exact rationals, then one
    correct bf16 rounding; non-square so that a transposed operand fails."""
    rng = np.random.default_rng(seed)
    t, n_out, k = 3, 5, 12
    dy = _random_bf16_bits(rng, (t, n_out))
    c = rng.integers(-1, 2, size=(n_out, k)).astype(np.int8)
    g = np.float32(0.0137)
    got = np.asarray(impl.ste_grad_x(dy, c, g))
    assert got.shape == (t, k)
    for i in range(t):
        for j in range(k):
            exact = sum((_bf16_value(dy[i, nn]) * Fraction(float(g)) * int(c[nn, j]) for nn in range(n_out)),
                        Fraction(0))
            assert _bf16_value(got[i, j]) == fraction_to_bf16_value(exact), (i, j)


def check_ste_grad_w_exact(impl, seed=42):
    """dW[n, k] = sum_t dY[t, n] Xq[t, k] s_t / 127, exact rationals, then one
    correct bf16 rounding."""
    rng = np.random.default_rng(seed)
    t, n_out, k = 4, 3, 7
    dy = _random_bf16_bits(rng, (t, n_out))
    q = rng.integers(-127, 128, size=(t, k)).astype(np.int8)
    sc = np.array([0.5, 3.25, 17.0, 1e-5], dtype=np.float32)
    got = np.asarray(impl.ste_grad_w(dy, q, sc))
    assert got.shape == (n_out, k)
    for nn in range(n_out):
        for j in range(k):
            exact = sum((_bf16_value(dy[i, nn]) * int(q[i, j]) * Fraction(float(sc[i])) / 127 for i in range(t)),
                        Fraction(0))
            assert _bf16_value(got[nn, j]) == fraction_to_bf16_value(exact), (nn, j)


def check_ste_one_hot(impl):
    """Closed forms: a one-hot dY at (t0, n0) gives dX[t0] = gamma C[n0] and
    dW[n0] = Xq[t0] s_t0 / 127, every other row zero."""
    t, n_out, k = 2, 3, 8
    c = np.array([[1, 0, -1, 1, 0, 0, -1, 1], [0, 1, 1, 0, -1, 1, 0, 0], [-1, -1, 0, 0, 1, 1, 1, 0]], np.int8)
    g = np.float32(0.25)
    q = np.array([[3, -127, 0, 64, 5, -5, 100, 1], [1, 2, 3, 4, 5, 6, 7, 8]], np.int8)
    sc = np.array([12.7, 0.127], dtype=np.float32)
    dy = np.zeros((t, n_out), np.uint16)
    dy[1, 2] = 0x3F80                                    # 1.0
    dx = bf16_to_f64(np.asarray(impl.ste_grad_x(dy, c, g)))
    assert np.all(dx[0] == 0) and np.array_equal(dx[1], 0.25 * c[2].astype(np.float64))
    dw = np.asarray(impl.ste_grad_w(dy, q, sc))
    assert np.all(bf16_to_f64(dw[:2]) == 0)
    for j in range(k):
        assert _bf16_value(dw[2, j]) == fraction_to_bf16_value(int(q[1, j]) * Fraction(float(sc[1])) / 127)


def check_ste_finite_difference(impl, seed=43):
    """The loss L = sum dY * (Xd Wd^T) is bilinear, so raising one entry of
    Xd (or Wd) by 1 changes L by exactly the matching gradient entry."""
    rng = np.random.default_rng(seed)
    t, n_out, k = 3, 4, 16
    dy = _random_bf16_bits(rng, (t, n_out))
    c = rng.integers(-1, 2, size=(n_out, k)).astype(np.int8)
    g = np.float32(0.021)
    q = rng.integers(-127, 128, size=(t, k)).astype(np.int8)
    sc = rng.uniform(0.5, 8.0, size=t).astype(np.float32)
    G = bf16_to_f64(dy)
    xd = q.astype(np.float64) * (sc.astype(np.float64)[:, None] / 127.0)
    wd = float(g) * c.astype(np.float64)

    def loss(a, b):
        return float(np.einsum("tn,tk,nk->", G, a, b))

    dx = bf16_to_f64(np.asarray(impl.ste_grad_x(dy, c, g)))
    dw = bf16_to_f64(np.asarray(impl.ste_grad_w(dy, q, sc)))
    base = loss(xd, wd)
    tol = 1e-9 * (1.0 + abs(base))
    for (i, j) in [(0, 0), (1, 7), (2, 15), (0, 9)]:
        xp = xd.copy()
        xp[i, j] += 1.0
        fd = loss(xp, wd) - base
        assert abs(dx[i, j] - fd) <= 2.0 ** -8 * abs(fd) + tol, (i, j)
    for (nn, j) in [(0, 0), (3, 5), (2, 11), (1, 15)]:
        wp = wd.copy()
        wp[nn, j] += 1.0
        fd = loss(xd, wp) - base
        assert abs(dw[nn, j] - fd) <= 2.0 ** -8 * abs(fd) + tol, (nn, j)


def check_ste_matches_forward(impl, w_bits, x_bits, n, m, seed=44):
    """The backward linearizes the forward the oracle computes: for the
    bilinear Y = Xd Wd^T, sum(Xd * dX) = sum(dY * Y) = sum(Wd * dW), with Y
    from the forward's exact accumulators (acc gamma s_t / 127). Masked
    codes, gamma and the dequantized activations must all be the forward's."""
    rng = np.random.default_rng(seed)
    cb, mb, g, mask, dense = _impl_quantize_weights(impl, w_bits, n, m)
    q, sc = impl.quantize_acts(x_bits)
    acc = np.asarray(impl.bitlinear_acc(q, dense)).astype(np.float64)
    y = acc * float(g) * (np.asarray(sc, np.float64)[:, None] / 127.0)
    dy = _random_bf16_bits(rng, y.shape)
    G = bf16_to_f64(dy)
    dx = bf16_to_f64(np.asarray(impl.ste_grad_x(dy, dense, g)))
    dw = bf16_to_f64(np.asarray(impl.ste_grad_w(dy, q, sc)))
    xd = np.asarray(q).astype(np.float64) * (np.asarray(sc, np.float64)[:, None] / 127.0)
    wd = dense.astype(np.float64) * float(g)
    gy = float(np.sum(G * y))
    # each gradient entry is within 2**-8 of its exact value, so each sum is
    # within 2**-8 of sum |operand| |gradient|
    assert abs(float(np.sum(xd * dx)) - gy) <= 2.0 ** -8 * float(np.sum(np.abs(xd) * np.abs(dx))) + 1e-9 * (1 + abs(gy))
    assert abs(float(np.sum(wd * dw)) - gy) <= 2.0 ** -8 * float(np.sum(np.abs(wd) * np.abs(dw))) + 1e-9 * (1 + abs(gy))
