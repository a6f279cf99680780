"""Plant plausible mistakes in copies of the oracle (CPU only) and check that
at least one pin catches each. This is what makes the pins worth trusting."""

import types

import numpy as np
import pytest

import oracle
import oracle.sbn_oracle as O
import pins
from sparse_linear_layers_fwd_b200 import synth


def _impl(**overrides):
    ns = types.SimpleNamespace(**{k: getattr(O, k) for k in O.__all__})
    for k, v in overrides.items():
        setattr(ns, k, v)
    return ns


# ---- mutants ---------------------------------------------------------------

def bins_no_subnormal(w_bits):
    mag = np.asarray(w_bits, np.uint16).reshape(-1) & np.uint16(0x7FFF)
    e = (mag >> 7).astype(np.int64)
    s = (mag & 0x7F).astype(np.int64) + 128          # mistake: 128 added to subnormals too
    bins = [0] * 255
    for eb in np.unique(np.maximum(e, 1)):
        bins[int(eb)] = int(s[np.maximum(e, 1) == eb].sum())
    return np.array(bins, dtype=object)


def gamma_no_subnormal(w_bits):
    return O.gamma_from_bins(bins_no_subnormal(w_bits), np.asarray(w_bits).size)


def gamma_exponent_off_by_one(w_bits):
    bins = O.gamma_bins(w_bits)
    shifted = [0] + [int(b) for b in bins[2:]] + [0]    # mistake: every bin one exponent low
    return O.gamma_from_bins(shifted, np.asarray(w_bits).size)


def gamma_signed_mean(w_bits):
    x = O.bf16_bits_to_f32(w_bits).astype(np.float64)
    return np.float32(max(np.float32(abs(x.mean())), O.EPS))    # mistake: mean of w, not |w|


def gamma_of_masked(w_bits):
    mask = O.nm_mask(w_bits, 2, 4) if np.asarray(w_bits).shape[1] % 4 == 0 else np.ones(np.shape(w_bits), bool)
    x = np.abs(O.bf16_bits_to_f32(w_bits).astype(np.float64))
    return np.float32(max(np.float32(x[mask].mean()), O.EPS))   # mistake: gamma after masking


def gamma_rms(w_bits):
    x = O.bf16_bits_to_f32(w_bits).astype(np.float64)
    return np.float32(max(np.float32(np.sqrt((x * x).mean())), O.EPS))


def mask_tie_high(w_bits, n, m):
    rows, k = np.asarray(w_bits).shape
    mag = (np.asarray(w_bits) & 0x7FFF).astype(np.int64).reshape(rows, k // m, m)
    rev = mag[..., ::-1]
    order = np.argsort(-rev, axis=-1, kind="stable")
    keep = np.zeros(mag.shape, bool)
    np.put_along_axis(keep, (m - 1) - order[..., :n], True, axis=-1)   # ties keep the HIGHER index
    return keep.reshape(rows, k)


def mask_signed(w_bits, n, m):
    rows, k = np.asarray(w_bits).shape
    v = O.bf16_bits_to_f32(w_bits).reshape(rows, k // m, m)     # mistake: ranks w, not |w|
    order = np.argsort(-v, axis=-1, kind="stable")
    keep = np.zeros(v.shape, bool)
    np.put_along_axis(keep, order[..., :n], True, axis=-1)
    return keep.reshape(rows, k)


def mask_smallest(w_bits, n, m):
    rows, k = np.asarray(w_bits).shape
    mag = (np.asarray(w_bits) & 0x7FFF).astype(np.int64).reshape(rows, k // m, m)
    order = np.argsort(mag, axis=-1, kind="stable")             # mistake: keeps the smallest
    keep = np.zeros(mag.shape, bool)
    np.put_along_axis(keep, order[..., :n], True, axis=-1)
    return keep.reshape(rows, k)


def mask_along_rows(w_bits, n, m):
    wt = np.ascontiguousarray(np.asarray(w_bits).T)              # mistake: groups along N_out
    if wt.shape[1] % m:
        return O.nm_mask(w_bits, n, m)
    return O.nm_mask(wt, n, m).T


def codes_multiply(w_bits, gamma, mask):
    w = O.bf16_bits_to_f32(w_bits)
    c = np.clip(np.rint(w * np.float32(gamma)), -1, 1).astype(np.int8)   # mistake: multiply
    c[~mask] = 0
    return c


def codes_half_up(w_bits, gamma, mask):
    w = O.bf16_bits_to_f32(w_bits)
    c = np.clip(np.floor(w / np.float32(gamma) + np.float32(0.5)), -1, 1).astype(np.int8)
    c[~mask] = 0
    return c


def codes_sign_flip(w_bits, gamma, mask):
    return (-O.ternary_codes(w_bits, gamma, mask)).astype(np.int8)


def codes_unmasked(w_bits, gamma, mask):
    return O.ternary_codes(w_bits, gamma, np.ones(np.shape(mask), bool))   # mistake: ignores mask


def pack_reversed_fields(codes, mask, n, m):
    cb, mb = O.pack_weights(codes, mask, n, m)
    f = [(cb >> (2 * i)) & 3 for i in range(4)]
    cb2 = (f[3] | (f[2] << 2) | (f[1] << 4) | (f[0] << 6)).astype(np.uint8)
    return cb2, mb


def pack_minus_as_10(codes, mask, n, m):
    cb, mb = O.pack_weights(codes, mask, n, m)
    out = cb.copy()
    for i in range(4):
        fld = (cb >> (2 * i)) & 3
        out = np.where(fld == 3, out ^ np.uint8(1 << (2 * i)), out).astype(np.uint8)
    return out, mb


def pack_meta_msb_first(codes, mask, n, m):
    cb, mb = O.pack_weights(codes, mask, n, m)
    if n != m:
        bits = np.packbits(mask, axis=1, bitorder="big")
        mb = mb.copy()
        mb[:, :bits.shape[1]] = bits
    return cb, mb


def acts_scale_128(x_bits):
    x = O.bf16_bits_to_f32(x_bits)
    s = np.maximum(np.abs(x).max(1), O.EPS).astype(np.float32)
    q = np.clip(np.rint(x * (np.float32(128) / s)[:, None]), -127, 127).astype(np.int8)
    return q, s


def acts_per_channel(x_bits):
    x = O.bf16_bits_to_f32(x_bits)
    s = np.maximum(np.abs(x).max(0), O.EPS).astype(np.float32)    # mistake: per channel
    q = np.clip(np.rint(x * (np.float32(127) / s)[None, :]), -127, 127).astype(np.int8)
    return q, np.maximum(np.abs(x).max(1), O.EPS).astype(np.float32)


def acts_truncate(x_bits):
    x = O.bf16_bits_to_f32(x_bits)
    s = np.maximum(np.abs(x).max(1), O.EPS).astype(np.float32)
    q = np.clip(np.trunc(x * (np.float32(127) / s)[:, None]), -127, 127).astype(np.int8)
    return q, s


def acc_transposed_codes(xq, dense):
    d = dense[::-1]                                   # mistake: wrong row index of W
    return O.bitlinear_acc(xq, np.ascontiguousarray(d))


def acc_dropped_last_k(xq, dense):
    return O.bitlinear_acc(xq[:, :-1], dense[:, :-1])   # mistake: dropped term


def dequant_no_s(acc, s, gamma):
    return O.dequant_bf16(acc, np.full_like(s, 127.0), gamma)


def dequant_truncate(acc, s, gamma):
    y = acc.astype(np.float64) * float(gamma) * (s.astype(np.float64)[:, None] / 127)
    return (np.asarray(y, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _entropy_pack_with(rank_fn=None, digit_order=1, bits_fn=None):
    """entropy_pack with one step replaced (for the mutants below)."""
    def pack(mask, dense, n, m):
        rows, k = mask.shape
        bits = (bits_fn or O.entropy_group_bits)(n, m)
        out = np.zeros((rows, O.entropy_row_bytes(k, n, m)), np.uint8)
        for r in range(rows):
            stream = 0
            for g in range(k // m):
                offs = [j for j in range(m) if mask[r, g * m + j]]
                word = (rank_fn or O.colex_rank)(offs) * 3 ** n
                for i, j in enumerate(offs[::digit_order]):
                    word += (int(dense[r, g * m + j]) + 1) * 3 ** i
                stream |= word << (g * bits)
            nbytes = (k // m * bits + 7) // 8
            out[r, :nbytes] = np.frombuffer(stream.to_bytes(nbytes, "little"), np.uint8)
        return out
    return pack


def _lex_rank(offs):
    import itertools as it
    m = 4 if max(offs, default=0) < 4 else 16
    return list(it.combinations(range(m), len(offs))).index(tuple(offs))


def ste_dx_no_gamma(dy_bits, dense_codes, gamma):
    return O.ste_grad_x(dy_bits, dense_codes, np.float32(1.0))       # mistake: gamma dropped


def ste_dx_transposed(dy_bits, dense_codes, gamma):
    dy = O.bf16_bits_to_f32(dy_bits).astype(np.float64)
    return O.bf16_bits_from_f64_rne(dy @ (float(gamma) * dense_codes.astype(np.float64)).T)


def ste_dx_sign_flip(dy_bits, dense_codes, gamma):
    return O.ste_grad_x(dy_bits, -np.asarray(dense_codes), gamma)


def ste_dw_no_127(dy_bits, xq, s):
    return O.ste_grad_w(dy_bits, xq, np.asarray(s, np.float64) * 127.0)   # mistake: Xq s, not Xq s/127


def ste_dw_unscaled(dy_bits, xq, s):
    return O.ste_grad_w(dy_bits, xq, np.full(np.shape(s), 127.0))         # mistake: raw Xq


def ste_dw_transposed_dy(dy_bits, xq, s):
    dy = O.bf16_bits_to_f32(dy_bits).astype(np.float64)
    xd = np.asarray(xq).astype(np.float64) * (np.asarray(s, np.float64)[:, None] / O.Q_ACT)
    return O.bf16_bits_from_f64_rne(dy @ xd.T)


MUTANTS = {
    "gamma_no_subnormal": dict(absmean_gamma=gamma_no_subnormal, gamma_bins=bins_no_subnormal),
    "gamma_exponent_off_by_one": dict(absmean_gamma=gamma_exponent_off_by_one),
    "gamma_signed_mean": dict(absmean_gamma=gamma_signed_mean),
    "gamma_of_masked": dict(absmean_gamma=gamma_of_masked),
    "gamma_rms": dict(absmean_gamma=gamma_rms),
    "mask_tie_high": dict(nm_mask=mask_tie_high),
    "mask_signed": dict(nm_mask=mask_signed),
    "mask_smallest": dict(nm_mask=mask_smallest),
    "mask_along_rows": dict(nm_mask=mask_along_rows),
    "codes_multiply": dict(ternary_codes=codes_multiply),
    "codes_half_up": dict(ternary_codes=codes_half_up),
    "codes_sign_flip": dict(ternary_codes=codes_sign_flip),
    "codes_unmasked": dict(ternary_codes=codes_unmasked),
    "pack_reversed_fields": dict(pack_weights=pack_reversed_fields),
    "pack_minus_as_10": dict(pack_weights=pack_minus_as_10),
    "pack_meta_msb_first": dict(pack_weights=pack_meta_msb_first),
    "acts_scale_128": dict(quantize_acts=acts_scale_128),
    "acts_per_channel": dict(quantize_acts=acts_per_channel),
    "acts_truncate": dict(quantize_acts=acts_truncate),
    "acc_transposed_codes": dict(bitlinear_acc=acc_transposed_codes),
    "acc_dropped_last_k": dict(bitlinear_acc=acc_dropped_last_k),
    "dequant_no_s": dict(dequant_bf16=dequant_no_s),
    "dequant_truncate": dict(dequant_bf16=dequant_truncate),
    "entropy_lex_rank": dict(entropy_pack=_entropy_pack_with(rank_fn=_lex_rank)),
    "entropy_digits_msb_first": dict(entropy_pack=_entropy_pack_with(digit_order=-1)),
    "entropy_bits_undersized": dict(entropy_group_bits=lambda n, m: O.entropy_group_bits(n, m) - 1),
    "ste_dx_no_gamma": dict(ste_grad_x=ste_dx_no_gamma),
    "ste_dx_transposed": dict(ste_grad_x=ste_dx_transposed),
    "ste_dx_sign_flip": dict(ste_grad_x=ste_dx_sign_flip),
    "ste_dw_no_127": dict(ste_grad_w=ste_dw_no_127),
    "ste_dw_unscaled": dict(ste_grad_w=ste_dw_unscaled),
    "ste_dw_transposed_dy": dict(ste_grad_w=ste_dw_transposed_dy),
}


def all_pins(impl):
    """Every pin, in order; returns the names of those that failed."""
    small = synth.layer_small()
    w = synth.latent_weights(64, 256, seed=0)
    wide = np.random.default_rng(3).integers(0, 0x7F7F, size=(16, 64)).astype(np.uint16)
    checks = [
        ("gamma_constant", lambda: pins.check_gamma_constant(impl)),
        ("gamma_floor", lambda: pins.check_gamma_floor(impl)),
        ("gamma_subnormal", lambda: pins.check_gamma_subnormal_scale(impl)),
        ("gamma_exact", lambda: pins.check_gamma_exact_mean(impl, w)),
        ("gamma_exact_wide", lambda: pins.check_gamma_exact_mean(impl, wide)),
        ("gamma_gaussian", lambda: pins.check_gamma_gaussian(impl)),
        ("mask_hand", lambda: pins.check_mask_hand(impl)),
        ("mask_brute", lambda: pins.check_mask_bruteforce(impl)),
        ("mask_inv", lambda: pins.check_mask_invariants(impl, w, 6, 8)),
        ("codes_exact", lambda: pins.check_codes_exact(impl, w, 2, 4)),
        ("codes_zero_frac", lambda: pins.check_codes_zero_fraction(impl)),
        ("codes_constant", lambda: pins.check_codes_constant(impl)),
        ("pack_hand", lambda: pins.check_pack_hand(impl)),
        ("pack_random", lambda: pins.check_pack_random(impl)),
        ("acts", lambda: pins.check_acts(impl, small["x"])),
        ("acts_zero_row", lambda: pins.check_acts_zero_row(impl)),
        ("acc_brute", lambda: pins.check_acc_bruteforce(impl)),
        ("acc_extremes", lambda: pins.check_acc_extremes(impl)),
        ("dequant", lambda: pins.check_dequant(impl)),
        ("layer", lambda: pins.check_layer_vs_float(impl, small["w"], small["x"], 2, 4)),
        ("entropy_accounting", lambda: pins.check_entropy_accounting(impl)),
        ("entropy_hand", lambda: pins.check_entropy_hand(impl)),
        ("entropy_bijection", lambda: pins.check_entropy_bijection(impl)),
        ("ste_dx_exact", lambda: pins.check_ste_grad_x_exact(impl)),
        ("ste_dw_exact", lambda: pins.check_ste_grad_w_exact(impl)),
        ("ste_one_hot", lambda: pins.check_ste_one_hot(impl)),
        ("ste_finite_difference", lambda: pins.check_ste_finite_difference(impl)),
        ("ste_forward", lambda: pins.check_ste_matches_forward(impl, small["w"], small["x"], 2, 4)),
    ]
    failed = []
    for name, fn in checks:
        try:
            fn()
        except (AssertionError, ValueError, IndexError):
            failed.append(name)
    return failed


def test_real_oracle_passes_every_pin():
    assert all_pins(oracle) == []


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    failed = all_pins(_impl(**MUTANTS[name]))
    assert failed, f"mutant {name} passed every pin"
