"""The CPU oracle against its pins (no GPU)."""

import math
from pathlib import Path

import numpy as np
import pytest

import oracle
import pins
from sparse_linear_layers_fwd_b200 import synth


def test_gamma_constant():
    pins.check_gamma_constant(oracle)


def test_gamma_floor():
    pins.check_gamma_floor(oracle)


def test_gamma_subnormals():
    pins.check_gamma_subnormal_scale(oracle)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_gamma_exact_mean_random(seed):
    w = synth.latent_weights(64, 256, seed=seed)
    pins.check_gamma_exact_mean(oracle, w)
    pins.check_gamma_fsum(oracle, w)


def test_gamma_wide_exponent_range():
    rng = np.random.default_rng(3)
    w = rng.integers(0, 0x7F7F, size=(16, 64)).astype(np.uint16)   # finite, any exponent
    w |= (rng.integers(0, 2, size=w.shape).astype(np.uint16) << 15)
    pins.check_gamma_exact_mean(oracle, w)
    pins.check_gamma_fsum(oracle, w)


def test_gamma_gaussian():
    pins.check_gamma_gaussian(oracle)


def test_mask_hand():
    pins.check_mask_hand(oracle)


@pytest.mark.parametrize("seed", [0, 1])
def test_mask_bruteforce(seed):
    pins.check_mask_bruteforce(oracle, seed)


@pytest.mark.parametrize("nm", [(2, 4), (4, 8), (6, 8), (8, 16), (8, 8)])
def test_mask_invariants(nm):
    w = synth.latent_weights(32, 512, seed=4)
    pins.check_mask_invariants(oracle, w, *nm)


@pytest.mark.parametrize("nm", [(2, 4), (6, 8), (8, 16), (8, 8)])
def test_codes_exact(nm):
    w = synth.latent_weights(64, 512, seed=5)
    pins.check_codes_exact(oracle, w, *nm)


def test_codes_zero_fraction():
    pins.check_codes_zero_fraction(oracle)


def test_codes_constant():
    pins.check_codes_constant(oracle)


def test_pack_hand():
    pins.check_pack_hand(oracle)


def test_pack_random():
    pins.check_pack_random(oracle)


def test_acts_layer_small():
    pins.check_acts(oracle, synth.layer_small()["x"])


def test_acts_heavy_tail():
    pins.check_acts(oracle, synth.activations(8, 896, seed=1, heavy_tail_channels=14))


def test_acts_zero_row():
    pins.check_acts_zero_row(oracle)


def test_acc_bruteforce():
    pins.check_acc_bruteforce(oracle)


def test_acc_extremes():
    pins.check_acc_extremes(oracle)


def test_dequant():
    pins.check_dequant(oracle)


@pytest.mark.parametrize("nm", [(2, 4), (6, 8), (8, 8)])
def test_layer_small_vs_float(nm):
    d = synth.layer_small()
    pins.check_layer_vs_float(oracle, d["w"], d["x"], *nm)


def test_sampled_matches_full():
    d = synth.layer_small()
    cb, mb, g, mask, dense = oracle.quantize_weights(d["w"], 2, 4)
    q, s = oracle.quantize_acts(d["x"])
    y, acc = oracle.bitlinear(q, s, cb, mb, g, 256, 2, 4)
    rng = np.random.default_rng(0)
    ti = rng.integers(0, 16, 50)
    ni = rng.integers(0, 256, 50)
    ys, accs = oracle.bitlinear_at(q, s, dense, g, ti, ni)
    assert np.array_equal(accs, acc[ti, ni]) and np.array_equal(ys, y[ti, ni])


def test_layer_small_zero_fraction_reported():
    """Synthetic N(0, 0.02) weights: ~31% ternary zeros before masking, not
    the 42.3% of the trained model in Figure 1 of the Sparse-BitNet page."""
    w = synth.latent_weights(256, 256, seed=0)
    g = oracle.absmean_gamma(w)
    c = oracle.ternary_codes(w, g, np.ones(w.shape, bool))
    assert 0.29 < float(np.mean(c == 0)) < 0.33


# ---- mask flip rate --------------------------------------------------------

def test_mask_flips_brute_force_and_invariants():
    rng = np.random.default_rng(31)
    for (n, m) in [(2, 4), (6, 8), (8, 16), (1, 4)]:
        w1 = rng.integers(0, 0x4000, size=(7, 64)).astype(np.uint16)
        w2 = w1.copy()
        sel = rng.random(w2.shape) < 0.2
        w2[sel] = rng.integers(0, 0x4000, size=int(sel.sum())).astype(np.uint16)
        a, b = oracle.nm_mask(w1, n, m), oracle.nm_mask(w2, n, m)
        # brute force: a plain loop over positions
        brute = 0
        for i in range(a.shape[0]):
            for j in range(a.shape[1]):
                brute += 1 if bool(a[i, j]) != bool(b[i, j]) else 0
        assert oracle.mask_flips(a, b) == brute
        # every group keeps exactly n in both masks: flips come in pairs per group
        per_group = (a != b).reshape(a.shape[0], -1, m).sum(axis=2)
        assert np.all(per_group % 2 == 0)
        assert np.all(per_group <= 2 * min(n, m - n))
        assert oracle.mask_flips(a, a) == 0
        assert oracle.mask_flip_rate(a, b) == brute / a.size


def test_mask_flips_complement_within_2of4_groups():
    # keep {0,1} vs keep {2,3} in every group of four: every position flips
    w1 = np.tile(np.array([0x3F80, 0x3F80, 0x3C00, 0x3C00], np.uint16), (3, 32))
    w2 = np.tile(np.array([0x3C00, 0x3C00, 0x3F80, 0x3F80], np.uint16), (3, 32))
    a, b = oracle.nm_mask(w1, 2, 4), oracle.nm_mask(w2, 2, 4)
    assert oracle.mask_flips(a, b) == a.size
    assert oracle.mask_flip_rate(a, b) == 1.0


# ---- entropy-tight packed format ---------------------------------------------

def test_mask_index_bits_match_the_pages_accounting():
    # "From 2:4 to 8:16 sparsity patterns ...", Abstract: 0.75 vs 0.875 bits/element
    assert oracle.mask_index_bits(2, 4) / 4 == 0.75
    assert oracle.mask_index_bits(8, 16) / 16 == 0.875
    assert oracle.entropy_group_bits(6, 8) == 15           # 28 * 729 = 20412 < 2^15


def test_colex_rank_order_for_2of4():
    order = [(0, 1), (0, 2), (1, 2), (0, 3), (1, 3), (2, 3)]
    for r, offs in enumerate(order):
        assert oracle.colex_rank(list(offs)) == r
        assert oracle.colex_unrank(r, 2, 4) == list(offs)


@pytest.mark.parametrize("nm", [(1, 4), (2, 4), (3, 4), (4, 4), (2, 8), (6, 8)])
def test_entropy_words_are_a_bijection(nm):
    import itertools
    n, m = nm
    bits = oracle.entropy_group_bits(n, m)
    seen = set()
    for offs in itertools.combinations(range(m), n):
        for digits in itertools.product((-1, 0, 1), repeat=n):
            mask = np.zeros((1, m), bool)
            dense = np.zeros((1, m), np.int8)
            for j, d in zip(offs, digits):
                mask[0, j] = True
                dense[0, j] = d
            packed = oracle.entropy_pack(mask, dense, n, m)
            word = int.from_bytes(bytes(packed[0]), "little")
            assert word < (1 << bits)
            seen.add(word)
            d2, m2 = oracle.entropy_unpack(packed, m, n, m)
            assert np.array_equal(d2, dense) and np.array_equal(m2, mask)
    assert len(seen) == math.comb(m, n) * 3 ** n


def test_entropy_hand_example():
    text = (Path(__file__).parent / "golden" / "entropy_hand.txt").read_text().splitlines()
    rows = {ln.split(":")[0]: ln.split(":")[1].split() for ln in text if ln and not ln.startswith("#")}
    dense = np.array([[int(v) for v in rows["codes"]]], np.int8)
    mask = np.array([[v == "1" for v in rows["mask"]]])
    want = [int(v, 16) for v in rows["bytes"]]
    packed = oracle.entropy_pack(mask, dense, 2, 4)
    assert list(packed[0, :len(want)]) == want and not packed[0, len(want):].any()
    assert packed.shape[1] == 16


@pytest.mark.parametrize("nm", [(2, 4), (6, 8), (8, 16), (4, 8), (8, 8), (12, 16)])
def test_entropy_round_trip_on_quantized_layers(nm):
    n, m = nm
    w = synth.latent_weights(9, 256, seed=41, tag=f"ent{nm}")
    cb, mb, gamma, mask, dense = oracle.quantize_weights(w, n, m)
    packed = oracle.entropy_pack(mask, dense, n, m)
    assert packed.shape == (9, oracle.entropy_row_bytes(256, n, m))
    d2, m2 = oracle.entropy_unpack(packed, 256, n, m)
    assert np.array_equal(d2, dense) and np.array_equal(m2, mask)


# ---- backward: straight-through estimator ------------------------------------

def test_ste_grad_x_exact_rationals():
    pins.check_ste_grad_x_exact(oracle)


def test_ste_grad_w_exact_rationals():
    pins.check_ste_grad_w_exact(oracle)


def test_ste_one_hot_closed_forms():
    pins.check_ste_one_hot(oracle)


def test_ste_finite_differences():
    pins.check_ste_finite_difference(oracle)


@pytest.mark.parametrize("nm", [(2, 4), (6, 8)])
def test_ste_linearizes_the_forward(nm):
    d = synth.layer_small()
    pins.check_ste_matches_forward(oracle, d["w"], d["x"], *nm)
