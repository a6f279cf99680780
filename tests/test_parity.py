"""CUDA path against the oracle, element by element (needs a B200).

Bar: bit-exact gamma, masks (meta), packed codes, INT8 activations, scales
and int32 accumulators; bf16 outputs within 1e-2 relative.
"""

import numpy as np
import pytest

import oracle
from gpu_util import (assert_weights_exact, assert_y_close, full_parity, run_layer,
                      run_quantize_weights, packed_to_numpy, to_dev_bf16, bf16_tensor_bits)
from sparse_linear_layers_fwd_b200 import synth

pytestmark = pytest.mark.gpu

SUPPORTED = [(1, 4), (2, 4), (3, 4), (4, 4), (2, 8), (4, 8), (6, 8), (8, 8),
             (4, 16), (8, 16), (12, 16), (16, 16)]
SHAPES = [(1, 128, 1), (5, 384, 7), (17, 1024, 130), (33, 256, 64), (100, 512, 257)]


@pytest.fixture(autouse=True)
def _lib(sbn_lib, cuda_ok):
    return sbn_lib


def test_layer_small_full_parity():
    d = synth.layer_small()
    full_parity(d["w"], d["x"], d["n"], d["m"])


@pytest.mark.parametrize("nm", SUPPORTED)
@pytest.mark.parametrize("shape", SHAPES)
def test_patterns_and_ragged_shapes(nm, shape):
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=1, tag=f"p{nm}{shape}")
    x = synth.activations(t, k, seed=1, tag=f"p{nm}{shape}", outlier_channels=2)
    full_parity(w, x, *nm)


@pytest.mark.parametrize("nm", SUPPORTED)
@pytest.mark.parametrize("shape", [s for s in SHAPES if s[0] > 16])
def test_tensor_core_without_workspace(nm, shape):
    """T > 16 without a workspace: the weights are expanded inside the
    tensor-core kernel instead of into the workspace first."""
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=13, tag=f"nows{nm}{shape}")
    x = synth.activations(t, k, seed=13, tag=f"nows{nm}{shape}", outlier_channels=2)
    full_parity(w, x, *nm, workspace=False)


@pytest.mark.parametrize("which", ["up", "down"])
def test_prefill_full_without_workspace(which):
    """Config-3 shapes (2:4, T=4096) with the weights expanded inside the
    sparse tensor-core kernel: every accumulator and output compared."""
    d = synth.prefill(which)
    full_parity(d["w"], d["x"], d["n"], d["m"], workspace=False)


# 2:4 runs on the sparse tensor-core MMA: token tiles of 224, output-feature
# tiles of 128, K stages of 128 positions; ragged tails on both tile axes
SPARSE24_SHAPES = [(17, 128, 1), (224, 256, 128), (225, 384, 129), (449, 640, 300), (700, 128, 77),
                   (300, 2560, 260)]


@pytest.mark.parametrize("shape", SPARSE24_SHAPES)
@pytest.mark.parametrize("ws", [None, False], ids=["workspace", "in_kernel"])
def test_sparse24_tensor_core_tiles(shape, ws):
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=5, tag=f"sp24{shape}")
    x = synth.activations(t, k, seed=5, tag=f"sp24{shape}", outlier_channels=2)
    full_parity(w, x, 2, 4, workspace=ws)


# Dense patterns on CTA pairs: 128-token tiles where 256-token ones would
# leave pairs idle, 256-token tiles otherwise (the host picks by the number
# of tile rounds); ragged token, row and K tails for both.
DENSE_PAIR_CASES = [
    ((1000, 384, 4000), (6, 8)),    # wide tiles: 64 of them fill one round
    ((300, 640, 520), (4, 8)),      # narrow tiles
    ((129, 1152, 257), (8, 16)),    # narrow tiles, one token past a tile
    ((2048, 896, 128), (6, 8)),     # narrow, a single 256-row pair tile half empty
]


@pytest.mark.parametrize("shape,nm", DENSE_PAIR_CASES, ids=[f"{c[0]}_{c[1][0]}of{c[1][1]}" for c in DENSE_PAIR_CASES])
def test_dense_pair_tiles(shape, nm):
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=6, tag=f"dp{shape}")
    x = synth.activations(t, k, seed=6, tag=f"dp{shape}", outlier_channels=2)
    full_parity(w, x, *nm)


@pytest.mark.parametrize("ws", [None, False], ids=["workspace", "in_kernel"])
def test_sparse24_every_group_mask(ws):
    """Rows whose 2:4 groups run through all six kept-position pairs (each
    one a different metadata nibble), with kept zeros, ties and both signs."""
    rng = np.random.default_rng(8)
    pairs = [(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)]
    n_out, k, t = 150, 768, 230
    mag = np.full((n_out, k), 0.001, np.float32)
    for r in range(n_out):
        for g in range(k // 4):
            a, b = pairs[(r + 7 * g) % 6]
            mag[r, 4 * g + a] = rng.choice([0.03, 0.05, 0.0011])   # 0.0011: kept, codes to 0
            mag[r, 4 * g + b] = rng.choice([0.03, 0.05])
    mag[::5, :8] = 0.02                                            # four-way ties: keep positions 0, 1
    sign = np.where(rng.random((n_out, k)) < 0.5, -1.0, 1.0).astype(np.float32)
    w = ((mag * sign).view(np.uint32) >> 16).astype(np.uint16)
    x = synth.activations(t, k, seed=8, outlier_channels=2)
    full_parity(w, x, 2, 4, workspace=ws)


def _fused_check(w, x, n, m):
    """sbn_bitlinear_x against the oracle: Xq and s bit-exact, y within tolerance."""
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    pw = run_quantize_weights(w, n, m)
    xd = to_dev_bf16(x)
    t, k = x.shape
    oq = torch.empty((t, k), dtype=torch.int8, device="cuda")
    os_ = torch.empty((t,), dtype=torch.float32, device="cuda")
    y = sbn.bitlinear_x(xd, pw, out_q=oq, out_s=os_)
    torch.cuda.synchronize()
    assert sbn.get_device_error() == 0
    cb, mb, gamma, mask, dense = oracle.quantize_weights(w, n, m)
    q, s = oracle.quantize_acts(x)
    assert np.array_equal(oq.cpu().numpy(), q) and np.array_equal(os_.cpu().numpy(), s)
    acc = oracle.bitlinear_acc(q, dense)
    assert_y_close(bf16_tensor_bits(y), oracle.dequant_bf16(acc, s, gamma))
    # without the optional outputs
    y2 = sbn.bitlinear_x(xd, pw)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_tensor_bits(y2), bf16_tensor_bits(y))
    return bf16_tensor_bits(y)


@pytest.mark.parametrize("nm", SUPPORTED)
@pytest.mark.parametrize("shape", SHAPES)
def test_fused_act_quant_contraction(nm, shape):
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=14, tag=f"fx{nm}{shape}")
    x = synth.activations(t, k, seed=14, tag=f"fx{nm}{shape}", outlier_channels=2)
    _fused_check(w, x, *nm)


# decode GEMV: token counts on both sides of 8, ragged row tiles, K with a
# half 256-position item at the end, and rows spread over many CTAs
GEMV_SHAPES = [(9, 640, 50), (16, 1152, 33), (3, 2560, 200), (8, 256, 16), (12, 384, 4099)]


@pytest.mark.parametrize("nm", SUPPORTED)
@pytest.mark.parametrize("shape", GEMV_SHAPES)
def test_gemv_shapes(nm, shape):
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=21, tag=f"gv{nm}{shape}")
    x = synth.activations(t, k, seed=21, tag=f"gv{nm}{shape}", outlier_channels=2)
    g = full_parity(w, x, *nm)
    # the fused route multiplies the same accumulators by the same scales
    assert np.array_equal(_fused_check(w, x, *nm), g["y"])


@pytest.mark.parametrize("t", synth.DECODE_TOKENS)
def test_fused_decode_full(t):
    _fused_check(synth.decode_weights(), synth.decode_acts(t), 6, 8)


def test_fused_zero_rows_and_streaming_fallback():
    w = synth.latent_weights(40, 11008, seed=15)
    x = synth.activations(16, 11008, seed=15)       # X does not fit: two-step route
    x[3] = 0
    _fused_check(w, x, 6, 8)
    x2 = synth.activations(5, 512, seed=16)
    x2[0] = 0
    x2[1] = 0x8000
    _fused_check(synth.latent_weights(64, 512, seed=16), x2, 2, 4)


def _tie_scales():
    """bf16 scales s in [1, 256) for which fl32(s/2 * fl32(127/s)) is exactly
    63.5 although the exact product is not: rounding the product first (as
    the definition does) gives the even 64, a fused multiply-add of the
    product and the rounding constant would give 63 for half of them."""
    out = []
    for bits in range(0x3F80, 0x4380):
        sv = np.uint32(bits << 16).view(np.float32)
        p = np.float32(np.float32(sv / np.float32(2)) * np.float32(np.float32(127) / sv))
        if p == np.float32(63.5):
            out.append(bits)
    return out


def _tie_rows(scales, k, seed):
    # row r: its maximum s_r first, then +-s_r/2 (exact in bf16) everywhere
    rng = np.random.default_rng(seed)
    x = np.empty((len(scales), k), dtype=np.uint16)
    for r, sb in enumerate(scales):
        row = np.full(k, sb - 0x80, dtype=np.uint16)
        row[rng.random(k) < 0.5] |= np.uint16(0x8000)
        row[0] = sb
        x[r] = row
    return x


def test_activation_rounding_ties_quantize_acts():
    from sparse_linear_layers_fwd_b200 import sbn
    import torch
    scales = _tie_scales()
    assert len(scales) > 500
    for k in (256, 2560, 4096):
        x = _tie_rows(scales, k, seed=k)
        q, sc = oracle.quantize_acts(x)
        assert np.count_nonzero(np.abs(q.astype(np.int32)) == 64) > 0
        xq, xs = sbn.quantize_acts(to_dev_bf16(x))
        torch.cuda.synchronize()
        assert np.array_equal(xs.cpu().numpy(), sc) and np.array_equal(xq.cpu().numpy(), q)


@pytest.mark.parametrize("t,k", [(20000, 128), (9000, 896), (8000, 1536), (6000, 2560), (5000, 3072), (3000, 6912),
                                 (2000, 12288), (700, 17408)])
def test_quantize_acts_rows_beyond_one_wave(t, k):
    """More rows than one wave of CTAs holds: each warp (K <= 2560) or CTA
    (longer rows) takes several rows in turn."""
    from sparse_linear_layers_fwd_b200 import sbn
    import torch
    x = synth.activations(t, k, seed=3, tag=f"qawave{t}_{k}", outlier_channels=1)
    q, sc = oracle.quantize_acts(x)
    xq, xs = sbn.quantize_acts(to_dev_bf16(x))
    torch.cuda.synchronize()
    assert np.array_equal(xs.cpu().numpy(), sc), "scales differ"
    assert np.array_equal(xq.cpu().numpy(), q), "INT8 activations differ"


@pytest.mark.parametrize("t,k", [(16, 2560), (9, 640), (1, 1152), (16, 384)])
def test_activation_rounding_ties_fused(t, k):
    # the fused decode path, 16 (or t) tie scales per call, all of them in turn
    scales = _tie_scales()
    w = synth.latent_weights(40, k, seed=23, tag="ties")
    for i in range(0, len(scales), 16 * 9):
        x = _tie_rows(scales[i:i + t], k, seed=i)
        _fused_check(w, x, 6, 8)


@pytest.mark.parametrize("nm", [(2, 4), (6, 8), (8, 16), (8, 8)])
def test_all_zero_weights(nm):
    w = np.zeros((40, 256), np.uint16)
    w[::3] = 0x8000                                      # negative zeros too
    x = synth.activations(3, 256, seed=2)
    g = full_parity(w, x, *nm)
    assert g["gamma"] == np.float32(1e-5)


@pytest.mark.parametrize("nm", [(2, 4), (6, 8), (8, 16)])
def test_constant_weights_tie_everywhere(nm):
    w = np.full((24, 384), 0x3C23, np.uint16)            # 0.00995..., all equal magnitude
    w[1::2] ^= 0x8000                                    # alternate signs, same magnitude
    x = synth.activations(9, 384, seed=3)
    full_parity(w, x, *nm)


def test_exact_half_ties_in_codes():
    # half the weights 0.25, half 0.75 in magnitude: gamma = 0.5 exactly and
    # 0.25/gamma = 0.5 rounds (half to even) to 0
    row = np.array([0.25, -0.75, 0.75, -0.25] * 64, dtype=np.float32)
    w = np.tile((row.view(np.uint32) >> 16).astype(np.uint16), (16, 1))
    x = synth.activations(4, 256, seed=4)
    g = full_parity(w, x, 8, 8)
    assert g["gamma"] == np.float32(0.5)


def test_zero_and_tiny_activation_rows():
    w = synth.latent_weights(64, 512, seed=5)
    x = synth.activations(6, 512, seed=5)
    x[0] = 0
    x[1] = 0x8000
    x[2] = 0x0001                                        # smallest subnormal everywhere
    x[3, 7] = 0x7F7F                                     # largest finite bf16 in one channel
    full_parity(w, x, 2, 4)


def test_wide_exponent_weights():
    rng = np.random.default_rng(6)
    w = rng.integers(0, 0x7F00, size=(32, 512)).astype(np.uint16)   # every exponent, no inf
    w |= (rng.integers(0, 2, size=w.shape).astype(np.uint16) << 15)
    x = synth.activations(8, 512, seed=6)
    g = run_layer(w, x, 6, 8, want_acc=False)
    cb, mb, gamma, mask, dense = oracle.quantize_weights(w, 6, 8)
    assert_weights_exact(g, cb, mb, gamma)


def test_subnormal_and_large_weights_gamma():
    rng = np.random.default_rng(7)
    w = synth.latent_weights(16, 256, seed=7)
    w[0, :64] = rng.integers(1, 0x80, size=64).astype(np.uint16)      # subnormals
    w[1, :8] = 0x7A00                                                 # ~1.7e35
    w[2, :8] = 0x2000                                                 # ~1e-19
    g = run_layer(w, synth.activations(2, 256, seed=7), 2, 4, want_acc=False)
    cb, mb, gamma, _, _ = oracle.quantize_weights(w, 2, 4)
    assert_weights_exact(g, cb, mb, gamma)


def test_repeated_calls_reuse_workspace():
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    w1 = synth.latent_weights(256, 1024, seed=8, tag="a")
    w2 = synth.latent_weights(256, 1024, seed=8, tag="b")
    ws = torch.full((sbn.workspace_bytes(256, 1024),), 0xAB, dtype=torch.uint8, device="cuda")
    out = sbn.alloc_packed(256, 1024, 6, 8, "cuda")
    for w in [w1, w2, w1]:
        sbn.quantize_weights(to_dev_bf16(w), 6, 8, out=out, workspace=ws)
        c, mt, g = packed_to_numpy(out)
        rc, rm, rg, _, _ = oracle.quantize_weights(w, 6, 8)
        assert g == rg and np.array_equal(c, rc) and np.array_equal(mt, rm)


# ---------------------------------------------------------------------------
# the workloads at full size
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("shape,nm", [((16, 11008, 40), (6, 8)), ((9, 11008, 17), (8, 16)),
                                      ((12, 11008, 33), (8, 8))])
def test_decode_streaming_kernel(shape, nm):
    """Token counts and K whose activations do not fit next to the weights in
    shared memory take the streaming decode kernel."""
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=12, tag=f"stream{shape}")
    x = synth.activations(t, k, seed=12, tag=f"stream{shape}", outlier_channels=3)
    full_parity(w, x, *nm)


@pytest.fixture(scope="module")
def decode_ref():
    w = synth.decode_weights()
    cb, mb, gamma, mask, dense = oracle.quantize_weights(w, 6, 8)
    return w, cb, mb, gamma, dense


@pytest.mark.parametrize("t", synth.DECODE_TOKENS)
def test_decode_full_parity(decode_ref, t):
    w, cb, mb, gamma, dense = decode_ref
    x = synth.decode_acts(t)
    g = run_layer(w, x, 6, 8)
    assert_weights_exact(g, cb, mb, gamma)
    q, s = oracle.quantize_acts(x)
    assert np.array_equal(g["xq"], q) and np.array_equal(g["s"], s)
    acc = oracle.bitlinear_acc(q, dense)
    assert np.array_equal(g["acc"], acc)
    assert_y_close(g["y"], oracle.dequant_bf16(acc, s, gamma))


def _sampled_check(g, q, s, dense, gamma, t, n_out, seed, nsamp=4096):
    rng = np.random.default_rng(seed)
    ti = rng.integers(0, t, nsamp)
    ni = rng.integers(0, n_out, nsamp)
    # plus one full output row and one full output column
    tr, nc = int(rng.integers(0, t)), int(rng.integers(0, n_out))
    ti = np.concatenate([ti, np.full(n_out, tr), np.arange(t)])
    ni = np.concatenate([ni, np.arange(n_out), np.full(t, nc)])
    y_ref, acc_ref = oracle.bitlinear_at(q, s, dense, gamma, ti, ni)
    assert np.array_equal(g["acc"][ti, ni], acc_ref)
    assert_y_close(g["y"][ti, ni], y_ref)


@pytest.mark.parametrize("which", ["up", "down"])
def test_prefill_full(which):
    """Config-3 shapes (2:4, T=4096, compressed workspace route): every
    accumulator and output against the oracle's exact fp64 product."""
    d = synth.prefill(which)
    full_parity(d["w"], d["x"], d["n"], d["m"])


@pytest.mark.parametrize("proj", [p for p, _, _ in synth.QWEN05B_PROJ])
def test_qwen_layer0_full(proj):
    d = synth.qwen05b_layer(0, proj)
    full_parity(d["w"], d["x"], d["n"], d["m"])


@pytest.mark.parametrize("layer", [7, 23])
def test_qwen_other_layers_sampled(layer):
    for proj in ["q", "down"]:
        d = synth.qwen05b_layer(layer, proj)
        g = run_layer(d["w"], d["x"], 6, 8)
        cb, mb, gamma, mask, dense = oracle.quantize_weights(d["w"], 6, 8)
        assert_weights_exact(g, cb, mb, gamma)
        q, s = oracle.quantize_acts(d["x"])
        assert np.array_equal(g["xq"], q)
        _sampled_check(g, q, s, dense, gamma, d["x"].shape[0], d["w"].shape[0], seed=layer)


@pytest.mark.parametrize("nm", synth.FFN3B_PATTERNS)
@pytest.mark.parametrize("proj", ["gate", "down"])
def test_ffn3b_patterns(nm, proj):
    for t in synth.FFN3B_TOKENS:
        d = synth.ffn3b(proj, t, *nm)
        g = run_layer(d["w"], d["x"], *nm)
        if t == synth.FFN3B_TOKENS[0]:
            cb, mb, gamma, mask, dense = oracle.quantize_weights(d["w"], *nm)
            assert_weights_exact(g, cb, mb, gamma)
        q, s = oracle.quantize_acts(d["x"])
        assert np.array_equal(g["xq"], q) and np.array_equal(g["s"], s)
        if t <= 64:
            acc = oracle.bitlinear_acc(q, dense)
            assert np.array_equal(g["acc"], acc)
            assert_y_close(g["y"], oracle.dequant_bf16(acc, s, gamma))
        else:
            _sampled_check(g, q, s, dense, gamma, t, d["w"].shape[0], seed=t)


def test_bitlinear_module_matches_calls():
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    d = synth.layer_small()
    w = to_dev_bf16(d["w"])
    layer = sbn.BitLinear(256, 256, n=2, m=4, weight=w.clone())
    x = to_dev_bf16(d["x"]).reshape(2, 8, 256)
    y = layer(x)
    torch.cuda.synchronize()
    cb, mb, gamma, mask, dense = oracle.quantize_weights(d["w"], 2, 4)
    q, s = oracle.quantize_acts(d["x"])
    ref = oracle.dequant_bf16(oracle.bitlinear_acc(q, dense), s, gamma)
    assert y.shape == (2, 8, 256)
    assert_y_close(bf16_tensor_bits(y.reshape(16, 256)), ref)


def test_gamma_fp32_midpoint_exact_path():
    """2^24 weights, all 1.0 but one 2.0: the exact mean 1 + 2^-24 lies exactly
    halfway between two fp32 values, so no approximate sum can decide the
    rounding and the kernel must take its exact path; ties go to even (1.0)."""
    w = np.full((4096, 4096), 0x3F80, np.uint16)
    w[123, 456] = 0x4000
    x = synth.activations(2, 4096, seed=9)
    g = run_layer(w, x, 6, 8, want_acc=False)
    cb, mb, gamma, _, _ = oracle.quantize_weights(w, 6, 8)
    assert gamma == np.float32(1.0)
    assert_weights_exact(g, cb, mb, gamma)


def test_gamma_midpoint_plus_tiny_follows_fp64_rounding():
    """S = 2^24 + 1 + 2^-30 over 2^24 weights (all 1.0 except 2.0, 1.5, 1.5 and
    2^-30): the fp64 rounding of S drops the 2^-30 (half an ulp of 2^24 is
    2^-29), leaving the exact midpoint 1 + 2^-24 again, which goes to even.
    This pins the defined order fl32(fl64(fl64(S) / N)) on the exact path."""
    w = np.full((4096, 4096), 0x3F80, np.uint16)
    w[7, 9] = 0x4000          # 2.0
    w[8, 10] = 0x3FC0         # 1.5
    w[9, 11] = 0x3FC0         # 1.5
    w[10, 12] = 0x3080        # 2^-30
    x = synth.activations(2, 4096, seed=10)
    g = run_layer(w, x, 6, 8, want_acc=False)
    cb, mb, gamma, _, _ = oracle.quantize_weights(w, 6, 8)
    assert gamma == np.float32(1.0)
    assert_weights_exact(g, cb, mb, gamma)


@pytest.mark.parametrize("nm", [(2, 4), (6, 8), (8, 16), (1, 4), (12, 16)])
@pytest.mark.parametrize("shape", [(7, 128), (130, 1024), (6912, 2560)])
def test_mask_flips(nm, shape):
    """Keep-bit flips between two versions of a layer (a perturbed copy)."""
    n_out, k = shape
    w1 = synth.latent_weights(n_out, k, seed=17, tag=f"flip{shape}")
    rng = np.random.default_rng(17)
    w2 = w1.copy()
    sel = rng.random(w1.shape) < 0.05
    w2[sel] = synth.latent_weights(n_out, k, seed=18, tag=f"flip{shape}")[sel]
    from sparse_linear_layers_fwd_b200 import sbn
    p1 = run_quantize_weights(w1, *nm)
    p2 = run_quantize_weights(w2, *nm)
    got = int(sbn.mask_flips(p1, p2).cpu().item())
    assert got == oracle.mask_flips(oracle.nm_mask(w1, *nm), oracle.nm_mask(w2, *nm))
    assert int(sbn.mask_flips(p1, p1).cpu().item()) == 0


ENT_DECODE = [(1, 4), (2, 4), (3, 4), (2, 8), (4, 8), (6, 8)]


@pytest.mark.parametrize("nm", SUPPORTED)
@pytest.mark.parametrize("shape", [(7, 128), (130, 1024), (257, 512), (3, 1152)])
def test_pack_entropy_matches_oracle(nm, shape):
    n_out, k = shape
    w = synth.latent_weights(n_out, k, seed=19, tag=f"entp{nm}{shape}")
    from sparse_linear_layers_fwd_b200 import sbn
    import torch
    pw = run_quantize_weights(w, *nm)
    # every byte, row padding included, is written by the packer: start from 0xFF
    out = torch.full((n_out, sbn.entropy_row_bytes(k, *nm)), 255, dtype=torch.uint8, device="cuda")
    got = sbn.pack_entropy(pw, out=out).cpu().numpy()
    cb, mb, gamma, mask, dense = oracle.quantize_weights(w, *nm)
    assert np.array_equal(got, oracle.entropy_pack(mask, dense, *nm))


def _entropy_decode_check(w, x, n, m):
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    pw = run_quantize_weights(w, n, m)
    xq, s = sbn.quantize_acts(to_dev_bf16(x))
    ent = sbn.pack_entropy(pw)
    y_ent = sbn.bitlinear_entropy(xq, s, ent, pw)
    acc_ent = sbn.bitlinear_entropy_acc32(xq, ent, pw)
    y_can = sbn.bitlinear(xq, s, pw)
    torch.cuda.synchronize()
    assert sbn.get_device_error() == 0
    cb, mb, gamma, mask, dense = oracle.quantize_weights(w, n, m)
    q, sc = oracle.quantize_acts(x)
    acc = oracle.bitlinear_acc(q, dense)
    assert np.array_equal(acc_ent.cpu().numpy(), acc)
    assert np.array_equal(bf16_tensor_bits(y_ent), bf16_tensor_bits(y_can))
    assert_y_close(bf16_tensor_bits(y_ent), oracle.dequant_bf16(acc, sc, gamma))
    _entropy_fused_check(x, ent, pw, q, sc, y_ent)


def _entropy_fused_check(x, ent, pw, q, sc, y_ent):
    """sbn_bitlinear_entropy_x: Xq and s bit-exact against the oracle, y
    bit-identical to sbn_quantize_acts followed by sbn_bitlinear_entropy."""
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    t, k = x.shape
    xd = to_dev_bf16(x)
    oq = torch.full((t, k), 99, dtype=torch.int8, device="cuda")
    os_ = torch.full((t,), -1.0, dtype=torch.float32, device="cuda")
    y_x = sbn.bitlinear_entropy_x(xd, ent, pw, out_q=oq, out_s=os_, workspace=False)
    y_x2 = sbn.bitlinear_entropy_x(xd, ent, pw)
    torch.cuda.synchronize()
    assert sbn.get_device_error() == 0
    assert np.array_equal(oq.cpu().numpy(), q) and np.array_equal(os_.cpu().numpy(), sc)
    assert np.array_equal(bf16_tensor_bits(y_x), bf16_tensor_bits(y_ent))
    assert np.array_equal(bf16_tensor_bits(y_x2), bf16_tensor_bits(y_ent))


@pytest.mark.parametrize("nm", ENT_DECODE)
@pytest.mark.parametrize("shape", [(1, 128, 1), (5, 384, 7), (16, 1024, 130), (9, 512, 257)])
def test_bitlinear_entropy(nm, shape):
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=20, tag=f"entd{nm}{shape}")
    x = synth.activations(t, k, seed=20, tag=f"entd{nm}{shape}", outlier_channels=2)
    _entropy_decode_check(w, x, *nm)


def test_bitlinear_entropy_x_two_step_route():
    # T = 16 bf16 rows of K = 6144 do not fit in shared memory beside the
    # int8 rows: quantize_acts, then the contraction over int8 activations
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    t, k, n_out, n, m = 16, 6144, 40, 2, 8
    w = synth.latent_weights(n_out, k, seed=21, tag="ent2step")
    x = synth.activations(t, k, seed=21, tag="ent2step", outlier_channels=2)
    _entropy_decode_check(w, x, n, m)
    pw = run_quantize_weights(w, n, m)
    ent = sbn.pack_entropy(pw)
    with pytest.raises(sbn.SbnError) as e:   # no workspace and no Xq / s outputs to quantize into
        sbn.bitlinear_entropy_x(to_dev_bf16(x), ent, pw, workspace=False)
    assert e.value.status == 5
    torch.cuda.synchronize()


@pytest.mark.parametrize("t", synth.DECODE_TOKENS)
def test_bitlinear_entropy_decode_full(t):
    _entropy_decode_check(synth.decode_weights(), synth.decode_acts(t), 6, 8)


# ---- backward (straight-through estimator) ------------------------------------
#
# Tolerance from the arithmetic: the kernels accumulate L products in fp32
# (error at most L * 2^-24 of the sum of |terms|) and both sides round once to
# bf16 (2^-9 relative each): |got - ref| <= 2^-7 |ref| + L 2^-22 sum|terms|.

def _grad_close(got_bits, ref_bits, abs_terms, length):
    g = oracle.bf16_bits_to_f32(got_bits).astype(np.float64)
    r = oracle.bf16_bits_to_f32(ref_bits).astype(np.float64)
    bad = np.abs(g - r) > 2.0 ** -7 * np.abs(r) + length * 2.0 ** -22 * abs_terms
    assert not bad.any(), f"{bad.sum()} of {bad.size} off; first {np.argwhere(bad)[:3]}"


def _grad_check(w, x, dy, n, m):
    import torch
    from sparse_linear_layers_fwd_b200 import sbn
    pw = run_quantize_weights(w, n, m)
    xq, s = sbn.quantize_acts(to_dev_bf16(x))
    dyd = to_dev_bf16(dy)
    dx = sbn.bitlinear_grad_x(dyd, pw)
    dw = sbn.bitlinear_grad_w(dyd, xq, s)
    torch.cuda.synchronize()
    assert sbn.get_device_error() == 0
    cb, mb, gamma, mask, dense = oracle.quantize_weights(w, n, m)
    q, sc = oracle.quantize_acts(x)
    g = np.abs(oracle.bf16_bits_to_f32(dy).astype(np.float64))
    _grad_close(bf16_tensor_bits(dx), oracle.ste_grad_x(dy, dense, gamma),
                g @ (np.abs(dense.astype(np.float64)) * float(gamma)), dy.shape[1])
    xd = np.abs(q.astype(np.float64)) * (sc.astype(np.float64)[:, None] / 127.0)
    _grad_close(bf16_tensor_bits(dw), oracle.ste_grad_w(dy, q, sc), g.T @ xd, dy.shape[0])


@pytest.mark.parametrize("nm", SUPPORTED)
@pytest.mark.parametrize("shape", SHAPES)
def test_backward_grads(nm, shape):
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=23, tag=f"bw{nm}{shape}")
    x = synth.activations(t, k, seed=23, tag=f"bw{nm}{shape}", outlier_channels=2)
    dy = synth.activations(t, n_out, seed=24, tag=f"dy{nm}{shape}")
    _grad_check(w, x, dy, *nm)


# N_out a multiple of 8: dX runs on the tensor cores (dY by TMA); token tiles
# of 128 and position tiles of 256 with ragged tails, feature stages of 64
BWD_TC_SHAPES = [(130, 384, 136), (300, 640, 72), (17, 256, 520), (257, 256, 8), (64, 1152, 264)]


@pytest.mark.parametrize("nm", [(2, 4), (6, 8), (8, 16), (8, 8), (1, 4)])
@pytest.mark.parametrize("shape", BWD_TC_SHAPES)
def test_backward_dx_tensor_core_tiles(nm, shape):
    t, k, n_out = shape
    w = synth.latent_weights(n_out, k, seed=27, tag=f"bwtc{nm}{shape}")
    x = synth.activations(t, k, seed=27, tag=f"bwtc{nm}{shape}", outlier_channels=2)
    dy = synth.activations(t, n_out, seed=28, tag=f"dytc{nm}{shape}")
    _grad_check(w, x, dy, *nm)


def test_backward_grads_decode_layer():
    # the decode layer's weights (6912 x 2560, 6:8) with 300 tokens
    w = synth.decode_weights()
    x = synth.activations(300, 2560, seed=25, tag="bwfull", outlier_channels=2)
    dy = synth.activations(300, 6912, seed=26, tag="dyfull")
    _grad_check(w, x, dy, 6, 8)
