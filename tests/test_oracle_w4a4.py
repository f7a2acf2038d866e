"""Pins of the oracle's W4A4 mode (NVFP4 expert inputs): the activation
quantiser against the E2M1 and E4M3 grids enumerated from their bit
definitions, hand-worked codes (ties to the even code, saturation), the
scale rule checked by brute force over the grid, the error bound the rule
implies, the fp16 rounding against numpy's binary16 cast, and the two
oracles' W4A4 blocks against each other."""
import numpy as np
import pytest

from latent_mixture_experts_softmax_b200 import synth
from oracle import lmoe_oracle as np_oracle
from oracle import native as cpp_oracle


def e4m3_grid() -> np.ndarray:
    """Positive E4M3 values by code 0x00..0x7E from the bit layout (bias 7,
    subnormals m/8 * 2^-6; 0x7F is NaN)."""
    c = np.arange(0x7F)
    e, m = (c >> 3) & 15, c & 7
    return np.where(e == 0, m / 8 * 2.0 ** -6, (1 + m / 8) * 2.0 ** (e - 7))


def e2m1_value(code: int) -> float:
    s, e, m = (code >> 3) & 1, (code >> 1) & 3, code & 1
    mag = 0.5 * m if e == 0 else (1 + 0.5 * m) * 2.0 ** (e - 1)
    return -mag if s else mag


def test_hand_worked_row():
    """Every E2M1 magnitude once with both signs, and 0.25: the block maximum
    6 sets G = 6 / 2688 and the scale to the top code 0x7E (448); each value
    keeps its own code except 0.25, halfway between 0 and 0.5, which goes to
    the even code 0."""
    x = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -0.5, 0.25])
    out, codes, scales, G = cpp_oracle.nvfp4_act_quantize(x)
    assert list(codes) == [0, 1, 2, 3, 4, 5, 6, 7, 15, 14, 13, 12, 11, 10, 9, 0]
    assert list(scales) == [0x7E]
    assert G == pytest.approx(6 / 2688, rel=1e-7)
    expect = np.array([e2m1_value(int(c)) for c in codes]) * 448.0 * G
    np.testing.assert_array_equal(out, expect)


def test_ties_go_to_the_even_code_and_values_saturate():
    """Block maximum 6: the fp32 block scale 448 * G rounds to exactly 1, so
    the midpoints 0.75, 1.25, 1.75, 2.5, 3.5 and 5 are exact ties and go to
    1, 1, 2, 2, 4, 4 (the even codes 2, 2, 4, 4, 6, 6)."""
    x = np.zeros(16)
    x[0] = 6.0
    x[1:7] = [0.75, 1.25, 1.75, 2.5, 3.5, 5.0]
    _, codes, _, _ = cpp_oracle.nvfp4_act_quantize(x)
    assert list(codes[1:7]) == [2, 2, 4, 4, 6, 6]


@pytest.mark.parametrize("seed", range(5))
def test_scale_codes_equal_brute_force_over_the_grid(seed):
    """Each block's scale code is the smallest E4M3 value (searched here by
    brute force over the enumerated grid, in fp32 like the rule) not below
    max|v| / (6 G)."""
    rng = np.random.default_rng(seed)
    grid = e4m3_grid().astype(np.float32)
    v = rng.normal(size=256) * np.exp(rng.normal(size=256) * 3)
    out, codes, scales, G = cpp_oracle.nvfp4_act_quantize(v)
    r = np.array([cpp_oracle.fp16_round(t) for t in v], np.float32)
    G32 = np.float32(G)
    for b in range(16):
        bmax = np.float32(np.abs(r[16 * b:16 * b + 16]).max())
        if bmax == 0:
            assert scales[b] == 0
            continue
        s = np.float32(bmax / np.float32(np.float32(6) * G32))
        want = next((c for c in range(1, 0x7F) if grid[c] >= s), 0x7E)
        assert scales[b] == min(want, 0x7E)


@pytest.mark.parametrize("seed", range(5))
def test_error_bound_of_one_term(seed):
    """Nearest E2M1 rounding leaves at most half the widest step (1 of the
    grid's 4..6 step) times the block scale, and the rounded-up E4M3 scale
    is at most 9/8 of max|v| / 6 (normal scales): |v - q| <= 0.1875 max|v|
    per block, on the fp16-rounded row."""
    rng = np.random.default_rng(100 + seed)
    v = rng.normal(size=512) * 10.0 ** rng.uniform(-3, 3)
    out, _, _, _ = cpp_oracle.nvfp4_act_quantize(v)
    r = np.array([cpp_oracle.fp16_round(t) for t in v])
    for b in range(32):
        blk = r[16 * b:16 * b + 16]
        assert np.abs(blk - out[16 * b:16 * b + 16]).max() <= 0.1875 * np.abs(blk).max() * (1 + 1e-6)


def test_zero_rows_and_blocks():
    out, codes, scales, G = cpp_oracle.nvfp4_act_quantize(np.zeros(64))
    assert not out.any() and not codes.any() and not scales.any() and G == 1.0
    v = np.concatenate([np.zeros(16), np.ones(16)])
    out, _, scales, _ = cpp_oracle.nvfp4_act_quantize(v)
    assert scales[0] == 0 and not out[:16].any()


def test_fp16_rounding_matches_numpy_binary16():
    rng = np.random.default_rng(7)
    v = np.concatenate([rng.normal(size=500) * 10.0 ** rng.uniform(-9, 5, 500),
                        [65504.0, 65519.99, 65520.0, 2.0 ** -24 * 1.5, 2.0 ** -25, -0.0]])
    ours = np.array([cpp_oracle.fp16_round(t) for t in v])
    with np.errstate(over="ignore"):
        ref = v.astype(np.float16).astype(np.float64)
    np.testing.assert_array_equal(ours, ref)


def test_cpp_and_numpy_quantisers_agree():
    rng = np.random.default_rng(3)
    for t in range(100):
        v = rng.normal(size=96) * 10.0 ** rng.integers(-5, 4)
        if t % 5 == 0:
            v[16:32] = 0
        a = cpp_oracle.nvfp4_act_quantize(v)[0]
        np.testing.assert_array_equal(a, np_oracle.nvfp4_act(v))


def test_w4a4_block_cpp_and_numpy_agree_and_stay_near_w4a16():
    """The two oracles' W4A4 blocks agree; the W4A4 block differs from the
    W4A16 one (the activations are quantised) by a few percent, not more."""
    s = synth.LayerShape(hidden=256, latent=128, n_experts=24, top_k=5, n_groups=4, ffn=128, shared_ffn=64,
                         du_fmt=synth.Q8_0, router_dtype="bf16", act_fmt="nvfp4")
    wl = synth.Workload("w4a4", s, T=5, seed=23, bias_sigma=0.5, weight_sigma=0.05)
    layer = synth.make_layer(wl)
    xb = synth.make_x(wl)
    a = cpp_oracle.latent_moe_forward(s, layer, xb)
    b = np_oracle.latent_moe_forward(s, layer, xb)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-10, atol=1e-12)
    c = cpp_oracle.latent_moe_forward(synth.replace(s, act_fmt="fp16"), layer, xb)
    rel = np.linalg.norm(a[0] - c[0]) / np.linalg.norm(c[0])
    assert 1e-4 < rel < 0.1
