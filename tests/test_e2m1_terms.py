"""The activation encoding of the tensor-core expert kernels, checked on the
CPU: an fp16 row written as six E2M1 rows with E4M3 block scales (16
elements) and one fp32 scale per row and term,
    x ~= sum_j G_j s_j[b] q_j,   G_j = max|x| / (6 * 448) * 5^-j,
each term quantising the residual the earlier ones left (the scale rounded
up to the E4M3 grid, the codes to the nearest E2M1 value).  The E2M1 and
E4M3 grids are enumerated here from their definitions (sign, exponent,
mantissa, bias 1 and 7); the kernels' error claim is that the sum matches
the row to 5e-5 of each block's maximum (blocks within 2^17 of the row
maximum), far under the fp16 rounding (2^-11) the row already carries, and
that no block scale leaves the E4M3 range."""
import zlib

import numpy as np
import pytest


def e4m3_grid() -> np.ndarray:
    """Positive E4M3 values by code 0x00..0x7E (0x7F is NaN): subnormals
    m/8 * 2^-6, normals (1 + m/8) * 2^(e - 7)."""
    c = np.arange(0x7F)
    e, m = (c >> 3) & 15, c & 7
    return np.where(e == 0, m / 8 * 2.0 ** -6, (1 + m / 8) * 2.0 ** (e - 7))


E4 = e4m3_grid()
E2 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])   # E2M1 magnitudes by code 0..7


def e4m3_up(s: np.ndarray) -> np.ndarray:
    return np.minimum(np.searchsorted(E4, s, side="left"), 0x7E)


def e2m1_rn(v: np.ndarray) -> np.ndarray:
    a = np.minimum(np.abs(v), 6.0)
    d = np.abs(a[..., None] - E2)
    tie = (d == d.min(-1, keepdims=True)).sum(-1) > 1
    even = np.argmax((d == d.min(-1, keepdims=True)) & (np.arange(8) % 2 == 0), -1)
    return np.sign(v) * E2[np.where(tie, even, np.argmin(d, -1))]


def encode(x: np.ndarray, J: int = 6):
    """(reconstruction, largest block scale used) of one row, in the
    kernels' order of operations (fp32 residual, scales rounded up)."""
    x = x.astype(np.float32)
    amax_row = float(np.abs(x).max())
    g0 = np.float32(amax_row / (6 * 448)) if amax_row > 0 else np.float32(1)
    r = x.reshape(-1, 16).copy()
    rec = np.zeros(r.shape, np.float64)
    smax = 0.0
    for j in range(J):
        g = np.float32(g0 * np.float32(0.2) ** j)
        amax = np.abs(r).max(1)
        c = np.where(amax > 0, e4m3_up((amax / (6 * g)).astype(np.float32)), 0)
        smax = max(smax, float(E4[c].max()))
        sd = (E4[c] * g).astype(np.float32)
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.where(sd[:, None] > 0, e2m1_rn(r * (np.float32(1) / sd)[:, None]), 0.0)
        r = (r - q * sd[:, None]).astype(np.float32)
        rec += q * sd[:, None]
    return rec.reshape(-1), smax


def test_grids_match_their_definitions():
    assert E4[0x7E] == 448.0 and E4[0x01] == 2.0 ** -9 and E4[0x08] == 2.0 ** -6
    assert np.all(np.diff(E4) > 0)                        # codes ordered by value
    assert E2[-1] == 6.0 and len(set(E2)) == 8


@pytest.mark.parametrize("kind", ["normal", "lognormal", "cauchy", "sparse_scaled", "max_fp16"])
def test_six_terms_reach_five_e_minus_five_of_the_block_maximum(kind):
    rng = np.random.default_rng(zlib.crc32(kind.encode()))
    for _ in range(20):
        K = 1792
        if kind == "normal":
            x = rng.normal(size=K)
        elif kind == "lognormal":
            x = rng.normal(size=K) * np.exp(rng.normal(size=K) * 4)
        elif kind == "cauchy":
            x = rng.standard_cauchy(size=K)
        elif kind == "sparse_scaled":
            x = rng.normal(size=K)
            x[rng.random(K) < 0.5] = 0
            x *= 10.0 ** rng.integers(-6, 4)
        else:
            x = rng.choice([-65504.0, 65504.0, 1e-7, 0.0, 3.0], size=K)
        x = np.clip(x, -65504, 65504).astype(np.float16).astype(np.float32)
        rec, smax = encode(x)
        assert smax <= 448.0
        blocks = np.abs(x.reshape(-1, 16)).max(1)
        err = np.abs(x - rec).reshape(-1, 16).max(1)
        near = blocks > np.abs(x).max() * 2.0 ** -17
        assert np.all(err[near] <= 5e-5 * blocks[near])
        assert np.all(err <= 5e-5 * np.abs(x).max())


def test_zero_row_encodes_to_zero():
    rec, smax = encode(np.zeros(256, np.float32))
    assert np.all(rec == 0) and smax == 0
