"""Pins of the fp64 oracle against things other than itself: figures the pages
print, library conversions, closed forms, special cases and brute force."""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lmoe_oracle as np_oracle
from oracle import native as cpp_oracle
from latent_mixture_experts_softmax_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


@pytest.fixture(params=["cpp", "numpy"])
def orc(request):
    """Every pin runs against both oracles: the C++ one (used by the parity
    tests and the CPU baseline) and the numpy one (a second witness)."""
    return cpp_oracle if request.param == "cpp" else np_oracle


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------
# storage formats: byte totals the pages print
# ----------------------------------------------------------------------------

def test_record_and_build_sizes_match_pages(orc):
    g = _gold("page_figures.json")
    H, E, G, F, NL = (g[k]["value"] for k in ("hidden", "experts_per_layer", "groups", "swiglu_width", "layers"))
    L145, L120 = g["latent_145b"]["value"], g["latent_120b"]["value"]
    assert 3 * L145 * F == g["expert_weights_latent1792"]["value"]
    assert 3 * H * F == g["expert_weights_base"]["value"]
    assert orc.expert_record_bytes(L145, F) == g["nvfp4_record_bytes_latent1792"]["value"]
    # 145B NVFP4 build = experts + Q8_0 D and U (8 groups each), 48 layers
    per_layer = E * orc.expert_record_bytes(L145, F) + G * (orc.du_matrix_bytes(orc.Q8_0, L145, H)
                                                            + orc.du_matrix_bytes(orc.Q8_0, H, L145))
    assert NL * per_layer == g["weights_145b_nvfp4_bytes"]["value"]
    # the model page prints 47.79 GiB for the same byte total (47.785 GiB; it rounds up)
    assert abs(NL * per_layer / 2 ** 30 - g["weights_145b_nvfp4_gib"]["value"]) < 0.01
    # 120B NVFP4 build with Q4_0 D/U
    per_layer = E * orc.expert_record_bytes(L120, F) + G * (orc.du_matrix_bytes(orc.Q4_0, L120, H)
                                                            + orc.du_matrix_bytes(orc.Q4_0, H, L120))
    assert round(NL * per_layer / 2 ** 30, 2) == g["weights_120b_nvfp4_gib"]["value"]
    # with Q8_0 D/U the 120B would not match the printed build size
    per_layer_q8 = E * orc.expert_record_bytes(L120, F) + 2 * G * orc.du_matrix_bytes(orc.Q8_0, L120, H)
    assert round(NL * per_layer_q8 / 2 ** 30, 2) != g["weights_120b_nvfp4_gib"]["value"]
    # D+U parameters per layer and routed parameters per layer
    assert round(2 * H * L145 * G / 1e6, 1) == g["du_params_per_layer_145b"]["value"] / 1e6
    assert round(NL * 2 * H * L145 * G / 1e9, 2) == g["du_params_48_layers_145b"]["value"] / 1e9
    assert round(g["top_k"]["value"] * 3 * L145 * F / 1e6, 1) == g["routed_params_per_layer_145b"]["value"] / 1e6


# ----------------------------------------------------------------------------
# scalar formats against library conversions and the spec table
# ----------------------------------------------------------------------------

def test_e2m1_all_codes_match_spec_table(orc):
    want = np.array(_gold("e2m1_values.json")["values"])
    got = orc.e2m1_to_f64(np.arange(16))
    np.testing.assert_array_equal(got, want)
    assert np.all(np.signbit(got[8:]))


def test_e4m3fn_all_codes_match_torch(orc):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = orc.e4m3fn_to_f64(np.arange(256))
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert nan.sum() == 2                               # 0x7F and 0xFF
    np.testing.assert_array_equal(got[~nan], ref[~nan])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6


def test_fp16_all_codes_match_numpy(orc):
    codes = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = codes.view(np.float16).astype(np.float64)
    got = orc.fp16_to_f64(codes)
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    np.testing.assert_array_equal(got[~nan], ref[~nan])


def test_bf16_matches_torch(orc):
    rng = np.random.default_rng(3)
    codes = rng.integers(0, 65536, size=20000).astype(np.uint16)
    codes = codes[((codes >> 7) & 0xFF) != 0xFF]        # finite values only
    ref = torch.from_numpy(codes.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(orc.bf16_to_f64(codes), ref)


# ----------------------------------------------------------------------------
# matrix formats: blobs packed element by element here, independently
# ----------------------------------------------------------------------------

def _fp16_bits(v):
    return int(np.array([v], np.float16).view(np.uint16)[0])


def test_decode_q8_0_hand_packed(orc):
    R, C = 3, 96
    rng = np.random.default_rng(1)
    q = rng.integers(-127, 128, size=(R, C))
    d = rng.choice([0.5, 0.25, 0.015625, 3.0, 0.0078125], size=(R, C // 32))
    blob = bytearray(R * C + R * C // 16)
    want = np.zeros((R, C))
    for r in range(R):
        for c in range(C):
            b, j = divmod(c, 32)
            blob[(b * R + r) * 32 + j] = int(q[r, c]) & 0xFF
            want[r, c] = q[r, c] * d[r, b]
        for b in range(C // 32):
            bits = _fp16_bits(d[r, b])
            off = R * C + 2 * (b * R + r)
            blob[off], blob[off + 1] = bits & 0xFF, bits >> 8
    got = orc.decode_q8_0(np.frombuffer(bytes(blob), np.uint8), R, C)
    np.testing.assert_array_equal(got, want)


def test_decode_q4_0_hand_packed(orc):
    R, C = 2, 64
    rng = np.random.default_rng(2)
    q = rng.integers(0, 16, size=(R, C))
    d = rng.choice([0.5, -0.25, 2.0, 0.125], size=(R, C // 32))
    blob = bytearray(R * C // 2 + R * C // 16)
    want = np.zeros((R, C))
    for r in range(R):
        for c in range(C):
            b, j = divmod(c, 32)
            pos = (b * R + r) * 16 + (j % 16)
            if j < 16:
                blob[pos] |= int(q[r, c])
            else:
                blob[pos] |= int(q[r, c]) << 4
            want[r, c] = (q[r, c] - 8) * d[r, b]
        for b in range(C // 32):
            bits = _fp16_bits(d[r, b])
            off = R * C // 2 + 2 * (b * R + r)
            blob[off], blob[off + 1] = bits & 0xFF, bits >> 8
    got = orc.decode_q4_0(np.frombuffer(bytes(blob), np.uint8), R, C)
    np.testing.assert_array_equal(got, want)


def test_decode_nvfp4_hand_packed(orc):
    R, C = 3, 128
    rng = np.random.default_rng(4)
    codes = rng.integers(0, 16, size=(R, C))
    scodes = rng.integers(0x08, 0x7E, size=(R, C // 16))
    ts = np.float32(0.0123)
    table = _gold("e2m1_values.json")["values"]
    s_val = torch.tensor(scodes.reshape(-1), dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy().reshape(R, C // 16)
    qb = bytearray(R * C // 2)
    sb = bytearray(R * C // 16)
    want = np.zeros((R, C))
    for r in range(R):
        for c in range(C):
            pos = ((c // 32) * R + r) * 16 + (c % 32) // 2
            qb[pos] |= int(codes[r, c]) << (4 * (c % 2))
            want[r, c] = table[codes[r, c]] * s_val[r, c // 16] * float(ts)
        for b in range(C // 16):
            sb[((b // 4) * R + r) * 4 + b % 4] = int(scodes[r, b])
    got = orc.decode_nvfp4(np.frombuffer(bytes(qb), np.uint8), np.frombuffer(bytes(sb), np.uint8), ts, R, C)
    np.testing.assert_array_equal(got, want)


def test_generator_round_trip_within_quantisation_error(orc):
    """Bytes from the generator decode to the matrix it was asked to encode,
    within each format's rounding step."""
    rng = np.random.default_rng(5)
    w = rng.normal(0, 0.02, size=(64, 128))
    for fmt, steps in ((orc.Q8_0, 127.0), (orc.Q4_0, 8.0)):
        back = orc.decode_du(fmt, synth.qmatrix_encode(fmt, w), 64, 128)
        amax = np.abs(w).reshape(64, 4, 32).max(axis=2)
        bound = np.repeat(amax / steps, 32, axis=1) * 0.5 * 1.01 + 1e-12
        if fmt == orc.Q4_0:
            bound = np.repeat(amax / 8.0, 32, axis=1) * 1.01 + 1e-12   # asymmetric range: up to one step
        assert np.all(np.abs(back - w) <= bound)
    wg, wu, wd = rng.normal(0, 0.02, (64, 128)), rng.normal(0, 0.02, (64, 128)), rng.normal(0, 0.02, (128, 64))
    rec = synth.expert_record_encode(wg, wu, wd)
    g2, u2, d2 = orc.decode_expert(rec, 128, 64)
    for a, b in ((wg, g2), (wu, u2), (wd, d2)):
        # E2M1 keeps values to within 1/4 of a grid step relative to the block max (6 levels)
        assert orc.rel_l2(b, a) < 0.15
        assert np.corrcoef(a.ravel(), b.ravel())[0, 1] > 0.99


# ----------------------------------------------------------------------------
# router
# ----------------------------------------------------------------------------

def _brute_route(logits_row, K):
    order = sorted(range(len(logits_row)), key=lambda e: (-logits_row[e], e))
    sel = order[:K]
    mx = max(logits_row[e] for e in sel)
    ex = [math.exp(logits_row[e] - mx) for e in sel]
    tot = sum(ex)
    return sel, [v / tot for v in ex]


def test_route_matches_full_sort_and_closed_form_weights(orc):
    rng = np.random.default_rng(7)
    T, E, H, K = 6, 40, 32, 10
    x = rng.normal(size=(T, H))
    Wr = rng.normal(0, 0.3, size=(E, H))
    b = rng.normal(0, 1.0, size=E)
    idx, w, gap, logits = orc.route(x, Wr, b, K)
    for t in range(T):
        lt = [float(sum(x[t, i] * Wr[e, i] for i in range(H)) + b[e]) for e in range(E)]
        sel, ws = _brute_route(lt, K)
        assert list(idx[t]) == sel
        np.testing.assert_allclose(w[t], ws, rtol=1e-12)
        assert abs(w[t].sum() - 1.0) < 1e-12
        srt = sorted(lt, reverse=True)
        assert abs(gap[t] - (srt[K - 1] - srt[K])) < 1e-12


def test_route_ties_lowest_index_and_bias_moves_selection(orc):
    E, K = 8, 3
    x = np.zeros((1, 4))
    Wr = np.zeros((E, 4))
    b = np.array([0.0, 1.0, 1.0, 1.0, 1.0, 0.5, 0.0, 2.0])
    idx, w, gap, _ = orc.route(x, Wr, b, K)
    assert list(idx[0]) == [7, 1, 2]          # 2.0 first, then the lowest indices among the tie at 1.0
    assert gap[0] == 0.0
    e2, e1 = math.exp(2.0), math.exp(1.0)
    np.testing.assert_allclose(w[0], [e2 / (e2 + 2 * e1), e1 / (e2 + 2 * e1), e1 / (e2 + 2 * e1)], rtol=1e-14)


def test_route_many_ties_lowest_index_wins(orc):
    """Hundreds of experts sharing a few logit values: the kept experts are
    the first K of a full sort by (logit descending, index ascending)."""
    rng = np.random.default_rng(12)
    E, K, T = 300, 10, 4
    x = np.zeros((T, 2))
    Wr = np.zeros((E, 2))
    for t in range(T):
        b = rng.choice([0.0, 0.5, 1.0], size=E, p=[0.5, 0.3, 0.2])
        idx, w, gap, _ = orc.route(x[t:t + 1], Wr, b, K)
        want, ws = _brute_route(b.tolist(), K)
        assert list(idx[0]) == want
        np.testing.assert_allclose(w[0], ws, rtol=1e-14)


def test_route_permutation_invariance(orc):
    rng = np.random.default_rng(8)
    T, E, H, K = 5, 32, 16, 4
    x = rng.normal(size=(T, H))
    Wr = rng.normal(size=(E, H))
    perm = rng.permutation(E)
    idx, w, _, _ = orc.route(x, Wr, None, K)
    idx_p, w_p, _, _ = orc.route(x, Wr[perm], None, K)
    for t in range(T):
        assert sorted(perm[idx_p[t]]) == sorted(idx[t])
        np.testing.assert_allclose(sorted(w_p[t]), sorted(w[t]), rtol=1e-12)


# ----------------------------------------------------------------------------
# block: brute force and special cases on tiny shapes
# ----------------------------------------------------------------------------

TINY = synth.LayerShape(hidden=128, latent=64, n_experts=12, top_k=3, n_groups=3, ffn=64, shared_ffn=64,
                        du_fmt=synth.Q8_0, router_dtype="f32")


def _tiny_layer(shape=TINY, seed=11, fmt=None):
    wl = synth.Workload("t", shape if fmt is None else synth.replace(shape, du_fmt=fmt), T=5, seed=seed,
                        groups="uniform", bias_sigma=0.5, weight_sigma=0.1)
    return wl, synth.make_layer(wl), synth.make_x(wl)


def _t(a):
    return torch.from_numpy(np.asarray(a, np.float64))


@pytest.mark.parametrize("fmt", [synth.Q8_0, synth.Q4_0])
def test_block_equals_dense_masked_brute_force(orc, fmt):
    wl, layer, xb = _tiny_layer(fmt=fmt)
    s = wl.shape
    y, idx, w, _ = orc.latent_moe_forward(s, layer, xb)
    # independent arrangement: every expert on every token, then a [T, E] mask of weights
    x = _t(orc.bf16_to_f64(xb))
    Wr = _t(layer["router_w"].astype(np.float64))
    logits = x @ Wr.T + _t(layer["router_b"].astype(np.float64))
    T = x.shape[0]
    M = torch.zeros(T, s.n_experts, dtype=torch.float64)
    for t in range(T):
        sel, ws = _brute_route(logits[t].tolist(), s.top_k)
        for e, v in zip(sel, ws):
            M[t, e] = v
    grp = layer["expert_group"].astype(np.int64)
    D = [_t(orc.decode_du(fmt, orc.du_slice(layer["D"], fmt, g, s.latent, s.hidden), s.latent, s.hidden))
         for g in range(s.n_groups)]
    U = [_t(orc.decode_du(fmt, orc.du_slice(layer["U"], fmt, g, s.hidden, s.latent), s.hidden, s.latent))
         for g in range(s.n_groups)]
    out_all = torch.zeros(T, s.n_experts, s.latent, dtype=torch.float64)
    for e in range(s.n_experts):
        Wg, Wu, Wd = (_t(m) for m in orc.decode_expert(orc.expert_slice(layer["experts"], e, s.latent, s.ffn),
                                                       s.latent, s.ffn))
        h = x @ D[grp[e]].T                                              # [T, latent]
        out_all[:, e] = (torch.nn.functional.silu(h @ Wg.T) * (h @ Wu.T)) @ Wd.T
    Wsg, Wsu = _t(orc.bf16_to_f64(layer["shared_gate"])), _t(orc.bf16_to_f64(layer["shared_up"]))
    Wsd = _t(orc.bf16_to_f64(layer["shared_down"]))
    y_bf = (torch.nn.functional.silu(x @ Wsg.T) * (x @ Wsu.T)) @ Wsd.T
    for g in range(s.n_groups):
        mask_g = M * torch.tensor(grp == g, dtype=torch.float64)[None, :]
        s_g = torch.einsum("te,tel->tl", mask_g, out_all)
        y_bf = y_bf + s_g @ U[g].T
    np.testing.assert_allclose(y, y_bf.numpy(), rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(M.numpy()[np.arange(T)[:, None], idx], w, rtol=1e-12)


def test_block_linearity_of_U(orc):
    """U_g applied to the per-group sum equals the sum of U_g applied to each
    weighted expert output (the pieces recomputed here in torch from the
    decoded matrices)."""
    wl, layer, xb = _tiny_layer()
    s = wl.shape
    y, idx, w, _ = orc.latent_moe_forward(s, layer, xb)
    W = orc.Weights(s, layer)
    F = torch.nn.functional
    x = _t(orc.bf16_to_f64(xb))
    y2 = (F.silu(x @ _t(W.Wsg).T) * (x @ _t(W.Wsu).T)) @ _t(W.Wsd).T
    for t in range(x.shape[0]):
        for k in range(s.top_k):
            e = int(idx[t, k])
            g = int(W.group[e])
            Wg, Wu, Wd = (_t(m) for m in W.expert(e))
            h = _t(W.D(g)) @ x[t]
            o = Wd @ (F.silu(Wg @ h) * (Wu @ h))
            y2[t] += _t(W.U(g)) @ (float(w[t, k]) * o)
    np.testing.assert_allclose(y, y2.numpy(), rtol=1e-10, atol=1e-13)


def test_block_single_expert_single_group_is_textbook_chain(orc):
    s = synth.replace(TINY, n_experts=1, top_k=1, n_groups=1)
    wl, layer, xb = _tiny_layer(shape=s)
    y, idx, w, _ = orc.latent_moe_forward(s, layer, xb)
    assert np.all(idx == 0) and np.all(w == 1.0)
    x = _t(orc.bf16_to_f64(xb))
    D = _t(orc.decode_q8_0(layer["D"], s.latent, s.hidden))
    U = _t(orc.decode_q8_0(layer["U"], s.hidden, s.latent))
    Wg, Wu, Wd = (_t(m) for m in orc.decode_expert(layer["experts"], s.latent, s.ffn))
    Wsg, Wsu = _t(orc.bf16_to_f64(layer["shared_gate"])), _t(orc.bf16_to_f64(layer["shared_up"]))
    Wsd = _t(orc.bf16_to_f64(layer["shared_down"]))
    F = torch.nn.functional
    h = x @ D.T
    want = (F.silu(h @ Wg.T) * (h @ Wu.T)) @ Wd.T @ U.T + (F.silu(x @ Wsg.T) * (x @ Wsu.T)) @ Wsd.T
    np.testing.assert_allclose(y, want.numpy(), rtol=1e-11, atol=1e-14)


def test_block_zero_input_gives_zero(orc):
    wl, layer, xb = _tiny_layer()
    y, _, _, _ = orc.latent_moe_forward(wl.shape, layer, np.zeros_like(xb))
    assert np.all(y == 0.0)


def test_block_zero_experts_gives_shared_only(orc):
    wl, layer, xb = _tiny_layer()
    layer = dict(layer)
    layer["experts"] = np.zeros_like(layer["experts"])
    y, _, _, _ = orc.latent_moe_forward(wl.shape, layer, xb)
    F = torch.nn.functional
    x = _t(orc.bf16_to_f64(xb))
    bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).double()
    want = (F.silu(x @ bf(layer["shared_gate"]).T) * (x @ bf(layer["shared_up"]).T)) @ bf(layer["shared_down"]).T
    # fp64 sums in another order: equal to rounding
    np.testing.assert_allclose(y, want.numpy(), rtol=1e-12, atol=1e-14)


def _identity_q8_0(n):
    """Q8_0 identity matrix [n, n] packed by hand: q = 1 on the diagonal, d = 1.0."""
    blob = bytearray(n * n + n * n // 16)
    for r in range(n):
        blob[((r // 32) * n + r) * 32 + r % 32] = 1
        for b in range(n // 32):
            off = n * n + 2 * (b * n + r)
            blob[off], blob[off + 1] = 0x00, 0x3C                  # fp16 1.0
    return np.frombuffer(bytes(blob), np.uint8)


def test_block_identity_latent_reduces_to_standard_moe(orc):
    s = synth.replace(TINY, latent=TINY.hidden)
    wl, layer, xb = _tiny_layer(shape=s)
    layer = dict(layer)
    I = _identity_q8_0(s.hidden)
    layer["D"] = np.concatenate([I] * s.n_groups)
    layer["U"] = np.concatenate([I] * s.n_groups)
    y, idx, w, _ = orc.latent_moe_forward(s, layer, xb)
    F = torch.nn.functional
    x = _t(orc.bf16_to_f64(xb))
    want = (F.silu(x @ _t(orc.bf16_to_f64(layer["shared_gate"])).T) * (x @ _t(orc.bf16_to_f64(layer["shared_up"])).T)) \
        @ _t(orc.bf16_to_f64(layer["shared_down"])).T
    for t in range(x.shape[0]):
        for k in range(s.top_k):
            Wg, Wu, Wd = (_t(m) for m in orc.decode_expert(orc.expert_slice(layer["experts"], int(idx[t, k]),
                                                                             s.latent, s.ffn), s.latent, s.ffn))
            want[t] += w[t, k] * (Wd @ (F.silu(Wg @ x[t]) * (Wu @ x[t])))
    np.testing.assert_allclose(y, want.numpy(), rtol=1e-11, atol=1e-14)


def test_block_injection_overrides_routing(orc):
    wl, layer, xb = _tiny_layer()
    s = wl.shape
    T = xb.shape[0]
    inj_idx = np.tile(np.arange(s.top_k), (T, 1))
    inj_w = np.full((T, s.top_k), 1.0 / s.top_k)
    y, idx, w, _ = orc.latent_moe_forward(s, layer, xb, inject_idx=inj_idx, inject_w=inj_w)
    assert np.array_equal(idx, inj_idx) and np.array_equal(w, inj_w)
    y_ref, _, _, _ = orc.latent_moe_forward(s, layer, xb)
    assert orc.rel_l2(y, y_ref) > 1e-3


def test_residual_adds(orc):
    wl, layer, xb = _tiny_layer()
    r = synth.bf16_normal(123, 1.0, xb.shape)
    y0, _, _, _ = orc.latent_moe_forward(wl.shape, layer, xb)
    y1, _, _, _ = orc.latent_moe_forward(wl.shape, layer, xb, residual_bits=r)
    np.testing.assert_allclose(y1 - y0, orc.bf16_to_f64(r), rtol=0, atol=1e-12)


def test_rmsnorm_closed_form(orc):
    v = np.array([[3.0, -4.0], [0.0, 0.0]])
    g = np.array([2.0, 0.5])
    out = orc.rmsnorm(v, g, 0.0 + 1e-30)
    r = math.sqrt((9 + 16) / 2)
    np.testing.assert_allclose(out[0], [2 * 3 / r, 0.5 * -4 / r], rtol=1e-15)
    assert np.all(out[1] == 0)
    np.testing.assert_allclose(orc.rmsnorm(np.array([[1.0, 1.0]]), np.ones(2), 1.0), [[1 / math.sqrt(2)] * 2])


def test_stack_layer_is_residual_plus_block_of_norm(orc):
    wl, layer, xb = _tiny_layer()
    s = wl.shape
    gamma = np.linspace(0.5, 1.5, s.hidden)
    y, _, _, _ = orc.stack_layer_forward(s, layer, xb, gamma, 1e-6)
    x = orc.bf16_to_f64(xb)
    ms = (x * x).mean(axis=1, keepdims=True)
    xn = gamma[None, :] * x / np.sqrt(ms + 1e-6)
    blk, _, _, _ = orc.latent_moe_forward(s, layer, None, x_f64=xn)
    np.testing.assert_allclose(y, x + blk, rtol=1e-13, atol=1e-14)


# ----------------------------------------------------------------------------
# slicing of the D / U blobs and of the expert array, against the generator
# ----------------------------------------------------------------------------

def test_slices_match_the_generators_own_draws(orc):
    """du_slice(g) and expert_slice(e) pick the bytes the generator wrote for
    group g and expert e: re-encoding that index's own fp64 draws gives the
    same bytes, and decoding the slice gives those draws back within each
    format's rounding step.  An off-by-one group or record, or a transposed
    decode, fails."""
    s = synth.LayerShape(hidden=128, latent=64, n_experts=7, top_k=2, n_groups=3, ffn=64, shared_ffn=64,
                         du_fmt=synth.Q8_0, router_dtype="bf16")
    for fmt in (synth.Q8_0, synth.Q4_0):
        wl = synth.Workload("slices", synth.replace(s, du_fmt=fmt), T=2, seed=21, weight_sigma=0.05)
        layer = synth.make_layer(wl)
        for name, R, C in (("D", s.latent, s.hidden), ("U", s.hidden, s.latent)):
            for g in range(s.n_groups):
                w = synth.f64_normal(synth.key(wl.seed, 0, name, g), wl.weight_sigma, (R, C))
                sl = orc.du_slice(layer[name], fmt, g, R, C)
                assert np.array_equal(sl, synth.qmatrix_encode(fmt, w)), (name, g)
                amax = np.abs(w).reshape(R, C // 32, 32).max(axis=2)
                step = np.repeat(amax / (127.0 if fmt == synth.Q8_0 else 8.0), 32, axis=1)
                assert np.all(np.abs(orc.decode_du(fmt, sl, R, C) - w) <= step * 1.01 + 1e-12), (name, g)
    wl = synth.Workload("slices", s, T=2, seed=22, weight_sigma=0.05)
    layer = synth.make_layer(wl)
    kx = synth.key(wl.seed, 0, "experts")
    for e in (0, 3, s.n_experts - 1):
        ws = [synth.f64_normal(synth.expert_key(kx, e, m), wl.weight_sigma, shp)
              for m, shp in enumerate([(s.ffn, s.latent), (s.ffn, s.latent), (s.latent, s.ffn)])]
        rec = orc.expert_slice(layer["experts"], e, s.latent, s.ffn)
        assert np.array_equal(rec, synth.expert_record_encode(*ws)), e
        for want, got in zip(ws, orc.decode_expert(rec, s.latent, s.ffn)):
            # E2M1 with its E4M3 block scale: within half the widest grid gap
            # (2 of the block's 6 levels) of the block maximum
            amax16 = np.repeat(np.abs(want).reshape(want.shape[0], -1, 16).max(axis=2), 16, axis=1)
            assert np.all(np.abs(got - want) <= amax16 / 6.0 * 1.0625 + 1e-12), e


# ----------------------------------------------------------------------------
# the stack: a closed-form two-layer case
# ----------------------------------------------------------------------------

def _exact_nvfp4_matrix(rng, R, C, unit):
    """Values e2m1 * unit with +-6 * unit at the head of every 16-block, so
    that NVFP4 encodes them exactly when unit / (6 * 448) * 6 is a power of
    two (unit = 7 / 256 gives the tensor scale 2^-14 and block scale 448)."""
    grid = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    v = grid[rng.integers(0, 8, size=(R, C))] * np.where(rng.random((R, C)) < 0.5, -1.0, 1.0)
    v[:, ::16] = 6.0 * np.where(rng.random((R, C // 16)) < 0.5, -1.0, 1.0)
    return v * unit


def test_stack_two_layers_closed_form(orc):
    """Two pre-norm residual layers with identity D and U (latent = hidden),
    one expert always chosen with weight 1 and exactly representable NVFP4
    weights: each layer is x + S(n(x)) + W_d(silu(W_g n(x)) * W_u n(x)) with
    n = RMSNorm, written out here in torch; the second layer reads the first
    layer's output rounded to bf16, as the stack keeps its residual stream."""
    H = 64
    s = synth.LayerShape(hidden=H, latent=H, n_experts=2, top_k=1, n_groups=1, ffn=64, shared_ffn=64,
                         du_fmt=synth.Q8_0, router_dtype="f32")
    rng = np.random.default_rng(31)
    unit = 7.0 / 256.0
    F = torch.nn.functional
    bf = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).double()
    xb = synth.bf16_normal(synth.key(9, 0, "x"), 1.0, (3, H))
    x_ref = bf(xb)
    eps = 1e-6
    for layer_i in range(2):
        wl = synth.Workload("stack2", s, T=3, seed=40 + layer_i, weight_sigma=0.1)
        layer = synth.make_layer(wl)
        layer["router_w"] = np.zeros((2, H), np.float32)
        layer["router_b"] = np.array([5.0, 0.0], np.float32)
        layer["expert_group"] = np.zeros(2, np.uint8)
        layer["D"] = _identity_q8_0(H)
        layer["U"] = _identity_q8_0(H)
        Wg, Wu, Wd = (_exact_nvfp4_matrix(rng, H, H, unit) for _ in range(3))
        rec = synth.expert_record_encode(Wg, Wu, Wd)
        layer["experts"] = np.concatenate([rec, np.zeros_like(rec)])
        gamma = np.linspace(0.5, 1.5, H) + 0.25 * layer_i
        y, idx, w, _ = orc.stack_layer_forward(s, layer, xb, gamma, eps)
        assert np.all(idx == 0) and np.all(w == 1.0)
        n = _t(gamma)[None, :] * x_ref / torch.sqrt((x_ref * x_ref).mean(dim=1, keepdim=True) + eps)
        shared = (F.silu(n @ bf(layer["shared_gate"]).T) * (n @ bf(layer["shared_up"]).T)) @ bf(layer["shared_down"]).T
        expert = (F.silu(n @ _t(Wg).T) * (n @ _t(Wu).T)) @ _t(Wd).T
        want = x_ref + shared + expert
        np.testing.assert_allclose(y, want.numpy(), rtol=1e-12, atol=1e-13)
        # the next layer's input: this layer's output rounded to bf16 (here, by torch)
        x_ref = want.to(torch.bfloat16).double()
        xb = want.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ----------------------------------------------------------------------------
# the two oracles against each other (independent implementations)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [synth.Q8_0, synth.Q4_0])
def test_cpp_and_numpy_oracles_agree(fmt):
    s = synth.LayerShape(hidden=256, latent=128, n_experts=24, top_k=5, n_groups=4, ffn=128, shared_ffn=64,
                         du_fmt=fmt, router_dtype="bf16")
    wl = synth.Workload("agree", s, T=7, seed=17, bias_sigma=0.5, weight_sigma=0.05)
    layer = synth.make_layer(wl)
    xb = synth.make_x(wl)
    res = synth.bf16_normal(synth.key(17, 0, "residual"), 1.0, xb.shape)
    a = cpp_oracle.latent_moe_forward(s, layer, xb, residual_bits=res)
    b = np_oracle.latent_moe_forward(s, layer, xb, residual_bits=res)
    assert np.array_equal(a[1], b[1])
    np.testing.assert_allclose(a[2], b[2], rtol=1e-13)
    np.testing.assert_allclose(a[0], b[0], rtol=1e-11, atol=1e-13)
    gamma = np.linspace(0.8, 1.2, s.hidden)
    c = cpp_oracle.stack_layer_forward(s, layer, xb, gamma, 1e-6)
    d = np_oracle.stack_layer_forward(s, layer, xb, gamma, 1e-6)
    np.testing.assert_allclose(c[0], d[0], rtol=1e-11, atol=1e-13)


# ----------------------------------------------------------------------------
# the reference-kernel ablation: Q8_1 activations, D over every group
# ----------------------------------------------------------------------------

def test_q8_1_quantisation_rule():
    """d = fp16(amax / 127), q = rint(x / d) (fp32): a hand case, a zero
    block, and the rounding bound |x - d q| <= d / 2 on random rows."""
    x = np.zeros((1, 64), np.float32)
    x[0, :4] = [1.0, -0.5, 0.25, 127.0 / 128.0]          # amax 1: d = fp16(1/127)
    q, d = cpp_oracle.quantize_q8_1(x)
    dv = float(np.array([d[0, 0]], np.uint16).view(np.float16)[0])
    assert dv == float(np.float16(np.float32(1.0) / np.float32(127.0)))
    want = [int(np.rint(np.float32(v) / np.float32(dv))) for v in x[0, :4]]
    assert q[0, :4].tolist() == want and want[0] == 127
    assert np.all(q[0, 32:] == 0) and d[0, 1] == 0       # an all-zero block
    rng = np.random.default_rng(41)
    x = rng.normal(size=(5, 256)).astype(np.float32)
    q, d = cpp_oracle.quantize_q8_1(x)
    dv = d.view(np.float16).astype(np.float64).repeat(32, axis=1)
    assert np.all(np.abs(q) <= 127)
    assert np.all(np.abs(x - dv * q) <= dv * 0.5 * (1 + 1e-6) + 1e-12)


@pytest.mark.parametrize("fmt", [synth.Q8_0, synth.Q4_0])
def test_dproj_q8_1_exact_inputs_equal_plain_projection(fmt):
    """Rows that Q8_1 represents exactly (d = 2^-6 and integer multiples,
    +-127 d in every block) give exactly D_g x, with D decoded by the pinned
    decoder and multiplied in torch."""
    G, L, H = 3, 64, 128
    wl = synth.Workload("abl", synth.LayerShape(hidden=H, latent=L, n_experts=4, top_k=2, n_groups=G, ffn=64,
                                                 shared_ffn=64, du_fmt=fmt), T=3, seed=7, weight_sigma=0.05)
    layer = synth.make_layer(wl)
    rng = np.random.default_rng(43)
    k = rng.integers(-127, 128, size=(3, H))
    k[:, ::32] = 127 * np.where(rng.random((3, H // 32)) < 0.5, -1, 1)
    x = (k * 2.0 ** -6).astype(np.float32)
    h = cpp_oracle.dproj_q8_1(fmt, layer["D"], G, L, H, x)
    for g in range(G):
        Dg = torch.from_numpy(np_oracle.decode_du(fmt, np_oracle.du_slice(layer["D"], fmt, g, L, H), L, H))
        want = torch.from_numpy(x.astype(np.float64)) @ Dg.T
        np.testing.assert_allclose(h[:, g], want.numpy(), rtol=1e-12, atol=1e-12)


def test_dproj_q8_1_equals_projection_of_the_dequantised_rows():
    G, L, H = 2, 64, 256
    wl = synth.Workload("abl", synth.LayerShape(hidden=H, latent=L, n_experts=4, top_k=2, n_groups=G, ffn=64,
                                                 shared_ffn=64, du_fmt=synth.Q4_0), T=4, seed=8, weight_sigma=0.05)
    layer = synth.make_layer(wl)
    x = np.random.default_rng(44).normal(size=(4, H)).astype(np.float32)
    q, d = cpp_oracle.quantize_q8_1(x)
    xq = torch.from_numpy(q.astype(np.float64) * d.view(np.float16).astype(np.float64).repeat(32, axis=1))
    h = cpp_oracle.dproj_q8_1(synth.Q4_0, layer["D"], G, L, H, x)
    for g in range(G):
        Dg = torch.from_numpy(np_oracle.decode_du(synth.Q4_0, np_oracle.du_slice(layer["D"], synth.Q4_0, g, L, H), L, H))
        np.testing.assert_allclose(h[:, g], (xq @ Dg.T).numpy(), rtol=1e-12, atol=1e-13)


# ----------------------------------------------------------------------------
# the Q3_K gate/up + IQ4_NL down expert build
# ----------------------------------------------------------------------------

def test_q3k_build_sizes_match_pages(orc):
    """The record sizes and build totals the pages print for the Q3_K build,
    with the Q8_0 (145B) and Q4_0 (120B) D/U of the NVFP4 builds."""
    g = _gold("page_figures.json")
    H, E, G, F, NL = (g[k]["value"] for k in ("hidden", "experts_per_layer", "groups", "swiglu_width", "layers"))
    L145, L120 = g["latent_145b"]["value"], g["latent_120b"]["value"]
    assert orc.expert_record_bytes(L145, F, "q3k") == g["q3k_record_bytes_latent1792"]["value"]
    assert 2 * (F * L145 // 256 * 110) == g["q3k_record_gateup_bytes_latent1792"]["value"]
    assert L145 * F // 32 * 18 == g["q3k_record_down_bytes_latent1792"]["value"]
    assert orc.expert_record_bytes(L120, F, "q3k") == g["q3k_record_bytes_latent1280"]["value"]
    b145 = NL * (E * orc.expert_record_bytes(L145, F, "q3k") + 2 * G * orc.du_matrix_bytes(orc.Q8_0, L145, H))
    b120 = NL * (E * orc.expert_record_bytes(L120, F, "q3k") + 2 * G * orc.du_matrix_bytes(orc.Q4_0, L120, H))
    assert round(b145 / 2 ** 30, 2) == g["weights_145b_q3k_gib"]["value"]
    assert round(b120 / 2 ** 30, 2) == g["weights_120b_q3k_gib"]["value"]


def test_iq4nl_levels_are_the_scaled_normal_quantiles(orc):
    from scipy.stats import norm
    z = norm.ppf((np.arange(16) + 0.5) / 16.0)
    np.testing.assert_array_equal(orc.iq4nl_levels(), np.rint(127.0 * z / z[-1]))
    assert orc.iq4nl_levels()[0] == -127 and orc.iq4nl_levels()[15] == 127


def test_decode_q3k_hand_packed(orc):
    """Codes, sub-block scales and super-block scales placed bit by bit from
    the documented arrangement; w = d * (sc - 32) * (q - 4)."""
    R, C = 3, 512
    rng = np.random.default_rng(51)
    q = rng.integers(0, 8, size=(R, C))
    sc = rng.integers(0, 64, size=(R, C // 16))
    d = rng.choice([0.5, 0.25, 0.0078125, 1.5], size=(R, C // 256))
    nh = C // 128
    lo = bytearray(nh * R * 32)
    hi = bytearray(nh * R * 16)
    scb = bytearray(nh * R * 6)
    db = bytearray(2 * (C // 256) * R)
    want = np.zeros((R, C))
    for r in range(R):
        for c in range(C):
            h, e = divmod(c, 128)
            lo[(h * R + r) * 32 + 4 * (e // 16) + e % 4] |= (int(q[r, c]) & 3) << (2 * ((e % 16) // 4))
            if q[r, c] & 4:
                hi[(h * R + r) * 16 + 4 * (e // 32) + e % 4] |= 1 << ((e % 32) // 4)
            want[r, c] = d[r, c // 256] * (sc[r, c // 16] - 32) * (q[r, c] - 4)
        for h in range(nh):
            word = sum(int(sc[r, h * 8 + j]) << (6 * j) for j in range(8))
            for k in range(6):
                scb[(h * R + r) * 6 + k] = (word >> (8 * k)) & 0xFF
        for sb in range(C // 256):
            bits = _fp16_bits(d[r, sb])
            db[2 * (sb * R + r)], db[2 * (sb * R + r) + 1] = bits & 0xFF, bits >> 8
    blob = np.frombuffer(bytes(lo + hi + scb + db), np.uint8)
    assert blob.size == R * C // 256 * 110
    np.testing.assert_array_equal(orc.decode_q3k(blob, R, C), want)


def test_decode_iq4nl_hand_packed(orc):
    R, C = 2, 64
    rng = np.random.default_rng(52)
    q = rng.integers(0, 16, size=(R, C))
    d = rng.choice([0.5, -0.25, 2.0 ** -10], size=(R, C // 32))
    from scipy.stats import norm
    z = norm.ppf((np.arange(16) + 0.5) / 16.0)
    lev = np.rint(127.0 * z / z[-1])
    blob = bytearray(R * C // 2 + R * C // 16)
    want = np.zeros((R, C))
    for r in range(R):
        for c in range(C):
            b, j = divmod(c, 32)
            blob[(b * R + r) * 16 + j % 16] |= int(q[r, c]) << (0 if j < 16 else 4)
            want[r, c] = lev[q[r, c]] * d[r, b]
        for b in range(C // 32):
            bits = _fp16_bits(d[r, b])
            off = R * C // 2 + 2 * (b * R + r)
            blob[off], blob[off + 1] = bits & 0xFF, bits >> 8
    np.testing.assert_array_equal(orc.decode_iq4nl(np.frombuffer(bytes(blob), np.uint8), R, C), want)


def test_q3k_generator_round_trip(orc):
    """The generator's Q3_K / IQ4_NL bytes decode to the matrices it encoded,
    within each format's grid: Q3_K within one sub-block step (|s| <= amax/4
    of the 16 elements, plus the 6-bit rounding of s), IQ4_NL within the
    widest half-gap of the levels (37/2 of d = amax/127)."""
    rng = np.random.default_rng(53)
    w = rng.normal(0, 0.02, size=(32, 512))
    back = orc.decode_q3k(synth.q3k_encode(w), 32, 512)
    amax16 = np.repeat(np.abs(w).reshape(32, -1, 16).max(axis=2), 16, axis=1)
    assert np.all(np.abs(back - w) <= amax16 * 0.35 + 1e-12)
    assert orc.rel_l2(back, w) < 0.2
    back = orc.decode_iq4nl(synth.iq4nl_encode(w), 32, 512)
    amax32 = np.repeat(np.abs(w).reshape(32, -1, 32).max(axis=2), 32, axis=1)
    assert np.all(np.abs(back - w) <= amax32 / 127.0 * 18.6 + 1e-12)
    assert orc.rel_l2(back, w) < 0.12


def test_q3k_block_equals_dense_masked_brute_force(orc):
    """The block with Q3_K experts: every expert on every token, masked by the
    routing weights, in torch from the decoded matrices."""
    s = synth.replace(TINY, latent=256, expert_fmt="q3k")
    wl, layer, xb = _tiny_layer(shape=s)
    y, idx, w, _ = orc.latent_moe_forward(s, layer, xb)
    F = torch.nn.functional
    x = _t(orc.bf16_to_f64(xb))
    logits = x @ _t(layer["router_w"].astype(np.float64)).T + _t(layer["router_b"].astype(np.float64))
    grp = layer["expert_group"].astype(np.int64)
    bf = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).double()
    want = (F.silu(x @ bf(layer["shared_gate"]).T) * (x @ bf(layer["shared_up"]).T)) @ bf(layer["shared_down"]).T
    for t in range(x.shape[0]):
        sel, ws = _brute_route(logits[t].tolist(), s.top_k)
        assert list(idx[t]) == sel
        for g in sorted({int(grp[e]) for e in sel}):
            Dg = _t(orc.decode_du(s.du_fmt, orc.du_slice(layer["D"], s.du_fmt, g, s.latent, s.hidden), s.latent, s.hidden))
            Ug = _t(orc.decode_du(s.du_fmt, orc.du_slice(layer["U"], s.du_fmt, g, s.hidden, s.latent), s.hidden, s.latent))
            h = Dg @ x[t]
            acc = torch.zeros(s.latent, dtype=torch.float64)
            for e, wk in zip(sel, ws):
                if grp[e] != g:
                    continue
                Wg, Wu, Wd = (_t(m) for m in orc.decode_expert(orc.expert_slice(layer["experts"], e, s.latent, s.ffn, "q3k"),
                                                               s.latent, s.ffn, "q3k"))
                acc += wk * (Wd @ (F.silu(Wg @ h) * (Wu @ h)))
            want[t] += Ug @ acc
    np.testing.assert_allclose(y, want.numpy(), rtol=1e-10, atol=1e-12)
