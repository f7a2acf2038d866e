"""CUDA path (through the C ABI) against the fp64 oracle on seeded inputs."""
import numpy as np
import pytest
import torch

from latent_mixture_experts_softmax_b200 import binding as B
from latent_mixture_experts_softmax_b200 import build, synth
from latent_mixture_experts_softmax_b200.layer import DeviceLayer, to_device
from oracle import native as orc

from parity import GAP, check_block, check_routing, small_workload, assert_close, bf16_bits_to_f64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    build.build_all()
    assert torch.cuda.is_available()


# ----------------------------------------------------------------------------
# storage-format decoders of the kernels, bit for bit
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", [synth.Q8_0, synth.Q4_0])
def test_decode_du_matches_oracle(fmt):
    R, C = 96, 256
    blob = synth.qmatrix(fmt, 77, 0.03, R, C)
    out = torch.empty(R, C, dtype=torch.float32, device="cuda")
    B.lmoe_debug_decode(fmt, to_device(blob, "cuda"), R, C, 1.0, out)
    ref = orc.decode_du(fmt, blob, R, C)
    np.testing.assert_array_equal(out.cpu().numpy().astype(np.float64), ref)


def test_decode_nvfp4_matches_oracle():
    L_, F_ = 128, 64
    rec = synth.experts_normal(5, 0.02, 1, L_, F_)
    nq, ns = L_ * F_ // 2, L_ * F_ // 16
    ts = np.frombuffer(rec[3 * nq + 3 * ns: 3 * nq + 3 * ns + 12].tobytes(), np.float32)
    for m, (R, C) in enumerate([(F_, L_), (F_, L_), (L_, F_)]):
        blob = np.concatenate([rec[m * nq:(m + 1) * nq], rec[3 * nq + m * ns:3 * nq + (m + 1) * ns]])
        out = torch.empty(R, C, dtype=torch.float32, device="cuda")
        B.lmoe_debug_decode(B.LMOE_NVFP4_DEBUG, to_device(blob, "cuda"), R, C, float(ts[m]), out)
        ref = orc.decode_nvfp4(blob[:nq], blob[nq:], ts[m], R, C)
        np.testing.assert_allclose(out.cpu().numpy().astype(np.float64), ref, rtol=2.0 ** -23, atol=0)


# ----------------------------------------------------------------------------
# router
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("name", ["tiny", "edge0_120b_decode", "edge0_145b_decode"])
def test_route_matches_oracle(name):
    wl = synth.WORKLOADS[name]
    layer = synth.make_layer(wl)
    dev = DeviceLayer(wl.shape, layer)
    n_ok = 0
    for draw in range(4):
        xb = synth.make_x(wl, T=16, draw=draw)
        ws = dev.workspace(16)
        idx, w = dev.route(to_device(xb, "cuda"), ws)
        W = orc.Weights(wl.shape, layer)
        idx_r, w_r, gap, _ = orc.route(orc.bf16_to_f64(xb), W.Wr, W.b, wl.shape.top_k)
        n_ok += check_routing(idx.cpu().numpy(), w.cpu().numpy(), idx_r, w_r, gap)
        # selection order is logit-descending: the weights must be non-increasing
        assert np.all(np.diff(w.cpu().numpy(), axis=1) <= 1e-7)
    assert n_ok >= 48


def test_route_ties_pick_lowest_index():
    s = synth.replace(synth.WORKLOADS["tiny"].shape, n_experts=64, top_k=4)
    wl = synth.Workload("ties", s, T=3, bias_sigma=None)
    layer = synth.make_layer(wl)
    layer["router_w"] = np.zeros_like(layer["router_w"])
    layer["router_b"] = np.zeros(64, np.float32)
    layer["router_b"][[5, 9, 17, 33, 40]] = 1.0          # five-way tie for four places
    dev = DeviceLayer(s, layer)
    idx, w = dev.route(to_device(synth.make_x(wl), "cuda"), dev.workspace(3))
    assert idx.cpu().tolist() == [[5, 9, 17, 33]] * 3
    np.testing.assert_allclose(w.cpu().numpy(), 0.25, rtol=1e-6)


# ----------------------------------------------------------------------------
# the block
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 2, 3, 4, 5, 8, 13, 37])
def test_block_small_shape_ragged_tokens(T):
    wl = small_workload(T)
    layer = synth.make_layer(wl)
    check_block(wl.shape, layer, synth.make_x(wl), what=f"T={T}")


@pytest.mark.parametrize("fmt", [synth.Q8_0, synth.Q4_0])
def test_block_small_shape_formats_with_residual(fmt):
    wl = small_workload(11, du_fmt=fmt, router_dtype="f32")
    layer = synth.make_layer(wl)
    res = synth.bf16_normal(synth.key(1, 0, "residual"), 1.0, (11, wl.shape.hidden))
    check_block(wl.shape, layer, synth.make_x(wl), residual_bits=res, what=f"fmt={fmt}")


def test_block_one_hot_expert_and_unhit_groups():
    """Every token routes to the same experts (one expert holds all T tokens,
    more than one pass of the token chunk) and most groups are never hit."""
    wl = small_workload(21)
    layer = synth.make_layer(wl)
    layer["router_b"] = np.full(wl.shape.n_experts, -50.0, np.float32)
    layer["router_b"][:wl.shape.top_k] = 50.0 + np.arange(wl.shape.top_k, dtype=np.float32)
    layer["expert_group"][:wl.shape.top_k] = 1
    out = check_block(wl.shape, layer, synth.make_x(wl), what="one-hot")
    assert np.all(np.sort(out["idx_gpu"], axis=1) == np.arange(wl.shape.top_k))


@pytest.mark.parametrize("T", [1, 8])
def test_block_few_tokens_one_hot_expert_and_unhit_groups(T):
    """The few-token path with every token on the same experts, all in one
    group: the other groups' h is computed and never read, one expert holds
    every token, and most warps of most CTAs get no steps."""
    wl = small_workload(T)
    layer = synth.make_layer(wl)
    layer["router_b"] = np.full(wl.shape.n_experts, -50.0, np.float32)
    layer["router_b"][:wl.shape.top_k] = 50.0 + np.arange(wl.shape.top_k, dtype=np.float32)
    layer["expert_group"][:] = 0
    layer["expert_group"][:wl.shape.top_k] = 2
    out = check_block(wl.shape, layer, synth.make_x(wl), what=f"few-token one-hot T={T}")
    assert np.all(np.sort(out["idx_gpu"], axis=1) == np.arange(wl.shape.top_k))


@pytest.mark.parametrize("fmt,T", [(synth.Q8_0, 3), (synth.Q4_0, 7)])
def test_block_few_tokens_ragged_steps(fmt, T):
    """Few tokens with step counts that do not divide the reductions (down:
    6 of 8 chunks in its only step) and a shared expert whose U items take
    more steps than the groups' (5 against 2 or 3)."""
    wl = small_workload(T, hidden=512, latent=384, n_experts=96, top_k=8, n_groups=6, ffn=192, shared_ffn=320,
                        du_fmt=fmt)
    layer = synth.make_layer(wl)
    res = synth.bf16_normal(synth.key(2, 0, "residual"), 1.0, (T, wl.shape.hidden))
    check_block(wl.shape, layer, synth.make_x(wl), residual_bits=res, what=f"ragged steps fmt={fmt} T={T}")


@pytest.mark.parametrize("T", [2, 8])
def test_block_wide_hidden_few_token_steps(T):
    """hidden 4096 (the D kernel's activation cache at its widest) with
    latent 256 and ffn 128 (one 256-column stage per gate/up item, a
    half-filled stage per down item on the tensor-core expert kernels), at 2
    and 8 tokens, against the oracle."""
    wl = small_workload(T, hidden=4096, latent=256, n_experts=48, top_k=6, n_groups=4, ffn=128, shared_ffn=128)
    layer = synth.make_layer(wl)
    check_block(wl.shape, layer, synth.make_x(wl), what=f"hidden 4096 T={T}")


def test_block_tiny_config():
    wl = synth.WORKLOADS["tiny"]
    check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl), what="tiny")


@pytest.mark.parametrize("name", ["edge0_120b_decode", "edge0_145b_decode"])
def test_block_decode_configs(name):
    wl = synth.WORKLOADS[name]
    layer = synth.make_layer(wl)
    dev = DeviceLayer(wl.shape, layer)
    W = orc.Weights(wl.shape, layer, max_cached_experts=16)
    for draw in range(3):
        check_block(wl.shape, layer, synth.make_x(wl, draw=draw), dev=dev, weights=W, what=f"{name} draw {draw}")


def _cover_rows(idx_all: np.ndarray, tile: int, per_tile: int) -> np.ndarray:
    """Rows to recompute on the CPU: per_tile rows from every `tile`-token
    tile, each picked (greedily, within its tile) to add the most experts not
    yet covered, so that the sample reaches nearly every expert the batch
    routes to and every tile of the tensor-core GEMMs."""
    T = idx_all.shape[0]
    covered = set()
    rows = []
    for t0 in range(0, T, tile):
        cand = list(range(t0, min(T, t0 + tile)))
        for _ in range(min(per_tile, len(cand))):
            best = max(cand, key=lambda t: (len(set(idx_all[t].tolist()) - covered), -t))
            cand.remove(best)
            rows.append(best)
            covered |= set(idx_all[best].tolist())
    return np.array(sorted(rows))


def _check_prefill_sampled(wl, T, per_tile, min_expert_cover):
    layer = synth.make_layer(wl)
    xb = synth.make_x(wl, T=T)
    dev = DeviceLayer(wl.shape, layer)
    idx, _ = dev.route(to_device(xb, "cuda"), dev.workspace(T))
    idx_all = idx.cpu().numpy()
    rows = _cover_rows(idx_all, 256, per_tile)
    assert len({r // 256 for r in rows}) == (T + 255) // 256           # every token tile
    routed = set(idx_all.reshape(-1).tolist())
    cover = set(idx_all[rows].reshape(-1).tolist())
    assert len(cover) >= min_expert_cover * len(routed), (len(cover), len(routed))
    out = check_block(wl.shape, layer, xb, tokens=rows, dev=dev, what=f"prefill T={T} sample")
    return out, rows


def test_block_prefill_config_sampled_tokens():
    """T=4096 through the same launch sequence the benchmark times; the oracle
    recomputes 128 rows (8 per 256-token tile) that reach >= 90% of the
    experts the batch routes to (the block is per token)."""
    wl = synth.WORKLOADS["edge0_145b_prefill"]
    _check_prefill_sampled(wl, 4096, 8, 0.9)


def test_forward_host_matches_device_call():
    wl = small_workload(6)
    layer = synth.make_layer(wl)
    dev = DeviceLayer(wl.shape, layer)
    xb = synth.make_x(wl)
    ws = dev.workspace(6)
    y_dev = dev.forward(to_device(xb, "cuda"), ws)
    x_h = torch.from_numpy(xb.view(np.int16)).pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    B.lmoe_forward_host(dev.cfg, x_h, dev.router_w, dev.router_b, dev.expert_group, dev.D, dev.U, dev.experts,
                        dev.shared, y_h, 6, ws)
    assert torch.equal(y_h, y_dev.cpu())


def test_forward_is_deterministic():
    wl = small_workload(37)
    layer = synth.make_layer(wl)
    dev = DeviceLayer(wl.shape, layer)
    x = to_device(synth.make_x(wl), "cuda")
    ws = dev.workspace(37)
    a = dev.forward(x, ws).clone()
    b = dev.forward(x, ws).clone()
    assert torch.equal(a, b)


def test_empty_batch_is_noop():
    wl = small_workload(4)
    dev = DeviceLayer(wl.shape, synth.make_layer(wl))
    y = torch.full((0, wl.shape.hidden), 7, dtype=torch.int16, device="cuda")
    x = torch.zeros((0, wl.shape.hidden), dtype=torch.int16, device="cuda")
    ws = dev.workspace(1)
    # zero-size tensors may have a null data pointer: pass a valid one
    B.lmoe_forward(dev.cfg, ws, dev.router_w, dev.expert_group, dev.D, dev.U, dev.experts, dev.shared, ws, 0, ws)


def test_bad_group_label_is_reported_not_faulted():
    wl = small_workload(4)
    layer = synth.make_layer(wl)
    layer["expert_group"][:] = 200                      # >= n_groups
    dev = DeviceLayer(wl.shape, layer)
    ws = dev.workspace(4)
    dev.forward(to_device(synth.make_x(wl), "cuda"), ws)
    assert B.lmoe_last_device_status(ws) == B.LMOE_ERR_DEVICE_CHECK
    assert B.lmoe_last_device_status(ws) == B.LMOE_OK       # read clears it


def test_stack_layers_against_oracle_layer_by_layer():
    wl = small_workload(5).with_(n_layers=3)
    s = wl.shape
    layers = [synth.make_layer(wl, layer=l) for l in range(wl.n_layers)]
    gammas = [synth.bf16_bits_from_f32(np.linspace(0.5, 1.5, s.hidden).astype(np.float32) + 0.1 * l)
              for l in range(wl.n_layers)]
    devs = [DeviceLayer(s, ly, gamma=g) for ly, g in zip(layers, gammas)]
    xb = synth.make_x(wl)
    x = to_device(xb, "cuda")
    ws = devs[0].workspace(wl.T)
    eps = 1e-6
    # layer by layer through the stack call with 1..n layers: each output is
    # checked against the oracle fed the GPU's own input of that layer
    cur = xb
    for l in range(wl.n_layers):
        y = torch.empty_like(x)
        B.lmoe_stack_forward(devs[0].cfg, [d.as_c_layer() for d in devs[:l + 1]], x, y, wl.T, eps, ws)
        torch.cuda.synchronize()
        y_ref, _, _, gap = orc.stack_layer_forward(s, layers[l], cur, orc.bf16_to_f64(gammas[l]), eps)
        assert np.all(gap >= GAP)
        assert_close(bf16_bits_to_f64(y), y_ref, f"stack layer {l}")
        cur = y.cpu().numpy().view(np.uint16)


# ----------------------------------------------------------------------------
# many tokens: the tensor-core path (every row compared)
# ----------------------------------------------------------------------------

def prefill_workload(T, seed=5, **kw):
    shape = synth.LayerShape(hidden=256, latent=128, n_experts=128, top_k=6, n_groups=4, ffn=128, shared_ffn=64,
                             du_fmt=synth.Q8_0, router_dtype="bf16")
    return synth.Workload("prefill_small", synth.replace(shape, **kw), T=T, seed=seed, groups="uniform",
                          bias_sigma=0.5, weight_sigma=0.05)


@pytest.mark.parametrize("T", [64, 300, 777])
def test_prefill_path_small_shape_all_rows(T):
    wl = prefill_workload(T)
    check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl), what=f"prefill T={T}")


@pytest.mark.parametrize("fmt", [synth.Q8_0, synth.Q4_0])
def test_prefill_path_formats_with_residual(fmt):
    wl = prefill_workload(260, du_fmt=fmt, latent=256)
    res = synth.bf16_normal(synth.key(2, 0, "residual"), 1.0, (260, wl.shape.hidden))
    check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl), residual_bits=res, what=f"prefill fmt={fmt}")


@pytest.mark.parametrize("latent,ffn", [(384, 192), (128, 320)])
def test_prefill_path_odd_row_tile_counts(latent, ffn):
    """The expert GEMMs take two 128-row weight tiles per item (gate/up: 64
    output features of gate and of up per tile; down: 128 rows of h); an odd
    number of tiles leaves the last item of each matrix with one."""
    wl = prefill_workload(200, latent=latent, ffn=ffn)
    check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl), what=f"prefill latent={latent} ffn={ffn}")


def test_prefill_path_skewed_expert_spans_several_tiles():
    """One expert takes every token (several 128-slot tiles of the expert GEMMs)."""
    wl = prefill_workload(400)
    layer = synth.make_layer(wl)
    layer["router_b"][7] = 40.0
    out = check_block(wl.shape, layer, synth.make_x(wl), what="skewed")
    assert np.all(out["idx_gpu"][:, 0] == 7)


def test_prefill_route_matches_oracle():
    wl = prefill_workload(500)
    layer = synth.make_layer(wl)
    dev = DeviceLayer(wl.shape, layer)
    xb = synth.make_x(wl)
    idx, w = dev.route(to_device(xb, "cuda"), dev.workspace(500))
    W = orc.Weights(wl.shape, layer)
    idx_r, w_r, gap, _ = orc.route(orc.bf16_to_f64(xb), W.Wr, W.b, wl.shape.top_k)
    assert check_routing(idx.cpu().numpy(), w.cpu().numpy(), idx_r, w_r, gap) >= 490


def test_prefill_stack_layers():
    wl = prefill_workload(130).with_(n_layers=2)
    s = wl.shape
    layers = [synth.make_layer(wl, layer=l) for l in range(2)]
    gammas = [synth.bf16_bits_from_f32(np.linspace(0.5, 1.5, s.hidden).astype(np.float32) + 0.2 * l) for l in range(2)]
    devs = [DeviceLayer(s, ly, gamma=g) for ly, g in zip(layers, gammas)]
    xb = synth.make_x(wl)
    x = to_device(xb, "cuda")
    ws = devs[0].workspace(wl.T)
    cur = xb
    for l in range(2):
        y = torch.empty_like(x)
        B.lmoe_stack_forward(devs[0].cfg, [d.as_c_layer() for d in devs[:l + 1]], x, y, wl.T, 1e-6, ws)
        torch.cuda.synchronize()
        y_ref, _, _, gap = orc.stack_layer_forward(s, layers[l], cur, orc.bf16_to_f64(gammas[l]), 1e-6)
        assert np.all(gap >= GAP)
        assert_close(bf16_bits_to_f64(y), y_ref, f"prefill stack layer {l}")
        cur = y.cpu().numpy().view(np.uint16)
    assert B.lmoe_last_device_status(ws) == B.LMOE_OK


def test_prefill_16384_tokens_sampled():
    """The largest configuration: 16384 tokens of the Edge0-145B-shaped layer,
    one oracle row per 256-token tile (64 rows) chosen to reach the most
    experts."""
    wl = synth.WORKLOADS["edge0_145b_prefill"].with_(T=16384)
    _check_prefill_sampled(wl, 16384, 1, 0.6)


# ----------------------------------------------------------------------------
# Edge0 shapes on the 9-63-token kernels and the full-shape stack
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("name,T", [("edge0_120b_decode", 16), ("edge0_145b_decode", 16),
                                    ("edge0_120b_decode", 48), ("edge0_145b_decode", 48)])
def test_block_edge0_shapes_between_9_and_63_tokens(name, T):
    """Routing and output at the Edge0 shapes on the kernels that take 9-63
    tokens in passes of 8 (every row compared)."""
    wl = synth.WORKLOADS[name]
    check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl, T=T, draw=7), what=f"{name} T={T}")


def test_stack_full_shape_145b_layer_by_layer():
    """Three Edge0-145B-shaped layers (hidden 2560, latent 1792, 512 experts,
    Q8_0 D/U) at T=4 through the stack call; each layer's output against the
    oracle fed the GPU's own input of that layer."""
    wl = synth.WORKLOADS["edge0_145b_stack"].with_(n_layers=3)
    s = wl.shape
    layers = [synth.make_layer(wl, layer=l) for l in range(wl.n_layers)]
    gammas = [synth.bf16_bits_from_f32((np.linspace(0.8, 1.2, s.hidden) + 0.05 * l).astype(np.float32))
              for l in range(wl.n_layers)]
    devs = [DeviceLayer(s, ly, gamma=g) for ly, g in zip(layers, gammas)]
    xb = synth.make_x(wl)
    x = to_device(xb, "cuda")
    ws = devs[0].workspace(wl.T)
    eps = 1e-6
    cur = xb
    for l in range(wl.n_layers):
        y = torch.empty_like(x)
        B.lmoe_stack_forward(devs[0].cfg, [d.as_c_layer() for d in devs[:l + 1]], x, y, wl.T, eps, ws)
        torch.cuda.synchronize()
        assert B.lmoe_last_device_status(ws) == B.LMOE_OK
        y_ref, _, _, gap = orc.stack_layer_forward(s, layers[l], cur, orc.bf16_to_f64(gammas[l]), eps)
        assert np.all(gap >= GAP)
        assert_close(bf16_bits_to_f64(y), y_ref, f"145B stack layer {l}")
        cur = y.cpu().numpy().view(np.uint16)


# ----------------------------------------------------------------------------
# inputs outside the fp16 range of the staged activations
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("T", [4, 16, 300])
def test_input_beyond_fp16_range_is_reported(T):
    """A block input of 1e5 (representable in bf16, not in fp16) is reported
    as LMOE_ERR_DEVICE_CHECK on every dispatch path (few tokens, 9-63
    tokens, tensor cores) instead of running on as inf."""
    wl = prefill_workload(T) if T >= 64 else small_workload(T)
    layer = synth.make_layer(wl)
    dev = DeviceLayer(wl.shape, layer)
    xb = synth.make_x(wl)
    xb[T // 2, 7] = synth.bf16_bits_from_f32(np.array([1e5], np.float32))[0]
    ws = dev.workspace(T)
    dev.forward(to_device(xb, "cuda"), ws)
    assert B.lmoe_last_device_status(ws) == B.LMOE_ERR_DEVICE_CHECK
    # the same call on an in-range input is clean again
    dev.forward(to_device(synth.make_x(wl), "cuda"), ws)
    assert B.lmoe_last_device_status(ws) == B.LMOE_OK


# ----------------------------------------------------------------------------
# the reference-kernel ablation of D_g
# ----------------------------------------------------------------------------

def _d_only(name):
    wl = synth.WORKLOADS[name]
    s = wl.shape
    D = np.concatenate([synth.qmatrix(s.du_fmt, synth.key(wl.seed, 0, "D", g), wl.weight_sigma, s.latent, s.hidden)
                        for g in range(s.n_groups)])
    return wl, s, D


@pytest.mark.parametrize("name", ["edge0_145b_decode", "edge0_120b_decode"])
@pytest.mark.parametrize("T", [1, 4, 11])
def test_dproj_ablation_matches_oracle(name, T):
    """Q8_1 activations over every group against the oracle's Q8_1 reading
    (integer products exact on both sides, fp32 sums on the GPU), and fp16
    activations over a subset of groups against D_g x (other groups left
    untouched)."""
    wl, s, D = _d_only(name)
    xb = synth.make_x(wl, T=T, draw=3)
    x32 = orc.bf16_to_f64(xb).astype(np.float32)
    cfg = B.make_cfg(s)
    ws = torch.zeros(B.lmoe_workspace_bytes(cfg, T), dtype=torch.uint8, device="cuda")
    Dd, xd = to_device(D, "cuda"), to_device(xb, "cuda")
    G, L, H = s.n_groups, s.latent, s.hidden
    h = torch.full((T, G, L), float("nan"), dtype=torch.float32, device="cuda")
    B.lmoe_dproj_ablation(cfg, xd, Dd, 1, (1 << G) - 1, h, T, ws)
    ref = orc.dproj_q8_1(s.du_fmt, D, G, L, H, x32)
    got = h.cpu().numpy().astype(np.float64)
    assert orc.rel_l2(got, ref) < 1e-5 and orc.max_abs_over_rms(got, ref) < 1e-4
    mask = 0b10110101 & ((1 << G) - 1)
    h.fill_(float("nan"))
    B.lmoe_dproj_ablation(cfg, xd, Dd, 0, mask, h, T, ws)
    got = h.cpu().numpy().astype(np.float64)
    for g in range(G):
        if mask >> g & 1:
            ref_g = orc.du_apply(s.du_fmt, orc.du_slice(D, s.du_fmt, g, L, H), L, H, x32)
            assert orc.rel_l2(got[:, g], ref_g) < 1e-4, g
        else:
            assert np.all(np.isnan(got[:, g])), g


# ----------------------------------------------------------------------------
# the Q3_K gate/up + IQ4_NL down expert build
# ----------------------------------------------------------------------------

def test_decode_q3k_iq4nl_match_oracle_bit_for_bit():
    rng = np.random.default_rng(61)
    w = rng.normal(0, 0.03, size=(48, 512))
    for fmt, blob, dec in ((B.LMOE_Q3K_DEBUG, synth.q3k_encode(w), orc.decode_q3k),
                           (B.LMOE_IQ4NL_DEBUG, synth.iq4nl_encode(w), orc.decode_iq4nl)):
        out = torch.empty(48, 512, dtype=torch.float32, device="cuda")
        B.lmoe_debug_decode(fmt, to_device(blob, "cuda"), 48, 512, 1.0, out)
        np.testing.assert_array_equal(out.cpu().numpy().astype(np.float64), dec(blob, 48, 512))


@pytest.mark.parametrize("T", [1, 4, 8, 13, 37])
def test_block_q3k_experts_few_tokens(T):
    """The few-token step with Q3_K gate/up and IQ4_NL down records (T <= 8:
    the weight-streaming kernels), and the same step on passes of 8 tokens
    (9-63)."""
    wl = small_workload(T, latent=256, expert_fmt="q3k")
    check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl), what=f"q3k T={T}")


def test_block_q3k_experts_tensor_cores():
    wl = prefill_workload(300, latent=256, expert_fmt="q3k")
    res = synth.bf16_normal(synth.key(4, 0, "residual"), 1.0, (300, wl.shape.hidden))
    check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl), residual_bits=res, what="q3k prefill")


def test_block_q3k_145b_decode_config():
    wl = synth.WORKLOADS["edge0_145b_q3k_decode"]
    layer = synth.make_layer(wl)
    dev = DeviceLayer(wl.shape, layer)
    for draw in range(2):
        check_block(wl.shape, layer, synth.make_x(wl, draw=draw), dev=dev, what=f"145B q3k draw {draw}")
