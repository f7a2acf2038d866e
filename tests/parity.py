"""Parity helpers: run the CUDA path through the C ABI and the fp64 oracle on
the same seeded inputs, and compare them with the block's tolerance."""
from __future__ import annotations

import numpy as np
import torch

from latent_mixture_experts_softmax_b200 import synth
from latent_mixture_experts_softmax_b200.layer import DeviceLayer, to_device
from oracle import native as orc

# Tolerance of the block's output for bf16 activations with fp32 accumulation:
# relative L2 error and the largest error relative to the output's RMS.
REL_L2 = 5e-3
MAX_OVER_RMS = 2e-2
# Routing: below this gap between the K-th and (K+1)-th logit the fp32 router
# may legitimately order the two experts differently from the fp64 oracle; the
# oracle's routing is then injected into the CUDA run.
GAP = 1e-4
W_RTOL = 1e-5


def bf16_bits_to_f64(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.bfloat16).double().cpu().numpy()


def assert_close(y_gpu: np.ndarray, y_ref: np.ndarray, what: str = ""):
    r = orc.rel_l2(y_gpu, y_ref)
    m = orc.max_abs_over_rms(y_gpu, y_ref)
    assert r <= REL_L2 and m <= MAX_OVER_RMS, f"{what}: rel_l2={r:.3e} max/rms={m:.3e}"
    return r, m


def check_routing(idx_gpu, w_gpu, idx_ref, w_ref, gap):
    """Selected sets bit-exact for tokens whose top-K boundary is resolvable;
    weights within W_RTOL (same expert order)."""
    idx_gpu = np.asarray(idx_gpu)
    w_gpu = np.asarray(w_gpu, np.float64)
    n_checked = 0
    for t in range(idx_ref.shape[0]):
        if gap[t] < GAP:
            continue
        assert sorted(idx_gpu[t].tolist()) == sorted(idx_ref[t].tolist()), f"token {t}"
        o_g = np.argsort(idx_gpu[t], kind="stable")
        o_r = np.argsort(idx_ref[t], kind="stable")
        np.testing.assert_allclose(w_gpu[t][o_g], w_ref[t][o_r], rtol=W_RTOL, atol=1e-7)
        n_checked += 1
    return n_checked


def run_block(shape, layer_np: dict, x_bits: np.ndarray, residual_bits: np.ndarray | None = None,
              tokens: np.ndarray | None = None, dev: DeviceLayer | None = None, weights: orc.Weights | None = None):
    """Run both sides.  `tokens` restricts the oracle to a subset of rows (the
    block is per token).  Returns dict with y_gpu, y_ref, routing."""
    dev = dev or DeviceLayer(shape, layer_np)
    T = x_bits.shape[0]
    x = to_device(x_bits, "cuda")
    res = to_device(residual_bits, "cuda") if residual_bits is not None else None
    ws = dev.workspace(T)
    y, idx, w = dev.forward(x, ws, residual=res, want_routing=True)
    torch.cuda.synchronize()
    idx_g, w_g = idx.cpu().numpy(), w.cpu().numpy()
    rows = np.arange(T) if tokens is None else np.asarray(tokens)
    W = weights or orc.Weights(shape, layer_np, max_cached_experts=16)
    y_ref, idx_r, w_r, gap = orc.latent_moe_forward(shape, layer_np, x_bits[rows],
                                                     None if residual_bits is None else residual_bits[rows],
                                                     weights=W)
    out = {"idx_gpu": idx_g[rows], "w_gpu": w_g[rows], "idx_ref": idx_r, "w_ref": w_r, "gap": gap, "rows": rows}
    if np.any(gap < GAP):
        # inject the oracle routing for the whole batch (only the sampled rows are known)
        inj_i = idx.clone()
        inj_w = w.clone()
        inj_i[torch.from_numpy(rows).cuda()] = torch.from_numpy(idx_r.astype(np.int32)).cuda()
        inj_w[torch.from_numpy(rows).cuda()] = torch.from_numpy(w_r.astype(np.float32)).cuda()
        y = dev.forward(x, ws, residual=res, inject=(inj_i, inj_w))
        torch.cuda.synchronize()
        out["injected"] = True
    out["y_gpu"] = bf16_bits_to_f64(y)[rows]
    out["y_ref"] = y_ref
    out["status"] = dev_status(ws)
    return out


def dev_status(ws):
    from latent_mixture_experts_softmax_b200 import binding as B
    return B.lmoe_last_device_status(ws)


def check_block(shape, layer_np, x_bits, residual_bits=None, tokens=None, what="", **kw):
    out = run_block(shape, layer_np, x_bits, residual_bits, tokens, **kw)
    assert out["status"] == 0, f"device status {out['status']}"
    check_routing(out["idx_gpu"], out["w_gpu"], out["idx_ref"], out["w_ref"], out["gap"])
    out["rel_l2"], out["max_over_rms"] = assert_close(out["y_gpu"], out["y_ref"], what)
    return out


def small_shape(**kw):
    """Several tiles of every kernel with short loops: hidden 256, latent 128."""
    base = synth.LayerShape(hidden=256, latent=128, n_experts=40, top_k=6, n_groups=4, ffn=128, shared_ffn=64,
                            du_fmt=synth.Q8_0, router_dtype="bf16")
    return synth.replace(base, **kw)


def small_workload(T, seed=3, **kw):
    return synth.Workload("small", small_shape(**kw), T=T, seed=seed, groups="uniform", bias_sigma=0.5,
                          weight_sigma=0.05)
