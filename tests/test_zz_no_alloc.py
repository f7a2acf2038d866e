"""The router entry point that allocates nothing, against the ordinary one.

Some callers cannot call cudaMalloc (a host framework that owns all device
memory, or a path with no workspace to hand in); lmoe_route_noalloc keeps its
scratch in a fixed array inside the library.  This file is collected last so
that a run stopping at the first failure has already run every other test."""
import numpy as np
import pytest
import torch

from latent_mixture_experts_softmax_b200 import binding as B
from latent_mixture_experts_softmax_b200 import build, synth
from latent_mixture_experts_softmax_b200.layer import DeviceLayer, to_device

from parity import W_RTOL

pytestmark = pytest.mark.gpu


def test_route_noalloc_matches_route_on_two_calls():
    build.build_all()
    wl = synth.WORKLOADS["edge0_120b_decode"]
    layer = synth.make_layer(wl)
    dev = DeviceLayer(wl.shape, layer)
    K = wl.shape.top_k
    for call, T in enumerate((4, 33)):            # two calls in a row, different sizes
        xb = synth.make_x(wl, T=T, draw=500 + call)
        x = to_device(xb, "cuda")
        ref_idx, ref_w = dev.route(x, dev.workspace(T))
        idx = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
        w = torch.full((T, K), -1.0, dtype=torch.float32, device="cuda")
        B.lmoe_route_noalloc(dev.cfg, x, dev.router_w, dev.router_b, T, idx, w)
        torch.cuda.synchronize()
        assert torch.equal(idx.cpu(), ref_idx.cpu()), f"call {call}"
        np.testing.assert_allclose(w.cpu().numpy(), ref_w.cpu().numpy(), rtol=W_RTOL, atol=1e-7)


def test_route_noalloc_rejects_sizes_beyond_its_scratch():
    build.build_all()
    wl = synth.WORKLOADS["edge0_120b_decode"]
    dev = DeviceLayer(wl.shape, synth.make_layer(wl))
    T = 65
    x = to_device(synth.make_x(wl, T=T), "cuda")
    idx = torch.empty((T, wl.shape.top_k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.shape.top_k), dtype=torch.float32, device="cuda")
    with pytest.raises(B.LmoeError) as err:
        B.lmoe_route_noalloc(dev.cfg, x, dev.router_w, dev.router_b, T, idx, w)
    assert err.value.status == B.LMOE_ERR_WORKSPACE
