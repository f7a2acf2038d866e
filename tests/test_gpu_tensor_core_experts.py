"""The few-token NVFP4 expert phases on the tensor cores
(LMOE_FEW_TOKEN_EXPERTS=tensor_cores: tcgen05 kind::mxf4nvf4 with the
weights as stored and each activation row as six E2M1 terms), against the
fp64 oracle on the same tolerance as every block test.  The shapes span:
one and several 256-column K stages per item, a half-filled last stage
(ffn 640: down's third stage holds two of four MMA steps), items cut between
CTAs (their partial sums meet through tickets) and whole items, 1 to 8
tokens (B columns 16, 32 and 48)."""
import numpy as np
import pytest

from latent_mixture_experts_softmax_b200 import synth
from parity import check_block, small_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def tensor_core_experts(monkeypatch):
    monkeypatch.setenv("LMOE_FEW_TOKEN_EXPERTS", "tensor_cores")


@pytest.mark.parametrize("T", [1, 3, 8])
def test_small_shape(T):
    wl = small_workload(T, latent=256, ffn=128, n_experts=48)
    check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl), what=f"tensor-core experts small T={T}")


def test_one_stage_items_with_residual():
    wl = small_workload(5, latent=128, ffn=256)
    res = synth.bf16_normal(synth.key(6, 0, "residual"), 1.0, (5, wl.shape.hidden))
    check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl), residual_bits=res,
                what="tensor-core experts latent 128, ffn 256")


@pytest.mark.parametrize("name,T", [("edge0_145b_decode", 4), ("edge0_145b_decode", 1),
                                    ("edge0_120b_decode", 4), ("edge0_145b_decode", 8)])
def test_edge0_shapes(name, T):
    wl = synth.WORKLOADS[name].with_(T=T)
    out = check_block(wl.shape, synth.make_layer(wl), synth.make_x(wl, T=T), what=f"tensor-core experts {name} T={T}")
    assert np.isfinite(out["y_gpu"]).all()
