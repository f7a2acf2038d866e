"""The seeded generator: determinism, per-element regeneration and the
distributions the workloads ask for."""
import numpy as np

from latent_mixture_experts_softmax_b200 import synth


def test_counter_based_elements_regenerate_alone():
    L = synth.lib()
    a = synth.f32_normal(99, 1.0, (1000,))
    for i in (0, 1, 2, 3, 517, 999):
        assert a[i] == np.float32(L.lmoe_synth_normal(99, i))


def test_normal_moments():
    a = synth.f32_normal(5, 0.02, (200000,)).astype(np.float64)
    assert abs(a.mean()) < 0.02 * 0.01
    assert abs(a.std() / 0.02 - 1.0) < 0.01


def test_streams_differ_and_repeat():
    k1, k2 = synth.key(0, 0, "D", 0), synth.key(0, 0, "D", 1)
    assert k1 != k2
    assert np.array_equal(synth.qmatrix(8, k1, 0.02, 32, 64), synth.qmatrix(8, k1, 0.02, 32, 64))
    assert not np.array_equal(synth.qmatrix(8, k1, 0.02, 32, 64), synth.qmatrix(8, k2, 0.02, 32, 64))


def test_groups():
    wl = synth.WORKLOADS["tiny"]
    assert list(synth.expert_groups(wl)[:10]) == [0, 1, 2, 3, 4, 5, 6, 7, 0, 1]
    g = synth.expert_groups(synth.WORKLOADS["edge0_145b_decode"])
    assert g.min() == 0 and g.max() == 7 and len(set(g.tolist())) == 8


def test_tiny_layer_sizes():
    wl = synth.WORKLOADS["tiny"]
    s = wl.shape
    layer = synth.make_layer(wl)
    assert layer["router_w"].dtype == np.float32 and layer["router_b"] is None
    assert layer["D"].size == s.n_groups * s.latent * s.hidden * 18 // 32
    assert layer["experts"].size == s.n_experts * synth.expert_record_bytes(s.latent, s.ffn)
