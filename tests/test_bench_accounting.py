"""The benchmark's algorithmic byte and FLOP counts (the numerators of its
roofline fractions) against the sizes of the arrays the layer is actually
stored in and a brute-force count of the routed work.  CPU only."""
import importlib.util
import os
import sys

import numpy as np
import pytest

from latent_mixture_experts_softmax_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    argv = sys.argv
    sys.argv = ["bench.py"]
    try:
        spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
    finally:
        sys.argv = argv
    return mod


def routing(shape, T, seed):
    """T tokens' top-k expert indices, distinct within a token."""
    rng = np.random.default_rng(seed)
    return np.stack([rng.choice(shape.n_experts, shape.top_k, replace=False) for _ in range(T)]).astype(np.int32)


@pytest.mark.parametrize("name,T", [("tiny", 1), ("tiny", 4), ("tiny", 8)])
def test_decode_bytes_match_stored_arrays(bench, name, T):
    """Few tokens: every hit group's D_g and U_g blocks, every routed expert's
    record (its 16-byte tensor-scale tail aside), the router and the shared
    expert, each read once, plus the activations in and out."""
    wl = synth.WORKLOADS[name]
    s = wl.shape
    layer = synth.make_layer(wl)
    groups = layer["expert_group"]
    idx = routing(s, T, seed=T)
    c = bench.step_cost(s, idx, groups, T, prefill=False)
    hit = sorted({int(groups[e]) for e in idx.reshape(-1)})
    distinct = sorted(set(idx.reshape(-1).tolist()))
    per_group_d = layer["D"].nbytes // s.n_groups
    per_group_u = layer["U"].nbytes // s.n_groups
    per_record = layer["experts"].nbytes // s.n_experts - 16
    shared = layer["shared_gate"].nbytes + layer["shared_up"].nbytes + layer["shared_down"].nbytes
    act = T * s.hidden * 2          # bf16 x in
    expect = (layer["router_w"].nbytes + shared + len(hit) * (per_group_d + per_group_u)
              + len(distinct) * per_record
              + act                   # router kernel stages x
              + act                   # D reads x
              + 2 * act)              # U: two T x H bf16 activation streams (the bench's count)
    assert c["n_distinct"] == len(distinct) and c["n_groups_hit"] == len(hit)
    assert c["bytes_total"] == pytest.approx(expect, rel=0, abs=0)


def test_prefill_flops_match_brute_force(bench):
    """Many tokens: 2 x the multiply-adds of every contraction, counted pair
    by pair from the routing (D and U only for the (token, group) pairs a
    token hits)."""
    wl = synth.WORKLOADS["tiny"]
    s = wl.shape
    layer = synth.make_layer(wl)
    groups = layer["expert_group"]
    T = 37
    idx = routing(s, T, seed=11)
    c = bench.step_cost(s, idx, groups, T, prefill=True)
    H, L, E, F, Fs = s.hidden, s.latent, s.n_experts, s.ffn, s.shared_ffn
    macs = 0
    for t in range(T):
        macs += E * H                               # router logits
        macs += 2 * Fs * H + H * Fs                 # shared gate, up, down
        for g in {int(groups[e]) for e in idx[t]}:
            macs += L * H + H * L                   # D_g and U_g of a hit group
        for e in idx[t]:
            macs += 2 * F * L + L * F               # the expert's gate, up and down
    assert c["flops_total"] == pytest.approx(2.0 * macs, rel=1e-12)


def test_traffic_is_keyed_by_sources_and_expert_inputs(bench):
    """A DRAM-traffic figure is reported only for the sources it was taken
    from, and W4A4 workloads have their own entries."""
    wl = synth.WORKLOADS["edge0_145b_prefill"]
    w4 = wl.with_(shape=synth.replace(wl.shape, act_fmt="nvfp4"))
    key16 = ("edge0_145b_prefill", 4096, "gateup")
    key4 = ("edge0_145b_prefill+w4a4", 4096, "gateup")
    table = dict(bench.NCU_TRAFFIC)
    try:
        bench.NCU_TRAFFIC[key16] = (111, bench.cuda_source_hash())
        bench.NCU_TRAFFIC[key4] = (222, bench.cuda_source_hash())
        assert bench.ncu_traffic(wl, 4096, "gateup") == 111
        assert bench.ncu_traffic(w4, 4096, "gateup") == 222
        bench.NCU_TRAFFIC[key16] = (111, "000000000000")
        assert bench.ncu_traffic(wl, 4096, "gateup") is None
        assert bench.ncu_traffic(wl, 4096, "no_such_kernel") is None
    finally:
        bench.NCU_TRAFFIC.clear()
        bench.NCU_TRAFFIC.update(table)
