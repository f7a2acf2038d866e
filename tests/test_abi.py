"""The C-ABI library: it loads, exports every declared symbol, and its host
side (shape checks, sizes, argument errors) behaves without a GPU."""
import ctypes
import os
import re

import pytest

from latent_mixture_experts_softmax_b200 import binding as B
from latent_mixture_experts_softmax_b200 import build, synth
from oracle import lmoe_oracle as orc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build_all()
    return B.lib()


def _declared():
    src = open(os.path.join(ROOT, "include", "lmoe.h")).read()
    return set(re.findall(r"LMOE_API\s+[\w\s\*]+?\b(lmoe_\w+)\s*\(", src))


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert len(names) >= 12
    for n in names:
        assert hasattr(L, n), n
    assert names == set(B.EXPORTS)


def test_cfg_check_and_sizes(L):
    for name in ("tiny", "edge0_120b_decode", "edge0_145b_decode", "edge0_145b_prefill"):
        s = synth.WORKLOADS[name].shape
        cfg = B.make_cfg(s)
        assert B.lmoe_cfg_check(cfg) == B.LMOE_OK
        assert B.lmoe_expert_record_bytes(cfg) == orc.expert_record_bytes(s.latent, s.ffn)
        assert B.lmoe_du_bytes(cfg) == s.n_groups * orc.du_matrix_bytes(s.du_fmt, s.latent, s.hidden)
        assert B.lmoe_workspace_bytes(cfg, 4) > 0
    bad = B.make_cfg(synth.replace(synth.SHAPE_145B, latent=1800))
    assert B.lmoe_cfg_check(bad) == B.LMOE_ERR_UNSUPPORTED
    assert B.lmoe_workspace_bytes(bad, 4) == 0
    bad = B.make_cfg(synth.replace(synth.SHAPE_145B, du_fmt=5))
    assert B.lmoe_cfg_check(bad) == B.LMOE_ERR_UNSUPPORTED
    bad = B.make_cfg(synth.replace(synth.SHAPE_145B, top_k=600))
    assert B.lmoe_cfg_check(bad) == B.LMOE_ERR_UNSUPPORTED
    assert L.lmoe_cfg_check(None) == B.LMOE_ERR_ARG


def test_argument_errors_launch_nothing(L):
    cfg = B.make_cfg(synth.SHAPE_145B)
    sh = B.lmoe_shared(16, 32, 48)
    # null x
    st = L.lmoe_forward(ctypes.byref(cfg), None, 16, 16, 16, 16, 16, ctypes.byref(sh), 16, 4, 256, 1 << 30, None)
    assert st == B.LMOE_ERR_ARG
    # misaligned router weights
    st = L.lmoe_forward(ctypes.byref(cfg), 16, 18, 16, 16, 16, 16, ctypes.byref(sh), 16, 4, 256, 1 << 30, None)
    assert st == B.LMOE_ERR_ARG
    # workspace too small
    st = L.lmoe_forward(ctypes.byref(cfg), 16, 16, 16, 16, 16, 16, ctypes.byref(sh), 16, 4, 256, 1024, None)
    assert st == B.LMOE_ERR_WORKSPACE
    # empty batch is a valid no-op
    st = L.lmoe_forward(ctypes.byref(cfg), 16, 16, 16, 16, 16, 16, ctypes.byref(sh), 16, 0, None, 0, None)
    assert st == B.LMOE_OK
    # negative T
    st = L.lmoe_forward(ctypes.byref(cfg), 16, 16, 16, 16, 16, 16, ctypes.byref(sh), 16, -1, 256, 1 << 30, None)
    assert st == B.LMOE_ERR_ARG
    # inject_idx without inject_w
    st = L.lmoe_forward_ex(ctypes.byref(cfg), 16, 16, None, 16, 16, 16, 16, ctypes.byref(sh), None, 16, None,
                           None, None, 16, 4, 256, 1 << 30, None)
    assert st == B.LMOE_ERR_ARG
    assert "workspace" in B.status_str(B.LMOE_ERR_WORKSPACE)


def test_stack_needs_gamma(L):
    cfg = B.make_cfg(synth.SHAPE_145B)
    layer = B.lmoe_layer(16, None, 16, 16, 16, 16, B.lmoe_shared(16, 16, 16), None)
    arr = (B.lmoe_layer * 1)(layer)
    assert L.lmoe_stack_forward(ctypes.byref(cfg), 1, arr, 16, 32, 4, 1e-6, 256, 1 << 30, None) == B.LMOE_ERR_ARG


def test_w4a4_needs_nvfp4_records_and_128_multiples():
    """lmoe_cfg.act_fmt = LMOE_ACT_NVFP4 (W4A4) runs on the tensor-core expert
    kernels: NVFP4 records, latent and ffn multiples of 128 up to 2048."""
    from parity import small_workload
    ok = small_workload(4, latent=256, ffn=128, act_fmt="nvfp4")
    assert B.lmoe_cfg_check(B.make_cfg(ok.shape)) == B.LMOE_OK
    for kw in ({"ffn": 192}, {"latent": 2176}, {"expert_fmt": "q3k"}):
        wl = small_workload(4, **{"latent": 256, "ffn": 128, "act_fmt": "nvfp4", **kw})
        assert B.lmoe_cfg_check(B.make_cfg(wl.shape)) == B.LMOE_ERR_UNSUPPORTED, kw
    cfg = B.make_cfg(ok.shape)
    cfg.act_fmt = 2
    assert B.lmoe_cfg_check(cfg) == B.LMOE_ERR_UNSUPPORTED
