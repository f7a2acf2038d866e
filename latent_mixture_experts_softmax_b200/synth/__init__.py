"""Seeded synthetic workloads for the latent mixture-of-experts FFN block.

Only random draws and packing into storage formats live here (the C file
next to this one does the work).  Nothing in this module decodes a format or
computes any part of the block, so the CUDA path and the fp64 test oracle
can both be fed from it without sharing arithmetic.

Workloads follow the shapes of the Edge0 145B / 120B model page ("Model
profile" and the two architecture tables: hidden 2560, 512 experts, top-10,
8 D/U groups, latent 1792 or 1280, SwiGLU width 640, one shared expert) and
the record sizes of the teardown article "Edge0-145B: a Qwen MoE with its
experts squeezed" (section "What is 4-bit").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass, field, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lmoe_synth.c")
_LIB_PATH = os.path.join(_HERE, "liblmoe_synth.so")
_lib = None

Q8_0 = 8
Q4_0 = 4


def build(force: bool = False) -> str:
    """Compile the generator (plain C, OpenMP) in place."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, _SRC, "-lm"])
    return _LIB_PATH


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        u64, i32, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.lmoe_synth_bits.restype = u64
        L.lmoe_synth_bits.argtypes = [u64, u64]
        L.lmoe_synth_key.restype = u64
        L.lmoe_synth_key.argtypes = [u64, u64]
        L.lmoe_synth_normal.restype = dbl
        L.lmoe_synth_normal.argtypes = [u64, u64]
        L.lmoe_synth_uniform.restype = dbl
        L.lmoe_synth_uniform.argtypes = [u64, u64]
        L.lmoe_synth_bf16.argtypes = [u64, dbl, vp, i64]
        L.lmoe_synth_f32.argtypes = [u64, dbl, vp, i64]
        L.lmoe_synth_f64.argtypes = [u64, dbl, vp, i64]
        L.lmoe_synth_groups_uniform.argtypes = [u64, i32, i32, vp]
        L.lmoe_synth_q8_0.argtypes = [u64, dbl, i32, i32, vp]
        L.lmoe_synth_q4_0.argtypes = [u64, dbl, i32, i32, vp]
        L.lmoe_synth_q8_0_encode.argtypes = [vp, i32, i32, vp]
        L.lmoe_synth_q4_0_encode.argtypes = [vp, i32, i32, vp]
        L.lmoe_synth_nvfp4_record_bytes.restype = ctypes.c_size_t
        L.lmoe_synth_nvfp4_record_bytes.argtypes = [i32, i32]
        L.lmoe_synth_nvfp4_experts.argtypes = [u64, dbl, i32, i32, i32, vp]
        L.lmoe_synth_nvfp4_encode.restype = ctypes.c_float
        L.lmoe_synth_nvfp4_encode.argtypes = [vp, i32, i32, vp, vp]
        for n in ("lmoe_synth_q3k_bytes", "lmoe_synth_iq4nl_bytes", "lmoe_synth_q3k_record_bytes"):
            getattr(L, n).restype = ctypes.c_size_t
            getattr(L, n).argtypes = [i32, i32]
        L.lmoe_synth_q3k_encode.argtypes = [vp, i32, i32, vp]
        L.lmoe_synth_iq4nl_encode.argtypes = [vp, i32, i32, vp]
        L.lmoe_synth_q3k_experts.argtypes = [u64, dbl, i32, i32, i32, vp]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return ctypes.c_void_p(a.ctypes.data)


# ----------------------------------------------------------------------------
# shapes and workloads
# ----------------------------------------------------------------------------

@dataclass(frozen=True)
class LayerShape:
    hidden: int = 2560
    latent: int = 1792
    n_experts: int = 512
    top_k: int = 10
    n_groups: int = 8
    ffn: int = 640
    shared_ffn: int = 640
    du_fmt: int = Q8_0          # 8: Q8_0, 4: Q4_0
    router_dtype: str = "bf16"  # "f32" or "bf16"
    expert_fmt: str = "nvfp4"   # "nvfp4", or "q3k" (Q3_K gate/up + IQ4_NL down)
    act_fmt: str = "fp16"       # expert inputs: "fp16" (as computed), or "nvfp4" (W4A4)


@dataclass(frozen=True)
class Workload:
    name: str
    shape: LayerShape
    T: int
    seed: int = 0
    groups: str = "uniform"        # "mod" (e % G) or "uniform"
    bias_sigma: float | None = None
    weight_sigma: float = 0.02
    x_sigma: float = 1.0
    n_layers: int = 1
    extra: dict = field(default_factory=dict, compare=False)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


SHAPE_120B = LayerShape(latent=1280, du_fmt=Q4_0)
SHAPE_145B = LayerShape(latent=1792, du_fmt=Q8_0)
SHAPE_145B_Q3K = LayerShape(latent=1792, du_fmt=Q8_0, expert_fmt="q3k")

WORKLOADS = {
    # 8 tokens, 64 experts, latent 1280, Q4_0 D/U, fp32 router, no bias, expert_group = e % 8
    "tiny": Workload("tiny", replace(SHAPE_120B, n_experts=64, router_dtype="f32"), T=8,
                     seed=0, groups="mod", bias_sigma=None),
    # Edge0-120B-shaped layer, MTP verify window of 4 tokens
    "edge0_120b_decode": Workload("edge0_120b_decode", SHAPE_120B, T=4, groups="uniform", bias_sigma=1.0),
    # Edge0-145B-shaped layer, MTP verify window of 4 tokens
    "edge0_145b_decode": Workload("edge0_145b_decode", SHAPE_145B, T=4, groups="uniform", bias_sigma=1.0),
    # Edge0-145B-shaped layer, prefill of 4096 (and 16384) tokens
    "edge0_145b_prefill": Workload("edge0_145b_prefill", SHAPE_145B, T=4096, groups="uniform", bias_sigma=0.5),
    # the same layer with the other expert build (Q3_K gate/up + IQ4_NL down)
    "edge0_145b_q3k_decode": Workload("edge0_145b_q3k_decode", SHAPE_145B_Q3K, T=4, groups="uniform",
                                      bias_sigma=1.0),
    "edge0_145b_q3k_prefill": Workload("edge0_145b_q3k_prefill", SHAPE_145B_Q3K, T=4096, groups="uniform",
                                       bias_sigma=0.5),
    # 48 stacked Edge0-145B-shaped layers with pre-RMSNorm and residual
    "edge0_145b_stack": Workload("edge0_145b_stack", SHAPE_145B, T=4, groups="uniform", bias_sigma=1.0,
                                 n_layers=48),
}

# tensor tags of the key tree: key(seed, layer, tag[, index])
TAG = {"x": 1, "router_w": 2, "router_b": 3, "groups": 4, "D": 5, "U": 6, "experts": 7,
       "shared_gate": 8, "shared_up": 9, "shared_down": 10, "residual": 11}


def key(seed: int, layer: int, tag: str, index: int | None = None) -> int:
    L = lib()
    k = L.lmoe_synth_key(L.lmoe_synth_key(seed, layer), TAG[tag])
    if index is not None:
        k = L.lmoe_synth_key(k, index)
    return k


# ----------------------------------------------------------------------------
# byte sizes of the storage formats
# ----------------------------------------------------------------------------

def du_matrix_bytes(fmt: int, rows: int, cols: int) -> int:
    """One Q8_0 (34 B per 32) or Q4_0 (18 B per 32) matrix."""
    per32 = 34 if fmt == Q8_0 else 18
    return rows * cols // 32 * per32


def expert_record_bytes(latent: int, ffn: int, expert_fmt: str = "nvfp4") -> int:
    if expert_fmt == "q3k":
        return int(lib().lmoe_synth_q3k_record_bytes(latent, ffn))
    return int(lib().lmoe_synth_nvfp4_record_bytes(latent, ffn))


# ----------------------------------------------------------------------------
# generators
# ----------------------------------------------------------------------------

def bf16_normal(k: int, sigma: float, shape) -> np.ndarray:
    out = np.empty(shape, np.uint16)
    lib().lmoe_synth_bf16(k, sigma, _p(out), out.size)
    return out


def f32_normal(k: int, sigma: float, shape) -> np.ndarray:
    out = np.empty(shape, np.float32)
    lib().lmoe_synth_f32(k, sigma, _p(out), out.size)
    return out


def f64_normal(k: int, sigma: float, shape) -> np.ndarray:
    """The unrounded draws sigma * normal(k, i) behind every generated tensor
    (element i in row-major order)."""
    out = np.empty(shape, np.float64)
    lib().lmoe_synth_f64(k, sigma, _p(out), out.size)
    return out


def expert_key(k: int, e: int, m: int) -> int:
    """Key of matrix m (0 gate, 1 up, 2 down) of expert e in experts_normal(k, ...)."""
    L = lib()
    return L.lmoe_synth_key(L.lmoe_synth_key(k, e), m)


def qmatrix(fmt: int, k: int, sigma: float, rows: int, cols: int) -> np.ndarray:
    out = np.zeros(du_matrix_bytes(fmt, rows, cols), np.uint8)
    (lib().lmoe_synth_q8_0 if fmt == Q8_0 else lib().lmoe_synth_q4_0)(k, sigma, rows, cols, _p(out))
    return out


def qmatrix_encode(fmt: int, w: np.ndarray) -> np.ndarray:
    """Pack a given matrix [rows, cols] into Q8_0 / Q4_0 (for structured test weights)."""
    w = np.ascontiguousarray(w, np.float64)
    rows, cols = w.shape
    out = np.zeros(du_matrix_bytes(fmt, rows, cols), np.uint8)
    (lib().lmoe_synth_q8_0_encode if fmt == Q8_0 else lib().lmoe_synth_q4_0_encode)(_p(w), rows, cols, _p(out))
    return out


def experts_normal(k: int, sigma: float, E: int, latent: int, ffn: int) -> np.ndarray:
    out = np.zeros(E * expert_record_bytes(latent, ffn), np.uint8)
    lib().lmoe_synth_nvfp4_experts(k, sigma, E, latent, ffn, _p(out))
    return out


def expert_record_encode(w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """Pack one expert from given matrices gate [F, L], up [F, L], down [L, F]."""
    F, L = w_gate.shape
    nq, ns = L * F // 2, L * F // 16
    rec = np.zeros(expert_record_bytes(L, F), np.uint8)
    ts = np.zeros(4, np.float32)
    for m, w in enumerate((w_gate, w_up, w_down)):
        w = np.ascontiguousarray(w, np.float64)
        q = np.zeros(nq, np.uint8)
        s = np.zeros(ns, np.uint8)
        ts[m] = lib().lmoe_synth_nvfp4_encode(_p(w), w.shape[0], w.shape[1], _p(q), _p(s))
        rec[m * nq:(m + 1) * nq] = q
        rec[3 * nq + m * ns:3 * nq + (m + 1) * ns] = s
    rec[3 * nq + 3 * ns:] = ts.view(np.uint8)
    return rec


def q3k_encode(w: np.ndarray) -> np.ndarray:
    """Pack a matrix [rows, cols] (cols a multiple of 256) into the Q3_K planes."""
    w = np.ascontiguousarray(w, np.float64)
    out = np.zeros(int(lib().lmoe_synth_q3k_bytes(*w.shape)), np.uint8)
    lib().lmoe_synth_q3k_encode(_p(w), w.shape[0], w.shape[1], _p(out))
    return out


def iq4nl_encode(w: np.ndarray) -> np.ndarray:
    """Pack a matrix [rows, cols] (cols a multiple of 32) into the IQ4_NL planes."""
    w = np.ascontiguousarray(w, np.float64)
    out = np.zeros(int(lib().lmoe_synth_iq4nl_bytes(*w.shape)), np.uint8)
    lib().lmoe_synth_iq4nl_encode(_p(w), w.shape[0], w.shape[1], _p(out))
    return out


def q3k_record_encode(w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """One expert of the Q3_K build from given gate [F, L], up [F, L], down [L, F]."""
    return np.concatenate([q3k_encode(w_gate), q3k_encode(w_up), iq4nl_encode(w_down)])


def q3k_experts(k: int, sigma: float, E: int, latent: int, ffn: int) -> np.ndarray:
    out = np.zeros(E * expert_record_bytes(latent, ffn, "q3k"), np.uint8)
    lib().lmoe_synth_q3k_experts(k, sigma, E, latent, ffn, _p(out))
    return out


def expert_groups(wl: Workload, layer: int = 0) -> np.ndarray:
    E, G = wl.shape.n_experts, wl.shape.n_groups
    if wl.groups == "mod":
        return (np.arange(E) % G).astype(np.uint8)
    out = np.empty(E, np.uint8)
    lib().lmoe_synth_groups_uniform(key(wl.seed, layer, "groups"), E, G, _p(out))
    return out


def make_x(wl: Workload, T: int | None = None, draw: int = 0) -> np.ndarray:
    """Token activations [T, hidden] as bf16 bits; `draw` selects another sample."""
    T = wl.T if T is None else T
    return bf16_normal(key(wl.seed, 0, "x", draw), wl.x_sigma, (T, wl.shape.hidden))


def make_layer(wl: Workload, layer: int = 0) -> dict:
    """All weights of one layer (numpy, host).  bf16 tensors are uint16 bit patterns."""
    s, seed, sig = wl.shape, wl.seed, wl.weight_sigma
    H, L, E, G, F, Fs = s.hidden, s.latent, s.n_experts, s.n_groups, s.ffn, s.shared_ffn
    out = {}
    if s.router_dtype == "f32":
        out["router_w"] = f32_normal(key(seed, layer, "router_w"), sig, (E, H))
    else:
        out["router_w"] = bf16_normal(key(seed, layer, "router_w"), sig, (E, H))
    out["router_b"] = (f32_normal(key(seed, layer, "router_b"), wl.bias_sigma, (E,))
                       if wl.bias_sigma is not None else None)
    out["expert_group"] = expert_groups(wl, layer)
    out["D"] = np.concatenate([qmatrix(s.du_fmt, key(seed, layer, "D", g), sig, L, H) for g in range(G)])
    out["U"] = np.concatenate([qmatrix(s.du_fmt, key(seed, layer, "U", g), sig, H, L) for g in range(G)])
    if s.expert_fmt == "q3k":
        out["experts"] = q3k_experts(key(seed, layer, "experts"), sig, E, L, F)
    else:
        out["experts"] = experts_normal(key(seed, layer, "experts"), sig, E, L, F)
    out["shared_gate"] = bf16_normal(key(seed, layer, "shared_gate"), sig, (Fs, H))
    out["shared_up"] = bf16_normal(key(seed, layer, "shared_up"), sig, (Fs, H))
    out["shared_down"] = bf16_normal(key(seed, layer, "shared_down"), sig, (H, Fs))
    return out


def bf16_bits_from_f32(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to bf16 bit patterns (nearest even)."""
    u = np.ascontiguousarray(a, np.float32).view(np.uint32).astype(np.uint64)
    u = u + 0x7FFF + ((u >> 16) & 1)
    return (u >> 16).astype(np.uint16)
