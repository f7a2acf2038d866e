"""ctypes facade over the C++ fp64 oracle (lmoe_oracle.cpp, this directory).

TEST INFRASTRUCTURE.  Only the test suite, the smoke check and the
CPU-baseline legs of the benchmark may import this module.  The functions
have the names and signatures of the numpy oracle next to it
(lmoe_oracle.py), so that every pin runs against both implementations; all
arithmetic happens in the C++ library, this file only marshals arrays.

The block it computes is the layer equation of the teardown article
"Edge0-145B: a Qwen MoE with its experts squeezed, and a 51B table left on
the SSD", section "A latent in front of the experts", read per group (model
page "Edge0 145B and Edge0 120B", "Model profile" and architecture tables);
the steps are listed in the header of lmoe_oracle.cpp.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

from . import lmoe_oracle as _np_oracle

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lmoe_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "liblmoe_oracle.so")
_lib = None

Q8_0 = 8
Q4_0 = 4

# test metrics, not oracle arithmetic
rel_l2 = _np_oracle.rel_l2
max_abs_over_rms = _np_oracle.max_abs_over_rms


def build(force: bool = False) -> str:
    """Compile the oracle in place (plain g++, OpenMP, IEEE fp64: no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        subprocess.check_call(["g++", "-O2", "-std=c++17", "-fopenmp", "-fPIC", "-shared", "-o", _LIB_PATH, _SRC])
    return _LIB_PATH


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("hidden", "latent", "n_experts", "top_k", "n_groups", "ffn",
                                            "shared_ffn", "du_fmt", "router_bf16", "expert_fmt", "act_fmt")]


class _Layer(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("router_w", "router_b", "expert_group", "D", "U", "experts",
                                               "shared_gate", "shared_up", "shared_down")]


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_double
        L.orc_threads.restype = i32
        for n in ("orc_du_matrix_bytes", "orc_expert_record_bytes", "orc_du_offset", "orc_expert_offset"):
            getattr(L, n).restype = i64
        L.orc_du_matrix_bytes.argtypes = [i32, i32, i32]
        L.orc_expert_record_bytes.argtypes = [i32, i32]
        L.orc_du_offset.argtypes = [i32, i32, i32, i32]
        L.orc_expert_offset.argtypes = [i32, i32, i32]
        for n in ("orc_bf16_to_f64", "orc_fp16_to_f64", "orc_e2m1_to_f64", "orc_e4m3fn_to_f64"):
            getattr(L, n).argtypes = [vp, i64, vp]
        L.orc_decode_du.restype = i32
        L.orc_decode_du.argtypes = [i32, vp, i32, i32, vp]
        L.orc_decode_nvfp4.restype = i32
        L.orc_decode_nvfp4.argtypes = [vp, vp, dbl, i32, i32, vp]
        L.orc_decode_expert.argtypes = [vp, i32, i32, vp, vp, vp]
        L.orc_route.argtypes = [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp]
        L.orc_shared_expert.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Layer), vp, i32, vp]
        L.orc_expert_apply.argtypes = [vp, i32, i32, vp, i32, vp]
        L.orc_du_apply.argtypes = [i32, vp, i32, i32, vp, i32, vp]
        L.orc_forward.restype = i32
        L.orc_forward.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Layer), vp, vp, vp, vp, i32, vp, vp, vp, vp]
        L.orc_rmsnorm.argtypes = [vp, vp, dbl, i32, i32, vp]
        L.orc_quantize_q8_1.argtypes = [vp, i32, i32, vp, vp]
        L.orc_decode_q3k_iq4nl.restype = i32
        L.orc_decode_q3k_iq4nl.argtypes = [i32, vp, i32, i32, vp]
        L.orc_iq4nl_levels.argtypes = [vp]
        L.orc_expert_record_bytes_fmt.restype = i64
        L.orc_expert_record_bytes_fmt.argtypes = [i32, i32, i32]
        L.orc_expert_offset_fmt.restype = i64
        L.orc_expert_offset_fmt.argtypes = [i32, i32, i32, i32]
        L.orc_decode_expert_fmt.argtypes = [i32, vp, i32, i32, vp, vp, vp]
        L.orc_dproj_q8_1.argtypes = [i32, vp, i32, i32, i32, vp, i32, vp]
        L.orc_nvfp4_act_quantize.argtypes = [vp, i32, vp, vp, vp, vp]
        L.orc_fp16_round.restype = dbl
        L.orc_fp16_round.argtypes = [dbl]
        L.orc_stack_layer.restype = i32
        L.orc_stack_layer.argtypes = [ctypes.POINTER(_Shape), ctypes.POINTER(_Layer), vp, vp, dbl, vp, vp, i32, vp,
                                      vp, vp, vp]
        _lib = L
    return _lib


def threads() -> int:
    """OpenMP threads the oracle spreads its rows, tokens and experts over."""
    return int(lib().orc_threads())


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a, ctypes.c_void_p(a.ctypes.data) if a.size else ctypes.c_void_p(0)


def _ptr(a):
    return ctypes.c_void_p(a.ctypes.data) if a is not None and a.size else None


# ----------------------------------------------------------------------------
# scalar and matrix formats
# ----------------------------------------------------------------------------

def _scalar(fn, dtype, codes):
    c, p = _c(codes, dtype)
    out = np.empty(c.shape, np.float64)
    getattr(lib(), fn)(p, c.size, _ptr(out))
    return out


def bf16_to_f64(bits):
    return _scalar("orc_bf16_to_f64", np.uint16, bits)


def fp16_to_f64(bits):
    return _scalar("orc_fp16_to_f64", np.uint16, np.asarray(bits).astype(np.int64) & 0xFFFF)


def e2m1_to_f64(code):
    return _scalar("orc_e2m1_to_f64", np.uint8, np.asarray(code).astype(np.int64) & 0xFF)


def e4m3fn_to_f64(code):
    return _scalar("orc_e4m3fn_to_f64", np.uint8, np.asarray(code).astype(np.int64) & 0xFF)


def du_matrix_bytes(fmt: int, rows: int, cols: int) -> int:
    return int(lib().orc_du_matrix_bytes(fmt, rows, cols))


def _efmt(expert_fmt) -> int:
    return 1 if expert_fmt == "q3k" else 0


def expert_record_bytes(latent: int, ffn: int, expert_fmt: str = "nvfp4") -> int:
    return int(lib().orc_expert_record_bytes_fmt(_efmt(expert_fmt), latent, ffn))


def iq4nl_levels() -> np.ndarray:
    out = np.empty(16)
    lib().orc_iq4nl_levels(_ptr(out))
    return out


def decode_q3k(blob, rows: int, cols: int) -> np.ndarray:
    b, p = _c(blob, np.uint8)
    out = np.empty((rows, cols))
    if lib().orc_decode_q3k_iq4nl(1, p, rows, cols, _ptr(out)) != 0:
        raise ValueError("Q3_K columns must be a multiple of 256")
    return out


def decode_iq4nl(blob, rows: int, cols: int) -> np.ndarray:
    b, p = _c(blob, np.uint8)
    out = np.empty((rows, cols))
    if lib().orc_decode_q3k_iq4nl(2, p, rows, cols, _ptr(out)) != 0:
        raise ValueError("IQ4_NL columns must be a multiple of 32")
    return out


def decode_du(fmt: int, blob, rows: int, cols: int) -> np.ndarray:
    b, p = _c(blob, np.uint8)
    assert b.size >= du_matrix_bytes(fmt, rows, cols)
    out = np.empty((rows, cols), np.float64)
    if lib().orc_decode_du(fmt, p, rows, cols, _ptr(out)) != 0:
        raise ValueError(f"unknown D/U format {fmt}")
    return out


def decode_q8_0(blob, rows, cols):
    return decode_du(Q8_0, blob, rows, cols)


def decode_q4_0(blob, rows, cols):
    return decode_du(Q4_0, blob, rows, cols)


def decode_nvfp4(qbytes, sbytes, ts, rows: int, cols: int) -> np.ndarray:
    q, pq = _c(qbytes, np.uint8)
    s, ps = _c(sbytes, np.uint8)
    assert q.size >= rows * cols // 2 and s.size >= rows * cols // 16
    out = np.empty((rows, cols), np.float64)
    if lib().orc_decode_nvfp4(pq, ps, float(ts), rows, cols, _ptr(out)) != 0:
        raise ValueError("NVFP4 columns must be a multiple of 64")
    return out


def decode_expert(record, latent: int, ffn: int, expert_fmt: str = "nvfp4"):
    r, p = _c(record, np.uint8)
    assert r.size >= expert_record_bytes(latent, ffn, expert_fmt)
    wg = np.empty((ffn, latent))
    wu = np.empty((ffn, latent))
    wd = np.empty((latent, ffn))
    lib().orc_decode_expert_fmt(_efmt(expert_fmt), p, latent, ffn, _ptr(wg), _ptr(wu), _ptr(wd))
    return wg, wu, wd


def expert_slice(experts: np.ndarray, e: int, latent: int, ffn: int, expert_fmt: str = "nvfp4") -> np.ndarray:
    o = int(lib().orc_expert_offset_fmt(_efmt(expert_fmt), e, latent, ffn))
    return experts[o:o + expert_record_bytes(latent, ffn, expert_fmt)]


def du_slice(blob: np.ndarray, fmt: int, g: int, rows: int, cols: int) -> np.ndarray:
    o = int(lib().orc_du_offset(fmt, g, rows, cols))
    return blob[o:o + du_matrix_bytes(fmt, rows, cols)]


# ----------------------------------------------------------------------------
# router and block
# ----------------------------------------------------------------------------

def route(x, Wr, b, top_k: int):
    """-> (idx [T, K] int64, w [T, K], gap [T], logits [T, E])."""
    x, px = _c(x, np.float64)
    Wr, pw = _c(Wr, np.float64)
    T, H = x.shape
    E = Wr.shape[0]
    bb = None if b is None else np.ascontiguousarray(b, np.float64)
    idx = np.empty((T, top_k), np.int64)
    w = np.empty((T, top_k))
    gap = np.empty(T)
    logits = np.empty((T, E))
    lib().orc_route(px, pw, _ptr(bb), T, H, E, top_k, _ptr(idx), _ptr(w), _ptr(gap), _ptr(logits))
    return idx, w, gap, logits


def _shape(shape) -> _Shape:
    return _Shape(shape.hidden, shape.latent, shape.n_experts, shape.top_k, shape.n_groups, shape.ffn,
                  shape.shared_ffn, shape.du_fmt, 1 if shape.router_dtype == "bf16" else 0,
                  _efmt(getattr(shape, "expert_fmt", "nvfp4")), 1 if getattr(shape, "act_fmt", "fp16") == "nvfp4" else 0)


class _LayerRef:
    """The layer's arrays, kept alive for as long as the C struct points at them."""

    def __init__(self, shape, layer: dict):
        rw = layer["router_w"]
        self.arrays = {
            "router_w": np.ascontiguousarray(rw, np.uint16 if shape.router_dtype == "bf16" else np.float32),
            "router_b": None if layer.get("router_b") is None else np.ascontiguousarray(layer["router_b"], np.float32),
            "expert_group": np.ascontiguousarray(layer["expert_group"], np.uint8),
            "D": np.ascontiguousarray(layer["D"], np.uint8),
            "U": np.ascontiguousarray(layer["U"], np.uint8),
            "experts": np.ascontiguousarray(layer["experts"], np.uint8),
            "shared_gate": np.ascontiguousarray(layer["shared_gate"], np.uint16),
            "shared_up": np.ascontiguousarray(layer["shared_up"], np.uint16),
            "shared_down": np.ascontiguousarray(layer["shared_down"], np.uint16),
        }
        self.c = _Layer(*[_ptr(self.arrays[n]) for n, _ in _Layer._fields_])


def latent_moe_forward(shape, layer: dict, x_bits, residual_bits=None, inject_idx=None, inject_w=None,
                       weights=None, x_f64=None):
    """One latent-MoE block on x [T, H] (bf16 bits, or fp64 via x_f64).
    Returns (y [T, H] fp64, idx, w, gap).  `weights` is accepted for the
    numpy oracle's signature and not used (the C++ oracle decodes on use)."""
    x = bf16_to_f64(x_bits) if x_f64 is None else np.ascontiguousarray(x_f64, np.float64)
    T = x.shape[0]
    K = shape.top_k
    ref = _LayerRef(shape, layer)
    res = None if residual_bits is None else np.ascontiguousarray(residual_bits, np.uint16)
    ii = None if inject_idx is None else np.ascontiguousarray(inject_idx, np.int64)
    iw = None if inject_w is None else np.ascontiguousarray(inject_w, np.float64)
    y = np.empty((T, shape.hidden))
    idx = np.empty((T, K), np.int64)
    w = np.empty((T, K))
    gap = np.empty(T)
    rc = lib().orc_forward(ctypes.byref(_shape(shape)), ctypes.byref(ref.c), _ptr(x), _ptr(res), _ptr(ii), _ptr(iw),
                           T, _ptr(y), _ptr(idx), _ptr(w), _ptr(gap))
    if rc != 0:
        raise ValueError("routed expert index or group label out of range")
    return y, idx, w, gap


def rmsnorm(v, gamma, eps: float) -> np.ndarray:
    v = np.ascontiguousarray(v, np.float64)
    g = np.ascontiguousarray(gamma, np.float64)
    out = np.empty_like(v)
    lib().orc_rmsnorm(_ptr(v), _ptr(g), float(eps), v.shape[0], v.shape[1], _ptr(out))
    return out


def stack_layer_forward(shape, layer: dict, x_bits, gamma, eps: float, weights=None, inject_idx=None, inject_w=None):
    """x + block(RMSNorm(x)), x as bf16 bits.  Returns (y fp64, idx, w, gap)."""
    xb = np.ascontiguousarray(x_bits, np.uint16)
    T = xb.shape[0]
    K = shape.top_k
    ref = _LayerRef(shape, layer)
    g = np.ascontiguousarray(gamma, np.float64)
    ii = None if inject_idx is None else np.ascontiguousarray(inject_idx, np.int64)
    iw = None if inject_w is None else np.ascontiguousarray(inject_w, np.float64)
    y = np.empty((T, shape.hidden))
    idx = np.empty((T, K), np.int64)
    w = np.empty((T, K))
    gap = np.empty(T)
    rc = lib().orc_stack_layer(ctypes.byref(_shape(shape)), ctypes.byref(ref.c), _ptr(xb), _ptr(g), float(eps),
                               _ptr(ii), _ptr(iw), T, _ptr(y), _ptr(idx), _ptr(w), _ptr(gap))
    if rc != 0:
        raise ValueError("routed expert index or group label out of range")
    return y, idx, w, gap


def silu(a):
    a = np.asarray(a, np.float64)
    return a / (1.0 + np.exp(-a))


def shared_expert_layer(shape, layer: dict, x) -> np.ndarray:
    """The shared expert of a layer on fp64 x [T, H]."""
    x = np.ascontiguousarray(x, np.float64)
    ref = _LayerRef(shape, layer)
    y = np.empty_like(x)
    lib().orc_shared_expert(ctypes.byref(_shape(shape)), ctypes.byref(ref.c), _ptr(x), x.shape[0], _ptr(y))
    return y


def expert_apply_record(record, latent: int, ffn: int, h) -> np.ndarray:
    """One stored expert on latent vectors h [n, latent]."""
    r, pr = _c(record, np.uint8)
    h = np.ascontiguousarray(np.atleast_2d(h), np.float64)
    o = np.empty_like(h)
    lib().orc_expert_apply(pr, latent, ffn, _ptr(h), h.shape[0], _ptr(o))
    return o


def du_apply(fmt: int, blob, rows: int, cols: int, x) -> np.ndarray:
    """A stored Q8_0 / Q4_0 matrix [rows, cols] on vectors x [n, cols]."""
    b, pb = _c(blob, np.uint8)
    x = np.ascontiguousarray(np.atleast_2d(x), np.float64)
    y = np.empty((x.shape[0], rows))
    lib().orc_du_apply(fmt, pb, rows, cols, _ptr(x), x.shape[0], _ptr(y))
    return y


class Weights:
    """Decoded view of one layer's weights (the numpy oracle's interface):
    Wr, b, group, Wsg, Wsu, Wsd and D(g), U(g), expert(e) decoded by the
    C++ library on first use."""

    def __init__(self, shape, layer: dict, max_cached_experts: int = 64):
        self.s = shape
        self.layer = layer
        H, Fs = shape.hidden, shape.shared_ffn
        rw = layer["router_w"]
        self.Wr = bf16_to_f64(rw) if rw.dtype == np.uint16 else np.asarray(rw, np.float64)
        self.b = None if layer.get("router_b") is None else np.asarray(layer["router_b"], np.float64)
        self.group = np.asarray(layer["expert_group"], np.int64)
        self.Wsg = bf16_to_f64(layer["shared_gate"]).reshape(Fs, H)
        self.Wsu = bf16_to_f64(layer["shared_up"]).reshape(Fs, H)
        self.Wsd = bf16_to_f64(layer["shared_down"]).reshape(H, Fs)
        self._D, self._U, self._E = {}, {}, {}
        self._max = max_cached_experts

    def D(self, g: int) -> np.ndarray:
        if g not in self._D:
            s = self.s
            self._D[g] = decode_du(s.du_fmt, du_slice(self.layer["D"], s.du_fmt, g, s.latent, s.hidden), s.latent, s.hidden)
        return self._D[g]

    def U(self, g: int) -> np.ndarray:
        if g not in self._U:
            s = self.s
            self._U[g] = decode_du(s.du_fmt, du_slice(self.layer["U"], s.du_fmt, g, s.hidden, s.latent), s.hidden, s.latent)
        return self._U[g]

    def expert(self, e: int):
        if e not in self._E:
            if len(self._E) >= self._max:
                self._E.pop(next(iter(self._E)))
            s = self.s
            f = getattr(s, "expert_fmt", "nvfp4")
            self._E[e] = decode_expert(expert_slice(self.layer["experts"], e, s.latent, s.ffn, f), s.latent, s.ffn, f)
        return self._E[e]


# ----------------------------------------------------------------------------
# ablation: D over all groups with Q8_1 activations
# ----------------------------------------------------------------------------

def quantize_q8_1(x):
    """fp32 rows [T, H] -> (q int8 [T, H], d fp16 bits [T, H/32]), Q8_1 as read
    in lmoe_oracle.cpp (every rounding an fp32 operation)."""
    x = np.ascontiguousarray(x, np.float32)
    T, H = x.shape
    q = np.empty((T, H), np.int8)
    d = np.empty((T, H // 32), np.uint16)
    lib().orc_quantize_q8_1(_ptr(x), T, H, _ptr(q), _ptr(d))
    return q, d


def dproj_q8_1(fmt: int, D, G: int, L: int, H: int, x) -> np.ndarray:
    """h [T, G, L] = D_g applied to the Q8_1 reading of x [T, H] (fp32), every group."""
    Db, pD = _c(D, np.uint8)
    x = np.ascontiguousarray(x, np.float32)
    h = np.empty((x.shape[0], G, L))
    lib().orc_dproj_q8_1(fmt, pD, G, L, H, _ptr(x), x.shape[0], _ptr(h))
    return h


def nvfp4_act_quantize(v):
    """One activation row as the W4A4 mode quantises it: (values fp64 [K],
    E2M1 codes [K], E4M3 scale codes [K/16], G)."""
    v = np.ascontiguousarray(v, np.float64)
    K = v.size
    assert K % 16 == 0
    out = np.empty(K, np.float64)
    codes = np.empty(K, np.uint8)
    scales = np.empty(K // 16, np.uint8)
    G = np.empty(1, np.float32)
    lib().orc_nvfp4_act_quantize(_ptr(v), K, _ptr(out), _ptr(codes), _ptr(scales), _ptr(G))
    return out, codes, scales, float(G[0])


def fp16_round(x: float) -> float:
    return float(lib().orc_fp16_round(float(x)))
