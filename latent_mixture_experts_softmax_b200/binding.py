"""ctypes binding of liblmoe.so: one Python function per C entry point, with
the same name, doing argument marshalling only.  Device buffers are torch
tensors (or raw integer addresses); every step of the block runs in the
library's kernels.  Importing this module never falls back to anything: if
the library is missing the first call raises."""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "liblmoe.so")

LMOE_OK = 0
LMOE_ERR_ARG = -1
LMOE_ERR_UNSUPPORTED = -2
LMOE_ERR_CUDA = -3
LMOE_ERR_WORKSPACE = -4
LMOE_ERR_TIMEOUT = -5
LMOE_ERR_DEVICE_CHECK = -6
LMOE_Q8_0 = 8
LMOE_Q4_0 = 4
LMOE_F32 = 0
LMOE_BF16 = 1
LMOE_NVFP4_DEBUG = 1
LMOE_Q3K_DEBUG = 2
LMOE_IQ4NL_DEBUG = 3
LMOE_EXPERTS_NVFP4 = 0
LMOE_EXPERTS_Q3K = 1
LMOE_ACT_FP16 = 0
LMOE_ACT_NVFP4 = 1

# every symbol include/lmoe.h declares
EXPORTS = ("lmoe_cfg_check", "lmoe_expert_record_bytes", "lmoe_du_bytes", "lmoe_workspace_bytes", "lmoe_route",
           "lmoe_forward", "lmoe_forward_ex", "lmoe_forward_host", "lmoe_stack_forward", "lmoe_last_device_status",
           "lmoe_status_str", "lmoe_debug_decode", "lmoe_debug_act_quant", "lmoe_profile_stage_events",
           "lmoe_route_noalloc", "lmoe_dproj_ablation")


class LmoeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_str(status)} ({status})")
        self.status = status


class lmoe_cfg(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("hidden", "latent", "n_experts", "top_k", "n_groups", "ffn",
                                            "shared_ffn", "du_fmt", "router_dtype", "expert_fmt", "act_fmt")]


class lmoe_shared(ctypes.Structure):
    _fields_ = [("gate", ctypes.c_void_p), ("up", ctypes.c_void_p), ("down", ctypes.c_void_p)]


class lmoe_layer(ctypes.Structure):
    _fields_ = [("router_w", ctypes.c_void_p), ("router_b", ctypes.c_void_p), ("expert_group", ctypes.c_void_p),
                ("D", ctypes.c_void_p), ("U", ctypes.c_void_p), ("experts", ctypes.c_void_p),
                ("shared", lmoe_shared), ("norm_gamma", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run latent_mixture_experts_softmax_b200.build.build_all()")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, sz, f32 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_float
        cfgp = ctypes.POINTER(lmoe_cfg)
        L.lmoe_cfg_check.argtypes = [cfgp]
        L.lmoe_cfg_check.restype = i32
        for n in ("lmoe_expert_record_bytes", "lmoe_du_bytes"):
            getattr(L, n).argtypes = [cfgp]
            getattr(L, n).restype = sz
        L.lmoe_workspace_bytes.argtypes = [cfgp, i32]
        L.lmoe_workspace_bytes.restype = sz
        L.lmoe_route.argtypes = [cfgp, vp, vp, vp, i32, vp, vp, vp, sz, vp]
        L.lmoe_route.restype = i32
        L.lmoe_forward.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(lmoe_shared), vp, i32, vp, sz, vp]
        L.lmoe_forward.restype = i32
        L.lmoe_forward_ex.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(lmoe_shared), vp, vp, vp,
                                      vp, vp, vp, i32, vp, sz, vp]
        L.lmoe_forward_ex.restype = i32
        L.lmoe_forward_host.argtypes = [cfgp, vp, vp, vp, vp, vp, vp, vp, ctypes.POINTER(lmoe_shared), vp, i32, vp,
                                        sz, vp]
        L.lmoe_forward_host.restype = i32
        L.lmoe_stack_forward.argtypes = [cfgp, i32, ctypes.POINTER(lmoe_layer), vp, vp, i32, f32, vp, sz, vp]
        L.lmoe_stack_forward.restype = i32
        L.lmoe_last_device_status.argtypes = [vp, sz, vp]
        L.lmoe_last_device_status.restype = i32
        L.lmoe_status_str.argtypes = [i32]
        L.lmoe_status_str.restype = ctypes.c_char_p
        L.lmoe_debug_decode.argtypes = [i32, vp, i32, i32, f32, vp, vp]
        L.lmoe_debug_decode.restype = i32
        L.lmoe_debug_act_quant.argtypes = [vp, i32, i32, vp, vp, vp, vp]
        L.lmoe_debug_act_quant.restype = i32
        L.lmoe_profile_stage_events.argtypes = [ctypes.POINTER(ctypes.c_void_p), i32]
        L.lmoe_profile_stage_events.restype = i32
        L.lmoe_route_noalloc.argtypes = [cfgp, vp, vp, vp, i32, vp, vp, vp]
        L.lmoe_route_noalloc.restype = i32
        L.lmoe_dproj_ablation.argtypes = [cfgp, vp, vp, i32, ctypes.c_uint32, vp, i32, vp, sz, vp]
        L.lmoe_dproj_ablation.restype = i32
        _lib = L
    return _lib


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _ptr(a):
    """Device (or host) address of a tensor, an int address, or None."""
    if a is None:
        return None
    if isinstance(a, int):
        return a
    return a.data_ptr()


def _nbytes(a):
    return a.numel() * a.element_size()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, what: str) -> int:
    if status < 0:
        raise LmoeError(status, what)
    return status


def make_cfg(shape) -> lmoe_cfg:
    """lmoe_cfg from any object with the shape fields (see synth.LayerShape)."""
    rd = shape.router_dtype
    if isinstance(rd, str):
        rd = LMOE_BF16 if rd == "bf16" else LMOE_F32
    ef = getattr(shape, "expert_fmt", "nvfp4")
    if isinstance(ef, str):
        ef = LMOE_EXPERTS_Q3K if ef == "q3k" else LMOE_EXPERTS_NVFP4
    af = getattr(shape, "act_fmt", "fp16")
    if isinstance(af, str):
        af = LMOE_ACT_NVFP4 if af == "nvfp4" else LMOE_ACT_FP16
    return lmoe_cfg(shape.hidden, shape.latent, shape.n_experts, shape.top_k, shape.n_groups, shape.ffn,
                    shape.shared_ffn, shape.du_fmt, rd, ef, af)


def make_shared(gate, up, down) -> lmoe_shared:
    return lmoe_shared(_ptr(gate), _ptr(up), _ptr(down))


# ----------------------------------------------------------------------------
# entry points
# ----------------------------------------------------------------------------

def status_str(status: int) -> str:
    return lib().lmoe_status_str(status).decode()


lmoe_status_str = status_str


def lmoe_cfg_check(cfg: lmoe_cfg) -> int:
    return lib().lmoe_cfg_check(ctypes.byref(cfg))


def lmoe_expert_record_bytes(cfg: lmoe_cfg) -> int:
    return lib().lmoe_expert_record_bytes(ctypes.byref(cfg))


def lmoe_du_bytes(cfg: lmoe_cfg) -> int:
    return lib().lmoe_du_bytes(ctypes.byref(cfg))


def lmoe_workspace_bytes(cfg: lmoe_cfg, T_max: int) -> int:
    return lib().lmoe_workspace_bytes(ctypes.byref(cfg), T_max)


def lmoe_route(cfg, x, router_w, router_b, T, topk_idx, topk_w, ws, stream=None):
    return _check(lib().lmoe_route(ctypes.byref(cfg), _ptr(x), _ptr(router_w), _ptr(router_b), T, _ptr(topk_idx),
                                   _ptr(topk_w), _ptr(ws), _nbytes(ws), _stream(stream)), "lmoe_route")


def lmoe_forward(cfg, x, router_w, expert_group, D, U, experts, shared: lmoe_shared, y, T, ws, stream=None):
    return _check(lib().lmoe_forward(ctypes.byref(cfg), _ptr(x), _ptr(router_w), _ptr(expert_group), _ptr(D), _ptr(U),
                                     _ptr(experts), ctypes.byref(shared), _ptr(y), T, _ptr(ws), _nbytes(ws),
                                     _stream(stream)), "lmoe_forward")


def lmoe_forward_ex(cfg, x, router_w, router_b, expert_group, D, U, experts, shared: lmoe_shared, residual,
                    inject_idx, inject_w, out_idx, out_w, y, T, ws, stream=None):
    return _check(lib().lmoe_forward_ex(ctypes.byref(cfg), _ptr(x), _ptr(router_w), _ptr(router_b), _ptr(expert_group),
                                        _ptr(D), _ptr(U), _ptr(experts), ctypes.byref(shared), _ptr(residual),
                                        _ptr(inject_idx), _ptr(inject_w), _ptr(out_idx), _ptr(out_w), _ptr(y), T,
                                        _ptr(ws), _nbytes(ws), _stream(stream)), "lmoe_forward_ex")


def lmoe_forward_host(cfg, x_host, router_w, router_b, expert_group, D, U, experts, shared: lmoe_shared, y_host, T,
                      ws, stream=None):
    return _check(lib().lmoe_forward_host(ctypes.byref(cfg), _ptr(x_host), _ptr(router_w), _ptr(router_b),
                                          _ptr(expert_group), _ptr(D), _ptr(U), _ptr(experts), ctypes.byref(shared),
                                          _ptr(y_host), T, _ptr(ws), _nbytes(ws), _stream(stream)),
                  "lmoe_forward_host")


def lmoe_stack_forward(cfg, layers, x, y, T, rms_eps, ws, stream=None):
    arr = (lmoe_layer * len(layers))(*layers)
    return _check(lib().lmoe_stack_forward(ctypes.byref(cfg), len(layers), arr, _ptr(x), _ptr(y), T, rms_eps,
                                           _ptr(ws), _nbytes(ws), _stream(stream)), "lmoe_stack_forward")


def lmoe_last_device_status(ws, stream=None) -> int:
    return lib().lmoe_last_device_status(_ptr(ws), _nbytes(ws), _stream(stream))


def lmoe_debug_act_quant(src, n, cols, codes, scales, G, stream=None):
    return _check(lib().lmoe_debug_act_quant(_ptr(src), n, cols, _ptr(codes), _ptr(scales), _ptr(G), _stream(stream)),
                  "lmoe_debug_act_quant")


def lmoe_debug_decode(fmt, blob, rows, cols, ts, out, stream=None):
    return _check(lib().lmoe_debug_decode(fmt, _ptr(blob), rows, cols, float(ts), _ptr(out), _stream(stream)),
                  "lmoe_debug_decode")


def lmoe_profile_stage_events(events) -> int:
    """events: list of torch.cuda.Event (created, not yet recorded) or [] to stop."""
    handles = []
    for ev in events:
        ev.record()          # materialise the handle; re-recorded by the library
        handles.append(ev.cuda_event)
    arr = (ctypes.c_void_p * max(1, len(handles)))(*handles)
    return _check(lib().lmoe_profile_stage_events(arr, len(handles)), "lmoe_profile_stage_events")


def lmoe_route_noalloc(cfg, x, router_w, router_b, T, topk_idx, topk_w, stream=None):
    """Router without a workspace (scratch is a fixed array inside the library)."""
    return _check(lib().lmoe_route_noalloc(ctypes.byref(cfg), _ptr(x), _ptr(router_w), _ptr(router_b), T,
                                           _ptr(topk_idx), _ptr(topk_w), _stream(stream)), "lmoe_route_noalloc")


def lmoe_dproj_ablation(cfg, x, D, act_fmt, group_mask, h, T, ws, stream=None):
    """D_g x for the groups of group_mask, fp16 (act_fmt 0) or Q8_1 (1) activations."""
    return _check(lib().lmoe_dproj_ablation(ctypes.byref(cfg), _ptr(x), _ptr(D), int(act_fmt), int(group_mask),
                                            _ptr(h), T, _ptr(ws), _nbytes(ws), _stream(stream)),
                  "lmoe_dproj_ablation")
