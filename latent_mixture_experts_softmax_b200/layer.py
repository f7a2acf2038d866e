"""Device-resident weights of one latent-MoE layer and a workspace, held as
torch tensors, with thin calls into the C ABI.  torch provides the memory
and the stream; all arithmetic runs in liblmoe.so."""
from __future__ import annotations

import numpy as np
import torch

from . import binding as B


def to_device(a: np.ndarray | None, device) -> torch.Tensor | None:
    """Host numpy array -> device tensor with the same bytes (uint16 goes as int16)."""
    if a is None:
        return None
    if a.dtype == np.uint16:
        a = a.view(np.int16)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


class DeviceLayer:
    """One layer's weights on the device (see include/lmoe.h for the layouts)."""

    def __init__(self, shape, layer: dict, device="cuda", gamma: np.ndarray | None = None):
        self.shape = shape
        self.cfg = B.make_cfg(shape)
        self.device = torch.device(device)
        self.router_w = to_device(layer["router_w"], device)
        self.router_b = to_device(layer.get("router_b"), device)
        self.expert_group = to_device(layer["expert_group"], device)
        self.D = to_device(layer["D"], device)
        self.U = to_device(layer["U"], device)
        self.experts = to_device(layer["experts"], device)
        self.shared_gate = to_device(layer["shared_gate"], device)
        self.shared_up = to_device(layer["shared_up"], device)
        self.shared_down = to_device(layer["shared_down"], device)
        self.shared = B.make_shared(self.shared_gate, self.shared_up, self.shared_down)
        self.gamma = to_device(gamma, device) if gamma is not None else None

    def weight_bytes(self) -> int:
        ts = [self.router_w, self.router_b, self.expert_group, self.D, self.U, self.experts, self.shared_gate,
              self.shared_up, self.shared_down]
        return sum(t.numel() * t.element_size() for t in ts if t is not None)

    def as_c_layer(self) -> B.lmoe_layer:
        if self.gamma is None:
            raise ValueError("a stack layer needs its RMSNorm gamma")
        p = B._ptr
        return B.lmoe_layer(p(self.router_w), p(self.router_b), p(self.expert_group), p(self.D), p(self.U),
                            p(self.experts), self.shared, p(self.gamma))

    def workspace(self, T_max: int) -> torch.Tensor:
        n = B.lmoe_workspace_bytes(self.cfg, T_max)
        if n == 0:
            raise B.LmoeError(B.LMOE_ERR_UNSUPPORTED, "lmoe_workspace_bytes")
        ws = torch.empty(n, dtype=torch.uint8, device=self.device)
        ws[:4096].zero_()
        return ws

    def forward(self, x: torch.Tensor, ws: torch.Tensor, y: torch.Tensor | None = None,
                residual: torch.Tensor | None = None, inject: tuple | None = None, want_routing: bool = False,
                stream=None):
        """y = block(x) (+ residual).  x, y: int16 tensors holding bf16 [T][hidden]."""
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        out_idx = out_w = None
        if want_routing:
            out_idx = torch.empty((T, self.shape.top_k), dtype=torch.int32, device=self.device)
            out_w = torch.empty((T, self.shape.top_k), dtype=torch.float32, device=self.device)
        inj_idx, inj_w = inject if inject is not None else (None, None)
        B.lmoe_forward_ex(self.cfg, x, self.router_w, self.router_b, self.expert_group, self.D, self.U, self.experts,
                          self.shared, residual, inj_idx, inj_w, out_idx, out_w, y, T, ws, stream)
        if want_routing:
            return y, out_idx, out_w
        return y

    def route(self, x: torch.Tensor, ws: torch.Tensor, stream=None):
        T = x.shape[0]
        idx = torch.empty((T, self.shape.top_k), dtype=torch.int32, device=self.device)
        w = torch.empty((T, self.shape.top_k), dtype=torch.float32, device=self.device)
        B.lmoe_route(self.cfg, x, self.router_w, self.router_b, T, idx, w, ws, stream)
        return idx, w


def bf16_bits_to_float(t: torch.Tensor) -> torch.Tensor:
    """int16 tensor of bf16 bit patterns -> float32 values (on the same device)."""
    return t.view(torch.bfloat16).float()
