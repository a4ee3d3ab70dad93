"""Device-side marshalling for the C ABI: uploads a layer's host arrays into torch CUDA
tensors, fills ``moe_weights`` with their addresses and owns the handle and workspaces.

Torch provides memory and streams only; every computation runs in ``libmoe.so``.
"""
from __future__ import annotations

import numpy as np
import torch

from . import (MOE_FMT_INT4_ROWSCALE, MOE_FMT_NVFP4, moe_combine, moe_expert_ffn,
               moe_forward, moe_forward_fused, moe_forward_host, moe_group, moe_layer_create, moe_layer_desc,
               moe_layer_destroy, moe_route, moe_route_static, moe_weights, moe_workspace_size)

# host array key -> moe_weights field
_FIELD = {
    "Wr": "router_w", "bias": "router_bias", "g": "gate", "u": "up", "d": "down",
    "sg": "gate_scale", "su": "up_scale", "sd": "down_scale",
    "bg": "gate_bscale", "bu": "up_bscale", "bd": "down_bscale",
    "tg": "gate_tscale", "tu": "up_tscale", "td": "down_tscale",
    "sh_g": "shared_gate", "sh_u": "shared_up", "sh_d": "shared_down",
    "sh_sg": "shared_gate_scale", "sh_su": "shared_up_scale", "sh_sd": "shared_down_scale",
    "sh_bg": "shared_gate_bscale", "sh_bu": "shared_up_bscale", "sh_bd": "shared_down_bscale",
    "sh_tg": "shared_gate_tscale", "sh_tu": "shared_up_tscale", "sh_td": "shared_down_tscale",
}


def make_desc(d: dict, max_tokens: int) -> moe_layer_desc:
    return moe_layer_desc(hidden=d["H"], inter=d["I"], inter_shared=d["I_sh"], n_experts=d["E"],
                          top_k=d["k"], n_shared=d["n_shared"], routed_scaling=d["scaling"],
                          format=d["fmt"], max_tokens=max_tokens, top_p=float(d.get("top_p", 0.0)))


def _to_device(a, device) -> torch.Tensor:
    a = np.ascontiguousarray(np.asarray(a))
    if a.ndim == 0:
        a = a.reshape(1)
    return torch.from_numpy(a).to(device)


class DeviceLayer:
    """One layer resident in HBM plus its handle."""

    def __init__(self, desc: dict, host: dict | None = None, max_tokens: int = 1,
                 device="cuda", tensors: dict | None = None):
        self.d = dict(desc)
        self.device = torch.device(device)
        self.max_tokens = max_tokens
        if tensors is None:
            tensors = {k: _to_device(v, self.device) for k, v in host.items() if k in _FIELD}
        self.t = tensors
        w = moe_weights()
        for k, v in self.t.items():
            setattr(w, _FIELD[k], v.data_ptr())
        self.weights = w
        self.desc = make_desc(self.d, max_tokens)
        self.handle = moe_layer_create(self.desc, self.weights)

    def clone_weights(self) -> "DeviceLayer":
        """A second layer with the same values at different HBM addresses."""
        return DeviceLayer(self.d, max_tokens=self.max_tokens, device=self.device,
                           tensors={k: v.clone() for k, v in self.t.items()})

    def close(self):
        if getattr(self, "handle", None):
            moe_layer_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # ------------------------------------------------------------------ workspace
    def workspace(self, T: int) -> torch.Tensor:
        n = moe_workspace_size(self.handle, T)
        if n == 0:
            raise ValueError(f"T={T} out of range for this handle")
        return torch.zeros(n, dtype=torch.uint8, device=self.device)

    # ------------------------------------------------------------------ calls
    @staticmethod
    def _stream(stream):
        return (stream or torch.cuda.current_stream()).cuda_stream

    def forward(self, x: torch.Tensor, ws: torch.Tensor, y: torch.Tensor | None = None,
                stream=None, fused: bool = False) -> torch.Tensor:
        """The layer (moe_forward); fused=True: the one-launch decode path
        (moe_forward_fused, T <= 16)."""
        T = x.shape[0]
        if y is None:
            y = torch.empty_like(x)
        fn = moe_forward_fused if fused else moe_forward
        fn(self.handle, x.data_ptr(), T, y.data_ptr(), ws.data_ptr(), ws.numel(), self._stream(stream))
        return y

    def forward_host(self, x_host: torch.Tensor, y_host: torch.Tensor, ws: torch.Tensor,
                     stream=None):
        moe_forward_host(self.handle, x_host.data_ptr(), x_host.shape[0], y_host.data_ptr(),
                         ws.data_ptr(), ws.numel(), self._stream(stream))

    def route(self, x, T, ws, logits_in=None, want_logits=False, stream=None):
        k, E = self.d["k"], self.d["E"]
        idx = torch.empty((T, k), dtype=torch.int32, device=self.device)
        w = torch.empty((T, k), dtype=torch.float32, device=self.device)
        lo = torch.empty((T, E), dtype=torch.float32, device=self.device) if want_logits else None
        moe_route(self.handle, x.data_ptr() if x is not None else None, T,
                  logits_in.data_ptr() if logits_in is not None else None,
                  lo.data_ptr() if lo is not None else None, idx.data_ptr(), w.data_ptr(),
                  ws.data_ptr(), ws.numel(), self._stream(stream))
        return idx, w, lo

    def route_static(self, x, T, logits_in=None, want_logits=False, stream=None):
        """moe_route with the library's static scratch instead of a workspace."""
        k, E = self.d["k"], self.d["E"]
        idx = torch.empty((T, k), dtype=torch.int32, device=self.device)
        w = torch.empty((T, k), dtype=torch.float32, device=self.device)
        lo = torch.empty((T, E), dtype=torch.float32, device=self.device) if want_logits else None
        moe_route_static(self.handle, x.data_ptr() if x is not None else None, T,
                         logits_in.data_ptr() if logits_in is not None else None,
                         lo.data_ptr() if lo is not None else None, idx.data_ptr(), w.data_ptr(),
                         self._stream(stream))
        return idx, w, lo

    def group(self, topk_idx, T, ws, stream=None):
        E = self.d["E"]
        dev = self.device
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        perm = torch.empty(max(T * self.d["k"], 1), dtype=torch.int32, device=dev)
        unique = torch.empty(E, dtype=torch.int32, device=dev)
        nu = torch.empty(1, dtype=torch.int32, device=dev)
        moe_group(self.handle, topk_idx.data_ptr(), T, counts.data_ptr(), offsets.data_ptr(),
                  perm.data_ptr(), unique.data_ptr(), nu.data_ptr(), ws.data_ptr(), ws.numel(),
                  self._stream(stream))
        return counts, offsets, perm, unique, nu

    def expert_ffn(self, x, T, offsets, perm, ws, stream=None):
        H, k = self.d["H"], self.d["k"]
        ya = torch.empty((T * k, H), dtype=torch.float32, device=self.device)
        ys = torch.empty((T, H), dtype=torch.float32, device=self.device) if self.d["n_shared"] else None
        moe_expert_ffn(self.handle, x.data_ptr(), T, offsets.data_ptr(), perm.data_ptr(),
                       ya.data_ptr(), ys.data_ptr() if ys is not None else None, ws.data_ptr(),
                       ws.numel(), self._stream(stream))
        return ya, ys

    def combine(self, y_assign, y_shared, topk_w, T, stream=None):
        y = torch.empty((T, self.d["H"]), dtype=torch.uint16, device=self.device)
        moe_combine(self.handle, y_assign.data_ptr(),
                    y_shared.data_ptr() if y_shared is not None else None, topk_w.data_ptr(), T,
                    y.data_ptr(), self._stream(stream))
        return y


def fp16_bits_to_float(y_bits: torch.Tensor) -> np.ndarray:
    return y_bits.cpu().numpy().view(np.float16).astype(np.float64)
