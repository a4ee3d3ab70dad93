"""W4A16 quantized-expert MoE decode layer for NVIDIA B200 (sm_100a).

A thin ctypes binding of the C ABI in ``include/moe.h`` (``libmoe.so``): the functions
below carry the C names and only marshal arguments; every step of the layer runs in the
library's CUDA kernels.  PyTorch is used by callers for device memory and streams only.
There is no CPU fallback: if ``libmoe.so`` is missing, ``lib()`` raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_DEVICE_TIMEOUT = 5
MOE_ERR_DEVICE_BOUNDS = 6

MOE_FMT_INT4_ROWSCALE = 0
MOE_FMT_NVFP4 = 1
MOE_FMT_INT8_ROWSCALE = 2
MOE_FMT_INT2_ROWSCALE = 3
MOE_PLAN_DECODE = 0
MOE_PLAN_F16_BATCH = 1
MOE_PLAN_TENSOR_MEMORY = 2

vp = ctypes.c_void_p
c_int = ctypes.c_int
c_size = ctypes.c_size_t


class moe_layer_desc(ctypes.Structure):
    _fields_ = [("hidden", c_int), ("inter", c_int), ("inter_shared", c_int),
                ("n_experts", c_int), ("top_k", c_int), ("n_shared", c_int),
                ("routed_scaling", ctypes.c_float), ("format", c_int), ("max_tokens", c_int),
                ("top_p", ctypes.c_float)]


WEIGHT_FIELDS = ["router_w", "router_bias", "gate", "up", "down",
                 "gate_scale", "up_scale", "down_scale",
                 "gate_bscale", "up_bscale", "down_bscale",
                 "gate_tscale", "up_tscale", "down_tscale",
                 "shared_gate", "shared_up", "shared_down",
                 "shared_gate_scale", "shared_up_scale", "shared_down_scale",
                 "shared_gate_bscale", "shared_up_bscale", "shared_down_bscale",
                 "shared_gate_tscale", "shared_up_tscale", "shared_down_tscale"]


class moe_weights(ctypes.Structure):
    _fields_ = [(f, vp) for f in WEIGHT_FIELDS]


class moe_ws_routing(ctypes.Structure):
    _fields_ = [(f, c_size) for f in ("logits", "topk_idx", "topk_w", "counts", "offsets", "perm", "unique",
                                      "n_unique")]


class MoeError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: {status_string(code)} ({code})")
        self.code = code


_lib = None


def lib():
    """Load libmoe.so; raises if it has not been built (no fallback path exists)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m w4a16_quantized_expert_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        L.moe_version.restype = c_int
        L.moe_status_string.argtypes = [c_int]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_layer_create.argtypes = [ctypes.POINTER(moe_layer_desc), ctypes.POINTER(moe_weights),
                                       ctypes.POINTER(vp)]
        L.moe_layer_destroy.argtypes = [vp]
        L.moe_workspace_size.argtypes = [vp, c_int]
        L.moe_workspace_size.restype = c_size
        L.moe_route.argtypes = [vp, vp, c_int, vp, vp, vp, vp, vp, c_size, vp]
        L.moe_route_static.argtypes = [vp, vp, c_int, vp, vp, vp, vp, vp]
        L.moe_group.argtypes = [vp, vp, c_int, vp, vp, vp, vp, vp, vp, c_size, vp]
        L.moe_expert_ffn.argtypes = [vp, vp, c_int, vp, vp, vp, vp, vp, c_size, vp]
        L.moe_combine.argtypes = [vp, vp, vp, vp, c_int, vp, vp]
        L.moe_forward.argtypes = [vp, vp, c_int, vp, vp, c_size, vp]
        L.moe_forward_fused.argtypes = [vp, vp, c_int, vp, vp, c_size, vp]
        L.moe_forward_host.argtypes = [vp, vp, c_int, vp, vp, c_size, vp]
        L.moe_forward_timed.argtypes = [vp, vp, c_int, vp, vp, c_size, vp, ctypes.POINTER(vp),
                                        ctypes.POINTER(c_int)]
        L.moe_get_device_status.argtypes = [vp, ctypes.POINTER(c_int)]
        L.moe_debug_wait_timeout.argtypes = [vp, ctypes.c_longlong, vp]
        L.moe_workspace_routing.argtypes = [vp, c_int, ctypes.POINTER(moe_ws_routing)]
        L.moe_plan.argtypes = [ctypes.POINTER(moe_layer_desc), c_int, ctypes.POINTER(c_int)]
        for f in ("moe_layer_create", "moe_layer_destroy", "moe_route", "moe_route_static", "moe_group",
                  "moe_expert_ffn", "moe_combine", "moe_forward", "moe_forward_fused", "moe_forward_host", "moe_forward_timed",
                  "moe_get_device_status", "moe_debug_wait_timeout", "moe_workspace_routing", "moe_plan"):
            getattr(L, f).restype = c_int
        _lib = L
    return _lib


def _check(rc: int, what: str) -> None:
    if rc != MOE_OK:
        raise MoeError(rc, what)


def moe_status_string(code: int) -> str:
    return lib().moe_status_string(code).decode()


status_string = moe_status_string


def moe_version() -> int:
    return lib().moe_version()


def moe_layer_create(desc: moe_layer_desc, weights: moe_weights) -> int:
    h = vp()
    _check(lib().moe_layer_create(ctypes.byref(desc), ctypes.byref(weights), ctypes.byref(h)),
           "moe_layer_create")
    return h.value


def moe_layer_destroy(layer: int) -> None:
    _check(lib().moe_layer_destroy(layer), "moe_layer_destroy")


def moe_workspace_size(layer: int, T: int) -> int:
    return lib().moe_workspace_size(layer, T)


def moe_route(layer, x, T, logits_in, logits_out, topk_idx, topk_w, ws, ws_bytes, stream=0):
    _check(lib().moe_route(layer, x, T, logits_in, logits_out, topk_idx, topk_w, ws, ws_bytes,
                           stream), "moe_route")


def moe_route_static(layer, x, T, logits_in, logits_out, topk_idx, topk_w, stream=0):
    _check(lib().moe_route_static(layer, x, T, logits_in, logits_out, topk_idx, topk_w, stream),
           "moe_route_static")


def moe_group(layer, topk_idx, T, counts, offsets, perm, unique, n_unique, ws, ws_bytes, stream=0):
    _check(lib().moe_group(layer, topk_idx, T, counts, offsets, perm, unique, n_unique, ws,
                           ws_bytes, stream), "moe_group")


def moe_expert_ffn(layer, x, T, offsets, perm, y_assign, y_shared, ws, ws_bytes, stream=0):
    _check(lib().moe_expert_ffn(layer, x, T, offsets, perm, y_assign, y_shared, ws, ws_bytes,
                                stream), "moe_expert_ffn")


def moe_combine(layer, y_assign, y_shared, topk_w, T, y, stream=0):
    _check(lib().moe_combine(layer, y_assign, y_shared, topk_w, T, y, stream), "moe_combine")


def moe_forward(layer, x, T, y, ws, ws_bytes, stream=0):
    _check(lib().moe_forward(layer, x, T, y, ws, ws_bytes, stream), "moe_forward")


def moe_forward_fused(layer, x, T, y, ws, ws_bytes, stream=0):
    _check(lib().moe_forward_fused(layer, x, T, y, ws, ws_bytes, stream), "moe_forward_fused")


def moe_forward_host(layer, x_host, T, y_host, ws, ws_bytes, stream=0):
    _check(lib().moe_forward_host(layer, x_host, T, y_host, ws, ws_bytes, stream),
           "moe_forward_host")


def moe_forward_timed(layer, x, T, y, ws, ws_bytes, stream, events):
    """Returns (timed parts, kernels launched); see include/moe.h."""
    ev = (vp * 4)(*events)
    info = (c_int * 2)(0, 0)
    _check(lib().moe_forward_timed(layer, x, T, y, ws, ws_bytes, stream, ev, info), "moe_forward_timed")
    return int(info[0]), int(info[1])


def moe_get_device_status(layer) -> int:
    st = c_int(0)
    _check(lib().moe_get_device_status(layer, ctypes.byref(st)), "moe_get_device_status")
    return st.value


def moe_debug_wait_timeout(layer, max_iters, stream=0):
    _check(lib().moe_debug_wait_timeout(layer, max_iters, stream), "moe_debug_wait_timeout")


def moe_plan(desc: moe_layer_desc, T: int) -> tuple:
    """(kernel family, tokens per work item, int8 limbs) of a batch of T tokens; see
    include/moe.h."""
    plan = (c_int * 3)(0, 0, 0)
    _check(lib().moe_plan(ctypes.byref(desc), T, plan), "moe_plan")
    return int(plan[0]), int(plan[1]), int(plan[2])


def moe_workspace_routing(layer, T) -> dict:
    """Byte offsets of the routing and grouping arrays moe_forward leaves in the workspace."""
    r = moe_ws_routing()
    _check(lib().moe_workspace_routing(layer, T, ctypes.byref(r)), "moe_workspace_routing")
    return {f: getattr(r, f) for f, _ in moe_ws_routing._fields_}
