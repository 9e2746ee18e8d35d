"""Python binding of libmoe.so (argument marshalling only).

Every step of the layer runs in the library's CUDA kernels; this module only
turns torch tensors into the C structs of include/moe.h and checks status
codes.  There is no fallback: if libmoe.so is missing or fails to load, the
import-time loader raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_DEVICE_TIMEOUT = -5
MOE_ERR_DEVICE_INDEX = -6

# Every entry point declared in include/moe.h.
EXPORTS = ("moe_workspace_size", "moe_route", "moe_forward", "moe_decode", "moe_forward_host", "moe_forward_host_async",
           "moe_forward_stack", "moe_rmsnorm", "moe_forward_profiled", "moe_route_static", "moe_get_status",
           "moe_set_wait_limit", "moe_strerror")


class QMatC(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("biases", ctypes.c_void_p)]


class LayerC(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int), ("I", ctypes.c_int), ("I_shared", ctypes.c_int), ("E", ctypes.c_int),
                ("k", ctypes.c_int), ("group_size", ctypes.c_int), ("bits", ctypes.c_int), ("renorm", ctypes.c_int),
                ("w_router", ctypes.c_void_p), ("router_bias", ctypes.c_void_p),
                ("gate", QMatC), ("up", QMatC), ("down", QMatC),
                ("sh_gate", QMatC), ("sh_up", QMatC), ("sh_down", QMatC),
                ("w_shared_gate", ctypes.c_void_p)]


class RoutingC(ctypes.Structure):
    _fields_ = [("topk_idx", ctypes.c_void_p), ("topk_w", ctypes.c_void_p), ("counts", ctypes.c_void_p),
                ("offsets", ctypes.c_void_p), ("perm", ctypes.c_void_p), ("inv_perm", ctypes.c_void_p),
                ("sigma", ctypes.c_void_p)]


class MoEError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: status {code} ({strerror(code)})")
        self.code = code


_lib = None


def library() -> ctypes.CDLL:
    """Load libmoe.so (built in-tree by build.py); raise if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise ImportError(f"libmoe.so not built (expected at {_LIB_PATH}); run "
                          "python -m bit_quantized_expert_route_b200.build")
    lib = ctypes.CDLL(_LIB_PATH)
    P, I, S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    LP, RP = ctypes.POINTER(LayerC), ctypes.POINTER(RoutingC)
    lib.moe_workspace_size.argtypes = [LP, I, ctypes.POINTER(S)]
    lib.moe_route.argtypes = [LP, P, I, RP, P, S, P]
    lib.moe_forward.argtypes = [LP, P, I, P, RP, P, S, P]
    lib.moe_decode.argtypes = [LP, P, I, P, RP, P, S, P]
    lib.moe_forward_host.argtypes = [LP, P, I, P, P, S, P]
    lib.moe_forward_host_async.argtypes = [LP, P, I, P, P, S, P]
    lib.moe_rmsnorm.argtypes = [P, P, I, I, ctypes.c_float, P]
    lib.moe_forward_stack.argtypes = [LP, I, P, I, P, P, ctypes.c_float, P, S, P]
    lib.moe_forward_profiled.argtypes = [LP, P, I, P, P, S, P, ctypes.POINTER(ctypes.c_float),
                                         ctypes.POINTER(ctypes.c_int)]
    lib.moe_route_static.argtypes = [LP, P, I, RP, P]
    lib.moe_get_status.argtypes = [P, P]
    lib.moe_set_wait_limit.argtypes = [ctypes.c_longlong]
    lib.moe_strerror.argtypes = [I]
    lib.moe_strerror.restype = ctypes.c_char_p
    for name in EXPORTS:
        if name != "moe_strerror":
            getattr(lib, name).restype = I
    _lib = lib
    return lib


def strerror(code: int) -> str:
    return library().moe_strerror(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != MOE_OK:
        raise MoEError(code, where)


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ layers --

def _bits_tensor(a: np.ndarray, device) -> torch.Tensor:
    """Upload a uint16 (bf16 bits) or uint32 array as bf16 / int32 without changing a bit."""
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    if a.dtype == np.uint32:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int32)).to(device)
    if a.dtype == np.float32:
        return torch.from_numpy(np.ascontiguousarray(a)).to(device)
    raise TypeError(a.dtype)


@dataclass
class MoELayer:
    """A layer whose weights live in device memory, plus its C descriptor."""
    H: int
    I: int
    I_shared: int
    E: int
    k: int
    tensors: dict

    def __post_init__(self):
        t = self.tensors

        def qm(name):
            m = t[name]
            return QMatC(m["q"].data_ptr(), m["scales"].data_ptr(), m["biases"].data_ptr())

        self.desc = LayerC(self.H, self.I, self.I_shared, self.E, self.k, 64, 4, 1,
                           t["w_router"].data_ptr(), _ptr(t.get("router_bias")),
                           qm("gate"), qm("up"), qm("down"), qm("sh_gate"), qm("sh_up"), qm("sh_down"),
                           t["w_shared_gate"].data_ptr())

    @staticmethod
    def from_synth(layer, device="cuda") -> "MoELayer":
        """Upload a synth.Layer (numpy storage arrays) bit for bit."""
        d = layer.dims

        def q(m):
            return {"q": _bits_tensor(m.q, device), "scales": _bits_tensor(m.scales, device),
                    "biases": _bits_tensor(m.biases, device)}

        t = {"w_router": _bits_tensor(layer.w_router, device),
             "router_bias": None if layer.router_bias is None else _bits_tensor(layer.router_bias, device),
             "gate": q(layer.gate), "up": q(layer.up), "down": q(layer.down),
             "sh_gate": q(layer.sh_gate), "sh_up": q(layer.sh_up), "sh_down": q(layer.sh_down),
             "w_shared_gate": _bits_tensor(layer.w_shared_gate, device)}
        return MoELayer(d.H, d.I, d.I_s, d.E, d.k, t)

    @staticmethod
    def from_tensors(dims, tensors: dict) -> "MoELayer":
        return MoELayer(dims.H, dims.I, dims.I_s, dims.E, dims.k, tensors)


class Routing:
    """Device buffers for moe_route's outputs (see moe_routing in include/moe.h)."""

    def __init__(self, T: int, E: int, k: int, device="cuda"):
        n = T * k
        i32 = dict(dtype=torch.int32, device=device)
        self.topk_idx = torch.empty(n, **i32)
        self.topk_w = torch.empty(n, dtype=torch.float32, device=device)
        self.counts = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.perm = torch.empty(n, **i32)
        self.inv_perm = torch.empty(n, **i32)
        self.sigma = torch.empty(T, dtype=torch.float32, device=device)
        self.c = RoutingC(*(t.data_ptr() for t in (self.topk_idx, self.topk_w, self.counts, self.offsets,
                                                   self.perm, self.inv_perm, self.sigma)))


def moe_workspace_size(layer: MoELayer, T_max: int) -> int:
    n = ctypes.c_size_t(0)
    _check(library().moe_workspace_size(ctypes.byref(layer.desc), int(T_max), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def alloc_workspace(layer: MoELayer, T_max: int, device="cuda") -> torch.Tensor:
    """A zero-filled device workspace for calls with T <= T_max (torch allocations are 256-byte aligned)."""
    return torch.zeros(moe_workspace_size(layer, T_max), dtype=torch.uint8, device=device)


def moe_route(layer: MoELayer, x: torch.Tensor, routing: Routing, workspace: torch.Tensor, stream=None) -> None:
    T = x.shape[0]
    _check(library().moe_route(ctypes.byref(layer.desc), x.data_ptr(), T, ctypes.byref(routing.c),
                               workspace.data_ptr(), workspace.numel(), _stream(stream)), "moe_route")


def moe_route_static(layer: MoELayer, x: torch.Tensor, routing: Routing, stream=None) -> None:
    """moe_route without a workspace (scratch in a static device array of libmoe.so)."""
    T = x.shape[0]
    _check(library().moe_route_static(ctypes.byref(layer.desc), x.data_ptr(), T, ctypes.byref(routing.c),
                                      _stream(stream)), "moe_route_static")


def moe_forward(layer: MoELayer, x: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                routing: Routing | None = None, stream=None) -> None:
    T = x.shape[0]
    r = ctypes.byref(routing.c) if routing is not None else None
    _check(library().moe_forward(ctypes.byref(layer.desc), x.data_ptr(), T, out.data_ptr(), r,
                                 workspace.data_ptr(), workspace.numel(), _stream(stream)), "moe_forward")


def moe_decode(layer: MoELayer, x: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
               routing: Routing | None = None, stream=None) -> None:
    T = x.shape[0]
    r = ctypes.byref(routing.c) if routing is not None else None
    _check(library().moe_decode(ctypes.byref(layer.desc), x.data_ptr(), T, out.data_ptr(), r,
                                workspace.data_ptr(), workspace.numel(), _stream(stream)), "moe_decode")


def moe_forward_host(layer: MoELayer, x_host: torch.Tensor, out_host: torch.Tensor, workspace: torch.Tensor,
                     stream=None) -> None:
    T = x_host.shape[0]
    _check(library().moe_forward_host(ctypes.byref(layer.desc), x_host.data_ptr(), T, out_host.data_ptr(),
                                      workspace.data_ptr(), workspace.numel(), _stream(stream)), "moe_forward_host")


def moe_forward_host_async(layer: MoELayer, x_host: torch.Tensor, out_host: torch.Tensor, workspace: torch.Tensor,
                           stream=None) -> None:
    """moe_forward_host without the final wait (page-locked x_host/out_host for overlap)."""
    T = x_host.shape[0]
    _check(library().moe_forward_host_async(ctypes.byref(layer.desc), x_host.data_ptr(), T, out_host.data_ptr(),
                                            workspace.data_ptr(), workspace.numel(), _stream(stream)),
           "moe_forward_host_async")


class LayerStack:
    """A host array of layer descriptors for moe_forward_stack (keeps the layers' tensors alive)."""

    def __init__(self, layers):
        self.layers = list(layers)
        self.array = (LayerC * len(self.layers))(*(L.desc for L in self.layers))


def moe_forward_stack(stack: LayerStack, x: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                      trace: torch.Tensor | None = None, eps: float = 1e-6, stream=None) -> None:
    """len(stack.layers) layers joined by RMSNorm in one enqueued sequence (see include/moe.h)."""
    T = x.shape[0]
    _check(library().moe_forward_stack(stack.array, len(stack.layers), x.data_ptr(), T, out.data_ptr(),
                                       _ptr(trace), float(eps), workspace.data_ptr(), workspace.numel(),
                                       _stream(stream)), "moe_forward_stack")


def moe_rmsnorm(y: torch.Tensor, y_out: torch.Tensor, eps: float = 1e-6, stream=None) -> None:
    T, H = y.shape
    _check(library().moe_rmsnorm(y.data_ptr(), y_out.data_ptr(), T, H, float(eps), _stream(stream)), "moe_rmsnorm")


PREFILL_STAGES = ("router", "group", "gather", "gateup", "down", "combine")
MID_DECODE_STAGES = ("route", "gateup", "down", "combine")
FUSED_DECODE_STAGES = ("decode_fused",)


def moe_forward_profiled(layer: MoELayer, x: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor,
                         stream=None) -> dict:
    """moe_forward with per-stage device times (ms), keyed by stage name."""
    T = x.shape[0]
    ms = (ctypes.c_float * 8)()
    n = ctypes.c_int(0)
    _check(library().moe_forward_profiled(ctypes.byref(layer.desc), x.data_ptr(), T, out.data_ptr(),
                                          workspace.data_ptr(), workspace.numel(), _stream(stream), ms,
                                          ctypes.byref(n)), "moe_forward_profiled")
    names = {1: FUSED_DECODE_STAGES, len(MID_DECODE_STAGES): MID_DECODE_STAGES, len(PREFILL_STAGES): PREFILL_STAGES}[n.value]
    return {names[i]: float(ms[i]) for i in range(n.value)}


def moe_get_status(workspace: torch.Tensor | None, stream=None) -> int:
    """Status word of a workspace (None: of moe_route_static's static scratch); cleared when not MOE_OK."""
    return int(library().moe_get_status(_ptr(workspace), _stream(stream)))


def moe_set_wait_limit(cycles: int) -> None:
    """SM clock cycles before the kernels' bounded waits give up (<= 0: the default, about 2 s)."""
    _check(library().moe_set_wait_limit(int(cycles)), "moe_set_wait_limit")
