"""Python binding of libmoe.so's Gated DeltaNet decode step (include/deltanet.h):
argument marshalling only.  The step runs in the library's CUDA kernel; there
is no fallback."""
from __future__ import annotations

import ctypes

import torch

from . import moe

# Every entry point declared in include/deltanet.h.
GDN_EXPORTS = ("gdn_decode_step",)

_ready = False


def library() -> ctypes.CDLL:
    global _ready
    lib = moe.library()
    if not _ready:
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.gdn_decode_step.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P]
        lib.gdn_decode_step.restype = I
        _ready = True
    return lib


def gdn_decode_step(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, g: torch.Tensor, beta: torch.Tensor,
                    state: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """q, k: bf16 [B, H_k, d_k]; v, out: bf16 [B, H_v, d_v]; g, beta: FP32 [B, H_v];
    state: FP32 [B, H_v, d_v, d_k], updated in place.  All contiguous on one device."""
    for t in (q, k, v, g, beta, state, out):
        if not t.is_contiguous():
            raise ValueError("gdn_decode_step needs contiguous tensors")
    B, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    moe._check(library().gdn_decode_step(q.data_ptr(), k.data_ptr(), v.data_ptr(), g.data_ptr(), beta.data_ptr(),
                                         state.data_ptr(), out.data_ptr(), B, Hk, Hv, dk, dv, moe._stream(stream)),
               "gdn_decode_step")
