"""Python binding of libmoe.so's decode attention (include/attn.h): argument
marshalling only.  Every step runs in the library's CUDA kernels; there is no
fallback."""
from __future__ import annotations

import ctypes

import torch

from . import moe

MOE_ERR_DEVICE_INDEX = -6

# Every entry point declared in include/attn.h.
ATTN_EXPORTS = ("attn_decode_workspace_size", "attn_decode", "attn_decode_plan")

_ready = False


def library() -> ctypes.CDLL:
    global _ready
    lib = moe.library()
    if not _ready:
        P, I = ctypes.c_void_p, ctypes.c_int
        lib.attn_decode_workspace_size.argtypes = [I, I, I, I, I]
        lib.attn_decode_workspace_size.restype = ctypes.c_size_t
        lib.attn_decode.argtypes = [P, P, P, P, P, I, I, I, I, I, I, I, ctypes.c_float, P, P, ctypes.c_size_t, P]
        lib.attn_decode.restype = I
        lib.attn_decode_plan.argtypes = [I, I, I, I, ctypes.POINTER(I), ctypes.POINTER(I)]
        lib.attn_decode_plan.restype = I
        _ready = True
    return lib


def workspace_size(B: int, Hkv: int, D: int, block: int, max_blocks: int) -> int:
    return int(library().attn_decode_workspace_size(B, Hkv, D, block, max_blocks))


def alloc_workspace(B: int, Hkv: int, D: int, block: int, max_blocks: int, device="cuda") -> torch.Tensor:
    n = workspace_size(B, Hkv, D, block, max_blocks)
    if n == 0:
        raise moe.MoEError(moe.MOE_ERR_UNSUPPORTED, "attn_decode_workspace_size")
    return torch.zeros(n, dtype=torch.uint8, device=device)


def plan(B: int, Hkv: int, block: int, max_blocks: int) -> tuple[int, int]:
    """(ranges per sequence and key/value head, 16-position chunks per range)."""
    ns, cps = ctypes.c_int(0), ctypes.c_int(0)
    moe._check(library().attn_decode_plan(B, Hkv, block, max_blocks, ctypes.byref(ns), ctypes.byref(cps)),
               "attn_decode_plan")
    return ns.value, cps.value


def attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, block_table: torch.Tensor,
                ctx_len: torch.Tensor, out: torch.Tensor, workspace: torch.Tensor, scale: float = 0.0,
                stream=None) -> None:
    """q, out: bf16 [B, Hq, D]; caches: bf16 [n_blocks, Hkv, block, D]; block_table: int32 [B, max_blocks];
    ctx_len: int32 [B]; all contiguous on one device."""
    for t in (q, k_cache, v_cache, block_table, ctx_len, out, workspace):
        if not t.is_contiguous():
            raise ValueError("attn_decode needs contiguous tensors")
    B, Hq, D = q.shape
    n_blocks, Hkv, block, _ = k_cache.shape
    max_blocks = block_table.shape[1]
    moe._check(library().attn_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), block_table.data_ptr(),
                                     ctx_len.data_ptr(), B, Hq, Hkv, D, block, max_blocks, n_blocks, float(scale),
                                     out.data_ptr(), workspace.data_ptr(), workspace.numel(), moe._stream(stream)),
               "attn_decode")
