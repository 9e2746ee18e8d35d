"""Seeded synthetic inputs for one sparse-MoE layer.

This module only draws random numbers and stores them in the layer's storage
formats (bf16 bit patterns, packed 4-bit words).  It holds none of the layer's
arithmetic: no dequantisation, no routing, no expert math.  Both the CPU
oracle's tests and the CUDA path's tests and benchmark take their inputs from
here, so the two sides always see the same bytes.

Recipe (the workloads of the Qwen3.6-35B-A3B MoE layer; "The Model" section
of the Lily write-ups gives 256 experts, top-8, one shared expert, and MLX
affine 4-bit weights with groups of 64):

* x ~ N(0, 1), stored as bf16.
* Router W_r ~ N(0, 0.02), bf16, shape [E, H].
* Every expert matrix is a "q-matrix" [R, C]: 4-bit codes q ~ U{0..15}
  packed 8 per uint32 (code i of a word in bits 4i..4i+3), a bf16 scale
  ~ U(0.002, 0.006) and a bf16 bias = -8 * scale + N(0, 1e-3) per group of
  64 consecutive columns (the input dimension).
* Shared-expert gate vector w_sg ~ N(0, 0.02), bf16, shape [H].
* Skewed ("Zipf 1.2") routing adds a float32 router bias
  b_e = 1.5 * ln(1 / rank_e ** 1.2) with ranks a seeded permutation of 1..E.

Random streams: every layer's weights come from one PCG64 stream keyed by
(seed, layer); x from a stream keyed by (seed, 'x'); a redrawn row t of x
(attempt a) from a stream keyed by (seed, t, a).  Bit patterns are stored as
numpy uint16 (bf16) / uint32 (packed codes) / float32 (router bias).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

_KEY_W = 0x57455447      # stream tag for a layer's weights
_KEY_X = 0x58494E50      # stream tag for the activations
_KEY_ROW = 0x524F5752    # stream tag for a redrawn activation row


@dataclasses.dataclass(frozen=True)
class Dims:
    """Shape of one MoE layer (names follow the Qwen3.6-35B-A3B MoE block)."""
    H: int = 2048        # hidden size
    E: int = 256         # routed experts
    k: int = 8           # experts chosen per token
    I: int = 512         # routed expert intermediate size
    I_s: int = 512       # shared expert intermediate size
    group: int = 64      # quantisation group along the input dimension

    @staticmethod
    def tiny() -> "Dims":
        return Dims(H=256, E=16, k=2, I=128, I_s=128)


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(v) for v in key])))


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Store real numbers as bf16 bit patterns (torch's round-to-nearest-even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bf16_bits_as_f32(bits: np.ndarray) -> np.ndarray:
    """Reinterpret bf16 bit patterns as float32 values (exact widening)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


@dataclasses.dataclass
class QMat:
    """One (or a stack of) affine 4-bit matrices [.., R, C] in MLX storage."""
    q: np.ndarray        # uint32 [.., R, C/8]
    scales: np.ndarray   # uint16 (bf16 bits) [.., R, C/64]
    biases: np.ndarray   # uint16 (bf16 bits) [.., R, C/64]


def _qmat(rng: np.random.Generator, lead: tuple, R: int, C: int, group: int) -> QMat:
    q = rng.integers(0, 2**32, size=lead + (R, C // 8), dtype=np.uint32)
    s_bits = to_bf16_bits(rng.uniform(0.002, 0.006, size=lead + (R, C // group)))
    noise = rng.normal(0.0, 1e-3, size=s_bits.shape)
    b_bits = to_bf16_bits(-8.0 * bf16_bits_as_f32(s_bits).astype(np.float64) + noise)
    return QMat(q, s_bits, b_bits)


@dataclasses.dataclass
class Layer:
    """All weights of one MoE layer, in the layer's storage formats."""
    dims: Dims
    w_router: np.ndarray              # uint16 [E, H]
    router_bias: np.ndarray | None    # float32 [E] or None
    gate: QMat                        # [E, I, H]
    up: QMat                          # [E, I, H]
    down: QMat                        # [E, H, I]
    sh_gate: QMat                     # [I_s, H]
    sh_up: QMat                       # [I_s, H]
    sh_down: QMat                     # [H, I_s]
    w_shared_gate: np.ndarray         # uint16 [H]


def zipf_router_bias(rng: np.random.Generator, E: int) -> np.ndarray:
    """b_e = 1.5*ln(1/rank_e^1.2) for a seeded permutation of ranks 1..E."""
    rank = rng.permutation(E) + 1
    return np.array([1.5 * math.log(1.0 / float(r) ** 1.2) for r in rank], dtype=np.float32)


def make_layer(seed: int, layer: int, dims: Dims, zipf: bool = False) -> Layer:
    """Draw one layer's weights from the (seed, layer) stream."""
    d = dims
    rng = _rng(_KEY_W, seed, layer)
    w_router = to_bf16_bits(rng.normal(0.0, 0.02, size=(d.E, d.H)))
    router_bias = zipf_router_bias(rng, d.E) if zipf else None
    gate = _qmat(rng, (d.E,), d.I, d.H, d.group)
    up = _qmat(rng, (d.E,), d.I, d.H, d.group)
    down = _qmat(rng, (d.E,), d.H, d.I, d.group)
    sh_gate = _qmat(rng, (), d.I_s, d.H, d.group)
    sh_up = _qmat(rng, (), d.I_s, d.H, d.group)
    sh_down = _qmat(rng, (), d.H, d.I_s, d.group)
    w_sg = to_bf16_bits(rng.normal(0.0, 0.02, size=(d.H,)))
    return Layer(d, w_router, router_bias, gate, up, down, sh_gate, sh_up, sh_down, w_sg)


def make_x(seed: int, T: int, H: int) -> np.ndarray:
    """Activations x ~ N(0,1) as bf16 bits, shape [T, H]."""
    return to_bf16_bits(_rng(_KEY_X, seed).normal(0.0, 1.0, size=(T, H)))


def redraw_row(seed: int, t: int, attempt: int, H: int) -> np.ndarray:
    """A replacement for row t of x (attempt = 1, 2, ...), still N(0,1) bf16."""
    return to_bf16_bits(_rng(_KEY_ROW, seed, t, attempt).normal(0.0, 1.0, size=(H,)))


# --------------------------------------------------------------------------
# Device-side generation of the same recipe (benchmark only: fast, no parity
# claim rests on it).  Uses torch's own generator on the given device.
# --------------------------------------------------------------------------

def _dev_qmat(g: torch.Generator, shape_lead: tuple, R: int, C: int, group: int, device) -> dict:
    q = torch.randint(-2**31, 2**31, shape_lead + (R, C // 8), generator=g, device=device,
                      dtype=torch.int64).to(torch.int32)
    s = torch.empty(shape_lead + (R, C // group), device=device, dtype=torch.float32)
    s.uniform_(0.002, 0.006, generator=g)
    s = s.to(torch.bfloat16)
    b = (-8.0 * s.float() + torch.randn(s.shape, generator=g, device=device) * 1e-3).to(torch.bfloat16)
    return {"q": q, "scales": s, "biases": b}


def make_layer_on_device(seed: int, layer: int, dims: Dims, device, zipf: bool = False) -> dict:
    """Same distributions as make_layer, drawn by torch directly in device memory."""
    d = dims
    g = torch.Generator(device=device)
    g.manual_seed((seed * 1_000_003 + layer * 7919 + 17) & 0x7FFFFFFF)
    out = {
        "w_router": (torch.randn((d.E, d.H), generator=g, device=device) * 0.02).to(torch.bfloat16),
        "router_bias": None,
    }
    if zipf:
        out["router_bias"] = zipf_bias_on_device(seed, layer, d, device)
    out["gate"] = _dev_qmat(g, (d.E,), d.I, d.H, d.group, device)
    out["up"] = _dev_qmat(g, (d.E,), d.I, d.H, d.group, device)
    out["down"] = _dev_qmat(g, (d.E,), d.H, d.I, d.group, device)
    out["sh_gate"] = _dev_qmat(g, (), d.I_s, d.H, d.group, device)
    out["sh_up"] = _dev_qmat(g, (), d.I_s, d.H, d.group, device)
    out["sh_down"] = _dev_qmat(g, (), d.H, d.I_s, d.group, device)
    out["w_shared_gate"] = (torch.randn((d.H,), generator=g, device=device) * 0.02).to(torch.bfloat16)
    return out


def zipf_bias_on_device(seed: int, layer: int, dims: Dims, device) -> torch.Tensor:
    """The skewed workload's router bias of layer (seed, layer) as a float32 device tensor: the
    same bias make_layer_on_device(..., zipf=True) adds, so a uniform layer's tensors plus this
    bias form the skewed layer."""
    return torch.from_numpy(zipf_router_bias(_rng(_KEY_W, seed, layer), dims.E)).to(device)


def make_x_on_device(seed: int, T: int, H: int, device) -> torch.Tensor:
    g = torch.Generator(device=device)
    g.manual_seed((seed * 2_000_029 + 5) & 0x7FFFFFFF)
    return torch.randn((T, H), generator=g, device=device).to(torch.bfloat16)


# --------------------------------------------------------------------------
# Decode attention over a fixed-block KV cache: seeded q, paged K/V and a
# shuffled block table (no attention arithmetic here).
# --------------------------------------------------------------------------
_KEY_ATTN = 0x4154544E   # stream tag for an attention case


@dataclasses.dataclass
class AttnCase:
    """One decode-attention step's inputs in storage form."""
    q: np.ndarray             # uint16 (bf16) [B, Hq, D]
    k_cache: np.ndarray       # uint16 (bf16) [n_blocks, Hkv, block, D]
    v_cache: np.ndarray       # uint16 (bf16) [n_blocks, Hkv, block, D]
    block_table: np.ndarray   # int32 [B, max_blocks]: physical block of each logical block
    ctx_len: np.ndarray       # int32 [B]


def make_attention_case(seed: int, ctx_lens, Hq: int = 16, Hkv: int = 2, D: int = 256, block: int = 64,
                        spare_blocks: int = 3) -> AttnCase:
    """q, k, v ~ N(0, 1) as bf16; every sequence's logical blocks are mapped to physical
    blocks by one seeded permutation of all blocks (plus `spare_blocks` unused ones), so
    the table is scattered as a paged cache's would be."""
    rng = _rng(_KEY_ATTN, seed)
    ctx = np.asarray(list(ctx_lens), dtype=np.int32)
    B = len(ctx)
    per_seq = [(int(n) + block - 1) // block for n in ctx]
    max_blocks = max(per_seq)
    n_blocks = sum(per_seq) + spare_blocks
    phys = rng.permutation(n_blocks).astype(np.int32)
    table = np.full((B, max_blocks), -1, dtype=np.int32)
    pos = 0
    for b, nb in enumerate(per_seq):
        table[b, :nb] = phys[pos:pos + nb]
        pos += nb
    q = to_bf16_bits(rng.normal(0.0, 1.0, size=(B, Hq, D)))
    k = to_bf16_bits(rng.normal(0.0, 1.0, size=(n_blocks, Hkv, block, D)))
    v = to_bf16_bits(rng.normal(0.0, 1.0, size=(n_blocks, Hkv, block, D)))
    return AttnCase(q, k, v, table, ctx)


@dataclasses.dataclass
class AttnDeviceCase:
    """An attention case generated on the device (full-size inputs): torch tensors."""
    q: torch.Tensor             # bf16 [B, Hq, D]
    k_cache: torch.Tensor       # bf16 [n_blocks, Hkv, block, D]
    v_cache: torch.Tensor
    block_table: torch.Tensor   # int32 [B, max_blocks]
    ctx_len: torch.Tensor       # int32 [B]


def make_attention_case_on_device(seed: int, ctx_lens, device, Hq: int = 16, Hkv: int = 2, D: int = 256,
                                  block: int = 64, spare_blocks: int = 3) -> AttnDeviceCase:
    """The recipe of make_attention_case drawn by torch's generator on `device` (a different
    stream of numbers): q, k, v ~ N(0, 1) bf16, one seeded permutation of the physical blocks."""
    g = torch.Generator(device=device)
    g.manual_seed((seed * 3_000_017 + _KEY_ATTN) & 0x7FFFFFFF)
    ctx = [int(n) for n in ctx_lens]
    per_seq = [(n + block - 1) // block for n in ctx]
    n_blocks = sum(per_seq) + spare_blocks
    phys = torch.randperm(n_blocks, generator=g, device=device).to(torch.int32)
    table = torch.full((len(ctx), max(per_seq)), -1, dtype=torch.int32, device=device)
    pos = 0
    for b, nb in enumerate(per_seq):
        table[b, :nb] = phys[pos:pos + nb]
        pos += nb
    q = torch.randn((len(ctx), Hq, D), generator=g, device=device).to(torch.bfloat16)
    k = torch.randn((n_blocks, Hkv, block, D), generator=g, device=device).to(torch.bfloat16)
    v = torch.randn((n_blocks, Hkv, block, D), generator=g, device=device).to(torch.bfloat16)
    return AttnDeviceCase(q, k, v, table, torch.tensor(ctx, dtype=torch.int32, device=device))


def attention_case_to_host(c: AttnDeviceCase) -> AttnCase:
    """The same inputs in the storage form of make_attention_case (bf16 bit patterns)."""
    def bits(t):
        return t.detach().cpu().view(torch.int16).numpy().view(np.uint16).copy()
    return AttnCase(bits(c.q), bits(c.k_cache), bits(c.v_cache), c.block_table.cpu().numpy().copy(),
                    c.ctx_len.cpu().numpy().copy())


# --------------------------------------------------------------------------
# Gated DeltaNet decode step: seeded q, k, v (bf16), per-head log-decay and
# write strength, and an FP32 state (no recurrence arithmetic here).
# --------------------------------------------------------------------------
_KEY_DELTA = 0x474E4554   # stream tag for a recurrence case


@dataclasses.dataclass
class DeltaCase:
    """One recurrence step's inputs in storage form."""
    q: np.ndarray       # uint16 (bf16) [B, H_k, d_k]
    k: np.ndarray       # uint16 (bf16) [B, H_k, d_k]
    v: np.ndarray       # uint16 (bf16) [B, H_v, d_v]
    g: np.ndarray       # float32 [B, H_v]: log-decay, alpha = exp(g)
    beta: np.ndarray    # float32 [B, H_v]
    state: np.ndarray   # float32 [B, H_v, d_v, d_k]


def make_deltanet_case(seed: int, B: int, Hk: int = 16, Hv: int = 32, dk: int = 128, dv: int = 128,
                       step: int = 0) -> DeltaCase:
    """q, k, v ~ N(0, 1) as bf16; alpha ~ U(0.85, 0.999) (g = ln alpha); beta ~ U(0.05, 0.95);
    state ~ N(0, 0.05^2) FP32 (a state after many steps of unit-norm keys).  `step` draws a
    further token's inputs from the same case stream (the state is then ignored)."""
    rng = _rng(_KEY_DELTA, seed * 1000 + step)
    q = to_bf16_bits(rng.normal(0.0, 1.0, size=(B, Hk, dk)))
    k = to_bf16_bits(rng.normal(0.0, 1.0, size=(B, Hk, dk)))
    v = to_bf16_bits(rng.normal(0.0, 1.0, size=(B, Hv, dv)))
    g = np.log(rng.uniform(0.85, 0.999, size=(B, Hv))).astype(np.float32)
    beta = rng.uniform(0.05, 0.95, size=(B, Hv)).astype(np.float32)
    state = rng.normal(0.0, 0.05, size=(B, Hv, dv, dk)).astype(np.float32)
    return DeltaCase(q, k, v, g, beta, state)
