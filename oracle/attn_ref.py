"""CPU oracle for grouped-query decode attention over a fixed-block KV cache (float64).

TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
CUDA attention kernel is checked against.  Only the test suite and the
benchmark's CPU-baseline leg may import it; the library never does, and this
file imports nothing from the library.

What it follows.  "Perplexity's Lily: A Breakthrough Local Inference Engine
Tailored Exclusively for Apple Silicon" ([TD]), section "The Model:
Qwen3.6-35B-A3B in Focus": the model's full-attention layers use grouped-query
attention with 16 query heads and two key/value heads; section "How It Works:
Prefill and Decode Strategies": decode attention packs the query heads that
share a key/value head (GQA packing) and stores the key/value cache in fixed
blocks.  The pages give no formula; this is the plain definition of one
decode step of softmax attention, read as:
  * query head h uses key/value head h // (Hq / Hkv) (grouped-query attention);
  * o_h = sum_j softmax_j(scale * q_h . k_j) v_j over the sequence's first
    ctx_len cached positions j, scale = 1 / sqrt(D) (the textbook scaling;
    the pages fix none);
  * position j of sequence b lives in physical block block_table[b][j // bs]
    at row j % bs, with the cache laid out [block][kv head][row][D] (a
    block of one head is contiguous).
Everything is evaluated in float64 from the stored bf16 values.

Parity pins: tests/test_attn_oracle.py (single position gives v exactly,
equal keys give the mean of the values, a brute-force per-position loop,
torch's float64 scaled_dot_product_attention on the gathered keys and values,
physical-block permutation invariance, shift invariance of the scores).
"""
from __future__ import annotations

import numpy as np


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Value of bf16 bit patterns (uint16) as float64: the upper half of a float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def gather_kv(cache: np.ndarray, block_table: np.ndarray, b: int, g: int, n: int, block: int) -> np.ndarray:
    """The first n cached rows of kv head g of sequence b, in position order: [n, D] float64."""
    rows = []
    for j in range(n):
        blk = int(block_table[b][j // block])
        rows.append(bf16_to_f64(cache[blk, g, j % block]))
    return np.stack(rows) if rows else np.zeros((0, cache.shape[-1]))


def decode_attention(q_bits: np.ndarray, k_cache: np.ndarray, v_cache: np.ndarray, block_table: np.ndarray,
                     ctx_len: np.ndarray, scale: float | None = None) -> np.ndarray:
    """One decode step of grouped-query attention; returns o [B, Hq, D] in float64.

    q_bits: uint16 (bf16) [B, Hq, D]; k_cache, v_cache: uint16 [n_blocks, Hkv, block, D];
    block_table: int [B, max_blocks]; ctx_len: int [B] (>= 1).
    """
    B, Hq, D = q_bits.shape
    Hkv, block = k_cache.shape[1], k_cache.shape[2]
    assert Hq % Hkv == 0
    grp = Hq // Hkv
    s = 1.0 / np.sqrt(D) if scale is None else float(scale)
    q = bf16_to_f64(q_bits)
    out = np.zeros((B, Hq, D), dtype=np.float64)
    for b in range(B):
        n = int(ctx_len[b])
        for g in range(Hkv):
            K = gather_kv(k_cache, block_table, b, g, n, block)
            V = gather_kv(v_cache, block_table, b, g, n, block)
            for h in range(g * grp, (g + 1) * grp):
                logits = s * (K @ q[b, h])
                w = np.exp(logits - logits.max())
                out[b, h] = (w / w.sum()) @ V
    return out


def compare(out_gpu: np.ndarray, ref: np.ndarray) -> dict:
    """Relative L2 error and max-abs error relative to max|ref|."""
    d = np.asarray(out_gpu, dtype=np.float64) - ref
    nref = float(np.linalg.norm(ref))
    return {"rel_l2": float(np.linalg.norm(d)) / nref if nref > 0 else float(np.linalg.norm(d)),
            "max_err_rel": float(np.abs(d).max() / np.abs(ref).max()) if np.abs(ref).max() > 0 else float(np.abs(d).max())}


# Tolerance: bf16 output (2^-9 relative rounding), bf16 probabilities in the
# P.V product and FP32 accumulation; the same bounds as the MoE layer.
REL_L2_TOL = 5e-3
MAX_ERR_TOL = 2e-2
