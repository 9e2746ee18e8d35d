"""CPU oracle for one decode step of a Gated DeltaNet layer's recurrence (float64).

TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
CUDA recurrence kernel is checked against.  Only the test suite and the
benchmark's CPU-baseline leg may import it; the library never does, and this
file imports nothing from the library.

What it follows.  "Perplexity's Lily: A Breakthrough Local Inference Engine
Tailored Exclusively for Apple Silicon" ([TD]), section "The Model:
Qwen3.6-35B-A3B in Focus": besides its 10 attention layers the model has 30
Gated DeltaNet layers, a recurrence whose state has a fixed size.  The pages
give no formula.  The recurrence is the published gated delta rule (Yang,
Kautz and Hatamizadeh, "Gated Delta Networks: Improving Mamba2 with Delta
Rule", ICLR 2025), for one head with state S (d_v x d_k), read as:

    S_t = S_{t-1} (alpha_t (I - beta_t k_t k_t^T)) + beta_t v_t k_t^T
    o_t = S_t q_t

with k_t and q_t L2-normalised and q_t scaled by 1/sqrt(d_k) (the paper
normalises both; the scale is the usual one), alpha_t = exp(g_t) for a given
log-decay g_t <= 0, and beta_t in (0, 1).  The normalisation uses
x / sqrt(sum x^2 + 1e-6).  Value head hv reads key head hv // (H_v / H_k)
(key heads shared by groups of value heads, as the attention layers share
key/value heads).

`recurrent_step` evaluates the equation as printed: it forms the d_k x d_k
matrix alpha (I - beta k k^T) and multiplies.  Everything is evaluated in
float64 from the stored bf16 inputs and the float32 state.

Parity pins: tests/test_deltanet_oracle.py.
"""
from __future__ import annotations

import numpy as np

NORM_EPS = 1e-6


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Value of bf16 bit patterns (uint16) as float64: the upper half of a float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def l2_normalise(x: np.ndarray) -> np.ndarray:
    """x / sqrt(sum x^2 + 1e-6) along the last axis."""
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + NORM_EPS)


def recurrent_step(q_bits: np.ndarray, k_bits: np.ndarray, v_bits: np.ndarray, g: np.ndarray, beta: np.ndarray,
                   state: np.ndarray):
    """One token of every sequence and value head.

    q_bits, k_bits: uint16 (bf16) [B, H_k, d_k]; v_bits: uint16 [B, H_v, d_v];
    g (log-decay), beta: float [B, H_v]; state: float [B, H_v, d_v, d_k].
    Returns (o [B, H_v, d_v], new state [B, H_v, d_v, d_k]) in float64.
    """
    B, Hk, dk = q_bits.shape
    Hv, dv = v_bits.shape[1], v_bits.shape[2]
    assert Hv % Hk == 0
    grp = Hv // Hk
    q = l2_normalise(bf16_to_f64(q_bits)) / np.sqrt(dk)
    k = l2_normalise(bf16_to_f64(k_bits))
    v = bf16_to_f64(v_bits)
    S = np.asarray(state, dtype=np.float64)
    o = np.zeros((B, Hv, dv))
    S_new = np.zeros_like(S)
    eye = np.eye(dk)
    for b in range(B):
        for hv in range(Hv):
            hk = hv // grp
            kk = k[b, hk]
            alpha = np.exp(float(g[b, hv]))
            bt = float(beta[b, hv])
            transition = alpha * (eye - bt * np.outer(kk, kk))
            S_new[b, hv] = S[b, hv] @ transition + bt * np.outer(v[b, hv], kk)
            o[b, hv] = S_new[b, hv] @ q[b, hk]
    return o, S_new


def compare(got: np.ndarray, ref: np.ndarray) -> dict:
    """Relative L2 error and max-abs error relative to max|ref|."""
    d = np.asarray(got, dtype=np.float64) - ref
    nref = float(np.linalg.norm(ref))
    return {"rel_l2": float(np.linalg.norm(d)) / nref if nref > 0 else float(np.linalg.norm(d)),
            "max_err_rel": float(np.abs(d).max() / np.abs(ref).max()) if np.abs(ref).max() > 0 else
            float(np.abs(d).max())}


# Tolerances.  Output o is bf16 (2^-9 relative rounding) from FP32
# arithmetic; the state stays FP32 (FP32 dot products of 128 terms, a few
# ulps of the row's magnitude after each step).
O_REL_L2_TOL = 5e-3
O_MAX_ERR_TOL = 2e-2
STATE_REL_L2_TOL = 1e-5
