"""CPU oracle for the sparse-MoE layer with 4-bit affine experts (float64).

TEST INFRASTRUCTURE ONLY.  This file is the slow, plain reference that the
CUDA path is checked against.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import it; the library never does, and this
file imports nothing from the library.

What it follows.  The three Lily write-ups are cited by title:
  [TD] "Perplexity's Lily: A Breakthrough Local Inference Engine Tailored
       Exclusively for Apple Silicon" (technologiesdigest.com)
  [AT] "Perplexity Lily: Apple Silicon Local Inference" (atlectica-en)
  [AB] "Perplexity Open Sources Apple Chip Inference Engine Lily" (ababnews)
The layer is the Qwen3.6-35B-A3B MoE block ([TD] "The Model: Qwen3.6-35B-A3B
in Focus"; [AB] paragraph 5): a router scores 256 experts and keeps 8, and one
shared expert sees every token.  Weights are MLX affine 4-bit with one scale
and one bias per group of 64 weights ([TD] "The Model", [AB] paragraph 3).
The pages do not spell out softmax, renormalisation, SwiGLU, the sigmoid
shared-expert gate, the nibble order or tie-breaks; the readings taken here:
  * selection by logit, descending, lower expert index first on equal logits;
  * weights = softmax over the selected logits (= full softmax renormalised
    over the selected experts);
  * expert MLP = SwiGLU, silu(z) = z / (1 + exp(-z)), with the intermediate
    h rounded to bf16 (round to nearest even) before the down projection;
  * shared expert gated by sigmoid(x . w_sg);
  * code i of a packed uint32 word is bits 4i..4i+3 (LSB first);
  * stacked layers feed bf16(y / sqrt(mean(y^2) + 1e-6)) to the next layer.
Everything is evaluated in float64 from the stored bf16 / 4-bit values, so the
result is the layer's exact value up to float64 rounding, except for the one
deliberate bf16 rounding of h.

Parity pins: every function here is pinned by tests under tests/ (hand-worked
dequant words, brute-force full-sort top-k, closed-form zero-input case,
one-hot dense equivalence against torch's float64 SwiGLU, shared-only case,
token-permutation invariance, exact power-of-two scaling, routing-buffer
invariants, direct summation on the tiny layer, bf16 rounding against torch).
"""
from __future__ import annotations

import math

import numpy as np

GROUP = 64          # weights per quantisation group ([TD] "The Model")
CODES_PER_WORD = 8  # 4-bit codes per uint32 ([AB] paragraph 3: MLX affine 4bit)


# ---------------------------------------------------------------- formats --

def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    """Value of bf16 bit patterns (uint16) as float64: the upper half of a float32."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_to_bf16(v: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value, ties to even.

    bf16 keeps 8 significant bits (1 implicit + 7 stored) and float32's
    exponent range; below 2**-126 the spacing is fixed at 2**-133.  The result
    is returned as float64 (exactly representable in bf16).
    """
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    nz = v != 0
    m, e = np.frexp(v[nz])                 # v = m * 2**e, 0.5 <= |m| < 1
    q_exp = np.maximum(e - 8, -133)        # exponent of the last kept bit
    out[nz] = np.ldexp(np.rint(np.ldexp(v[nz], -q_exp)), q_exp)   # rint: ties to even
    return out


def f64_to_bf16_bits(v: np.ndarray) -> np.ndarray:
    """bf16 bit pattern of values that are already exactly bf16 (see round_to_bf16)."""
    f32 = np.asarray(v, dtype=np.float64).astype(np.float32)   # exact for bf16 values
    return (f32.view(np.uint32) >> 16).astype(np.uint16)


def unpack_codes(words: np.ndarray, cols: int) -> np.ndarray:
    """4-bit codes q[.., r, c] from packed words [.., r, cols/8].

    q[r, c] = (P[r, c // 8] >> 4*(c % 8)) & 0xF  (MLX affine 4-bit packing,
    [AB] paragraph 3; LSB-first order is the reading taken).
    """
    words = np.asarray(words, dtype=np.uint32)
    shifts = (4 * np.arange(CODES_PER_WORD, dtype=np.uint32))
    q = (words[..., :, :, None] >> shifts) & np.uint32(0xF)
    return q.reshape(words.shape[:-1] + (cols,)).astype(np.int64)


def dequant(q_words: np.ndarray, scales: np.ndarray, biases: np.ndarray) -> np.ndarray:
    """Dense float64 weights w[.., r, c] = scale[r, c//64] * q[r, c] + bias[r, c//64].

    Groupwise affine 4-bit reconstruction, one scale and one bias per group of
    64 weights along the input dimension ([TD] "The Model"; [AB] paragraph 3).
    Exact in float64 (bf16 scale times a 4-bit integer plus a bf16 bias).
    """
    cols = q_words.shape[-1] * CODES_PER_WORD
    q = unpack_codes(q_words, cols).astype(np.float64)
    s = np.repeat(bf16_to_f64(scales), GROUP, axis=-1)
    b = np.repeat(bf16_to_f64(biases), GROUP, axis=-1)
    return s * q + b


# ---------------------------------------------------------------- routing --

def router_logits(x: np.ndarray, w_router_bits: np.ndarray, router_bias=None) -> np.ndarray:
    """l[t, e] = sum_h x[t, h] * W_r[e, h] (+ b_e): the router's score of every expert.

    [TD] "The Model": a routing component scores all 256 experts per token.
    x is float64 (bf16 values); W_r is stored bf16; b_e (float32) is the
    optional per-expert bias of the skewed workload.
    """
    l = np.asarray(x, dtype=np.float64) @ bf16_to_f64(w_router_bits).T
    if router_bias is not None:
        l = l + np.asarray(router_bias, dtype=np.float32).astype(np.float64)[None, :]
    return l


def select_topk(logits: np.ndarray, k: int) -> np.ndarray:
    """Indices of the k chosen experts per token, in order (logit desc, index asc).

    [TD] "The Model" / [AB] paragraph 5: the router keeps 8 of the 256 experts.
    Softmax is monotone, so choosing on logits equals choosing on
    probabilities; equal logits go to the lower expert index.
    """
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int64)
    order_key = np.arange(E)
    for t in range(T):
        # stable sort on -logit keeps ascending expert index among equal logits
        order = np.argsort(-logits[t], kind="stable")
        idx[t] = order_key[order[:k]]
    return idx


def topk_weights(logits: np.ndarray, idx: np.ndarray) -> np.ndarray:
    """w[t, j] = exp(l[t, idx_j] - l[t, idx_0]) / sum_j' exp(l[t, idx_j'] - l[t, idx_0]).

    Softmax over all experts, then renormalised over the k chosen ones: the
    full-softmax denominator cancels, leaving a softmax over the chosen logits.
    """
    sel = np.take_along_axis(logits, idx, axis=1)
    z = np.exp(sel - sel[:, :1])
    return z / z.sum(axis=1, keepdims=True)


def boundary_gap(logits: np.ndarray, k: int) -> np.ndarray:
    """l_(k) - l_(k+1) per token: distance of the k-th chosen logit from the first unchosen one."""
    s = -np.sort(-logits, axis=1)
    if k >= logits.shape[1]:
        return np.full(logits.shape[0], np.inf)
    return s[:, k - 1] - s[:, k]


def routing_buffers(idx: np.ndarray, E: int):
    """Token-to-expert grouping built from the choices ([TD] "How It Works": histogram,
    prefix scan, scatter).

    counts[e]  = number of (t, j) with idx[t, j] = e;
    offsets    = exclusive prefix sum of counts, E + 1 entries;
    perm[pos]  = t*k + j, grouped by expert e ascending, tokens t ascending
                 inside an expert (a stable counting sort);
    inv_perm[t*k + j] = pos.
    """
    T, k = idx.shape
    counts = np.zeros(E, dtype=np.int64)
    for t in range(T):
        for j in range(k):
            counts[idx[t, j]] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + counts[e]
    perm = np.empty(T * k, dtype=np.int64)
    inv_perm = np.empty(T * k, dtype=np.int64)
    fill = offsets[:E].copy()
    for t in range(T):
        for j in range(k):
            e = idx[t, j]
            pos = fill[e]
            fill[e] += 1
            perm[pos] = t * k + j
            inv_perm[t * k + j] = pos
    return counts, offsets, perm, inv_perm


# ---------------------------------------------------------------- experts --

def silu(z: np.ndarray) -> np.ndarray:
    """silu(z) = z / (1 + exp(-z))."""
    return z / (1.0 + np.exp(-z))


def sigmoid(z: np.ndarray) -> np.ndarray:
    return 1.0 / (1.0 + np.exp(-z))


def swiglu_expert(x_rows: np.ndarray, w_gate: np.ndarray, w_up: np.ndarray, w_down: np.ndarray) -> np.ndarray:
    """One expert's SwiGLU MLP on rows of x, with dense float64 weights.

    g = x W_g^T, u = x W_u^T, h = bf16(silu(g) * u), y = h W_d^T.
    W_g, W_u: [I, H]; W_d: [H, I].  The bf16 rounding of h is the one rounding
    the layer fixes inside an expert.
    """
    g = x_rows @ w_gate.T
    u = x_rows @ w_up.T
    h = round_to_bf16(silu(g) * u)
    return h @ w_down.T


def shared_gate(x: np.ndarray, w_sg_bits: np.ndarray) -> np.ndarray:
    """sigma_t = sigmoid(x_t . w_sg): the always-on shared expert's gate ([TD] "The Model")."""
    return sigmoid(np.asarray(x, dtype=np.float64) @ bf16_to_f64(w_sg_bits))


def _expert_weights(layer, e: int):
    return (dequant(layer.gate.q[e], layer.gate.scales[e], layer.gate.biases[e]),
            dequant(layer.up.q[e], layer.up.scales[e], layer.up.biases[e]),
            dequant(layer.down.q[e], layer.down.scales[e], layer.down.biases[e]))


def _shared_weights(layer):
    return (dequant(layer.sh_gate.q, layer.sh_gate.scales, layer.sh_gate.biases),
            dequant(layer.sh_up.q, layer.sh_up.scales, layer.sh_up.biases),
            dequant(layer.sh_down.q, layer.sh_down.scales, layer.sh_down.biases))


def route(x_bits: np.ndarray, layer, k: int):
    """Routing only: logits, choices, weights, gap, buffers and the shared gate."""
    x = bf16_to_f64(x_bits)
    E = layer.w_router.shape[0]
    logits = router_logits(x, layer.w_router, layer.router_bias)
    idx = select_topk(logits, k)
    w = topk_weights(logits, idx)
    counts, offsets, perm, inv_perm = routing_buffers(idx, E)
    return {
        "logits": logits, "topk_idx": idx, "topk_w": w,
        "gap": boundary_gap(logits, k),
        "counts": counts, "offsets": offsets, "perm": perm, "inv_perm": inv_perm,
        "sigma": shared_gate(x, layer.w_shared_gate),
    }


def moe_layer(x_bits: np.ndarray, layer, k: int, tokens=None, idx_override=None) -> dict:
    """The MoE layer's output for the listed tokens (all tokens by default).

    out_t = sum_j w[t, j] * y_{t, j} + sigma_t * ys_t, summed in float64, where
    y_{t, j} is expert idx[t, j]'s SwiGLU output for x_t and ys_t the shared
    expert's.  Tokens are independent once routing is fixed, so a subset of
    tokens gives exactly those tokens' rows.  `idx_override` (rows of choices
    for some tokens) replaces the oracle's choices where a test has accepted
    another valid choice on a near tie; weights then follow those choices.
    """
    x = bf16_to_f64(x_bits)
    T = x.shape[0]
    r = route(x_bits, layer, k)
    idx, w = r["topk_idx"], r["topk_w"]
    if idx_override is not None:
        idx = idx.copy()
        for t, row in idx_override.items():
            idx[t] = row
        w = topk_weights(r["logits"], idx)
    toks = np.arange(T) if tokens is None else np.asarray(tokens, dtype=np.int64)
    H = x.shape[1]
    out = np.zeros((len(toks), H), dtype=np.float64)
    routed = np.zeros((len(toks), k, H), dtype=np.float64)
    # group the requested (token, slot) pairs by expert so each expert is dequantised once
    by_expert: dict[int, list] = {}
    for ti, t in enumerate(toks):
        for j in range(k):
            by_expert.setdefault(int(idx[t, j]), []).append((ti, j))
    for e in sorted(by_expert):
        wg, wu, wd = _expert_weights(layer, e)
        pairs = by_expert[e]
        rows = np.array([toks[ti] for ti, _ in pairs])
        y = swiglu_expert(x[rows], wg, wu, wd)
        for (ti, j), yrow in zip(pairs, y):
            routed[ti, j] = yrow
    swg, swu, swd = _shared_weights(layer)
    ys = swiglu_expert(x[toks], swg, swu, swd)
    sigma = r["sigma"][toks]
    for ti, t in enumerate(toks):
        acc = np.zeros(H, dtype=np.float64)
        for j in range(k):
            acc += w[t, j] * routed[ti, j]
        out[ti] = acc + sigma[ti] * ys[ti]
    r.update({"out": out, "tokens": toks, "topk_idx": idx, "topk_w": w})
    return r


def rmsnorm_bf16(y: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """Input of the next stacked layer: bf16(y / sqrt(mean(y^2) + eps)), weight 1, no residual."""
    y = np.asarray(y, dtype=np.float64)
    return round_to_bf16(y / np.sqrt(np.mean(y * y, axis=-1, keepdims=True) + eps))


def compare(out_gpu: np.ndarray, ref: np.ndarray) -> dict:
    """Relative L2 error and max-abs error relative to max|ref| (the layer's tolerance metrics)."""
    d = np.asarray(out_gpu, dtype=np.float64) - ref
    nref = float(np.linalg.norm(ref))
    return {
        "rel_l2": float(np.linalg.norm(d)) / nref if nref > 0 else float(np.linalg.norm(d)),
        "max_err_rel": float(np.abs(d).max() / np.abs(ref).max()) if np.abs(ref).max() > 0 else float(np.abs(d).max()),
    }


REL_L2_TOL = 5e-3      # relative L2 error bound on the layer output
MAX_ERR_TOL = 2e-2     # max |err| bound, relative to max |ref|
GAP_MIN = 1e-3         # smallest top-k boundary gap a routing comparison relies on
