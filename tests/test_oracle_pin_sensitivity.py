"""The oracle's pins catch plausible mistakes.

Each case below plants one slip in the oracle, on the CPU, by replacing one
function of the oracle module for the duration of the case (pytest's
monkeypatch restores it).  Every pin of tests/test_oracle.py then runs against
the altered oracle, and at least one of them must fail.  A slip that no pin
noticed would mean the oracle is not pinned at that point.  No GPU is used.
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import moe_ref
from tests import test_oracle as pins

SLOW_PIN = "test_direct_summation_tiny_layer"
CHEAP_PINS = sorted(n for n in dir(pins) if n.startswith("test_") and n != SLOW_PIN)


def _failing(names):
    failed = []
    for n in names:
        try:
            getattr(pins, n)()
        except Exception:     # a wrong value or a shape error both expose the slip
            failed.append(n)
    return failed


# ------------------------------------------------------------ planted slips --

def _unpack_msb_first(words, cols):
    words = np.asarray(words, dtype=np.uint32)
    shifts = np.uint32(28) - 4 * np.arange(8, dtype=np.uint32)
    q = (words[..., :, :, None] >> shifts) & np.uint32(0xF)
    return q.reshape(words.shape[:-1] + (cols,)).astype(np.int64)


def _topk_ties_to_higher_index(logits, k):
    T, E = logits.shape
    idx = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        order = (E - 1) - np.argsort(-logits[t, ::-1], kind="stable")
        idx[t] = order[:k]
    return idx


def _weights_over_all_experts(logits, idx):
    sel = np.take_along_axis(logits, idx, axis=1)
    m = logits.max(axis=1, keepdims=True)
    return np.exp(sel - m) / np.exp(logits - m).sum(axis=1, keepdims=True)


def _swiglu_without_h_rounding(x_rows, w_gate, w_up, w_down):
    g = x_rows @ w_gate.T
    u = x_rows @ w_up.T
    return (moe_ref.silu(g) * u) @ w_down.T


def _buffers_tokens_descending(idx, E):
    T, k = idx.shape
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.int64)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int64)
    perm = np.empty(T * k, dtype=np.int64)
    inv_perm = np.empty(T * k, dtype=np.int64)
    fill = offsets[:E].copy()
    for t in reversed(range(T)):
        for j in range(k):
            e = idx[t, j]
            perm[fill[e]] = t * k + j
            inv_perm[t * k + j] = fill[e]
            fill[e] += 1
    return counts, offsets, perm, inv_perm


def _buffers_inclusive_offsets(idx, E):
    counts, offsets, perm, inv_perm = _ORIG["routing_buffers"](idx, E)
    return counts, np.concatenate([offsets[1:], [offsets[-1]]]), perm, inv_perm


def _round_ties_away(v):
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros_like(v)
    nz = v != 0
    m, e = np.frexp(v[nz])
    q_exp = np.maximum(e - 8, -133)
    scaled = np.ldexp(v[nz], -q_exp)
    out[nz] = np.ldexp(np.sign(scaled) * np.floor(np.abs(scaled) + 0.5), q_exp)
    return out


_ORIG = {n: getattr(moe_ref, n) for n in ("unpack_codes", "dequant", "select_topk", "topk_weights", "silu",
                                            "sigmoid", "swiglu_expert", "router_logits", "routing_buffers",
                                            "shared_gate", "rmsnorm_bf16", "round_to_bf16")}

SLIPS = {
    "nibble order MSB first": ("unpack_codes", _unpack_msb_first),
    "dequant drops the bias": ("dequant", lambda q, s, b: _ORIG["dequant"](q, s, np.zeros_like(b))),
    "scale and bias swapped": ("dequant", lambda q, s, b: _ORIG["dequant"](q, b, s)),
    "equal logits go to the higher index": ("select_topk", _topk_ties_to_higher_index),
    "softmax not renormalised over the chosen": ("topk_weights", _weights_over_all_experts),
    "slot weights in reverse order": ("topk_weights", lambda l, i: _ORIG["topk_weights"](l, i)[:, ::-1]),
    "silu replaced by the sigmoid": ("silu", lambda z: 1.0 / (1.0 + np.exp(-z))),
    "silu with the wrong sign": ("silu", lambda z: z / (1.0 + np.exp(z))),
    "sigmoid with the wrong sign": ("sigmoid", lambda z: 1.0 / (1.0 + np.exp(z))),
    "gate and up projections swapped": ("swiglu_expert", lambda x, g, u, d: _ORIG["swiglu_expert"](x, u, g, d)),
    "h not rounded to bf16": ("swiglu_expert", _swiglu_without_h_rounding),
    "router bias dropped": ("router_logits", lambda x, w, b=None: _ORIG["router_logits"](x, w, None)),
    "router bias subtracted": ("router_logits",
                               lambda x, w, b=None: _ORIG["router_logits"](x, w, None if b is None else -np.asarray(b))),
    "tokens descending inside an expert": ("routing_buffers", _buffers_tokens_descending),
    "inclusive instead of exclusive offsets": ("routing_buffers", _buffers_inclusive_offsets),
    "shared gate 1 - sigma": ("shared_gate", lambda x, w: 1.0 - _ORIG["shared_gate"](x, w)),
    "rmsnorm without the square root": ("rmsnorm_bf16",
                                        lambda y, eps=1e-6: _ORIG["round_to_bf16"](
                                            y / (np.mean(np.asarray(y) ** 2, axis=-1, keepdims=True) + eps))),
    "bf16 rounding ties away from zero": ("round_to_bf16", _round_ties_away),
}


@pytest.mark.parametrize("slip", sorted(SLIPS))
def test_planted_slip_fails_a_pin(slip, monkeypatch):
    name, fn = SLIPS[slip]
    monkeypatch.setattr(moe_ref, name, fn)
    failed = _failing(CHEAP_PINS)
    if not failed:
        failed = _failing([SLOW_PIN])
    assert failed, f"no pin noticed the planted slip: {slip}"


def test_unaltered_oracle_passes_every_pin():
    assert _failing(CHEAP_PINS) == []
