"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign or index, a transposed operand, a wrong nibble order, a wrong
tie-break) fails at least one of them.  No GPU is used here.
"""
from __future__ import annotations

import dataclasses
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

from bit_quantized_expert_route_b200 import synth
from oracle import moe_ref
from tests.workloads import TINY, screen_rows, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bits(v):
    """bf16 bits of exactly representable values (test-side, via torch)."""
    return synth.to_bf16_bits(np.asarray(v, dtype=np.float64))


# ----------------------------------------------------------------- formats --

def test_round_to_bf16_matches_torch_rne():
    rng = np.random.default_rng(1)
    f32 = np.concatenate([
        rng.normal(0, 1, 20000).astype(np.float32),
        rng.normal(0, 1e-30, 2000).astype(np.float32),
        (rng.normal(0, 1, 2000) * 1e30).astype(np.float32),
    ])
    # exact ties: lower 16 bits = 0x8000, both parities of the kept bit
    tie = ((rng.integers(0x3F00, 0x4100, 4000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    f32 = np.concatenate([f32, tie, -tie])
    want = torch.from_numpy(f32).to(torch.bfloat16).to(torch.float64).numpy()
    got = moe_ref.round_to_bf16(f32.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_bf16_bits_roundtrip():
    vals = np.array([0.0, 1.0, -2.5, 0.00390625, 3.0e38, -1.0e-38])
    b = bits(vals)
    np.testing.assert_array_equal(moe_ref.f64_to_bf16_bits(moe_ref.bf16_to_f64(b)), b)


def _golden_words():
    rows = []
    with open(os.path.join(GOLDEN, "dequant_words.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            p = line.split()
            rows.append((int(p[0], 16), float(p[1]), float(p[2]), [float(v) for v in p[3:11]]))
    return rows


def test_dequant_golden_words():
    for word, scale, bias, want in _golden_words():
        # one row of 64 columns: the word in slot 0, zeros elsewhere
        q = np.zeros((1, 8), dtype=np.uint32)
        q[0, 0] = word
        w = moe_ref.dequant(q, bits([[scale]]), bits([[bias]]))
        np.testing.assert_array_equal(w[0, :8], np.array(want))
        np.testing.assert_array_equal(w[0, 8:], np.full(56, bias))


def test_dequant_extremes_and_groups():
    rng = np.random.default_rng(2)
    s = bits(rng.uniform(0.002, 0.006, (3, 4)))
    b = bits(rng.normal(0, 0.02, (3, 4)))
    S, B = moe_ref.bf16_to_f64(s), moe_ref.bf16_to_f64(b)
    zeros = np.zeros((3, 32), dtype=np.uint32)
    full = np.full((3, 32), 0xFFFFFFFF, dtype=np.uint32)
    np.testing.assert_array_equal(moe_ref.dequant(zeros, s, b), np.repeat(B, 64, axis=1))       # q=0 -> bias
    np.testing.assert_array_equal(moe_ref.dequant(full, s, b), np.repeat(15 * S + B, 64, axis=1))  # q=15
    const = np.full((3, 32), 0x55555555, dtype=np.uint32)                                      # q=5 everywhere
    w = moe_ref.dequant(const, s, b)
    for g in range(4):
        blk = w[:, 64 * g:64 * (g + 1)]
        assert np.all(blk == blk[:, :1])                                                        # constant per group
        np.testing.assert_array_equal(blk[:, 0], 5 * S[:, g] + B[:, g])


def test_dequant_stacked_matches_per_expert():
    lay = synth.make_layer(3, 0, TINY)
    allw = moe_ref.dequant(lay.down.q, lay.down.scales, lay.down.biases)
    assert allw.shape == (TINY.E, TINY.H, TINY.I)
    for e in (0, 7, TINY.E - 1):
        np.testing.assert_array_equal(allw[e], moe_ref.dequant(lay.down.q[e], lay.down.scales[e], lay.down.biases[e]))


# ----------------------------------------------------------------- routing --

def _brute_force_topk(l, k):
    """Rank of each expert = number of experts that beat it; no sorting used."""
    T, E = l.shape
    idx = np.empty((T, k), dtype=np.int64)
    for t in range(T):
        for e in range(E):
            rank = 0
            for f in range(E):
                if l[t, f] > l[t, e] or (l[t, f] == l[t, e] and f < e):
                    rank += 1
            if rank < k:
                idx[t, rank] = e
    return idx


def test_topk_brute_force_with_ties():
    rng = np.random.default_rng(4)
    l = rng.integers(-3, 4, size=(40, 16)).astype(np.float64)    # many exact ties
    for k in (1, 2, 5, 16):
        np.testing.assert_array_equal(moe_ref.select_topk(l, k), _brute_force_topk(l, k))


def test_topk_brute_force_full_size_rows():
    rng = np.random.default_rng(5)
    l = rng.normal(0, 1, size=(6, 256))
    np.testing.assert_array_equal(moe_ref.select_topk(l, 8), _brute_force_topk(l, 8))


def test_weights_are_renormalised_softmax():
    rng = np.random.default_rng(6)
    l = rng.normal(0, 2, size=(50, 256))
    idx = moe_ref.select_topk(l, 8)
    w = moe_ref.topk_weights(l, idx)
    p = scipy.special.softmax(l, axis=1)
    psel = np.take_along_axis(p, idx, axis=1)
    np.testing.assert_allclose(w, psel / psel.sum(axis=1, keepdims=True), rtol=1e-12, atol=0)
    assert np.all(np.abs(w.sum(axis=1) - 1.0) < 1e-12)
    assert np.all(np.diff(w, axis=1) <= 0)       # slot order is descending weight


def test_boundary_gap():
    l = np.array([[5.0, 1.0, 3.0, 2.9, 0.0]])
    assert moe_ref.boundary_gap(l, 2)[0] == pytest.approx(0.1)
    assert moe_ref.boundary_gap(l, 1)[0] == pytest.approx(2.0)


def test_routing_buffers_invariants():
    rng = np.random.default_rng(7)
    T, k, E = 300, 8, 64
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)])
    counts, offsets, perm, inv_perm = moe_ref.routing_buffers(idx, E)
    assert counts.sum() == T * k and offsets[0] == 0 and offsets[E] == T * k
    np.testing.assert_array_equal(np.bincount(idx.ravel(), minlength=E), counts)
    np.testing.assert_array_equal(np.sort(perm), np.arange(T * k))
    np.testing.assert_array_equal(inv_perm[perm], np.arange(T * k))
    for e in range(E):
        seg = perm[offsets[e]:offsets[e + 1]]
        assert np.all(idx.ravel()[seg] == e)
        assert np.all(np.diff(seg // k) > 0)      # tokens ascending within an expert


def test_zipf_bias_formula_values():
    rng = np.random.default_rng(0)
    b = synth.zipf_router_bias(rng, 256)
    ranks = np.rint(np.exp(-b.astype(np.float64) / 1.8)).astype(int)
    np.testing.assert_array_equal(np.sort(ranks), np.arange(1, 257))
    assert b.max() == 0.0 and b.min() == pytest.approx(-1.8 * math.log(256), rel=1e-6)


# ---------------------------------------------------------------- the layer --

def _dense(qm, e=None):
    if e is None:
        return moe_ref.dequant(qm.q, qm.scales, qm.biases)
    return moe_ref.dequant(qm.q[e], qm.scales[e], qm.biases[e])


def _torch_swiglu(x, wg, wu, wd):
    """Textbook SwiGLU MLP in torch float64: silu(x Wg^T) * (x Wu^T), rounded to bf16, then Wd."""
    X, G, U, D = (torch.from_numpy(a) for a in (x, wg, wu, wd))
    h = torch.nn.functional.silu(X @ G.T) * (X @ U.T)
    h = torch.from_numpy(moe_ref.round_to_bf16(h.numpy()))
    return (h @ D.T).numpy()


def test_zero_input_closed_form():
    lay = synth.make_layer(0, 0, TINY)
    x = np.zeros((5, TINY.H), dtype=np.uint16)
    r = moe_ref.moe_layer(x, lay, TINY.k)
    np.testing.assert_array_equal(r["topk_idx"], np.tile(np.arange(TINY.k), (5, 1)))   # ties -> lowest index
    np.testing.assert_array_equal(r["topk_w"], np.full((5, TINY.k), 1.0 / TINY.k))
    np.testing.assert_array_equal(r["sigma"], np.full(5, 0.5))
    np.testing.assert_array_equal(r["out"], np.zeros((5, TINY.H)))                     # silu(0)*0 = 0


def test_zero_input_with_router_bias_closed_form():
    """x = 0: the logits are the router bias itself, so the choice is the k largest
    bias entries (brute force), the weights their softmax, and the output 0."""
    lay = synth.make_layer(0, 0, TINY, zipf=True)
    bias = np.asarray(lay.router_bias, dtype=np.float32).astype(np.float64)
    x = np.zeros((3, TINY.H), dtype=np.uint16)
    r = moe_ref.moe_layer(x, lay, TINY.k)
    want_idx = _brute_force_topk(bias[None, :], TINY.k)[0]
    np.testing.assert_array_equal(r["topk_idx"], np.tile(want_idx, (3, 1)))
    want_w = scipy.special.softmax(bias[want_idx])
    np.testing.assert_allclose(r["topk_w"], np.tile(want_w, (3, 1)), rtol=1e-13, atol=0)
    np.testing.assert_array_equal(r["out"], np.zeros((3, TINY.H)))


def test_one_hot_routing_equals_dense_mlp():
    d = dataclasses.replace(TINY, k=1)
    lay, x, _ = workload(11, 12, d)
    r = moe_ref.moe_layer(x, lay, 1)
    X = moe_ref.bf16_to_f64(x)
    sig = 1.0 / (1.0 + np.exp(-(X @ moe_ref.bf16_to_f64(lay.w_shared_gate))))
    shared = _torch_swiglu(X, _dense(lay.sh_gate), _dense(lay.sh_up), _dense(lay.sh_down))
    for t in range(12):
        e = int(np.argmax(X[t] @ moe_ref.bf16_to_f64(lay.w_router).T))
        assert r["topk_idx"][t, 0] == e and r["topk_w"][t, 0] == 1.0
        want = _torch_swiglu(X[t:t + 1], _dense(lay.gate, e), _dense(lay.up, e), _dense(lay.down, e))[0]
        np.testing.assert_allclose(r["out"][t], want + sig[t] * shared[t], rtol=1e-11, atol=1e-14)


def test_identical_experts_equal_dense_mlp_any_routing():
    lay, x, _ = workload(12, 10, TINY)
    for name in ("gate", "up", "down"):
        qm = getattr(lay, name)
        for e in range(1, TINY.E):
            qm.q[e], qm.scales[e], qm.biases[e] = qm.q[0], qm.scales[0], qm.biases[0]
    r = moe_ref.moe_layer(x, lay, TINY.k)
    X = moe_ref.bf16_to_f64(x)
    sig = 1.0 / (1.0 + np.exp(-(X @ moe_ref.bf16_to_f64(lay.w_shared_gate))))
    routed = _torch_swiglu(X, _dense(lay.gate, 0), _dense(lay.up, 0), _dense(lay.down, 0))
    shared = _torch_swiglu(X, _dense(lay.sh_gate), _dense(lay.sh_up), _dense(lay.sh_down))
    np.testing.assert_allclose(r["out"], routed + sig[:, None] * shared, rtol=1e-11, atol=1e-14)


def test_shared_expert_only():
    lay, x, _ = workload(13, 9, TINY)
    for name in ("gate", "up", "down"):
        qm = getattr(lay, name)
        qm.scales[:] = 0
        qm.biases[:] = 0
    lay.w_shared_gate[:] = 0
    r = moe_ref.moe_layer(x, lay, TINY.k)
    X = moe_ref.bf16_to_f64(x)
    shared = _torch_swiglu(X, _dense(lay.sh_gate), _dense(lay.sh_up), _dense(lay.sh_down))
    np.testing.assert_array_equal(r["sigma"], np.full(9, 0.5))
    np.testing.assert_allclose(r["out"], 0.5 * shared, rtol=1e-12, atol=0)


def test_token_permutation_invariance():
    lay, x, _ = workload(14, 16, TINY)
    p = np.random.default_rng(0).permutation(16)
    a = moe_ref.moe_layer(x, lay, TINY.k)
    b = moe_ref.moe_layer(x[p], lay, TINY.k)
    np.testing.assert_array_equal(b["out"], a["out"][p])
    np.testing.assert_array_equal(b["counts"], a["counts"])
    np.testing.assert_array_equal(b["topk_idx"], a["topk_idx"][p])


def test_doubling_down_projection_doubles_output_exactly():
    lay, x, _ = workload(15, 8, TINY)
    a = moe_ref.moe_layer(x, lay, TINY.k)["out"]
    for qm in (lay.down, lay.sh_down):
        qm.scales[...] = bits(2 * moe_ref.bf16_to_f64(qm.scales))
        qm.biases[...] = bits(2 * moe_ref.bf16_to_f64(qm.biases))
    b = moe_ref.moe_layer(x, lay, TINY.k)["out"]
    np.testing.assert_array_equal(b, 2 * a)


def test_token_subset_equals_full_rows():
    lay, x, _ = workload(16, 16, TINY)
    full = moe_ref.moe_layer(x, lay, TINY.k)["out"]
    sub = moe_ref.moe_layer(x, lay, TINY.k, tokens=[3, 0, 15])["out"]
    np.testing.assert_array_equal(sub, full[[3, 0, 15]])


def test_direct_summation_tiny_layer():
    """Explicit loops over t, e, h with no BLAS, on a few tokens of the tiny layer."""
    d = TINY
    lay, x, _ = workload(0, 16, d)
    toks = [0, 5, 11]
    r = moe_ref.moe_layer(x, lay, d.k, tokens=toks)
    X = [[float(v) for v in row] for row in moe_ref.bf16_to_f64(x)]

    def deq(qm, e, row, col):
        q = qm.q if e is None else qm.q[e]
        s = qm.scales if e is None else qm.scales[e]
        b = qm.biases if e is None else qm.biases[e]
        word = int(q[row, col // 8])
        code = (word >> (4 * (col % 8))) & 0xF
        sv = float(moe_ref.bf16_to_f64(s[row, col // 64]))
        bv = float(moe_ref.bf16_to_f64(b[row, col // 64]))
        return sv * code + bv

    def mlp(xrow, e, gq, uq, dq, inter):
        hv = []
        for i in range(inter):
            g = sum(xrow[c] * deq(gq, e, i, c) for c in range(d.H))
            u = sum(xrow[c] * deq(uq, e, i, c) for c in range(d.H))
            hv.append(float(moe_ref.round_to_bf16(np.array([g / (1 + math.exp(-g)) * u]))[0]))
        return [sum(hv[i] * deq(dq, e, o, i) for i in range(inter)) for o in range(d.H)]

    Wr = moe_ref.bf16_to_f64(lay.w_router)
    wsg = moe_ref.bf16_to_f64(lay.w_shared_gate)
    for ti, t in enumerate(toks):
        logits = [sum(X[t][c] * Wr[e, c] for c in range(d.H)) for e in range(d.E)]
        order = sorted(range(d.E), key=lambda e: (-logits[e], e))[:d.k]
        assert list(r["topk_idx"][t]) == order
        z = [math.exp(logits[e] - logits[order[0]]) for e in order]
        wts = [v / sum(z) for v in z]
        out = [0.0] * d.H
        for j, e in enumerate(order):
            y = mlp(X[t], e, lay.gate, lay.up, lay.down, d.I)
            out = [o + wts[j] * yv for o, yv in zip(out, y)]
        sg = 1 / (1 + math.exp(-sum(X[t][c] * wsg[c] for c in range(d.H))))
        ys = mlp(X[t], None, lay.sh_gate, lay.sh_up, lay.sh_down, d.I_s)
        out = [o + sg * yv for o, yv in zip(out, ys)]
        np.testing.assert_allclose(r["out"][ti], np.array(out), rtol=1e-12, atol=1e-15)


def test_rmsnorm_against_torch_and_closed_form():
    rng = np.random.default_rng(8)
    y = rng.normal(0, 3, size=(7, 256))
    want = torch.nn.functional.rms_norm(torch.from_numpy(y), (256,), eps=1e-6).numpy()
    np.testing.assert_allclose(moe_ref.rmsnorm_bf16(y), moe_ref.round_to_bf16(want), rtol=0, atol=0)
    c = np.full((1, 256), -2.0)
    assert np.all(moe_ref.rmsnorm_bf16(c) == -1.0)            # -2/sqrt(4+1e-6) rounds to -1 in bf16


def test_screen_clears_gap():
    lay, x, red = workload(0, 64, TINY)
    logits = moe_ref.router_logits(moe_ref.bf16_to_f64(x), lay.w_router, lay.router_bias)
    assert moe_ref.boundary_gap(logits, TINY.k).min() >= moe_ref.GAP_MIN


def test_compare_metric():
    ref = np.array([[1.0, -2.0], [0.5, 0.0]])
    m = moe_ref.compare(ref + np.array([[0.0, 0.02], [0.0, 0.0]]), ref)
    assert m["max_err_rel"] == pytest.approx(0.01)
    assert m["rel_l2"] == pytest.approx(0.02 / math.sqrt(1 + 4 + 0.25))
