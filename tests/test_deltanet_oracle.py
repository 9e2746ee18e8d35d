"""Pins of the Gated DeltaNet recurrence oracle (oracle/deltanet_ref.py) against
what the delta rule and linear algebra fix, independent of the oracle's own
matrix-product evaluation."""
from __future__ import annotations

import numpy as np
import pytest

from bit_quantized_expert_route_b200 import synth
from oracle import deltanet_ref as dr


def _case(B=2, Hk=2, Hv=4, dk=16, dv=8, seed=3):
    return synth.make_deltanet_case(seed, B, Hk=Hk, Hv=Hv, dk=dk, dv=dv)


def _unit(x):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + 1e-6)


def test_no_decay_no_write_keeps_the_state():
    c = _case()
    g = np.zeros_like(c.g)
    beta = np.zeros_like(c.beta)
    o, S = dr.recurrent_step(c.q, c.k, c.v, g, beta, c.state)
    np.testing.assert_array_equal(S, c.state.astype(np.float64))
    q = _unit(dr.bf16_to_f64(c.q)) / np.sqrt(16)
    for b in range(2):
        for hv in range(4):
            np.testing.assert_allclose(o[b, hv], c.state[b, hv].astype(np.float64) @ q[b, hv // 2], rtol=1e-13,
                                       atol=1e-15)


def test_full_write_stores_the_value_under_its_key():
    """Delta rule: with alpha = beta = 1 the new state maps the (unit) key to the value."""
    c = _case()
    o, S = dr.recurrent_step(c.q, c.k, c.v, np.zeros_like(c.g), np.ones_like(c.beta), c.state)
    k = _unit(dr.bf16_to_f64(c.k))
    v = dr.bf16_to_f64(c.v)
    for b in range(2):
        for hv in range(4):
            np.testing.assert_allclose(S[b, hv] @ k[b, hv // 2], v[b, hv], rtol=0, atol=1e-6)


def test_full_decay_leaves_only_the_new_outer_product():
    c = _case()
    g = np.full_like(c.g, -60.0)      # alpha = e^-60
    o, S = dr.recurrent_step(c.q, c.k, c.v, g, c.beta, c.state)
    k = _unit(dr.bf16_to_f64(c.k))
    q = _unit(dr.bf16_to_f64(c.q)) / np.sqrt(16)
    v = dr.bf16_to_f64(c.v)
    for b in range(2):
        for hv in range(4):
            bt = float(c.beta[b, hv])
            np.testing.assert_allclose(S[b, hv], bt * np.outer(v[b, hv], k[b, hv // 2]), rtol=0, atol=1e-20)
            np.testing.assert_allclose(o[b, hv], bt * v[b, hv] * (k[b, hv // 2] @ q[b, hv // 2]), rtol=1e-12,
                                       atol=1e-20)


def test_row_form():
    """Expanded: S' = a S + u k^T with u = beta (v - a S k); o = a (S q) + u (k . q)."""
    c = _case(B=3, Hk=2, Hv=6, dk=32, dv=16)
    o, S = dr.recurrent_step(c.q, c.k, c.v, c.g, c.beta, c.state)
    k = _unit(dr.bf16_to_f64(c.k))
    q = _unit(dr.bf16_to_f64(c.q)) / np.sqrt(32)
    v = dr.bf16_to_f64(c.v)
    for b in range(3):
        for hv in range(6):
            a, bt = np.exp(float(c.g[b, hv])), float(c.beta[b, hv])
            S0 = c.state[b, hv].astype(np.float64)
            kk, qq = k[b, hv // 3], q[b, hv // 3]
            u = bt * (v[b, hv] - a * (S0 @ kk))
            np.testing.assert_allclose(S[b, hv], a * S0 + np.outer(u, kk), rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(o[b, hv], a * (S0 @ qq) + u * (kk @ qq), rtol=1e-11, atol=1e-13)


def _brute(q_bits, k_bits, v_bits, g, beta, state):
    """Element by element in plain Python loops."""
    B, Hk, dk = q_bits.shape
    Hv, dv = v_bits.shape[1], v_bits.shape[2]
    q0, k0, v = dr.bf16_to_f64(q_bits), dr.bf16_to_f64(k_bits), dr.bf16_to_f64(v_bits)
    o = np.zeros((B, Hv, dv))
    S_out = np.zeros((B, Hv, dv, dk))
    for b in range(B):
        for hv in range(Hv):
            hk = hv * Hk // Hv
            nk = sum(x * x for x in k0[b, hk]) + 1e-6
            nq = sum(x * x for x in q0[b, hk]) + 1e-6
            kk = [x / nk ** 0.5 for x in k0[b, hk]]
            qq = [x / nq ** 0.5 / dk ** 0.5 for x in q0[b, hk]]
            a, bt = float(np.exp(np.float64(g[b, hv]))), float(beta[b, hv])
            for i in range(dv):
                s = [float(x) for x in state[b, hv, i]]
                sk = sum(s[j] * kk[j] for j in range(dk))
                for j in range(dk):
                    # row i of S (alpha (I - beta k k^T)) + beta v_i k^T
                    S_out[b, hv, i, j] = a * (s[j] - bt * sk * kk[j]) + bt * v[b, hv, i] * kk[j]
                o[b, hv, i] = sum(S_out[b, hv, i, j] * qq[j] for j in range(dk))
    return o, S_out


def test_matches_brute_force_loops():
    c = _case(B=2, Hk=1, Hv=2, dk=4, dv=3, seed=9)
    o, S = dr.recurrent_step(c.q, c.k, c.v, c.g, c.beta, c.state)
    ob, Sb = _brute(c.q, c.k, c.v, c.g, c.beta, c.state)
    np.testing.assert_allclose(S, Sb, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(o, ob, rtol=1e-12, atol=1e-15)


def test_key_scale_does_not_matter():
    c = _case()
    o, S = dr.recurrent_step(c.q, c.k, c.v, c.g, c.beta, c.state)
    k2 = synth.to_bf16_bits(4.0 * dr.bf16_to_f64(c.k))     # exact in bf16: a power of two
    q2 = synth.to_bf16_bits(0.5 * dr.bf16_to_f64(c.q))
    o2, S2 = dr.recurrent_step(q2, k2, c.v, c.g, c.beta, c.state)
    np.testing.assert_allclose(S2, S, rtol=0, atol=1e-7)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-7)


def test_shared_key_heads_equal_duplicated_key_heads():
    c = _case(B=1, Hk=2, Hv=4)
    o, S = dr.recurrent_step(c.q, c.k, c.v, c.g, c.beta, c.state)
    qd, kd = np.repeat(c.q, 2, axis=1), np.repeat(c.k, 2, axis=1)      # one key head per value head
    od, Sd = dr.recurrent_step(qd, kd, c.v, c.g, c.beta, c.state)
    np.testing.assert_array_equal(o, od)
    np.testing.assert_array_equal(S, Sd)


# Planted slips in the oracle (on the CPU) must each fail a pin above.
def _slipped(kind):
    def recurrent_step(q_bits, k_bits, v_bits, g, beta, state):
        B, Hk, dk = q_bits.shape
        Hv, dv = v_bits.shape[1], v_bits.shape[2]
        grp = Hv // Hk
        q = dr.bf16_to_f64(q_bits) if kind == "no_norm" else dr.l2_normalise(dr.bf16_to_f64(q_bits))
        q = q if kind == "no_scale" else q / np.sqrt(dk)
        k = dr.bf16_to_f64(k_bits) if kind == "no_norm" else dr.l2_normalise(dr.bf16_to_f64(k_bits))
        v = dr.bf16_to_f64(v_bits)
        S = np.asarray(state, dtype=np.float64)
        o = np.zeros((B, Hv, dv))
        S_new = np.zeros_like(S)
        for b in range(B):
            for hv in range(Hv):
                hk = hv % Hk if kind == "group_mod" else hv // grp
                kk = k[b, hk]
                alpha, bt = np.exp(float(g[b, hv])), float(beta[b, hv])
                if kind == "decay_after":
                    S_new[b, hv] = alpha * (S[b, hv] @ (np.eye(dk) - bt * np.outer(kk, kk)) + bt * np.outer(v[b, hv], kk))
                elif kind == "no_beta_erase":
                    S_new[b, hv] = S[b, hv] @ (alpha * (np.eye(dk) - np.outer(kk, kk))) + bt * np.outer(v[b, hv], kk)
                elif kind == "transposed":
                    S_new[b, hv] = (alpha * (np.eye(dk) - bt * np.outer(kk, kk)))[:dv, :dv] @ S[b, hv] + \
                        bt * np.outer(v[b, hv], kk)
                else:
                    S_new[b, hv] = S[b, hv] @ (alpha * (np.eye(dk) - bt * np.outer(kk, kk))) + \
                        bt * np.outer(v[b, hv], kk)
                o[b, hv] = (S[b, hv] if kind == "old_state_out" else S_new[b, hv]) @ q[b, hk]
        return o, S_new
    return recurrent_step


@pytest.mark.parametrize("kind", ["no_norm", "no_scale", "group_mod", "decay_after", "no_beta_erase", "transposed",
                                  "old_state_out"])
def test_planted_slips_are_caught(kind, monkeypatch):
    monkeypatch.setattr(dr, "recurrent_step", _slipped(kind))
    pins = [test_no_decay_no_write_keeps_the_state, test_full_write_stores_the_value_under_its_key,
            test_full_decay_leaves_only_the_new_outer_product, test_row_form, test_matches_brute_force_loops,
            test_key_scale_does_not_matter, test_shared_key_heads_equal_duplicated_key_heads]
    failed = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed > 0, kind
