"""Pins of the decode-attention oracle (oracle/attn_ref.py) against what the
mathematics fixes, independent of the oracle's own code path."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from bit_quantized_expert_route_b200 import synth
from oracle import attn_ref


def _case(ctx, **kw):
    return synth.make_attention_case(7, ctx, **kw)


def test_single_position_returns_its_value_exactly():
    c = _case([1, 1], D=64)
    o = attn_ref.decode_attention(c.q, c.k_cache, c.v_cache, c.block_table, c.ctx_len)
    for b in range(2):
        blk = c.block_table[b][0]
        for h in range(16):
            np.testing.assert_array_equal(o[b, h], attn_ref.bf16_to_f64(c.v_cache[blk, h // 8, 0]))


def test_equal_keys_give_the_mean_of_the_values():
    c = _case([130], D=64)
    c.k_cache[...] = c.k_cache[0, 0, 0]            # every key the same: uniform weights
    o = attn_ref.decode_attention(c.q, c.k_cache, c.v_cache, c.block_table, c.ctx_len)
    for g in range(2):
        V = attn_ref.gather_kv(c.v_cache, c.block_table, 0, g, 130, 64)
        for h in range(8 * g, 8 * g + 8):
            np.testing.assert_allclose(o[0, h], V.mean(axis=0), rtol=0, atol=1e-12)


def _brute(q_bits, k_cache, v_cache, table, ctx, block):
    """Per position and per element in plain Python: scores, their maximum, weights, sums."""
    B, Hq, D = q_bits.shape
    Hkv = k_cache.shape[1]
    q = attn_ref.bf16_to_f64(q_bits)
    K = attn_ref.bf16_to_f64(k_cache)
    V = attn_ref.bf16_to_f64(v_cache)
    out = np.zeros((B, Hq, D))
    for b in range(B):
        for h in range(Hq):
            g = h // (Hq // Hkv)
            sc = []
            for j in range(int(ctx[b])):
                blk, row = table[b][j // block], j % block
                sc.append(sum(q[b, h, d] * K[blk, g, row, d] for d in range(D)) / D ** 0.5)
            m = max(sc)
            w = [np.exp(v - m) for v in sc]
            tot = sum(w)
            for d in range(D):
                out[b, h, d] = sum(w[j] * V[table[b][j // block], g, j % block, d] for j in range(len(w))) / tot
    return out


def test_matches_brute_force_loops():
    c = synth.make_attention_case(3, [5, 19], Hq=4, Hkv=2, D=8, block=4)
    o = attn_ref.decode_attention(c.q, c.k_cache, c.v_cache, c.block_table, c.ctx_len)
    np.testing.assert_allclose(o, _brute(c.q, c.k_cache, c.v_cache, c.block_table, c.ctx_len, 4), rtol=0, atol=1e-12)


@pytest.mark.parametrize("ctx", [[1], [63, 64, 65], [300]])
def test_matches_torch_sdpa_on_gathered_cache(ctx):
    c = _case(ctx, D=128)
    o = attn_ref.decode_attention(c.q, c.k_cache, c.v_cache, c.block_table, c.ctx_len)
    for b, n in enumerate(ctx):
        K = np.stack([attn_ref.gather_kv(c.k_cache, c.block_table, b, g, n, 64) for g in range(2)])
        V = np.stack([attn_ref.gather_kv(c.v_cache, c.block_table, b, g, n, 64) for g in range(2)])
        q = torch.from_numpy(attn_ref.bf16_to_f64(c.q[b]))[None, :, None, :]          # [1, Hq, 1, D]
        ref = torch.nn.functional.scaled_dot_product_attention(
            q, torch.from_numpy(K)[None], torch.from_numpy(V)[None], enable_gqa=True)
        np.testing.assert_allclose(o[b], ref[0, :, 0].numpy(), rtol=0, atol=1e-12)


def test_physical_block_order_does_not_matter():
    c = _case([200, 77], D=64)
    o = attn_ref.decode_attention(c.q, c.k_cache, c.v_cache, c.block_table, c.ctx_len)
    perm = np.random.default_rng(5).permutation(c.k_cache.shape[0])   # new physical slot of block i
    k2 = np.empty_like(c.k_cache)
    v2 = np.empty_like(c.v_cache)
    k2[perm] = c.k_cache
    v2[perm] = c.v_cache
    t2 = np.where(c.block_table >= 0, perm[np.maximum(c.block_table, 0)], -1)
    np.testing.assert_array_equal(attn_ref.decode_attention(c.q, k2, v2, t2, c.ctx_len), o)


def test_one_kv_head_per_query_head_is_plain_multi_head_attention():
    c = synth.make_attention_case(11, [90], Hq=4, Hkv=4, D=32, block=16)
    o = attn_ref.decode_attention(c.q, c.k_cache, c.v_cache, c.block_table, c.ctx_len)
    for h in range(4):
        K = attn_ref.gather_kv(c.k_cache, c.block_table, 0, h, 90, 16)
        V = attn_ref.gather_kv(c.v_cache, c.block_table, 0, h, 90, 16)
        s = K @ attn_ref.bf16_to_f64(c.q[0, h]) / np.sqrt(32)
        p = np.exp(s - s.max())
        np.testing.assert_allclose(o[0, h], (p / p.sum()) @ V, rtol=0, atol=1e-12)


# Planted slips in the oracle (on the CPU) must each fail a pin above.
def _slipped(kind):
    def decode_attention(q_bits, k_cache, v_cache, block_table, ctx_len, scale=None):
        B, Hq, D = q_bits.shape
        Hkv, block = k_cache.shape[1], k_cache.shape[2]
        grp = Hq // Hkv
        s = (1.0 if kind == "no_scale" else 1.0 / np.sqrt(D))
        q = attn_ref.bf16_to_f64(q_bits)
        out = np.zeros((B, Hq, D))
        for b in range(B):
            n = int(ctx_len[b]) + (1 if kind == "ctx_plus_one" else 0)
            for h in range(Hq):
                g = (h % Hkv) if kind == "group_mod" else h // grp
                K = attn_ref.gather_kv(k_cache, block_table, b, g, n, block)
                V = attn_ref.gather_kv(v_cache if kind != "k_for_v" else k_cache, block_table, b, g, n, block)
                lg = s * (K @ q[b, h])
                w = np.exp(lg - lg.max())
                out[b, h] = (w / w.sum()) @ V
        return out
    return decode_attention


@pytest.mark.parametrize("kind", ["no_scale", "group_mod", "k_for_v", "ctx_plus_one"])
def test_planted_slips_are_caught(kind, monkeypatch):
    """With a slip planted in the oracle, at least one pin above must fail."""
    monkeypatch.setattr(attn_ref, "decode_attention", _slipped(kind))
    pins = [test_single_position_returns_its_value_exactly, test_equal_keys_give_the_mean_of_the_values,
            test_matches_brute_force_loops, lambda: test_matches_torch_sdpa_on_gathered_cache([63, 64, 65]),
            test_physical_block_order_does_not_matter, test_one_kv_head_per_query_head_is_plain_multi_head_attention]
    failed = 0
    for pin in pins:
        try:
            pin()
        except (AssertionError, IndexError, ValueError):
            failed += 1
    assert failed > 0, kind
