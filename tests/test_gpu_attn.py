"""Decode attention on the GPU (include/attn.h) against the float64 oracle.

Cases span several 32-position chunks, ragged tails, blocks of 32, 64 and
128 rows, D = 128 and 256, GQA groups of 8, 4 and 1, batches whose sequences
have different lengths (so some key/value ranges are empty), one range per
sequence (large batch: the kernel writes the output itself) and many ranges
per sequence (the combine kernel merges them), and the full sizes the
benchmark times (one sequence of 32K and of 128K positions).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from bit_quantized_expert_route_b200 import attn, moe, synth
from oracle import attn_ref
from tests.gpu_util import bits_of, require_cuda, to_dev_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    require_cuda()


def _to_dev(c: synth.AttnCase):
    return (to_dev_bits(c.q), to_dev_bits(c.k_cache), to_dev_bits(c.v_cache),
            torch.from_numpy(c.block_table).cuda(), torch.from_numpy(c.ctx_len).cuda())


def _run(c: synth.AttnCase, scale=0.0):
    q, k, v, table, ctx = _to_dev(c)
    B, Hq, D = c.q.shape
    _, Hkv, block, _ = c.k_cache.shape
    out = torch.empty_like(q)
    ws = attn.alloc_workspace(B, Hkv, D, block, c.block_table.shape[1])
    attn.attn_decode(q, k, v, table, ctx, out, ws, scale=scale)
    torch.cuda.synchronize()
    return bits_of(out), moe.moe_get_status(ws)


def _check(c: synth.AttnCase, got_bits, scale=None):
    live = c.ctx_len > 0
    if live.any():
        ref = attn_ref.decode_attention(c.q[live], c.k_cache, c.v_cache, c.block_table[live], c.ctx_len[live],
                                        scale=scale)
        m = attn_ref.compare(attn_ref.bf16_to_f64(got_bits[live]), ref)
        assert m["rel_l2"] <= attn_ref.REL_L2_TOL and m["max_err_rel"] <= attn_ref.MAX_ERR_TOL, m
    # an empty context gives zeros
    assert np.all(got_bits[~live] == 0)


CASES = [
    # (ctx lens, Hq, Hkv, D, block)
    ([1], 16, 2, 256, 64),
    ([31], 16, 2, 256, 64),
    ([32], 16, 2, 256, 64),
    ([33], 16, 2, 256, 64),
    ([4097], 16, 2, 256, 64),
    ([100, 1, 257, 64], 16, 2, 256, 64),
    ([0, 500, 0, 63], 16, 2, 256, 64),
    ([1000, 77], 8, 2, 128, 32),
    ([333], 4, 4, 128, 128),
    ([700, 5], 16, 4, 256, 128),
    ([2048 + 17], 6, 2, 256, 64),
]


@pytest.mark.parametrize("ctx,Hq,Hkv,D,block", CASES)
def test_matches_oracle(ctx, Hq, Hkv, D, block):
    c = synth.make_attention_case(20 + len(ctx), ctx, Hq=Hq, Hkv=Hkv, D=D, block=block)
    got, status = _run(c)
    assert status == moe.MOE_OK
    _check(c, got)


def test_explicit_scale():
    c = synth.make_attention_case(31, [300, 45], D=128, block=64)
    got, status = _run(c, scale=0.3)
    assert status == moe.MOE_OK
    _check(c, got, scale=0.3)


def test_one_range_per_sequence_large_batch():
    B = 96                                    # 2 B >= the SM count: no split, no combine kernel
    ctx = [(37 * i) % 300 + 1 for i in range(B)]
    c = synth.make_attention_case(41, ctx, D=256, block=64)
    assert attn.plan(B, 2, 64, c.block_table.shape[1])[0] == 1
    got, status = _run(c)
    assert status == moe.MOE_OK
    _check(c, got)


def test_deterministic():
    c = synth.make_attention_case(43, [5000, 300], D=256, block=64)
    a, _ = _run(c)
    b, _ = _run(c)
    np.testing.assert_array_equal(a, b)


def test_never_reads_rows_past_the_context():
    """NaN bit patterns in the unused rows of the last block and in unused blocks change nothing."""
    c = synth.make_attention_case(47, [70, 129], D=256, block=64)
    ref_bits, _ = _run(c)
    nan = np.uint16(0x7FC1)
    for b, n in enumerate(c.ctx_len):
        last = c.block_table[b][(n - 1) // 64]
        c.k_cache[last, :, n % 64 or 64:] = nan
        c.v_cache[last, :, n % 64 or 64:] = nan
    used = set(c.block_table[c.block_table >= 0].tolist())
    for blk in range(c.k_cache.shape[0]):
        if blk not in used:
            c.k_cache[blk] = nan
            c.v_cache[blk] = nan
    got, status = _run(c)
    assert status == moe.MOE_OK
    np.testing.assert_array_equal(got, ref_bits)


def test_bad_block_index_is_reported_and_the_next_call_is_correct():
    c = synth.make_attention_case(53, [300], D=128, block=64)
    q, k, v, table, ctx = _to_dev(c)
    out = torch.empty_like(q)
    ws = attn.alloc_workspace(1, 2, 128, 64, c.block_table.shape[1])
    bad = table.clone()
    bad[0, 2] = c.k_cache.shape[0]            # one past the last block: checked, never loaded
    attn.attn_decode(q, k, v, bad, ctx, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_status(ws) == moe.MOE_ERR_DEVICE_INDEX
    assert moe.moe_get_status(ws) == moe.MOE_OK
    ctx_big = torch.tensor([c.block_table.shape[1] * 64 + 1], dtype=torch.int32, device="cuda")
    attn.attn_decode(q, k, v, table, ctx_big, out, ws)   # context beyond the table: clamped, reported
    torch.cuda.synchronize()
    assert moe.moe_get_status(ws) == moe.MOE_ERR_DEVICE_INDEX
    attn.attn_decode(q, k, v, table, ctx, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_status(ws) == moe.MOE_OK
    _check(c, bits_of(out))


def test_waits_run_out_and_the_next_call_is_correct():
    """Every CTA streams ~56 chunks through its 12-stage ring, so its waits are for copies just
    issued; with a one-cycle limit they give up, the copies in flight are drained, the CTA leaves."""
    c = synth.make_attention_case(59, [65536], D=256, block=64)
    q, k, v, table, ctx = _to_dev(c)
    out = torch.empty_like(q)
    ws = attn.alloc_workspace(1, 2, 256, 64, c.block_table.shape[1])
    moe.moe_set_wait_limit(1)
    try:
        attn.attn_decode(q, k, v, table, ctx, out, ws)
        torch.cuda.synchronize()
    finally:
        moe.moe_set_wait_limit(0)
    assert moe.moe_get_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    attn.attn_decode(q, k, v, table, ctx, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_status(ws) == moe.MOE_OK
    _check(c, bits_of(out))


@pytest.mark.parametrize("L", [32768, 131072])
def test_full_size_one_sequence(L):
    """The benchmark's configuration: 16 query heads, 2 key/value heads, D = 256, blocks of 64."""
    dev = torch.device("cuda")
    case = synth.make_attention_case_on_device(61, [L], dev)
    out = torch.empty_like(case.q)
    ws = attn.alloc_workspace(1, 2, 256, 64, case.block_table.shape[1])
    attn.attn_decode(case.q, case.k_cache, case.v_cache, case.block_table, case.ctx_len, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_status(ws) == moe.MOE_OK
    host = synth.attention_case_to_host(case)
    ref = attn_ref.decode_attention(host.q, host.k_cache, host.v_cache, host.block_table, host.ctx_len)
    m = attn_ref.compare(attn_ref.bf16_to_f64(bits_of(out)), ref)
    assert m["rel_l2"] <= attn_ref.REL_L2_TOL and m["max_err_rel"] <= attn_ref.MAX_ERR_TOL, m
