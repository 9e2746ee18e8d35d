"""GPU path vs the CPU oracle, through the C ABI.

Routing (indices, histogram, offsets, permutation) must be bit-exact on
screened inputs; the layer output must be within relative L2 5e-3 and
max |err| 2e-2 * max |ref| of the float64 oracle.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import pytest
import torch

from bit_quantized_expert_route_b200 import moe, synth
from oracle import moe_ref
from tests.gpu_util import assert_output_close, assert_routing_exact, bits_of, require_cuda, run_layer, to_dev_bits
from tests.workloads import FULL, TINY, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    require_cuda()


# ------------------------------------------------------------- tiny layer --

@pytest.mark.parametrize("T", [1, 3, 16, 17, 64, 65, 200, 700])
@pytest.mark.parametrize("zipf", [False, True])
def test_tiny_layer_all_tokens(T, zipf):
    lay, x, _ = workload(0 if not zipf else 1, T, TINY, zipf=zipf)
    ref = moe_ref.moe_layer(x, lay, TINY.k)
    gpu = run_layer(lay, x)
    assert gpu["status"] == 0
    assert_routing_exact(gpu, ref)
    assert_output_close(gpu["out"], ref["out"])


@pytest.mark.parametrize("T", [5, 300])
def test_route_only(T):
    lay, x, _ = workload(2, T, TINY)
    ref = moe_ref.route(x, lay, TINY.k)
    gpu = run_layer(lay, x, entry="route")
    assert_routing_exact(gpu, ref)


# One layer per expert split of the tensor-core router: clusters of 1, 2 or 4
# CTAs, each CTA owning a block of 16..128 experts (the last block ragged when
# E is not a multiple of it), lists of 1, 2, 4 or 8 candidates for k.
@pytest.mark.parametrize("E,k,zipf", [(64, 4, False), (160, 6, True), (200, 3, False), (250, 1, True),
                                      (256, 7, False), (256, 8, True)])
def test_route_expert_splits(E, k, zipf):
    dims = dataclasses.replace(TINY, E=E, k=k)
    lay, x, _ = workload(40 + E + k, 300, dims, zipf=zipf)
    ref = moe_ref.route(x, lay, k)
    gpu = run_layer(lay, x, entry="route")
    assert gpu["status"] == 0
    assert_routing_exact(gpu, ref)


# Degenerate layers: every token chooses every expert (E = k = 8), and a
# single expert (E = k = 1); both on the decode path (T <= 64) and prefill.
@pytest.mark.parametrize("E,k,T", [(8, 8, 5), (8, 8, 300), (1, 1, 3), (1, 1, 130)])
def test_degenerate_expert_counts(E, k, T):
    dims = dataclasses.replace(TINY, E=E, k=k)
    lay, x, _ = workload(60 + E + T, T, dims)
    ref = moe_ref.moe_layer(x, lay, k)
    gpu = run_layer(lay, x)
    assert gpu["status"] == 0
    assert_routing_exact(gpu, ref)
    assert_output_close(gpu["out"], ref["out"])


# Expert groups at the edges of the expert GEMMs' chunks of at most 160 rows:
# with E = k = 8 every expert, and the shared expert, receives exactly T rows
# (one full chunk, one full chunk plus a 1-row chunk, two full chunks, ...).
@pytest.mark.parametrize("T", [159, 160, 161, 320, 321])
def test_gemm_chunk_boundaries(T):
    dims = dataclasses.replace(TINY, E=8, k=8)
    lay, x, _ = workload(80 + T, T, dims)
    ref = moe_ref.moe_layer(x, lay, 8)
    gpu = run_layer(lay, x)
    assert gpu["status"] == 0
    assert_routing_exact(gpu, ref)
    assert_output_close(gpu["out"], ref["out"])


# Token counts at the edges of the router's 128-token tiles (one cluster each).
@pytest.mark.parametrize("T", [127, 128, 129, 256])
def test_router_tile_boundaries(T):
    lay, x, _ = workload(70 + T, T, TINY)
    ref = moe_ref.moe_layer(x, lay, TINY.k)
    gpu = run_layer(lay, x)
    assert gpu["status"] == 0
    assert_routing_exact(gpu, ref)
    assert_output_close(gpu["out"], ref["out"])


@pytest.mark.parametrize("T", [4, 100])
def test_zero_input_gives_exact_zero(T):
    lay = synth.make_layer(0, 0, TINY)
    x = np.zeros((T, TINY.H), dtype=np.uint16)
    gpu = run_layer(lay, x)
    np.testing.assert_array_equal(gpu["topk_idx"], np.tile(np.arange(TINY.k), (T, 1)))
    np.testing.assert_array_equal(gpu["topk_w"], np.full((T, TINY.k), 1.0 / TINY.k))
    assert np.all(moe_ref.bf16_to_f64(gpu["out"]) == 0.0)


@pytest.mark.parametrize("T", [7, 300])
def test_token_permutation(T):
    lay, x, _ = workload(3, T, TINY)
    p = np.random.default_rng(1).permutation(T)
    a = run_layer(lay, x)
    b = run_layer(lay, x[p])
    np.testing.assert_array_equal(b["counts"], a["counts"])
    np.testing.assert_array_equal(b["topk_idx"], a["topk_idx"][p])
    np.testing.assert_array_equal(b["out"], a["out"][p])        # rows are computed independently


@pytest.mark.parametrize("T", [6, 250])
def test_doubling_down_projection_doubles_output(T):
    lay, x, _ = workload(4, T, TINY)
    a = run_layer(lay, x)
    for qm in (lay.down, lay.sh_down):
        qm.scales[...] = synth.to_bf16_bits(2 * moe_ref.bf16_to_f64(qm.scales))
        qm.biases[...] = synth.to_bf16_bits(2 * moe_ref.bf16_to_f64(qm.biases))
    b = run_layer(lay, x)
    np.testing.assert_array_equal(moe_ref.bf16_to_f64(b["out"]), 2 * moe_ref.bf16_to_f64(a["out"]))


@pytest.mark.parametrize("T", [8, 129])
def test_run_to_run_bitwise(T):
    lay, x, _ = workload(5, T, TINY)
    a = run_layer(lay, x)
    b = run_layer(lay, x)
    for key in ("out", "topk_idx", "perm", "inv_perm", "counts"):
        np.testing.assert_array_equal(a[key], b[key])
    np.testing.assert_array_equal(a["topk_w"], b["topk_w"])


@pytest.mark.parametrize("T", [8, 333])
def test_forward_host_equals_device(T):
    lay, x, _ = workload(6, T, TINY)
    L = moe.MoELayer.from_synth(lay)
    dev = run_layer(lay, x, dev_layer=L)
    ws = moe.alloc_workspace(L, T)
    xh = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
    oh = torch.empty_like(xh).pin_memory()
    moe.moe_forward_host(L, xh, oh, ws)
    np.testing.assert_array_equal(oh.view(torch.int16).numpy().view(np.uint16), dev["out"])


@pytest.mark.parametrize("T", [5, 200])
def test_forward_host_async_two_streams(T):
    # alternating streams and workspaces, as a streaming caller would do
    lay, x_bits, _ = workload(60 + T, T, TINY)
    L = moe.MoELayer.from_synth(lay)
    x = to_dev_bits(x_bits)
    ref = torch.empty_like(x)
    moe.moe_forward(L, x, ref, moe.alloc_workspace(L, T))
    xh = x.cpu().pin_memory()
    outs = [torch.empty_like(xh).pin_memory() for _ in range(2)]
    wss = [moe.alloc_workspace(L, T) for _ in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for i in range(4):
        moe.moe_forward_host_async(L, xh, outs[i % 2], wss[i % 2], stream=streams[i % 2])
    torch.cuda.synchronize()
    for o in outs:
        np.testing.assert_array_equal(o.view(torch.int16).numpy(), bits_of(ref).view(np.int16))


def test_decode_entry_rejects_large_T():
    lay, x, _ = workload(7, 65, TINY)
    with pytest.raises(moe.MoEError) as e:
        run_layer(lay, x, entry="decode")
    assert e.value.code == moe.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("dims,T", [(TINY, 40), (FULL, 12)])
def test_decode_entry_and_forward_both_match_oracle(dims, T):
    # both entries run the mid-size decode path (mma.sync GEMVs over the active experts) at these T
    lay, x, _ = workload(8, T, dims)
    L = moe.MoELayer.from_synth(lay)
    ref = moe_ref.moe_layer(x, lay, dims.k)
    for entry in ("decode", "forward"):
        gpu = run_layer(lay, x, entry=entry, dev_layer=L)
        assert gpu["status"] == 0
        assert_routing_exact(gpu, ref)
        assert_output_close(gpu["out"], ref["out"])


# A second geometry for the mid-size decode path (H, I, I_shared multiples of
# 256): 8 groups per gate/up row and 4 per down row, and with 16 experts of
# which 4 are chosen every expert sees 16+ tokens at T >= 64 (several 8-token
# tiles per expert, the last one ragged).
MID = dataclasses.replace(TINY, H=512, E=16, k=4, I=256, I_s=256)


@pytest.mark.parametrize("T,zipf", [(9, False), (40, True), (64, False), (64, True)])
def test_mid_size_path_second_geometry(T, zipf):
    lay, x, _ = workload(70 + T, T, MID, zipf=zipf)
    ref = moe_ref.moe_layer(x, lay, MID.k)
    L = moe.MoELayer.from_synth(lay)
    assert len(moe.moe_forward_profiled(L, to_dev_bits(x), torch.empty((T, MID.H), dtype=torch.bfloat16,
                                                                         device="cuda"),
                                        moe.alloc_workspace(L, T))) == len(moe.MID_DECODE_STAGES)
    if T == 64:
        assert int(np.max(ref["counts"])) > 8
    for entry in ("forward", "decode"):
        gpu = run_layer(lay, x, entry=entry, dev_layer=L)
        assert gpu["status"] == 0
        assert_routing_exact(gpu, ref)
        assert_output_close(gpu["out"], ref["out"])


# The widest layer the ABI takes (H = 8192: a 131 KB staged token tile, one
# CTA per SM on the mid-size path) with I != I_shared and 2 groups per down
# row (pipeline blocks of 2); T = 65 runs the tensor-core path on it.
WIDE = dataclasses.replace(TINY, H=8192, E=16, k=4, I=128, I_s=256)


@pytest.mark.parametrize("T", [7, 64, 65])
def test_widest_layer(T):
    lay, x, _ = workload(90 + T, T, WIDE)
    ref = moe_ref.moe_layer(x, lay, WIDE.k)
    gpu = run_layer(lay, x)
    assert gpu["status"] == 0
    # the logits are FP32 sums of 8192 products, 4x the default's length: the
    # weight tolerance scales with H (worst-case linear growth), times 2
    assert_routing_exact(gpu, ref, w_atol=2e-6 * (WIDE.H / 2048) * 2)
    assert_output_close(gpu["out"], ref["out"])


def test_rmsnorm_matches_oracle():
    rng = np.random.default_rng(9)
    y_bits = synth.to_bf16_bits(rng.normal(0, 0.05, size=(37, 2048)))
    y = to_dev_bits(y_bits)
    out = torch.empty_like(y)
    moe.moe_rmsnorm(y, out, 1e-6)
    got = moe_ref.bf16_to_f64(bits_of(out))
    want = moe_ref.rmsnorm_bf16(moe_ref.bf16_to_f64(y_bits))
    diff = got != want
    # FP32 reciprocal square root vs float64 division: at most one bf16 step apart, rarely
    ulp = np.abs(want) * 2.0 ** -7
    assert np.all(np.abs(got - want) <= ulp + 1e-30)
    assert diff.mean() < 1e-3
    moe.moe_rmsnorm(y, y, 1e-6)            # in place
    np.testing.assert_array_equal(bits_of(y), bits_of(out))


# ------------------------------------------------------------- full layer --

@pytest.mark.parametrize("T,entry", [(1, "forward"), (2, "forward"), (3, "forward"), (5, "forward"),
                                     (8, "forward"), (9, "forward"), (16, "forward"), (33, "forward"),
                                     (64, "forward"), (65, "forward"), (128, "forward"), (3, "decode"),
                                     (8, "decode"), (9, "decode"), (64, "decode")])
def test_full_decode(T, entry):
    # T <= 3 runs the single-launch fused decode kernel (both entries); 4 <= T
    # <= 128 the mid-size decode path (small-T router, mma.sync GEMVs over the
    # active experts in 8-token tiles, fixed-order combine); moe_decode takes
    # T <= 64
    lay, x, _ = workload(10 + T, T, FULL)
    ref = moe_ref.moe_layer(x, lay, FULL.k)
    gpu = run_layer(lay, x, entry=entry)
    assert gpu["status"] == 0
    assert_routing_exact(gpu, ref)
    assert_output_close(gpu["out"], ref["out"])


@pytest.mark.parametrize("T", [1, 2, 8, 24, 64])
def test_full_decode_zipf(T):
    # at T = 24 and 64 the hot experts see more than 8 tokens: several token tiles per expert
    lay, x, _ = workload(30 + T, T, FULL, zipf=True)
    ref = moe_ref.moe_layer(x, lay, FULL.k)
    gpu = run_layer(lay, x, entry="decode")
    if T > 8:
        assert int(np.max(ref["counts"])) > 8
    assert gpu["status"] == 0
    assert_routing_exact(gpu, ref)
    assert_output_close(gpu["out"], ref["out"])


def test_full_decode_repeated_calls_one_workspace():
    # the fused kernel's grid barrier state lives in the workspace control
    # block: many calls in a row must keep giving the same bits
    lay, x_bits, _ = workload(41, 1, FULL)
    L = moe.MoELayer.from_synth(lay)
    x = to_dev_bits(x_bits)
    ws = moe.alloc_workspace(L, 1)
    outs = []
    for _ in range(5):
        out = torch.empty_like(x)
        moe.moe_decode(L, x, out, ws)
        outs.append(out)
    torch.cuda.synchronize()
    assert moe.moe_get_status(ws) == 0
    first = bits_of(outs[0])
    for o in outs[1:]:
        np.testing.assert_array_equal(bits_of(o), first)
    ref = moe_ref.moe_layer(x_bits, lay, FULL.k)
    assert_output_close(first, ref["out"])


@pytest.fixture(scope="module", params=["uniform", "zipf"])
def full_prefill(request):
    zipf = request.param == "zipf"
    lay, x, red = workload(20 if not zipf else 21, 4096, FULL, zipf=zipf)
    L = moe.MoELayer.from_synth(lay)
    gpu = run_layer(lay, x, dev_layer=L)
    return lay, x, L, gpu


def test_full_prefill_routing_all_tokens(full_prefill):
    lay, x, L, gpu = full_prefill
    ref = moe_ref.route(x, lay, FULL.k)
    assert_routing_exact(gpu, ref)
    assert gpu["status"] == 0


def test_full_prefill_sampled_outputs(full_prefill):
    lay, x, L, gpu = full_prefill
    sample = np.sort(np.random.default_rng(0).choice(4096, size=192, replace=False))
    sample = np.unique(np.concatenate([sample, [0, 4095]]))
    ref = moe_ref.moe_layer(x, lay, FULL.k, tokens=sample)
    assert_output_close(gpu["out"][sample], ref["out"])


def test_full_prefill_bitwise_repeatable(full_prefill):
    lay, x, L, gpu = full_prefill
    again = run_layer(lay, x, dev_layer=L)
    np.testing.assert_array_equal(again["out"], gpu["out"])
    np.testing.assert_array_equal(again["perm"], gpu["perm"])
