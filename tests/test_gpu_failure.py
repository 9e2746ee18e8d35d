"""Failure detection on the GPU without faulting it.

Two ways a call's status word comes to hold MOE_ERR_DEVICE_TIMEOUT, neither of
which faults, traps or hangs the device:

* injected on the host: the test writes the error code into the workspace's
  status word, as a kernel whose bounded wait gave up would;
* a real bounded wait that runs out: the test shortens every bounded wait of
  the kernels to one SM clock cycle (moe_set_wait_limit), so the router's
  epilogue gives up waiting for its accumulator long before the tensor cores
  can fill it; the router drains the copies it has issued and returns.

In both cases moe_get_status must return the error and clear the control
block, the kernels that read routing indices must have done nothing (out keeps
its sentinel), and the next call on the same workspace must match the oracle.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from bit_quantized_expert_route_b200 import moe
from oracle import moe_ref
from tests.gpu_util import assert_output_close, bits_of, require_cuda, to_dev_bits
from tests.workloads import FULL, TINY, workload

pytestmark = pytest.mark.gpu

SENTINEL = 0x7FC1   # a bf16 NaN pattern no kernel writes


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    require_cuda()


def _setup(seed, T):
    lay, x, _ = workload(seed, T, TINY)
    L = moe.MoELayer.from_synth(lay)
    xd = to_dev_bits(x)
    out = torch.empty_like(xd)
    ws = moe.alloc_workspace(L, T)
    return lay, x, L, xd, out, ws


def _fill_sentinel(out):
    out.view(torch.int16).fill_(SENTINEL)


def _assert_untouched(out):
    assert np.all(bits_of(out) == SENTINEL)


def _assert_next_call_correct(lay, x, L, xd, out, ws):
    moe.moe_forward(L, xd, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_status(ws) == moe.MOE_OK
    assert_output_close(bits_of(out), moe_ref.moe_layer(x, lay, TINY.k)["out"])


def test_injected_status_is_reported_cleared_and_skips_the_layer():
    T = 300
    lay, x, L, xd, out, ws = _setup(80, T)
    moe.moe_forward(L, xd, out, ws)
    torch.cuda.synchronize()
    assert moe.moe_get_status(ws) == moe.MOE_OK
    # a recorded error: the next call routes but leaves out unwritten
    ws[:4].view(torch.int32).fill_(moe.MOE_ERR_DEVICE_TIMEOUT)
    _fill_sentinel(out)
    moe.moe_forward(L, xd, out, ws)
    torch.cuda.synchronize()
    _assert_untouched(out)
    assert moe.moe_get_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    assert int(ws[:16].count_nonzero()) == 0          # control block cleared
    assert moe.moe_get_status(ws) == moe.MOE_OK
    _assert_next_call_correct(lay, x, L, xd, out, ws)


def test_router_wait_runs_out_and_the_next_call_is_correct():
    T = 300
    lay, x, L, xd, out, ws = _setup(81, T)
    _fill_sentinel(out)
    moe.moe_set_wait_limit(1)
    try:
        moe.moe_forward(L, xd, out, ws)
        torch.cuda.synchronize()
    finally:
        moe.moe_set_wait_limit(0)
    assert torch.cuda.is_available()                   # the context is still usable
    _assert_untouched(out)
    assert moe.moe_get_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    assert int(ws[:16].count_nonzero()) == 0
    _assert_next_call_correct(lay, x, L, xd, out, ws)


@pytest.mark.parametrize("T,entry", [(1, "forward"), (3, "forward"), (7, "stack")])
def test_fused_decode_waits_run_out_and_the_next_call_is_correct(T, entry):
    """The single-launch decode kernel's producer, consumers and grid barriers all give up
    after one cycle; every CTA leaves (its copies landed), the grid-barrier words are reset
    for the next launch, and the next call on the same workspace is correct.  A single
    layer runs the fused kernel up to T = 3, a stack (here of one layer) up to T = 7."""
    lay, x, _ = workload(82 + T, T, FULL)
    L = moe.MoELayer.from_synth(lay)
    xd = to_dev_bits(x)
    out = torch.empty_like(xd)
    ws = moe.alloc_workspace(L, T)

    def call():
        if entry == "stack":
            moe.moe_forward_stack(moe.LayerStack([L]), xd, out, ws, eps=1e-6)
        else:
            moe.moe_forward(L, xd, out, ws)

    assert len(moe.moe_forward_profiled(L, xd, out, ws)) == (1 if entry == "forward" else 4)
    moe.moe_set_wait_limit(1)
    try:
        call()
        torch.cuda.synchronize()
    finally:
        moe.moe_set_wait_limit(0)
    assert moe.moe_get_status(ws) == moe.MOE_ERR_DEVICE_TIMEOUT
    assert int(ws[:16].count_nonzero()) == 0
    for _ in range(2):
        call()
        torch.cuda.synchronize()
        assert moe.moe_get_status(ws) == moe.MOE_OK
        m = moe_ref.compare(moe_ref.bf16_to_f64(bits_of(out)), moe_ref.moe_layer(x, lay, FULL.k)["out"])
        assert m["rel_l2"] <= moe_ref.REL_L2_TOL and m["max_err_rel"] <= moe_ref.MAX_ERR_TOL, m
