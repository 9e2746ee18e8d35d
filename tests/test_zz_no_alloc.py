"""moe_route_static: routing for callers that cannot allocate device memory.

Some hosts give this library only the tensors it reads and writes (a plug-in
inside another runtime with no allocator to offer, a serving loop whose memory
plan forbids a cudaMalloc and the device synchronisation it can cause).  For
them moe_route_static keeps its scratch in a static device array inside
libmoe.so instead of a caller workspace.  This file checks, through the C ABI,
that two calls in a row give what moe_route gives, that its routing matches
the CPU oracle on both sides of T = 64 (where moe_route, and so this entry
point, switches from the one-launch small-T router to the tensor-core router),
that its status word reads back as MOE_OK, and that a call needing more than
the array holds is refused before anything is enqueued.  It is named to run
last so that a failure here cannot hide any other test's result.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from bit_quantized_expert_route_b200 import moe
from oracle import moe_ref
from tests.gpu_util import assert_routing_exact, require_cuda, to_dev_bits
from tests.workloads import FULL, TINY, workload

pytestmark = pytest.mark.gpu

FIELDS = ("topk_idx", "counts", "offsets", "perm", "inv_perm")


def _route(L, x_bits, static: bool, with_sigma: bool = True):
    T = x_bits.shape[0]
    x = to_dev_bits(x_bits)
    r = moe.Routing(T, L.E, L.k)
    if not with_sigma:
        r.c.sigma = None
    if static:
        moe.moe_route_static(L, x, r)
    else:
        ws = moe.alloc_workspace(L, T)
        moe.moe_route(L, x, r, ws)
    torch.cuda.synchronize()
    return {f: getattr(r, f).cpu().numpy() for f in FIELDS + ("topk_w", "sigma")}


@pytest.mark.parametrize("dims,T,seeds", [(TINY, 300, (40, 41)), (FULL, 4096, (42, 43))])
def test_static_route_matches_route_on_two_calls(dims, T, seeds):
    require_cuda()
    (lay_a, x_a, _), (lay_b, x_b, _) = (workload(s, T, dims) for s in seeds)
    La, Lb = moe.MoELayer.from_synth(lay_a), moe.MoELayer.from_synth(lay_b)
    want_a, want_b = _route(La, x_a, static=False), _route(Lb, x_b, static=False)
    got_a = _route(La, x_a, static=True)           # first call on this device sets up the scratch address
    got_b = _route(Lb, x_b, static=True)           # second call reuses the array left by the first
    for got, want in ((got_a, want_a), (got_b, want_b)):
        for f in FIELDS:
            np.testing.assert_array_equal(got[f], want[f])
        np.testing.assert_allclose(got["topk_w"], want["topk_w"], rtol=0, atol=2e-6)
        np.testing.assert_allclose(got["sigma"], want["sigma"], rtol=0, atol=2e-6)


@pytest.mark.parametrize("T", [1, 5, 64, 65, 300, 4096])
def test_static_route_matches_oracle(T):
    """Both routers behind the entry point (T <= 64 and T > 64) against the oracle, bit for bit."""
    require_cuda()
    lay, x, _ = workload(50 + T % 7, T, FULL)
    L = moe.MoELayer.from_synth(lay)
    got = _route(L, x, static=True)
    assert moe.moe_get_status(None) == moe.MOE_OK
    ref = moe_ref.route(x, lay, FULL.k)
    gpu = {
        "topk_idx": got["topk_idx"].reshape(T, FULL.k).astype(np.int64),
        "topk_w": got["topk_w"].reshape(T, FULL.k).astype(np.float64),
        "counts": got["counts"].astype(np.int64), "offsets": got["offsets"].astype(np.int64),
        "perm": got["perm"].astype(np.int64), "inv_perm": got["inv_perm"].astype(np.int64),
        "sigma": got["sigma"].astype(np.float64),
    }
    assert_routing_exact(gpu, ref)


def test_static_route_without_sigma_output():
    require_cuda()
    lay, x, _ = workload(44, 129, TINY)
    L = moe.MoELayer.from_synth(lay)
    want = _route(L, x, static=False)
    got = _route(L, x, static=True, with_sigma=False)
    for f in FIELDS:
        np.testing.assert_array_equal(got[f], want[f])


def test_static_route_refuses_calls_beyond_its_scratch():
    require_cuda()
    lay, _, _ = workload(45, 1, FULL, screen=False)
    L = moe.MoELayer.from_synth(lay)
    T = 60000                                      # needs more than the 512 KiB static scratch
    x = torch.zeros((T, FULL.H), dtype=torch.bfloat16, device="cuda")
    r = moe.Routing(T, L.E, L.k)
    with pytest.raises(moe.MoEError) as e:
        moe.moe_route_static(L, x, r)
    assert e.value.code == moe.MOE_ERR_WORKSPACE
    st = moe.library().moe_route_static(ctypes.byref(L.desc), x.data_ptr(), T, None, None)
    assert st == moe.MOE_ERR_INVALID_ARG
