"""The GPU-vs-oracle comparison helpers, exercised on the CPU with planted results."""
from __future__ import annotations

import numpy as np
import pytest

from oracle import moe_ref
from tests.gpu_util import assert_routing_up_to_near_ties


def _fake_gpu(logits, idx, E):
    counts, offsets, perm, inv_perm = moe_ref.routing_buffers(idx, E)
    return {"topk_idx": idx, "counts": counts, "offsets": offsets, "perm": perm, "inv_perm": inv_perm,
            "topk_w": moe_ref.topk_weights(logits, idx), "sigma": np.zeros(len(idx))}


def _case():
    rng = np.random.default_rng(0)
    T, E, k = 50, 32, 4
    l = rng.normal(0, 1, (T, E))
    o = np.argsort(-l[3])
    l[3, o[2]] = l[3, o[1]] - 1e-4          # token 3: its 2nd and 3rd best are a near tie
    idx = moe_ref.select_topk(l, k)
    return l, idx, E, k, {"logits": l, "topk_idx": idx, "sigma": np.zeros(T)}


def test_near_tie_swap_is_accepted_and_fed_back():
    l, idx, E, k, ref = _case()
    got = idx.copy()
    got[3, [1, 2]] = got[3, [2, 1]]
    override = assert_routing_up_to_near_ties(_fake_gpu(l, got, E), ref, k)
    assert list(override) == [3]
    np.testing.assert_array_equal(override[3], got[3])


def test_swap_of_clearly_ordered_experts_fails():
    l, idx, E, k, ref = _case()
    got = idx.copy()
    got[5, [0, 1]] = got[5, [1, 0]]
    with pytest.raises(AssertionError):
        assert_routing_up_to_near_ties(_fake_gpu(l, got, E), ref, k)


def test_buffers_must_follow_the_accepted_choice():
    l, idx, E, k, ref = _case()
    got = idx.copy()
    got[3, [1, 2]] = got[3, [2, 1]]
    gpu = _fake_gpu(l, got, E)
    gpu["perm"] = moe_ref.routing_buffers(idx, E)[2]      # buffers of the oracle's order, not the GPU's
    with pytest.raises(AssertionError):
        assert_routing_up_to_near_ties(gpu, ref, k)
