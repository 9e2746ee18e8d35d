"""Gated DeltaNet decode step on the GPU (include/deltanet.h) against the float64
oracle: single steps over several head geometries, a sequence of steps carried
in the state, the special cases of the delta rule, determinism, and the full
size the benchmark times."""
from __future__ import annotations

import numpy as np
import pytest
import torch

from bit_quantized_expert_route_b200 import deltanet, synth
from oracle import deltanet_ref as dr
from tests.gpu_util import bits_of, require_cuda, to_dev_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    require_cuda()


def _dev(c: synth.DeltaCase):
    f = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    return to_dev_bits(c.q), to_dev_bits(c.k), to_dev_bits(c.v), f(c.g), f(c.beta), f(c.state)


def _step(c: synth.DeltaCase, state_dev=None):
    q, k, v, g, beta, state = _dev(c)
    if state_dev is not None:
        state = state_dev
    out = torch.empty_like(v)
    deltanet.gdn_decode_step(q, k, v, g, beta, state, out)
    torch.cuda.synchronize()
    return bits_of(out), state


def _check(o_bits, state, o_ref, s_ref):
    m = dr.compare(dr.bf16_to_f64(o_bits), o_ref)
    assert m["rel_l2"] <= dr.O_REL_L2_TOL and m["max_err_rel"] <= dr.O_MAX_ERR_TOL, m
    ms = dr.compare(state.cpu().numpy().astype(np.float64), s_ref)
    assert ms["rel_l2"] <= dr.STATE_REL_L2_TOL, ms


@pytest.mark.parametrize("B,Hk,Hv,dk,dv", [(1, 16, 32, 128, 128), (3, 2, 4, 64, 64), (2, 4, 4, 256, 128),
                                            (5, 1, 2, 128, 32), (2, 2, 6, 64, 48)])
def test_one_step_matches_oracle(B, Hk, Hv, dk, dv):
    c = synth.make_deltanet_case(11 + B, B, Hk=Hk, Hv=Hv, dk=dk, dv=dv)
    o_bits, state = _step(c)
    o_ref, s_ref = dr.recurrent_step(c.q, c.k, c.v, c.g, c.beta, c.state)
    _check(o_bits, state, o_ref, s_ref)


def test_eight_steps_carried_in_the_state():
    c0 = synth.make_deltanet_case(21, 2, Hk=4, Hv=8, dk=128, dv=128)
    state_dev = torch.from_numpy(c0.state.copy()).cuda()
    s_ref = c0.state.astype(np.float64)
    for t in range(8):
        c = synth.make_deltanet_case(21, 2, Hk=4, Hv=8, dk=128, dv=128, step=t)
        o_bits, state_dev = _step(c, state_dev)
        o_ref, s_ref = dr.recurrent_step(c.q, c.k, c.v, c.g, c.beta, s_ref)
        _check(o_bits, state_dev, o_ref, s_ref)


def test_no_decay_no_write_keeps_the_state_bitwise():
    c = synth.make_deltanet_case(23, 2, Hk=2, Hv=4, dk=128, dv=64)
    c.g[...] = 0.0
    c.beta[...] = 0.0
    _, state = _step(c)
    np.testing.assert_array_equal(state.cpu().numpy(), c.state)


def test_full_decay_full_write_gives_the_outer_product():
    c = synth.make_deltanet_case(29, 1, Hk=2, Hv=4, dk=64, dv=64)
    c.g[...] = -100.0          # alpha = e^-100 = 0 in FP32
    c.beta[...] = 1.0
    o_bits, state = _step(c)
    o_ref, s_ref = dr.recurrent_step(c.q, c.k, c.v, c.g, c.beta, c.state)
    _check(o_bits, state, o_ref, s_ref)


def test_deterministic():
    c = synth.make_deltanet_case(31, 4, dk=128, dv=128)
    a, sa = _step(c)
    b, sb = _step(c)
    np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(sa.cpu().numpy(), sb.cpu().numpy())


def test_full_size_batch_of_64():
    """The benchmark's largest batch: 64 sequences, 16 key heads, 32 value heads, 128 x 128 state."""
    c = synth.make_deltanet_case(37, 64)
    o_bits, state = _step(c)
    o_ref, s_ref = dr.recurrent_step(c.q, c.k, c.v, c.g, c.beta, c.state)
    _check(o_bits, state, o_ref, s_ref)
