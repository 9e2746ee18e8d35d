"""The seeded input generators follow the stated recipe (CPU only).

Recipe: x ~ N(0, 1); W_r and w_sg ~ N(0, 0.02); codes uniform on 0..15;
scales ~ U(0.002, 0.006); bias = -8 * scale + N(0, 1e-3); all stored as bf16
bit patterns (codes as packed uint32).  The host draws (make_layer, make_x)
feed every parity test; the device draws (make_layer_on_device, run here on
the CPU device) feed the benchmark and must have the same shapes, storage
types and distributions.
"""
from __future__ import annotations

import numpy as np
import torch

from bit_quantized_expert_route_b200 import synth
from tests.workloads import TINY


def _f(bits):
    return synth.bf16_bits_as_f32(np.asarray(bits)).astype(np.float64)


# ends of the scale range as stored: U(0.002, 0.006) rounded to bf16
S_LO, S_HI = (float(v) for v in synth.bf16_bits_as_f32(synth.to_bf16_bits(np.array([0.002, 0.006]))))


def _codes(words):
    w = np.asarray(words, dtype=np.uint32)
    return ((w[..., None] >> (4 * np.arange(8, dtype=np.uint32))) & 0xF).ravel()


def test_host_layer_shapes_and_types():
    d = TINY
    lay = synth.make_layer(5, 2, d, zipf=True)
    assert lay.w_router.shape == (d.E, d.H) and lay.w_router.dtype == np.uint16
    assert lay.router_bias.shape == (d.E,) and lay.router_bias.dtype == np.float32
    for qm, lead, R, C in ((lay.gate, (d.E,), d.I, d.H), (lay.up, (d.E,), d.I, d.H), (lay.down, (d.E,), d.H, d.I),
                           (lay.sh_gate, (), d.I_s, d.H), (lay.sh_up, (), d.I_s, d.H), (lay.sh_down, (), d.H, d.I_s)):
        assert qm.q.shape == lead + (R, C // 8) and qm.q.dtype == np.uint32
        assert qm.scales.shape == lead + (R, C // 64) and qm.scales.dtype == np.uint16
        assert qm.biases.shape == qm.scales.shape and qm.biases.dtype == np.uint16
    assert lay.w_shared_gate.shape == (d.H,)


def test_host_layer_distributions():
    lay = synth.make_layer(6, 0, synth.Dims())
    wr = _f(lay.w_router)
    assert abs(wr.mean()) < 5e-4 and abs(wr.std() - 0.02) < 5e-4
    s = _f(lay.gate.scales)
    assert s.min() >= S_LO and s.max() <= S_HI
    assert abs(s.mean() - 0.004) < 5e-5
    resid = _f(lay.gate.biases) - (-8.0 * s)
    assert abs(resid.mean()) < 5e-5 and abs(resid.std() - 1e-3) < 1e-4
    counts = np.bincount(_codes(lay.up.q[:4]), minlength=16)
    expected = counts.sum() / 16
    assert np.all(np.abs(counts - expected) < 6 * np.sqrt(expected))   # uniform on 0..15


def test_x_distribution_and_redraw():
    x = _f(synth.make_x(7, 512, 2048))
    assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    r1 = synth.redraw_row(7, 3, 1, 2048)
    r2 = synth.redraw_row(7, 3, 2, 2048)
    assert r1.shape == (2048,) and not np.array_equal(r1, r2)
    assert abs(_f(r1).std() - 1.0) < 0.05


def test_draws_are_seeded_and_distinct():
    a = synth.make_layer(8, 1, TINY)
    b = synth.make_layer(8, 1, TINY)
    c = synth.make_layer(8, 2, TINY)
    np.testing.assert_array_equal(a.down.q, b.down.q)
    np.testing.assert_array_equal(a.w_router, b.w_router)
    assert not np.array_equal(a.down.q, c.down.q)
    np.testing.assert_array_equal(synth.make_x(3, 4, 256), synth.make_x(3, 4, 256))


def test_device_draws_follow_the_same_recipe():
    d = synth.Dims()
    t = synth.make_layer_on_device(9, 0, d, "cpu")
    assert t["w_router"].dtype == torch.bfloat16 and tuple(t["w_router"].shape) == (d.E, d.H)
    wr = t["w_router"].float().numpy()
    assert abs(wr.std() - 0.02) < 5e-4
    g = t["gate"]
    assert tuple(g["q"].shape) == (d.E, d.I, d.H // 8) and g["q"].dtype == torch.int32
    s = g["scales"].float().numpy()
    assert s.min() >= S_LO and s.max() <= S_HI
    resid = g["biases"].float().numpy() - (-8.0 * s)
    assert abs(resid.std() - 1e-3) < 1e-4
    counts = np.bincount(_codes(g["q"][:4].numpy().view(np.uint32)), minlength=16)
    expected = counts.sum() / 16
    assert np.all(np.abs(counts - expected) < 6 * np.sqrt(expected))
    x = synth.make_x_on_device(2, 256, d.H, "cpu").float().numpy()
    assert abs(x.std() - 1.0) < 0.02
