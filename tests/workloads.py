"""The seeded workloads the tests use, with the near-tie screen.

Routing is compared bit for bit, which is only meaningful where the k-th and
(k+1)-th logits of a token are not within rounding of each other.  Rows of x
whose oracle boundary gap l_(k) - l_(k+1) is below 1e-3 are redrawn from the
row's own stream (seed, t, attempt) until every token clears the gap; the rows
stay N(0, 1) bf16.  The screen uses the oracle's float64 logits.
"""
from __future__ import annotations

import numpy as np

from bit_quantized_expert_route_b200 import synth
from oracle import moe_ref

TINY = synth.Dims.tiny()            # T=16 layer: H=256, E=16, k=2, I=I_s=128
FULL = synth.Dims()                 # H=2048, E=256, k=8, I=I_s=512


def screen_rows(seed: int, x_bits: np.ndarray, layer, k: int, max_attempts: int = 64):
    """Redraw rows of x until every token's top-k boundary gap is >= 1e-3."""
    x_bits = x_bits.copy()
    H = x_bits.shape[1]
    redrawn = set()
    for attempt in range(1, max_attempts + 1):
        logits = moe_ref.router_logits(moe_ref.bf16_to_f64(x_bits), layer.w_router, layer.router_bias)
        bad = np.nonzero(moe_ref.boundary_gap(logits, k) < moe_ref.GAP_MIN)[0]
        if bad.size == 0:
            return x_bits, sorted(redrawn)
        for t in bad:
            x_bits[t] = synth.redraw_row(seed, int(t), attempt, H)
            redrawn.add(int(t))
    raise RuntimeError("near-tie screen did not converge")


def workload(seed: int, T: int, dims: synth.Dims, zipf: bool = False, layer_index: int = 0, screen: bool = True):
    layer = synth.make_layer(seed, layer_index, dims, zipf=zipf)
    x = synth.make_x(seed, T, dims.H)
    redrawn = []
    if screen:
        x, redrawn = screen_rows(seed, x, layer, dims.k)
    return layer, x, redrawn
