"""Helpers for the GPU tests: run the layer through the C ABI and fetch results."""
from __future__ import annotations

import numpy as np
import torch

from bit_quantized_expert_route_b200 import moe
from oracle import moe_ref


def require_cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    moe.library()


def to_dev_bits(a: np.ndarray) -> torch.Tensor:
    return moe._bits_tensor(a, "cuda")


def bits_of(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().view(torch.int16).numpy().view(np.uint16).copy()


def run_layer(layer_np, x_bits: np.ndarray, entry: str = "forward", dev_layer=None):
    """Run moe_forward / moe_decode / moe_route on the GPU; return out bits and routing arrays."""
    L = dev_layer if dev_layer is not None else moe.MoELayer.from_synth(layer_np)
    T = x_bits.shape[0]
    x = to_dev_bits(x_bits)
    out = torch.empty_like(x)
    ws = moe.alloc_workspace(L, T)
    r = moe.Routing(T, L.E, L.k)
    if entry == "forward":
        moe.moe_forward(L, x, out, ws, routing=r)
    elif entry == "decode":
        moe.moe_decode(L, x, out, ws, routing=r)
    elif entry == "route":
        moe.moe_route(L, x, r, ws)
    else:
        raise ValueError(entry)
    torch.cuda.synchronize()
    status = moe.moe_get_status(ws)
    res = {
        "out": None if entry == "route" else bits_of(out),
        "topk_idx": r.topk_idx.view(T, L.k).cpu().numpy().astype(np.int64),
        "topk_w": r.topk_w.view(T, L.k).cpu().numpy().astype(np.float64),
        "counts": r.counts.cpu().numpy().astype(np.int64),
        "offsets": r.offsets.cpu().numpy().astype(np.int64),
        "perm": r.perm.cpu().numpy().astype(np.int64),
        "inv_perm": r.inv_perm.cpu().numpy().astype(np.int64),
        "sigma": r.sigma.cpu().numpy().astype(np.float64),
        "status": status,
    }
    return res


def assert_routing_exact(gpu: dict, ref: dict, tokens=None, w_atol: float = 2e-6):
    """Routing must match the oracle bit for bit on screened inputs.

    w_atol bounds the FP32 weights and gates; the default is set for H = 2048,
    and the error of an FP32 dot product grows with its length H."""
    idx = ref["topk_idx"]
    np.testing.assert_array_equal(gpu["topk_idx"], idx)
    np.testing.assert_array_equal(gpu["counts"], ref["counts"])
    np.testing.assert_array_equal(gpu["offsets"], ref["offsets"])
    np.testing.assert_array_equal(gpu["perm"], ref["perm"])
    np.testing.assert_array_equal(gpu["inv_perm"], ref["inv_perm"])
    # weights: FP32 softmax over the chosen FP32 logits vs float64
    np.testing.assert_allclose(gpu["topk_w"], ref["topk_w"], rtol=0, atol=w_atol)
    np.testing.assert_allclose(gpu["sigma"], ref["sigma"], rtol=0, atol=w_atol)
    assert np.all(np.abs(gpu["topk_w"].sum(axis=1) - 1.0) < 1e-6)


def assert_routing_up_to_near_ties(gpu: dict, ref: dict, k: int) -> dict:
    """Routing vs the oracle where FP32 logits may order a near tie either way.

    Exact wherever the oracle's float64 logits separate each token's k + 1 best
    experts by at least GAP_MIN.  Elsewhere the GPU's choice must be a valid
    order of the oracle's logits (k distinct experts, each chosen logit >= the
    next one - GAP_MIN, none below an unchosen one - GAP_MIN).  The oracle's
    buffers (counts, offsets, perm, inv_perm) and weights are then rebuilt from
    the accepted choices and must match bit for bit.  Returns the accepted
    choices that differ from the oracle's, keyed by token, for idx_override.
    """
    logits, idx = ref["logits"], ref["topk_idx"].copy()
    T, E = logits.shape
    m = min(k + 1, E)
    top = -np.sort(-logits, axis=1)[:, :m]
    min_gap = (top[:, :-1] - top[:, 1:]).min(axis=1) if m > 1 else np.full(T, np.inf)
    clear = min_gap >= moe_ref.GAP_MIN
    np.testing.assert_array_equal(gpu["topk_idx"][clear], idx[clear])
    override = {}
    for t in np.nonzero(~clear)[0]:
        got = gpu["topk_idx"][t]
        if np.array_equal(got, idx[t]):
            continue
        lt = logits[t]
        assert len(set(got.tolist())) == k
        assert np.all(lt[got[:-1]] >= lt[got[1:]] - moe_ref.GAP_MIN)
        rest = np.setdiff1d(np.arange(E), got)
        if rest.size:
            assert lt[got].min() >= lt[rest].max() - moe_ref.GAP_MIN
        idx[t] = got
        override[int(t)] = got
    counts, offsets, perm, inv_perm = moe_ref.routing_buffers(idx, E)
    np.testing.assert_array_equal(gpu["counts"], counts)
    np.testing.assert_array_equal(gpu["offsets"], offsets)
    np.testing.assert_array_equal(gpu["perm"], perm)
    np.testing.assert_array_equal(gpu["inv_perm"], inv_perm)
    np.testing.assert_allclose(gpu["topk_w"], moe_ref.topk_weights(logits, idx), rtol=0, atol=2e-6)
    assert np.all(np.abs(gpu["topk_w"].sum(axis=1) - 1.0) < 1e-6)
    np.testing.assert_allclose(gpu["sigma"], ref["sigma"], rtol=0, atol=2e-6)
    return override


def assert_output_close(out_bits: np.ndarray, ref_out: np.ndarray):
    m = moe_ref.compare(moe_ref.bf16_to_f64(out_bits), ref_out)
    assert m["rel_l2"] <= moe_ref.REL_L2_TOL, m
    assert m["max_err_rel"] <= moe_ref.MAX_ERR_TOL, m
    return m
