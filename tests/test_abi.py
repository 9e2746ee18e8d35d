"""The C-ABI library loads, exports every declared entry point, sizes its
workspace, and rejects bad arguments on the host before touching a GPU."""
from __future__ import annotations

import ctypes
import os
import re

import pytest

from bit_quantized_expert_route_b200 import build as moe_build
from bit_quantized_expert_route_b200 import moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return moe.library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "moe.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:MOE_API\s+)?(?:int|const char\*)\s+(moe_\w+)\s*\(", text, flags=re.M)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert set(names) == set(moe.EXPORTS), names
    for n in names:
        assert hasattr(lib, n)


def test_strerror(lib):
    for code in (0, -1, -2, -3, -4, -5):
        assert moe.strerror(code)
    assert "unknown" in moe.strerror(42)


FAKE = 0x10000   # a 16-byte-aligned non-NULL address; never dereferenced on these paths


def fake_layer(**over):
    qm = moe.QMatC(FAKE, FAKE, FAKE)
    fields = dict(H=2048, I=512, I_shared=512, E=256, k=8, group_size=64, bits=4, renorm=1)
    fields.update(over)
    return moe.LayerC(fields["H"], fields["I"], fields["I_shared"], fields["E"], fields["k"], fields["group_size"],
                      fields["bits"], fields["renorm"], FAKE, None, qm, qm, qm, qm, qm, qm, FAKE)


def ws_size(lib, layer, T):
    n = ctypes.c_size_t(0)
    st = lib.moe_workspace_size(ctypes.byref(layer), T, ctypes.byref(n))
    return st, n.value


def test_workspace_size_monotone(lib):
    L = fake_layer()
    sizes = []
    for T in (1, 8, 64, 512, 4096, 16384):
        st, n = ws_size(lib, L, T)
        assert st == 0
        sizes.append(n)
    assert sizes == sorted(sizes)
    # Y (bf16, (T*k + T) x H) dominates at T=4096
    assert sizes[4] >= 9 * 4096 * 2048 * 2


@pytest.mark.parametrize("over", [dict(), dict(H=256, E=16, k=2, I=128, I_shared=128),
                                  dict(H=1024, I=256, I_shared=256)])
def test_workspace_for_t_max_serves_every_smaller_t(lib, over):
    """The header promises a workspace for any T <= T_max.  The layout of a
    call grows with T within each kernel set, but T <= 7 also holds the fused
    decode kernel's exchange words and T <= 128 the small router's logits, so
    the size for T_max = 8 must still cover a call with T = 7: the reported
    sizes never decrease with T."""
    L = fake_layer(**over)
    prev = 0
    for T in list(range(1, 140)) + [255, 256, 257, 4095, 4096, 4097]:
        st, n = ws_size(lib, L, T)
        assert st == 0
        assert n >= prev, (T, n, prev)
        prev = n


@pytest.mark.parametrize("over,code", [
    (dict(bits=8), moe.MOE_ERR_UNSUPPORTED),
    (dict(group_size=128), moe.MOE_ERR_UNSUPPORTED),
    (dict(renorm=0), moe.MOE_ERR_UNSUPPORTED),
    (dict(k=9), moe.MOE_ERR_UNSUPPORTED),
    (dict(k=0), moe.MOE_ERR_UNSUPPORTED),
    (dict(E=300), moe.MOE_ERR_UNSUPPORTED),
    (dict(E=4, k=8), moe.MOE_ERR_UNSUPPORTED),
    (dict(H=200), moe.MOE_ERR_UNSUPPORTED),
    (dict(I=96), moe.MOE_ERR_UNSUPPORTED),
    (dict(I_shared=4096), moe.MOE_ERR_UNSUPPORTED),
])
def test_layer_validation(lib, over, code):
    st, _ = ws_size(lib, fake_layer(**over), 16)
    assert st == code


# The documented edges of the accepted layout (include/moe.h, moe_layer_desc):
# 1 <= k <= 8, k <= E <= 256, H a multiple of 128 up to 8192, I and I_shared
# multiples of 128 up to 2048.  Multiples of the group size (64) that are not
# multiples of 128 are refused on purpose (full 128-row weight tiles).
@pytest.mark.parametrize("over,code", [
    (dict(k=1, E=1), 0), (dict(k=8, E=8), 0), (dict(k=8, E=256), 0), (dict(E=257), moe.MOE_ERR_UNSUPPORTED),
    (dict(H=128), 0), (dict(H=8192), 0), (dict(H=8320), moe.MOE_ERR_UNSUPPORTED),
    (dict(H=192), moe.MOE_ERR_UNSUPPORTED), (dict(H=64), moe.MOE_ERR_UNSUPPORTED),
    (dict(I=128), 0), (dict(I=2048), 0), (dict(I=2176), moe.MOE_ERR_UNSUPPORTED), (dict(I=192), moe.MOE_ERR_UNSUPPORTED),
    (dict(I_shared=128), 0), (dict(I_shared=2048), 0), (dict(I_shared=320), moe.MOE_ERR_UNSUPPORTED),
])
def test_documented_layout_edges(lib, over, code):
    assert ws_size(lib, fake_layer(**over), 16)[0] == code


def test_null_and_misaligned_pointers(lib):
    L = fake_layer()
    L.gate = moe.QMatC(FAKE, None, FAKE)
    assert ws_size(lib, L, 4)[0] == moe.MOE_ERR_INVALID_ARG
    L = fake_layer()
    L.w_router = FAKE + 2
    assert ws_size(lib, L, 4)[0] == moe.MOE_ERR_INVALID_ARG
    L = fake_layer()
    assert ws_size(lib, L, 0)[0] == moe.MOE_ERR_INVALID_ARG
    assert ws_size(lib, L, 70000)[0] == moe.MOE_ERR_INVALID_ARG


def test_calls_reject_before_launch(lib):
    L = fake_layer()
    st, need = ws_size(lib, L, 16)
    out = FAKE
    # workspace too small / misaligned / missing
    assert lib.moe_forward(ctypes.byref(L), FAKE, 16, out, None, FAKE, need - 1, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_forward(ctypes.byref(L), FAKE, 16, out, None, FAKE + 16, need, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_forward(ctypes.byref(L), FAKE, 16, out, None, None, need, None) == moe.MOE_ERR_WORKSPACE
    # bad T, x, out
    assert lib.moe_forward(ctypes.byref(L), FAKE, 0, out, None, FAKE, need, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_forward(ctypes.byref(L), FAKE + 8, 16, out, None, FAKE, need, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_forward(ctypes.byref(L), FAKE, 16, None, None, FAKE, need, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_decode(ctypes.byref(L), FAKE, 65, out, None, FAKE, 1 << 40, None) == moe.MOE_ERR_INVALID_ARG
    # moe_route needs a routing struct, and a complete one
    assert lib.moe_route(ctypes.byref(L), FAKE, 16, None, FAKE, need, None) == moe.MOE_ERR_INVALID_ARG
    r = moe.RoutingC(FAKE, FAKE, FAKE, None, FAKE, FAKE, None)
    assert lib.moe_route(ctypes.byref(L), FAKE, 16, ctypes.byref(r), FAKE, need, None) == moe.MOE_ERR_INVALID_ARG
    # unsupported layout wins over everything else
    L8 = fake_layer(bits=8)
    assert lib.moe_forward(ctypes.byref(L8), FAKE, 16, out, None, FAKE, need, None) == moe.MOE_ERR_UNSUPPORTED
    assert lib.moe_forward_host(ctypes.byref(L), None, 16, out, FAKE, need, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host_async(ctypes.byref(L), None, 16, out, FAKE, need, None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host_async(ctypes.byref(L), FAKE, 16, out, FAKE, 16, None) == moe.MOE_ERR_WORKSPACE
    assert lib.moe_rmsnorm(FAKE, FAKE, 0, 2048, ctypes.c_float(1e-6), None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_rmsnorm(FAKE, FAKE + 4, 4, 2048, ctypes.c_float(1e-6), None) == moe.MOE_ERR_INVALID_ARG
    assert lib.moe_get_status(FAKE + 16, None) == moe.MOE_ERR_WORKSPACE
    # NULL reads moe_route_static's status word: with no CUDA device the lookup itself fails
    import torch
    if not torch.cuda.is_available():
        assert lib.moe_get_status(None, None) == moe.MOE_ERR_CUDA


def test_library_is_built_for_sm100a():
    moe_build.build()
    assert "arch=compute_100a,code=sm_100a" in " ".join(moe_build.NVCC_FLAGS)
    assert os.path.exists(moe_build.LIB)


def _static_route_need(T, E, k, sigma_given, seg=128, chunk=160):
    """Scratch bytes of moe_route_static as moe.h states them (each piece rounded to 256 B):
    per-segment counts of 128-token segments, a chunk list of <= 160-row chunks."""
    r = lambda b: (b + 255) // 256 * 256
    n = 256
    if T <= 64:
        n += r(T * (E + 1) * 4)
    else:
        n += r(-(-T // seg) * E * 4) + r((T * k // chunk + T // chunk + E + 2) * 16) + r(4)
    n += r((E + 1) * 4) + r(4)
    return n + (0 if sigma_given else r(T * 4))


def test_static_route_limits(lib):
    """moe_route_static admits T <= 58112 (sigma given) / 40099 (sigma NULL) for E=256, k=8,
    and rejects the next T on the host with MOE_ERR_WORKSPACE before any CUDA call.
    (Only the rejecting side is called: an accepted call would launch kernels.)"""
    L = fake_layer()
    for sigma, limit in ((FAKE, 58112), (None, 40099)):
        assert _static_route_need(limit, 256, 8, sigma is not None) <= 512 * 1024
        assert _static_route_need(limit + 1, 256, 8, sigma is not None) > 512 * 1024
        r = moe.RoutingC(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, sigma)
        assert lib.moe_route_static(ctypes.byref(L), FAKE, limit + 1, ctypes.byref(r), None) == moe.MOE_ERR_WORKSPACE
