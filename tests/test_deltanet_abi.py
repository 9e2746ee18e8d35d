"""The recurrence entry point of include/deltanet.h is exported and rejects bad
arguments on the host (no GPU needed)."""
from __future__ import annotations

import os
import re

import pytest

from bit_quantized_expert_route_b200 import build as moe_build
from bit_quantized_expert_route_b200 import deltanet, moe

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return deltanet.library()


def test_exports_every_declared_symbol(lib):
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "deltanet.h")).read(), flags=re.S)
    names = set(re.findall(r"^\s*MOE_API\s+[\w\s\*]+?\b(gdn_\w+)\s*\(", text, flags=re.M))
    assert names == set(deltanet.GDN_EXPORTS), names
    for n in names:
        assert hasattr(lib, n)


def _call(lib, B=1, Hk=16, Hv=32, dk=128, dv=128, state=FAKE, q=FAKE, out=FAKE):
    return lib.gdn_decode_step(q, FAKE, FAKE, FAKE, FAKE, state, out, B, Hk, Hv, dk, dv, None)


def test_host_rejections(lib):
    assert _call(lib, q=None) == moe.MOE_ERR_INVALID_ARG
    assert _call(lib, state=FAKE + 8) == moe.MOE_ERR_INVALID_ARG      # state not 16-byte aligned
    assert _call(lib, out=FAKE + 1) == moe.MOE_ERR_INVALID_ARG
    assert _call(lib, dk=96) == moe.MOE_ERR_UNSUPPORTED
    assert _call(lib, dv=24) == moe.MOE_ERR_UNSUPPORTED               # not a multiple of 16
    assert _call(lib, Hk=3, Hv=32) == moe.MOE_ERR_UNSUPPORTED         # value heads not a multiple
    assert _call(lib, B=0) == moe.MOE_ERR_UNSUPPORTED
    assert _call(lib, Hk=32, Hv=16) == moe.MOE_ERR_UNSUPPORTED
