"""The attention entry points of include/attn.h are exported, size their
workspace, and reject bad arguments on the host (no GPU needed)."""
from __future__ import annotations

import os
import re

import pytest

from bit_quantized_expert_route_b200 import attn, moe
from bit_quantized_expert_route_b200 import build as moe_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000   # aligned, non-NULL, never dereferenced on these paths


@pytest.fixture(scope="module")
def lib():
    moe_build.build()
    return attn.library()


def test_exports_every_declared_symbol(lib):
    text = re.sub(r"/\*.*?\*/", "", open(os.path.join(ROOT, "include", "attn.h")).read(), flags=re.S)
    names = set(re.findall(r"^\s*MOE_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", text, flags=re.M))
    assert names == set(attn.ATTN_EXPORTS), names
    for n in names:
        assert hasattr(lib, n)


def test_strerror_knows_the_index_status(lib):
    assert "index" in moe.strerror(attn.MOE_ERR_DEVICE_INDEX)


def test_plan_covers_every_chunk(lib):
    for B, Hkv, block, mb in [(1, 2, 64, 64), (1, 2, 64, 512), (1, 2, 64, 2048), (3, 2, 32, 7), (96, 2, 64, 5),
                              (1, 8, 128, 1), (200, 1, 64, 100)]:
        ns, cps = attn.plan(B, Hkv, block, mb)
        chunks = mb * block // 16
        assert ns >= 1 and cps >= 1
        assert (ns - 1) * cps < chunks <= ns * cps          # no empty trailing range, every chunk owned
        if B * Hkv >= 148:
            assert ns == 1


def test_workspace_size(lib):
    assert attn.workspace_size(1, 2, 256, 64, 2048) >= 256
    ns, _ = attn.plan(1, 2, 64, 2048)
    assert attn.workspace_size(1, 2, 256, 64, 2048) >= 256 + ns * 2 * 8 * 256 * 4
    assert attn.workspace_size(1, 2, 192, 64, 8) == 0       # unsupported D
    assert attn.workspace_size(1, 2, 256, 40, 8) == 0       # block not a multiple of 16


def _call(lib, B=1, Hq=16, Hkv=2, D=256, block=64, max_blocks=4, n_blocks=4, ws=FAKE, ws_bytes=1 << 30,
          q=FAKE, kc=FAKE, vc=FAKE, table=FAKE, ctx=FAKE, out=FAKE):
    return lib.attn_decode(q, kc, vc, table, ctx, B, Hq, Hkv, D, block, max_blocks, n_blocks, 0.0, out, ws,
                           ws_bytes, None)


def test_host_rejections(lib):
    assert _call(lib, q=None) == moe.MOE_ERR_INVALID_ARG
    assert _call(lib, kc=FAKE + 8) == moe.MOE_ERR_INVALID_ARG       # cache not 16-byte aligned
    assert _call(lib, table=FAKE + 2) == moe.MOE_ERR_INVALID_ARG    # int32 table misaligned
    assert _call(lib, D=192) == moe.MOE_ERR_UNSUPPORTED
    assert _call(lib, Hq=18, Hkv=2) == moe.MOE_ERR_UNSUPPORTED      # group of 9 heads
    assert _call(lib, Hq=15, Hkv=2) == moe.MOE_ERR_UNSUPPORTED      # not a multiple
    assert _call(lib, block=40) == moe.MOE_ERR_UNSUPPORTED
    assert _call(lib, B=0) == moe.MOE_ERR_UNSUPPORTED
    assert _call(lib, n_blocks=1 << 20, block=1024, Hkv=8, Hq=8) == moe.MOE_ERR_UNSUPPORTED   # rows >= 2^31
    assert _call(lib, ws=None) == moe.MOE_ERR_WORKSPACE
    assert _call(lib, ws=FAKE + 16) == moe.MOE_ERR_WORKSPACE        # not 256-byte aligned
    assert _call(lib, ws_bytes=255) == moe.MOE_ERR_WORKSPACE
