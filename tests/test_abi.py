"""The C-ABI library loads and exports every symbol include/v4moe.h declares;
host-side argument checks (no device work is launched here)."""
import ctypes
import os
import re

import pytest

from conftest import ROOT

import mxfp4_routed_expert_v4moe_b200 as V
from mxfp4_routed_expert_v4moe_b200 import build as B

HEADER = os.path.join(ROOT, "include", "v4moe.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(v4moe_[a-z_0-9]+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return V.load()


def test_library_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert len(syms) >= 7
    for s in syms:
        assert hasattr(lib, s), f"{s} declared in include/v4moe.h but not exported"
    assert set(V.EXPORTED) <= set(syms)


def test_status_strings(lib):
    for code in range(0, 7):
        assert V.status_string(code)
    assert V.status_string(99) == "unknown status"


def test_workspace_bytes_host_only(lib):
    cfg = V.make_config(4096, 2048, 256, 6, 2048)
    a = V.v4moe_workspace_bytes(cfg, 1)
    b = V.v4moe_workspace_bytes(cfg, 4096)
    assert 0 < a < b
    assert V.v4moe_workspace_bytes(cfg, -1) == 0
    bad = V.make_config(4000, 2048, 256, 6, 2048)  # H not a multiple of 128
    assert V.v4moe_workspace_bytes(bad, 4) == 0
    assert V.v4moe_workspace_bytes(V.make_config(4096, 2048, 256, 9, 2048), 4) == 0   # k > 8
    assert V.v4moe_workspace_bytes(V.make_config(4096, 2048, 4, 6, 2048), 4) == 0     # E < k


def test_invalid_arguments_rejected_before_launch(lib):
    cfg = V.make_config(512, 256, 16, 6, 256)
    ws_bytes = V.v4moe_workspace_bytes(cfg, 8)
    # null config
    assert lib.v4moe_route(None, 8, None, None, None, None, None, None, None, None, 0, None) == V.V4MOE_ERR_INVALID_ARG
    # learned routing with null x
    assert V.v4moe_route(cfg, 8, None, 16, 256, None, None, 256, 256, 256, ws_bytes, 0) == V.V4MOE_ERR_INVALID_ARG
    # both bias and hash table
    assert V.v4moe_route(cfg, 8, 16, 16, 256, 16, 16, 256, 256, 256, ws_bytes, 0) == V.V4MOE_ERR_INVALID_ARG
    # misaligned x
    assert V.v4moe_route(cfg, 8, 18, 16, 256, None, None, 256, 256, 256, ws_bytes, 0) == V.V4MOE_ERR_INVALID_ARG
    # workspace too small / misaligned
    assert V.v4moe_route(cfg, 8, 16, 16, 256, None, None, 256, 256, 256, ws_bytes - 1, 0) == V.V4MOE_ERR_WORKSPACE
    assert V.v4moe_route(cfg, 8, 16, 16, 256, None, None, 256, 256, 512 + 16, ws_bytes, 0) == V.V4MOE_ERR_INVALID_ARG
    w = V.make_weights(None, None, None, None)
    assert V.v4moe_forward(cfg, 8, 16, 16, 16, 16, 16, 16, w, 32, 256, ws_bytes, 0) == V.V4MOE_ERR_INVALID_ARG
    # out aliasing x
    w2 = V.make_weights(256, 256, 256, 256, 256, 256, 256, 256)
    assert V.v4moe_forward(cfg, 8, 512, 16, 16, 16, 16, 16, w2, 512, 256, ws_bytes, 0) == V.V4MOE_ERR_INVALID_ARG
    assert V.v4moe_permute(cfg, 8, None, 16, 16, 16, 16, 256, ws_bytes, 0) == V.V4MOE_ERR_INVALID_ARG
    assert V.v4moe_read_device_status(None, 0) == V.V4MOE_ERR_INVALID_ARG
    assert V.v4moe_clear_device_status(17, 0) == V.V4MOE_ERR_INVALID_ARG


def test_python_binding_has_the_c_names():
    for s in declared_symbols():
        assert callable(getattr(V, s)), s


def test_linear_w8a16_rejects_bad_shapes_before_any_launch():
    import mxfp4_routed_expert_v4moe_b200 as V
    assert V.v4moe_linear_w8a16_workspace_bytes(4, 64, 128) == 256 + 64 * 128 * 2
    assert V.v4moe_linear_w8a16_workspace_bytes(4, 0, 128) == 0
    # N % 32, K % 64, misaligned pointers: refused on the host
    assert V.v4moe_linear_w8a16(4, 48, 128, 16, 16, 16, 32, 256, 1 << 20, 0) == V.V4MOE_ERR_INVALID_ARG
    assert V.v4moe_linear_w8a16(4, 64, 96, 16, 16, 16, 32, 256, 1 << 20, 0) == V.V4MOE_ERR_INVALID_ARG
    assert V.v4moe_linear_w8a16(4, 64, 128, 16, 8, 16, 32, 256, 1 << 20, 0) == V.V4MOE_ERR_INVALID_ARG
    assert V.v4moe_linear_w8a16(4, 64, 128, 16, 16, 16, 32, 256, 100, 0) == V.V4MOE_ERR_WORKSPACE
    assert V.v4moe_linear_w8a16_grouped_workspace_bytes(4, 8, 64, 128) == 256 + 8 * 64 * 128 * 2
    assert V.v4moe_linear_w8a16_grouped_workspace_bytes(4, 0, 64, 128) == 0
    assert V.v4moe_linear_w8a16_grouped(4, 0, 64, 128, 16, 16, 16, 32, 256, 1 << 20, 0) == V.V4MOE_ERR_INVALID_ARG
    assert V.v4moe_linear_w8a16_grouped(4, 2, 48, 128, 16, 16, 16, 32, 256, 1 << 20, 0) == V.V4MOE_ERR_INVALID_ARG
    assert V.v4moe_linear_w8a16_grouped(4, 2, 64, 128, 16, 16, 16, 32, 256, 1000, 0) == V.V4MOE_ERR_WORKSPACE

