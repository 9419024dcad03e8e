"""Host-side checks of the C ABI: the library loads, exports every symbol the header
declares, and rejects bad arguments synchronously (no CUDA call is made for those, so
these run without a GPU)."""

import ctypes
import os
import re

import pytest

import ternary_weight_linear_03_b200 as bl
from ternary_weight_linear_03_b200 import build as blbuild

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "bitlinear.h")


@pytest.fixture(scope="module")
def lib():
    blbuild.build()
    return bl.load_library()


def header_symbols():
    with open(HEADER) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(bitlinear_\w+)\s*\(", text)))


def test_header_declares_what_binding_lists():
    assert header_symbols() == sorted(bl.EXPORTS)


def test_library_exports_every_header_symbol(lib):
    for name in header_symbols():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


def test_status_strings(lib):
    for code, name in bl.bitlinear.STATUS.items():
        assert bl.status_string(code) == name
    assert bl.status_string(99) == "BL_ERR_UNKNOWN"


def test_workspace_size_rules(lib):
    assert bl.workspace_size(1, 256, 256) > 0
    assert bl.workspace_size(4096, 28672, 8192) >= 4096 * 8192 + 8 * 4096  # xq + scale + rowsum
    assert bl.workspace_size(4, 4096, 100) == 0       # K % 64 != 0
    assert bl.workspace_size(0, 4096, 1536) == 0      # M < 1
    assert bl.workspace_size(1, 1 << 20, 1 << 12) == 0  # N * K >= 2^31
    assert bl.workspace_size(1, 4096, 1536) % 256 == 0


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails its checks first


def test_argument_errors_are_synchronous(lib):
    f = lib.bitlinear_quantize_weights
    assert f(None, 0, 16, 64, 1e-5, FAKE, FAKE, FAKE, 1 << 20, None) == 1   # null W
    assert f(FAKE, 5, 16, 64, 1e-5, FAKE, FAKE, FAKE, 1 << 20, None) == 1   # bad dtype
    assert f(FAKE, 0, 16, 64, -1.0, FAKE, FAKE, FAKE, 1 << 20, None) == 1   # eps < 0
    assert f(FAKE, 0, 16, 64, float("nan"), FAKE, FAKE, FAKE, 1 << 20, None) == 1
    assert f(FAKE, 0, 16, 96, 1e-5, FAKE, FAKE, FAKE, 1 << 20, None) == 2   # K % 64
    assert f(FAKE + 4, 0, 16, 64, 1e-5, FAKE, FAKE, FAKE, 1 << 20, None) == 3  # misaligned
    assert f(FAKE, 0, 16, 64, 1e-5, FAKE, FAKE, FAKE, 16, None) == 7        # workspace
    g = lib.bitlinear_forward
    assert g(FAKE, 0, FAKE, FAKE, FAKE, 2, 1, 16, 64, FAKE, 1 << 20, None) == 1   # y int32
    assert g(FAKE, 0, FAKE, FAKE, FAKE, 0, 0, 16, 64, FAKE, 1 << 20, None) == 2   # M = 0
    assert g(FAKE, 0, FAKE, FAKE, FAKE + 8, 0, 1, 16, 64, FAKE, 1 << 20, None) == 3
    assert g(FAKE, 0, FAKE, FAKE, FAKE, 0, 64, 16, 64, FAKE, 16, None) == 7       # GEMM ws
    h = lib.bitlinear_contract_i32
    assert h(None, FAKE, FAKE, 1, 16, 64, FAKE, 1 << 20, None) == 1
    assert h(FAKE, FAKE, FAKE, 64, 16, 64, None, 0, None) == 7
    q = lib.bitlinear_quantize_acts
    assert q(FAKE, 0, 1, 63, FAKE, FAKE, None) == 2
    assert q(FAKE, 3, 1, 64, FAKE, FAKE, None) == 1
    assert lib.bitlinear_debug_timeout_probe(10, None) == 1                      # < 1 us


def test_tensor_parallel_entry_points_check_arguments(lib):
    a = lib.bitlinear_weight_abssum
    assert a(None, 0, 16, 64, FAKE, FAKE, 1 << 20, None) == 1
    assert a(FAKE, 0, 16, 96, FAKE, FAKE, 1 << 20, None) == 2
    assert a(FAKE, 0, 16, 64, FAKE + 8, FAKE, 1 << 20, None) == 3
    assert a(FAKE, 0, 16, 64, FAKE, FAKE, 16, None) == 7
    f = lib.bitlinear_quantize_weights_from_abssum
    assert f(FAKE, 0, 16, 64, 16 * 64, None, 1e-5, FAKE, FAKE, None) == 1
    assert f(FAKE, 0, 16, 64, 16 * 64 - 1, FAKE, 1e-5, FAKE, FAKE, None) == 1  # n_total < N*K
    assert f(FAKE, 0, 16, 64, 16 * 64, FAKE, -1.0, FAKE, FAKE, None) == 1
    assert f(FAKE, 0, 16, 64, 16 * 64, FAKE, 1e-5, FAKE + 4, FAKE, None) == 3
    m = lib.bitlinear_act_absmax
    assert m(FAKE, 2, 1, 64, FAKE, None) == 1
    assert m(FAKE, 0, 1, 65, FAKE, None) == 2
    q = lib.bitlinear_quantize_acts_absmax
    assert q(FAKE, 0, 1, 64, None, FAKE, FAKE, None) == 1
    assert q(FAKE, 0, 1, 64, FAKE, FAKE + 1, FAKE, None) == 3
    r = lib.bitlinear_rescale
    assert r(FAKE, FAKE, FAKE, FAKE, 2, 1, 16, None) == 1   # int32 out is not a rescale
    assert r(FAKE, FAKE, FAKE, FAKE, 0, 0, 16, None) == 2
    assert r(FAKE, FAKE, FAKE, FAKE + 2, 0, 1, 16, None) == 3
