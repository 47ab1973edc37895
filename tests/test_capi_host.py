"""CPU-only checks of the C ABI: the library builds and loads, exports every symbol
include/nvfp4.h declares, and its host-side size queries and argument validation
behave as documented.  Nothing here launches a kernel or touches a GPU: every
call below is rejected by the host checks before the first CUDA call."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from conftest import ROOT

HEADER = os.path.join(ROOT, "include", "nvfp4.h")


@pytest.fixture(scope="module")
def lib():
    from nvfp4_bit_quantized_amax_b200 import build, capi
    build.build()
    return capi.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


def test_header_and_binding_agree():
    from nvfp4_bit_quantized_amax_b200 import capi
    assert declared_functions() == sorted(capi.EXPORTS)


def test_every_declared_symbol_is_exported(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_sizes(lib):
    from nvfp4_bit_quantized_amax_b200 import capi
    assert capi.packed_bytes(8192, 5120) == 8192 * 5120 // 2
    assert capi.scale_bytes(8192, 5120) == 8192 * 5120 // 16
    assert capi.scale_bytes(300, 160) == 384 * 12  # rows pad to 128, blocks to 4
    assert capi.quantize_workspace_bytes() >= 64
    ws = capi.linear_workspace_bytes(8192, 5120, 20480)
    M, K, N = 8192, 5120, 20480
    payload = 2 * (M * K + N * K + M * N) * 9 // 16  # two orientations each, 4.5 bits
    assert payload <= ws <= payload + 64 * 1024
    assert lib.nvfp4_version() >= 100
    for s in range(-8, 1):
        assert lib.nvfp4_status_string(s)


def test_argument_validation_before_launch(lib):
    from nvfp4_bit_quantized_amax_b200 import capi
    p = C.c_void_p(4096)  # never dereferenced: every call fails validation first
    q = lib.nvfp4_quantize
    assert q(None, 16, 16, 0, 0, 0, p, p, p, p, None) == capi.ERR_ARG
    assert q(p, 16, 16, 0, 0, 0, p, p, p, None, None) == capi.ERR_WORKSPACE
    assert q(p, 16, 24, 0, 0, 0, p, p, p, p, None) == capi.ERR_SHAPE      # cols % 16
    assert q(p, 24, 32, 1, 0, 0, p, p, p, p, None) == capi.ERR_SHAPE      # 16x16 rows % 16
    assert q(p, 16, 16, 2, 0, 0, p, p, p, p, None) == capi.ERR_ARG        # block mode
    assert q(p, 16, 16, 0, 7, 0, p, p, p, p, None) == capi.ERR_ARG        # rounding
    assert q(C.c_void_p(4098), 16, 16, 0, 0, 0, p, p, p, p, None) == capi.ERR_ALIGN
    g = lib.nvfp4_gemm
    assert g(p, p, p, p, None, None, 1.0, 128, 128, 96, p, None, None, None) == capi.ERR_SHAPE
    assert g(p, p, p, p, None, None, 1.0, 128, 12, 128, p, None, None, None) == capi.ERR_SHAPE
    assert g(p, p, p, p, None, None, 1.0, 128, 128, 128, None, None, None, None) == capi.ERR_ARG
    bad = np.array([1] * 15 + [0], dtype=np.int8)
    good = np.array([1, -1] * 8, dtype=np.int8)
    assert lib.nvfp4_rht(p, 16, 16, 1, bad.ctypes.data_as(C.c_void_p), 16, p, None) == capi.ERR_ARG
    assert lib.nvfp4_rht(p, 16, 16, 1, good.ctypes.data_as(C.c_void_p), 8, p, None) == capi.ERR_ARG
    assert lib.nvfp4_rht(p, 8, 16, 0, good.ctypes.data_as(C.c_void_p), 16, p, None) == capi.ERR_SHAPE
    f = lib.nvfp4_linear_fprop
    sp = good.ctypes.data_as(C.c_void_p)
    need = lib.nvfp4_linear_workspace_bytes(128, 128, 128)
    assert f(p, p, p, 128, 128, 96, sp, p, need, None) == capi.ERR_SHAPE
    assert f(p, p, p, 128, 128, 128, sp, p, need - 1, None) == capi.ERR_WORKSPACE
    assert f(p, p, p, 128, 128, 128, None, p, need, None) == capi.ERR_ARG
    opts = capi.QuantizeOpts(1, 0, 0, 0, 1, sp)  # RHT is only defined for 1x16 blocks
    t = capi.Tensor(4096, 4096, 4096, 0, 0)
    assert lib.nvfp4_quantize_2d(p, 32, 32, C.byref(opts), None, C.byref(t), p, None) == capi.ERR_ARG


def test_linear_operand_views(lib):
    from nvfp4_bit_quantized_amax_b200 import capi

    class FakeWs:
        def data_ptr(self):
            return 1 << 20

    M, K, N = 256, 512, 768
    seen = []
    for which, (r, c) in enumerate([(M, K), (K, M), (N, K), (K, N), (M, N), (N, M)]):
        t = capi.nvfp4_linear_operand(FakeWs(), M, K, N, which)
        assert (t.rows, t.cols) == (r, c)
        assert t.data % 256 == 0 and t.scales % 256 == 0
        seen.append((t.data, t.data + r * c // 2))
        seen.append((t.scales, t.scales + capi.scale_bytes(r, c)))
    seen.sort()
    for (a0, a1), (b0, b1) in zip(seen, seen[1:]):
        assert a1 <= b0  # no two operands overlap
    assert seen[-1][1] <= (1 << 20) + capi.linear_workspace_bytes(M, K, N)
