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


def test_argument_validation_recipes_mx_moe(lib):
    """The recipe options, MXFP4, grouped-MoE, gather/combine and allocation-free
    entry points reject bad arguments on the host with the documented codes.  Every
    call here carries at least one invalid argument, so none reaches the device."""
    from nvfp4_bit_quantized_amax_b200 import capi
    p = C.c_void_p(4096)
    odd = C.c_void_p(4100)  # 4-byte but not 16-byte aligned
    sp = np.array([1, -1] * 8, dtype=np.int8)
    spp = sp.ctypes.data_as(C.c_void_p)
    need = lib.nvfp4_linear_workspace_bytes(128, 128, 128)

    # recipe options: invalid values, and the Mosaic rotation without 1x16 weights
    for wbm, rht in ((2, 0), (0, 2), (1, 1), (-1, 0)):
        o = capi.LinearOpts(wbm, rht)
        assert lib.nvfp4_linear_fprop_ex(p, p, p, 128, 128, 128, spp, C.byref(o), p, need,
                                         None) == capi.ERR_ARG
        assert lib.nvfp4_linear_dgrad_ex(p, p, 128, 128, 128, 0, spp, C.byref(o), p, need,
                                         None) == capi.ERR_ARG
    ok = capi.LinearOpts(0, 1)
    assert lib.nvfp4_linear_fprop_ex(p, p, p, 128, 128, 96, spp, C.byref(ok), p, need,
                                     None) == capi.ERR_SHAPE

    # MXFP4: 32-element blocks, K % 128 for the GEMM
    assert lib.nvfp4_mx_scale_bytes(128, 48) == 0
    assert lib.nvfp4_mx_scale_bytes(300, 320) == 384 * 12  # rows pad to 128, blocks to 4
    assert lib.nvfp4_mx_quantize(None, 128, 64, p, p, None) == capi.ERR_ARG
    assert lib.nvfp4_mx_quantize(p, 128, 48, p, p, None) == capi.ERR_SHAPE
    assert lib.nvfp4_mx_quantize(odd, 128, 64, p, p, None) == capi.ERR_ALIGN
    mg = lib.nvfp4_mx_gemm
    assert mg(p, p, p, p, 1.0, 128, 128, 192, p, None, None, None) == capi.ERR_SHAPE   # K % 128
    assert mg(p, p, p, p, 1.0, 128, 12, 128, p, None, None, None) == capi.ERR_SHAPE    # N % 8
    assert mg(p, p, p, p, 1.0, 128, 128, 128, None, None, None, None) == capi.ERR_ARG  # no output
    assert mg(p, odd, p, p, 1.0, 128, 128, 128, p, None, None, None) == capi.ERR_ALIGN

    # grouped MoE: group sizes multiples of 128 (0 allowed), K, N multiples of 128
    def g_ws(groups, K=128, N=128):
        return capi.moe_grouped_workspace_bytes(np.array(groups, dtype=np.int64), K, N)
    assert g_ws([128, 0, 256]) > 0
    assert g_ws([128, 64]) == 0           # ragged group
    assert g_ws([0, 0]) == 0              # no rows at all
    assert g_ws([128], K=192) == 0        # K % 128
    assert g_ws([128], N=64) == 0         # N % 128
    assert g_ws([128] * 1025) == 0        # more groups than the kernels take
    assert g_ws([-128, 256]) == 0
    groups = np.array([128, 0, 256], dtype=np.int64)
    gp = groups.ctypes.data_as(C.c_void_p)
    gneed = g_ws([128, 0, 256])
    f = lib.nvfp4_moe_grouped_fprop
    assert f(None, p, p, gp, 3, 128, 128, spp, p, gneed, None) == capi.ERR_ARG
    assert f(odd, p, p, gp, 3, 128, 128, spp, p, gneed, None) == capi.ERR_ALIGN
    assert f(p, p, p, gp, 3, 128, 128, None, p, gneed, None) == capi.ERR_ARG          # signs
    assert f(p, p, p, gp, 3, 128, 96, spp, p, gneed, None) == capi.ERR_SHAPE
    assert f(p, p, p, gp, 3, 128, 128, spp, None, gneed, None) == capi.ERR_WORKSPACE
    assert f(p, p, p, gp, 3, 128, 128, spp, C.c_void_p(4096 + 16), gneed, None) == capi.ERR_ALIGN
    assert f(p, p, p, gp, 3, 128, 128, spp, p, gneed - 1, None) == capi.ERR_WORKSPACE
    d = lib.nvfp4_moe_grouped_dgrad
    assert d(p, p, gp, 0, 128, 128, 0, spp, p, gneed, None) == capi.ERR_ARG            # E = 0
    assert d(p, p, gp, 3, 128, 128, 0, spp, p, gneed - 1, None) == capi.ERR_WORKSPACE
    w = lib.nvfp4_moe_grouped_wgrad
    assert w(None, gp, 3, 128, 128, p, gneed, None) == capi.ERR_ARG
    assert w(p, gp, 3, 128, 128, p, gneed - 1, None) == capi.ERR_WORKSPACE

    # gather / combine
    assert lib.nvfp4_moe_gather(p, p, 16, 12, p, None) == capi.ERR_SHAPE              # cols % 8
    assert lib.nvfp4_moe_gather(p, odd, 16, 16, odd, None) == capi.ERR_ALIGN
    assert lib.nvfp4_moe_combine(p, p, 16, 0, 16, p, None) == capi.ERR_ARG            # topk
    assert lib.nvfp4_moe_combine(p, p, 0, 4, 16, p, None) == capi.ERR_SHAPE

    # allocation-free quantize: the same checks as nvfp4_quantize
    nq = lib.nvfp4_quantize_noalloc
    assert nq(None, 16, 16, 0, 0, 0, p, p, p, None) == capi.ERR_ARG
    assert nq(p, 16, 24, 0, 0, 0, p, p, p, None) == capi.ERR_SHAPE
    assert nq(p, 24, 32, 1, 0, 0, p, p, p, None) == capi.ERR_SHAPE
    assert nq(p, 16, 16, 0, 5, 0, p, p, p, None) == capi.ERR_ARG
    assert nq(odd, 16, 16, 0, 0, 0, p, p, p, None) == capi.ERR_ALIGN


def test_moe_grouped_operand_views(lib):
    """The grouped workspace's operand views: whole-tensor shapes (rows summed over
    the experts, W stacked by expert), 256-byte aligned, no two overlapping, all
    inside the workspace; a view's tensor scales are one fp32 per expert."""
    from nvfp4_bit_quantized_amax_b200 import capi

    class FakeWs:
        def data_ptr(self):
            return 1 << 24

    groups = [256, 0, 128, 384]
    E, R, K, N = len(groups), sum(groups), 256, 384
    total = capi.moe_grouped_workspace_bytes(np.array(groups, dtype=np.int64), K, N)
    shapes = [(R, K), (K, R), (E * N, K), (K, E * N), (R, N), (N, R)]
    spans = []
    for which, (r, c) in enumerate(shapes):
        t = capi.nvfp4_moe_grouped_operand(FakeWs(), groups, K, N, which)
        assert (t.rows, t.cols) == (r, c)
        assert t.data % 256 == 0 and t.scales % 256 == 0
        spans.append((t.data, t.data + r * c // 2))
        spans.append((t.scales, t.scales + capi.scale_bytes(r, c)))
        spans.append((t.tensor_scale, t.tensor_scale + 4 * E))
    spans = sorted(set(spans))
    for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
        assert a1 <= b0
    assert spans[0][0] >= (1 << 24) and spans[-1][1] <= (1 << 24) + total
    with pytest.raises(RuntimeError):
        capi.nvfp4_moe_grouped_operand(FakeWs(), groups, K, N, 6)


def test_tile_row_limit(lib):
    """Tensors quantized by the tile kernel (two orientations or 16x16 blocks) take at
    most 65535 x 64 rows; one row tile more is a shape error, found on the host."""
    from nvfp4_bit_quantized_amax_b200 import capi
    p = C.c_void_p(4096)
    big = 65535 * 64 + 64
    q = lib.nvfp4_quantize
    assert q(p, big, 16, 1, 0, 0, p, p, p, p, None) == capi.ERR_SHAPE
    assert lib.nvfp4_quantize_noalloc(p, big, 16, 1, 0, 0, p, p, p, None) == capi.ERR_SHAPE
    opts = capi.QuantizeOpts(0, 0, 0, 0, 0, None)
    t = capi.Tensor(4096, 4096, 4096, 0, 0)
    assert lib.nvfp4_quantize_2d(p, big, 16, C.byref(opts), C.byref(t), None, p, None) == capi.ERR_SHAPE
    sp = np.array([1, -1] * 8, dtype=np.int8).ctypes.data_as(C.c_void_p)
    assert lib.nvfp4_linear_fprop(p, p, p, big, 64, 64, sp, p, 1 << 62, None) == capi.ERR_SHAPE
    assert lib.nvfp4_linear_fprop(p, p, p, 64, 64, big, sp, p, 1 << 62, None) == capi.ERR_SHAPE
    assert capi.moe_grouped_workspace_bytes(np.array([65535 * 64 + 128], dtype=np.int64), 128, 128) == 0
    # W of all experts [E*N][K] is one tile launch too: 1024 x 4096 rows is 64 too many
    assert capi.moe_grouped_workspace_bytes(np.array([128] * 1024, dtype=np.int64), 128, 4096) == 0
    assert capi.moe_grouped_workspace_bytes(np.array([128] * 1024, dtype=np.int64), 128, 3968) > 0
    g = np.array([big], dtype=np.int64)
    assert lib.nvfp4_moe_linear_fprop(p, p, p, g.ctypes.data_as(C.c_void_p), 1, 64, 64, sp, p,
                                      1 << 62, None) == capi.ERR_SHAPE
