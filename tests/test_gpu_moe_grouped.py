"""Grouped expert layer (nvfp4_moe_grouped_*) against the per-expert calls
(nvfp4_moe_linear_*), which the oracle pins expert by expert (test_gpu_moe.py).  On
ragged 128-row groups, empty experts included, every quantized operand byte, every
per-expert tensor scale and every output element must be identical; an empty
expert's dW is zero."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, to_dev_bf16, u8
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def nan_bf16(*shape):
    return torch.full(shape, float("nan"), dtype=torch.bfloat16, device=DEV)


def bits(t):
    return t.view(torch.int16)


def ws_bytes(ws, ptr, n):
    base = ws.data_ptr()
    return u8(ws[ptr - base: ptr - base + n])


def grouped_view(ws, g, K, N, which):
    v = capi.nvfp4_moe_grouped_operand(ws, g, K, N, which)
    data = ws_bytes(ws, v.data, v.rows * v.cols // 2).reshape(v.rows, v.cols // 2)
    sf = ws_bytes(ws, v.scales, capi.scale_bytes(v.rows, v.cols))
    gs = np.frombuffer(ws_bytes(ws, v.tensor_scale, 4 * len(g)).tobytes(), dtype=np.float32)
    return v, data, sf, gs


def expert_view(ws, g, K, N, e, which):
    base, _ = capi.nvfp4_moe_expert_workspace(ws, g, K, N, e)

    class View:
        def data_ptr(self):
            return base
    v = capi.nvfp4_linear_operand(View(), int(g[e]), K, N, which)
    data = ws_bytes(ws, v.data, v.rows * v.cols // 2).reshape(v.rows, v.cols // 2)
    sf = ws_bytes(ws, v.scales, capi.scale_bytes(v.rows, v.cols))
    gs = np.frombuffer(ws_bytes(ws, v.tensor_scale, 4).tobytes(), dtype=np.float32)[0]
    return v, data, sf, gs


def atoms(sf, rows, cols):
    """Scale bytes as [128-row group][k atom][512]."""
    return sf.reshape((rows + 127) // 128, -1, 512)


def expert_slice(kind, gv, gdata, gsf, e, off, m, N):
    """The part of a grouped operand that belongs to expert e, in the per-expert layout."""
    if kind == "rows":       # [R][C]: the expert's rows
        r0, r1 = off, off + m
        return gdata[r0:r1], atoms(gsf, gv.rows, gv.cols)[r0 // 128: r1 // 128].ravel()
    if kind == "wrows":      # [E*N][K]: rows e*N ..
        r0, r1 = e * N, (e + 1) * N
        return gdata[r0:r1], atoms(gsf, gv.rows, gv.cols)[r0 // 128: r1 // 128].ravel()
    if kind == "cols":       # [C][R]: the expert's columns
        c0, c1 = off, off + m
    else:                    # "wcols": [K][E*N]: columns e*N ..
        c0, c1 = e * N, (e + 1) * N
    return (gdata[:, c0 // 2: c1 // 2],
            atoms(gsf, gv.rows, gv.cols)[:, c0 // 64: c1 // 64].ravel())


@pytest.mark.parametrize("group_rows,K,N", [
    ([256, 0, 128, 384, 128], 256, 384),
    ([128], 128, 128),
    ([0, 1152, 128, 0, 256, 640, 128, 128], 512, 256),
])
def test_grouped_equals_per_expert(group_rows, K, N):
    g = np.array(group_rows, dtype=np.int64)
    E, R = len(g), int(g.sum())
    offs = np.concatenate([[0], np.cumsum(g)]).astype(np.int64)
    X = to_dev_bf16(syn.normal_bf16((R, K), 11, outlier_prob=0.01))
    W = to_dev_bf16(syn.normal_bf16((E * N, K), 12, std=0.02)).view(E, N, K)
    dY = to_dev_bf16(syn.normal_bf16((R, N), 13, std=1e-3))
    signs = syn.rht_signs(5)
    seed = 123

    wsg = torch.empty(capi.moe_grouped_workspace_bytes(g, K, N), dtype=torch.uint8, device=DEV)
    Yg, dXg, dWg = nan_bf16(R, N), nan_bf16(R, K), nan_bf16(E, N, K)
    capi.nvfp4_moe_grouped_fprop(X, W, Yg, g, signs, wsg)
    capi.nvfp4_moe_grouped_dgrad(dY, dXg, g, seed, signs, wsg)
    capi.nvfp4_moe_grouped_wgrad(dWg, g, wsg)

    wsp = torch.empty(capi.moe_workspace_bytes(g, K, N), dtype=torch.uint8, device=DEV)
    Yp, dXp, dWp = nan_bf16(R, N), nan_bf16(R, K), nan_bf16(E, N, K)
    capi.nvfp4_moe_linear_fprop(X, W, Yp, g, signs, wsp)
    capi.nvfp4_moe_linear_dgrad(dY, dXp, g, seed, signs, wsp)
    capi.nvfp4_moe_linear_wgrad(dWp, g, seed, signs, wsp)
    torch.cuda.synchronize()
    assert capi.nvfp4_read_status(wsg) == 0

    assert torch.equal(bits(Yg), bits(Yp))
    assert torch.equal(bits(dXg), bits(dXp))
    for e in range(E):
        if g[e]:
            assert torch.equal(bits(dWg[e]), bits(dWp[e])), e
        else:
            assert int(bits(dWg[e]).abs().max()) == 0, e

    kinds = {capi.LIN_X_ROW: "rows", capi.LIN_X_COL: "cols", capi.LIN_W_ROW: "wrows",
             capi.LIN_W_COL: "wcols", capi.LIN_DY_ROW: "rows", capi.LIN_DY_COL: "cols"}
    for which, kind in kinds.items():
        gv, gdata, gsf, gg = grouped_view(wsg, g, K, N, which)
        for e in range(E):
            if not g[e]:
                continue
            _, pdata, psf, pg = expert_view(wsp, g, K, N, e, which)
            d, s = expert_slice(kind, gv, gdata, gsf, e, int(offs[e]), int(g[e]), N)
            assert np.array_equal(d, pdata), (which, e)
            assert np.array_equal(s, psf), (which, e)
            assert gg[e].view(np.uint32) == np.float32(pg).view(np.uint32), (which, e)


def test_grouped_rejects_unaligned_groups():
    g = np.array([128, 64], dtype=np.int64)
    assert capi.moe_grouped_workspace_bytes(g, 128, 128) == 0
    assert capi.moe_grouped_workspace_bytes(np.array([128], dtype=np.int64), 192, 128) == 0
