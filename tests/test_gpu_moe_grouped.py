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


def _many_groups():
    """1024 groups (the most a grouped call takes), nearly all empty: the group
    tables' scans cross every warp of their block, and the last group is used."""
    g = [0] * 1024
    g[3], g[517], g[1000], g[1023] = 128, 384, 256, 128
    return g


@pytest.mark.parametrize("group_rows,K,N", [
    ([256, 0, 128, 384, 128], 256, 384),
    ([128], 128, 128),
    ([0, 1152, 128, 0, 256, 640, 128, 128], 512, 256),
    (_many_groups(), 128, 128),
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


def test_grouped_config_vs_oracle(ora):
    """The grouped expert layer as the MoE benchmark runs it (64 experts, hidden 2048,
    expert FFN 1024, 16384 tokens, top-4 of Zipf(1.1), segments padded to 128 rows),
    checked against the oracle directly: for the largest, the smallest and a middle
    expert every grouped operand byte (codes and swizzled scales) and every tensor
    scale, and a 32 x 32 grid of sampled outputs of Y, dX and dW[e] within the bound.
    The largest expert's wgrad reduces over its whole row range (45+ k-tiles)."""
    s = syn.MOE
    E, K, N = s["experts"], s["hidden"], s["ffn"]
    d = syn.moe_inputs(s["tokens"], E, K, N, s["topk"], s["zipf_s"], seed=0, pad=128)
    g = d["group_rows"]
    R = int(g.sum())
    offs = np.concatenate([[0], np.cumsum(g)]).astype(np.int64)
    signs = syn.rht_signs(0)
    seed = 4242

    x_tok = to_dev_bf16(d["X"])
    W = to_dev_bf16(d["W"].reshape(E * N, K)).view(E, N, K)
    dY = to_dev_bf16(d["dY"])
    row_src = torch.from_numpy(d["row_src"]).to(DEV)
    Y, dX, dW = nan_bf16(R, N), nan_bf16(R, K), nan_bf16(E, N, K)
    ws = torch.empty(capi.moe_grouped_workspace_bytes(g, K, N), dtype=torch.uint8, device=DEV)
    # as the benchmark runs it: the gather fused into the quantization of X
    capi.nvfp4_moe_grouped_fprop_gather(x_tok, row_src, W, Y, g, signs, ws)
    capi.nvfp4_moe_grouped_dgrad(dY, dX, g, seed, signs, ws)
    capi.nvfp4_moe_grouped_wgrad(dW, g, ws)
    torch.cuda.synchronize()
    assert capi.nvfp4_read_status(ws) == 0

    # the routed tokens' rows in expert order (padding rows zero), gathered on the host
    rs = d["row_src"]
    xp = np.zeros((R, K), np.uint16)
    xp[rs >= 0] = d["X"][rs[rs >= 0]]

    views = {w: grouped_view(ws, g, K, N, w) for w in range(6)}
    kinds = {capi.LIN_X_ROW: "rows", capi.LIN_X_COL: "cols", capi.LIN_W_ROW: "wrows",
             capi.LIN_W_COL: "wcols", capi.LIN_DY_ROW: "rows", capi.LIN_DY_COL: "cols"}
    order = np.argsort(g)
    for e in (int(order[-1]), int(order[0]), int(order[len(order) // 2])):
        off, m = int(offs[e]), int(g[e])
        Xe, We, dYe = xp[off:off + m], d["W"][e], d["dY"][off:off + m]
        specs = {capi.LIN_X_ROW: (Xe, 0, False, 0, 0, 0), capi.LIN_X_COL: (Xe, 1, True, 0, 0, 0),
                 capi.LIN_W_ROW: (We, 0, False, 1, 0, 0), capi.LIN_W_COL: (We, 1, False, 1, 0, 0),
                 capi.LIN_DY_ROW: (dYe, 0, False, 0, 1, seed + e),
                 capi.LIN_DY_COL: (dYe, 1, True, 0, 1, seed + e)}
        ref = {}
        for which, (src, orient, rht, bm, rnd, sd) in specs.items():
            p, sf, gg, _ = ora.quantize(src, orient, rht, signs, bm, rnd, sd)
            gv, gdata, gsf, gscale = views[which]
            dd, ss = expert_slice(kinds[which], gv, gdata, gsf, e, off, m, N)
            assert np.array_equal(dd, p), (e, which)
            assert np.array_equal(ss, ora.sf_swizzle(sf, p.shape[1] * 2)), (e, which)
            assert gscale[e].view(np.uint32) == np.float32(gg).view(np.uint32), (e, which)
            ref[which] = (p, sf, float(gg))
        rng = np.random.default_rng(e)
        for out, a, b, alpha in ((Y[off:off + m], capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0),
                                 (dX[off:off + m], capi.LIN_DY_ROW, capi.LIN_W_COL, 1.0),
                                 (dW[e], capi.LIN_DY_COL, capi.LIN_X_COL, 1.0 / 16)):
            pa, sa, ga = ref[a]
            pb, sb, gb = ref[b]
            mi = np.repeat(rng.choice(pa.shape[0], 32, replace=pa.shape[0] < 32), 32)
            ni = np.tile(rng.choice(pb.shape[0], 32, replace=False), 32)
            r, bound = ora.gemm_pairs(pa, sa, pb, sb, alpha * ga * gb, mi, ni)
            got = out.float()[torch.from_numpy(mi).to(DEV), torch.from_numpy(ni).to(DEV)]
            got = got.cpu().numpy().astype(np.float64)
            # fp32 value v within 1e-4 * bound of the exact r, then one bf16 rounding:
            # half an ulp of v, at most 2^-8 |v| (8 significant bits)
            lim = 1e-4 * bound * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(r) + 1e-30
            assert (np.abs(got - r) <= lim).all(), (e, a)


def test_fused_gather_equals_gather_then_grouped():
    """nvfp4_moe_grouped_fprop_gather (X's rows read through row_src inside the
    quantizer) leaves the same X and W operands, tensor scales and Y as the gather
    kernel followed by nvfp4_moe_grouped_fprop; an index past the token rows is
    reported as NVFP4_ERR_INDEX and read as a zero row."""
    E, K, N, T, k = 6, 256, 384, 300, 2
    d = syn.moe_inputs(T, E, K, N, k, 1.1, seed=5, pad=128)
    g = d["group_rows"]
    R = int(g.sum())
    signs = syn.rht_signs(1)
    x_tok = to_dev_bf16(d["X"])
    W = to_dev_bf16(d["W"].reshape(E * N, K)).view(E, N, K)
    row_src = torch.from_numpy(d["row_src"]).to(DEV)

    ws_a = torch.empty(capi.moe_grouped_workspace_bytes(g, K, N), dtype=torch.uint8, device=DEV)
    ws_b = torch.empty_like(ws_a)
    X_perm = torch.empty((R, K), dtype=torch.bfloat16, device=DEV)
    Ya, Yb = nan_bf16(R, N), nan_bf16(R, N)
    capi.nvfp4_moe_gather(x_tok, row_src, X_perm)
    capi.nvfp4_moe_grouped_fprop(X_perm, W, Ya, g, signs, ws_a)
    capi.nvfp4_moe_grouped_fprop_gather(x_tok, row_src, W, Yb, g, signs, ws_b)
    torch.cuda.synchronize()
    assert capi.nvfp4_read_status(ws_a) == 0 and capi.nvfp4_read_status(ws_b) == 0
    assert torch.equal(bits(Ya), bits(Yb))
    for which in (capi.LIN_X_ROW, capi.LIN_X_COL, capi.LIN_W_ROW, capi.LIN_W_COL):
        _, da, sa, ga = grouped_view(ws_a, g, K, N, which)
        _, db, sb, gb = grouped_view(ws_b, g, K, N, which)
        assert np.array_equal(da, db) and np.array_equal(sa, sb), which
        assert np.array_equal(ga.view(np.uint32), gb.view(np.uint32)), which

    bad = d["row_src"].copy()
    first_real = int(np.nonzero(bad >= 0)[0][0])
    bad[first_real] = T + 7  # past the token rows
    capi.nvfp4_moe_grouped_fprop_gather(x_tok, torch.from_numpy(bad).to(DEV), W, Yb, g, signs, ws_b)
    torch.cuda.synchronize()
    assert capi.nvfp4_read_status(ws_b) == capi.ERR_INDEX
