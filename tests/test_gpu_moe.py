"""GPU parity of the mixture-of-experts expert layer (nvfp4_moe_*): routing gather and
combine, and per-expert NVFP4 fprop / dgrad / wgrad with per-expert tensor scales,
against the oracle applied expert by expert on the same padded segments."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, f32_bits, operand_tensor, to_dev_bf16
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu
TOL = 1e-4
BF16_REL = 2.0 ** -8


def run_moe(d, K, N, signs, seed):
    T = d["X"].shape[0]
    E = d["W"].shape[0]
    rows = int(d["group_rows"].sum())
    x_tok = to_dev_bf16(d["X"])
    W = to_dev_bf16(d["W"].reshape(E * N, K)).view(E, N, K)
    dY = to_dev_bf16(d["dY"])
    row_src = torch.from_numpy(d["row_src"]).to(DEV)
    slots = torch.from_numpy(d["slots"]).to(DEV)
    X_perm = torch.empty((rows, K), dtype=torch.bfloat16, device=DEV)
    Y = torch.empty((rows, N), dtype=torch.bfloat16, device=DEV)
    dX = torch.empty((rows, K), dtype=torch.bfloat16, device=DEV)
    dX_tok = torch.empty((T, K), dtype=torch.bfloat16, device=DEV)
    dW = torch.empty((E, N, K), dtype=torch.bfloat16, device=DEV)
    ws = torch.empty(capi.moe_workspace_bytes(d["group_rows"], K, N), dtype=torch.uint8, device=DEV)
    capi.nvfp4_moe_gather(x_tok, row_src, X_perm)
    capi.nvfp4_moe_linear_fprop(X_perm, W, Y, d["group_rows"], signs, ws)
    capi.nvfp4_moe_linear_dgrad(dY, dX, d["group_rows"], seed, signs, ws)
    capi.nvfp4_moe_combine(dX, slots, dX_tok)
    capi.nvfp4_moe_linear_wgrad(dW, d["group_rows"], seed, signs, ws)
    torch.cuda.synchronize()
    return ws, X_perm, Y, dX, dX_tok, dW


def expert_operand(ws, group_rows, K, N, e, which):
    base, nbytes = capi.nvfp4_moe_expert_workspace(ws, group_rows, K, N, e)

    class View:
        def data_ptr(self):
            return base
    v = capi.nvfp4_linear_operand(View(), int(group_rows[e]), K, N, which)
    d, s, g = operand_tensor(v, v.rows * v.cols // 2, capi.scale_bytes(v.rows, v.cols), ws)
    return d.reshape(v.rows, v.cols // 2), s, g


def check_expert(ora, d, ws, outs, K, N, e, signs, seed, full=True, nsamp=16):
    X_perm, Y, dX, dW = outs
    g = d["group_rows"]
    off = int(np.concatenate([[0], np.cumsum(g)])[e])
    m = int(g[e])
    Xe = X_perm.view(torch.int16).cpu().numpy()[off:off + m].view(np.uint16)
    We = d["W"][e]
    dYe = d["dY"][off:off + m]
    specs = {capi.LIN_X_ROW: (Xe, 0, False, 0, 0, 0), capi.LIN_X_COL: (Xe, 1, True, 0, 0, 0),
             capi.LIN_W_ROW: (We, 0, False, 1, 0, 0), capi.LIN_W_COL: (We, 1, False, 1, 0, 0),
             capi.LIN_DY_ROW: (dYe, 0, False, 0, 1, seed + e),
             capi.LIN_DY_COL: (dYe, 1, True, 0, 1, seed + e)}
    ref = {}
    for which, (src, orient, rht, bm, rnd, sd) in specs.items():
        p, sf, gg, _ = ora.quantize(src, orient, rht, signs, bm, rnd, sd)
        gd, gs, ggpu = expert_operand(ws, g, K, N, e, which)
        assert np.array_equal(gd, p), f"expert {e} operand {which}"
        vc = p.shape[1] * 2
        assert np.array_equal(gs, ora.sf_swizzle(sf, vc)), f"expert {e} operand {which} scales"
        assert f32_bits(ggpu) == f32_bits(gg)
        ref[which] = (p, sf, float(gg))
    rng = np.random.default_rng(e)
    for out, a, b, alpha, rows_out in ((Y[off:off + m], capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0, m),
                                       (dX[off:off + m], capi.LIN_DY_ROW, capi.LIN_W_COL, 1.0, m),
                                       (dW[e], capi.LIN_DY_COL, capi.LIN_X_COL, 1.0 / 16, N)):
        pa, sa, ga = ref[a]
        pb, sb, gb = ref[b]
        ncols = pb.shape[0]
        if full:
            r, bound = ora.gemm(pa, sa, pb, sb, alpha * ga * gb)
            got = out.float().cpu().numpy().astype(np.float64)
        else:
            mi = rng.integers(0, rows_out, nsamp * nsamp)
            ni = rng.integers(0, ncols, nsamp * nsamp)
            r, bound = ora.gemm_pairs(pa, sa, pb, sb, alpha * ga * gb, mi, ni)
            got = out.float()[torch.from_numpy(mi).to(DEV), torch.from_numpy(ni).to(DEV)].cpu().numpy()
        assert (np.abs(got - r) <= TOL * bound + BF16_REL * np.abs(r) + 1e-30).all(), f"expert {e}"


def test_moe_small_full(ora):
    E, K, N, T, topk = 6, 128, 192, 200, 2
    d = syn.moe_inputs(T, E, K, N, topk, 1.1, seed=3)
    signs = syn.rht_signs(2)
    seed = 99
    ws, X_perm, Y, dX, dX_tok, dW = run_moe(d, K, N, signs, seed)
    # gather: exact row copies, zero padding
    xp = X_perm.view(torch.int16).cpu().numpy().view(np.uint16)
    rs = d["row_src"]
    assert np.array_equal(xp[rs >= 0], d["X"][rs[rs >= 0]])
    assert (xp[rs < 0] == 0).all()
    for e in range(E):
        if d["group_rows"][e]:
            check_expert(ora, d, ws, (X_perm, Y, dX, dW), K, N, e, signs, seed)
    # combine: fp32 sum of each token's routed rows, rounded to bf16
    dxp = dX.float().cpu().numpy().astype(np.float64)
    exact = dxp[d["slots"]].sum(axis=1)
    got = dX_tok.float().cpu().numpy()
    assert (np.abs(got - exact) <= 2.0 ** -8 * np.abs(exact) + 1e-6 * np.abs(dxp).max()).all()


def test_moe_config_sampled(ora):
    """64 experts, hidden 2048, expert FFN 1024, 16384 tokens, top-4 of Zipf(1.1): every
    operand of the largest, the smallest and a middle expert bit for bit, a grid of
    sampled outputs of each of their GEMMs within the bound."""
    s = syn.MOE
    d = syn.moe_inputs(s["tokens"], s["experts"], s["hidden"], s["ffn"], s["topk"], s["zipf_s"], seed=0)
    K, N = s["hidden"], s["ffn"]
    signs = syn.rht_signs(0)
    seed = 4242
    ws, X_perm, Y, dX, dX_tok, dW = run_moe(d, K, N, signs, seed)
    counts = d["group_rows"]
    order = np.argsort(counts)
    for e in (int(order[-1]), int(order[0]), int(order[len(order) // 2])):
        check_expert(ora, d, ws, (X_perm, Y, dX, dW), K, N, e, signs, seed, full=False)
