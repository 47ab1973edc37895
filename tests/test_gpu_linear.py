"""GPU parity of the NVFP4 linear training step (nvfp4_linear_fprop / dgrad / wgrad)
against the oracle: every quantized operand the step keeps in its workspace bit
for bit, and Y, dX, dW within the GEMM bound (bf16 outputs: the bound plus the
bf16 rounding of the fp32 value)."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, f32_bits, operand_tensor, to_dev_bf16
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu
TOL = 1e-4
BF16_REL = 2.0 ** -8  # round-to-nearest into 8 significant bits


def run_step(X, W, dY, signs, seed, wgrad_from_dy=False):
    M, K = X.shape
    N = W.shape[0]
    ws = torch.empty(capi.linear_workspace_bytes(M, K, N), dtype=torch.uint8, device=DEV)
    x, w, dy = to_dev_bf16(X), to_dev_bf16(W), to_dev_bf16(dY)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=DEV)
    dW = torch.empty((N, K), dtype=torch.bfloat16, device=DEV)
    capi.nvfp4_linear_fprop(x, w, Y, signs, ws)
    assert capi.nvfp4_read_status(ws) == 0
    capi.nvfp4_linear_dgrad(dy, dX, seed, signs, ws)
    assert capi.nvfp4_read_status(ws) == 0
    capi.nvfp4_linear_wgrad(dy if wgrad_from_dy else None, dW, M, seed, signs, ws)
    assert capi.nvfp4_read_status(ws) == 0
    torch.cuda.synchronize()
    return ws, Y, dX, dW


# (which, source tensor, orient, rht, block_mode, rounding, stream-seeded)
OPERANDS = {
    capi.LIN_X_ROW: ("X", 0, False, 0, 0),
    capi.LIN_X_COL: ("X", 1, True, 0, 0),
    capi.LIN_W_ROW: ("W", 0, False, 1, 0),
    capi.LIN_W_COL: ("W", 1, False, 1, 0),
    capi.LIN_DY_ROW: ("dY", 0, False, 0, 1),
    capi.LIN_DY_COL: ("dY", 1, True, 0, 1),
}


def ws_operand(ws, M, K, N, which):
    v = capi.nvfp4_linear_operand(ws, M, K, N, which)
    d, s, g = operand_tensor(v, v.rows * v.cols // 2, capi.scale_bytes(v.rows, v.cols), ws)
    return d.reshape(v.rows, v.cols // 2), s, g, (v.rows, v.cols)


def test_linear_256_outliers_full_parity(ora):
    """256^3 layer, N(0,1) with 1% x50 outliers: everything compared in full."""
    X, W, dY = syn.linear_small_inputs(0)
    signs = syn.rht_signs(0)
    seed = 0x5EED
    M, K = X.shape
    N = W.shape[0]
    ws, Y, dX, dW = run_step(X, W, dY, signs, seed)
    src = {"X": X, "W": W, "dY": dY}
    ref = {}
    for which, (name, orient, rht, bm, rnd) in OPERANDS.items():
        p, sf, g, amax = ora.quantize(src[name], orient, rht, signs, bm, rnd, seed)
        ref[which] = (p, sf, g)
        gd, gs, gg, (vr, vc) = ws_operand(ws, M, K, N, which)
        assert np.array_equal(gd, p), f"operand {which} codes"
        assert np.array_equal(gs, ora.sf_swizzle(sf, vc)), f"operand {which} scales"
        assert f32_bits(gg) == f32_bits(g), f"operand {which} tensor scale"

    def gemm_ref(a, b, alpha):
        pa, sa, ga = ref[a]
        pb, sb, gb = ref[b]
        return ora.gemm(pa, sa, pb, sb, alpha * float(ga) * float(gb))

    for out, (a, b, alpha) in ((Y, (capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0)),
                               (dX, (capi.LIN_DY_ROW, capi.LIN_W_COL, 1.0)),
                               (dW, (capi.LIN_DY_COL, capi.LIN_X_COL, 1.0 / 16))):
        r, bound = gemm_ref(a, b, alpha)
        got = out.float().cpu().numpy().astype(np.float64)
        assert (np.abs(got - r) <= TOL * bound + BF16_REL * np.abs(r) + 1e-30).all()

    # the fp32 values before the bf16 rounding, through nvfp4_gemm on the same operands
    for a, b, alpha, shape in ((capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0, (M, N)),
                               (capi.LIN_DY_COL, capi.LIN_X_COL, 1.0 / 16, (N, K))):
        va = capi.nvfp4_linear_operand(ws, M, K, N, a)
        vb = capi.nvfp4_linear_operand(ws, M, K, N, b)
        D = torch.empty(shape, dtype=torch.float32, device=DEV)
        lib = capi.load()
        rc = lib.nvfp4_gemm(va.data, va.scales, vb.data, vb.scales, va.tensor_scale,
                            vb.tensor_scale, alpha, va.rows, vb.rows, va.cols, None,
                            D.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
        assert rc == 0
        torch.cuda.synchronize()
        r, bound = gemm_ref(a, b, alpha)
        assert (np.abs(D.cpu().numpy().astype(np.float64) - r) <= TOL * bound + 1e-30).all()


def test_linear_wgrad_requantizes_same_dy(ora):
    X, W, dY = syn.linear_small_inputs(1)
    signs = syn.rht_signs(4)
    _, _, _, dW_a = run_step(X, W, dY, signs, 77)
    _, _, _, dW_b = run_step(X, W, dY, signs, 77, wgrad_from_dy=True)
    assert torch.equal(dW_a.view(torch.int16), dW_b.view(torch.int16))


def test_linear_rht_cancels(ora):
    """With the rotation the wgrad product still estimates dY^T X (the transform is
    undone by the 1/16); compare against the exact product of the bf16 inputs."""
    X, W, dY = syn.linear_small_inputs(2)
    _, _, _, dW = run_step(X, W, dY, syn.rht_signs(9), 3)
    exact = syn.bf16_bits_to_f32(dY).astype(np.float64).T @ syn.bf16_bits_to_f32(X)
    got = dW.float().cpu().numpy()
    assert np.linalg.norm(got - exact) / np.linalg.norm(exact) < 0.3


def test_linear_mlp_12b_sampled(ora):
    """The 8192 x 5120 -> 20480 up-projection step at full size: tensor scales
    exactly, 64 sampled rows of every operand bit for bit, 1024 sampled outputs of
    each GEMM within the bound."""
    s = syn.MLP_12B
    M, K, N = s["M"], s["K"], s["N"]
    X, W, dY = syn.mlp_inputs(M, K, N, seed=0)
    signs = syn.rht_signs(0)
    seed = 12345
    ws, Y, dX, dW = run_step(X, W, dY, signs, seed)
    src = {"X": X, "W": W, "dY": dY}
    rng = np.random.default_rng(0)
    amax = {}
    rows_cache = {}
    for which, (name, orient, rht, bm, rnd) in OPERANDS.items():
        key = (name, orient, rht)
        if key not in amax:
            amax[key] = ora.tensor_amax(src[name], orient, rht, signs)
        gd, gs, gg, (vr, vc) = ws_operand(ws, M, K, N, which)
        assert f32_bits(gg) == f32_bits(ora.tensor_scale(amax[key])), f"operand {which} g"
        step = 16 if bm == 1 else 1
        picks = np.sort(rng.choice(vr // step, 64 if step == 1 else 8, replace=False)) * step
        inner = None
        for r0 in picks:
            r1 = int(r0) + step
            p, sf = ora.quantize_rows(src[name], orient, rht, signs, bm, rnd, seed, amax[key],
                                      int(r0), r1)
            assert np.array_equal(gd[r0:r1], p), f"operand {which} rows {r0}"
            for i in range(r1 - int(r0)):
                offs = [ora.sf_offset(int(r0) + i, kb, vc) for kb in range(vc // 16)]
                assert np.array_equal(gs[offs], sf[i]), f"operand {which} scales row {r0 + i}"
        rows_cache[which] = (gd, gs, gg, vc)

    def sampled(out, a, b, alpha, nrows, ncols, bf16=True):
        # a 32 x 32 grid of outputs: 32 sampled rows of each operand, all pairs; bf16
        # outputs get the half-ulp of their rounding (8 significant bits: 2^-8 |r|)
        ra_idx = np.sort(rng.choice(nrows, 32, replace=False))
        rb_idx = np.sort(rng.choice(ncols, 32, replace=False))
        mi = np.repeat(ra_idx, 32)
        ni = np.tile(rb_idx, 32)
        Kred = rows_cache[a][3]
        # quantize exactly the rows the samples need (16-row groups for 16x16)
        def rows_of(which, idx):
            name, orient, rht, bm, rnd = OPERANDS[which]
            key = (name, orient, rht)
            out_p, out_s = [], []
            for r in idx:
                r0 = (int(r) // 16) * 16 if bm == 1 else int(r)
                p, sf = ora.quantize_rows(src[name], orient, rht, signs, bm, rnd, seed, amax[key],
                                          r0, r0 + (16 if bm == 1 else 1))
                out_p.append(p[int(r) - r0])
                out_s.append(sf[int(r) - r0])
            return np.array(out_p), np.array(out_s)
        ua, ia = np.unique(mi, return_inverse=True)
        ub, ib = np.unique(ni, return_inverse=True)
        pa, sa = rows_of(a, ua)
        pb, sb = rows_of(b, ub)
        ga, gb = rows_cache[a][2], rows_cache[b][2]
        ref, bound = ora.gemm_pairs(pa, sa, pb, sb, alpha * float(ga) * float(gb), ia, ib)
        got = out[torch.from_numpy(mi).to(DEV), torch.from_numpy(ni).to(DEV)].float().cpu().numpy()
        err = np.abs(got.astype(np.float64) - ref)
        assert (err <= TOL * bound + (BF16_REL * np.abs(ref) if bf16 else 0.0) + 1e-30).all()
        assert Kred == pa.shape[1] * 2

    sampled(Y, capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0, M, N)
    sampled(dX, capi.LIN_DY_ROW, capi.LIN_W_COL, 1.0, M, K)
    sampled(dW, capi.LIN_DY_COL, capi.LIN_X_COL, 1.0 / 16, N, K)

    # the fp32 values before the bf16 rounding: nvfp4_gemm with an fp32 output on the
    # step's own operands, at full size, sampled with the accumulation bound alone
    lib = capi.load()
    for a, b, alpha, shape in ((capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0, (M, N)),
                               (capi.LIN_DY_ROW, capi.LIN_W_COL, 1.0, (M, K)),
                               (capi.LIN_DY_COL, capi.LIN_X_COL, 1.0 / 16, (N, K))):
        va = capi.nvfp4_linear_operand(ws, M, K, N, a)
        vb = capi.nvfp4_linear_operand(ws, M, K, N, b)
        D = torch.empty(shape, dtype=torch.float32, device=DEV)
        rc = lib.nvfp4_gemm(va.data, va.scales, vb.data, vb.scales, va.tensor_scale,
                            vb.tensor_scale, alpha, va.rows, vb.rows, va.cols, None,
                            D.data_ptr(), None, torch.cuda.current_stream().cuda_stream)
        assert rc == 0
        torch.cuda.synchronize()
        sampled(D, a, b, alpha, shape[0], shape[1], bf16=False)
        del D
