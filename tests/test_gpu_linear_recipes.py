"""GPU parity of the linear layer's recipe options (nvfp4_linear_fprop_ex /
dgrad_ex) against the oracle: the 1D-weight recipe (W quantized 1x16 along K for
fprop and separately 1x16 along N for dgrad) and RHT on both dgrad operands (dY and
W^T rotated along N, alpha 1/16).  Quantized operands bit for bit, Y and dX within
the GEMM bound (plus the bf16 rounding of the fp32 value)."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, f32_bits, operand_tensor, to_dev_bf16
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu
TOL = 1e-4
BF16_REL = 2.0 ** -8


def ws_operand(ws, M, K, N, which):
    v = capi.nvfp4_linear_operand(ws, M, K, N, which)
    d, s, g = operand_tensor(v, v.rows * v.cols // 2, capi.scale_bytes(v.rows, v.cols), ws)
    return d.reshape(v.rows, v.cols // 2), s, g, (v.rows, v.cols)


@pytest.mark.parametrize("dgrad_rht", [0, 1])
@pytest.mark.parametrize("shape", [(256, 256, 256), (192, 320, 448)])
def test_recipe_options_parity(ora, dgrad_rht, shape):
    M, K, N = shape
    X = syn.normal_bf16((M, K), 31, outlier_prob=0.01)
    W = syn.normal_bf16((N, K), 32, std=0.02, outlier_prob=0.01)
    dY = syn.normal_bf16((M, N), 33, outlier_prob=0.01)
    signs = syn.rht_signs(8)
    seed = 0xABCD
    ws = torch.empty(capi.linear_workspace_bytes(M, K, N), dtype=torch.uint8, device=DEV)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=DEV)
    capi.nvfp4_linear_fprop_ex(to_dev_bf16(X), to_dev_bf16(W), Y, signs, ws,
                               weight_block_mode=capi.BLOCK_1X16, dgrad_rht=dgrad_rht)
    assert capi.nvfp4_read_status(ws) == 0
    capi.nvfp4_linear_dgrad_ex(to_dev_bf16(dY), dX, seed, signs, ws,
                               weight_block_mode=capi.BLOCK_1X16, dgrad_rht=dgrad_rht)
    assert capi.nvfp4_read_status(ws) == 0
    torch.cuda.synchronize()

    rot = bool(dgrad_rht)
    # (which, source, orient, rht, block_mode, rounding)
    specs = {capi.LIN_X_ROW: (X, 0, False, 0, 0),
             capi.LIN_W_ROW: (W, 0, False, 0, 0),
             capi.LIN_W_COL: (W, 1, rot, 0, 0),
             capi.LIN_DY_ROW: (dY, 0, rot, 0, 1),
             capi.LIN_DY_COL: (dY, 1, True, 0, 1)}
    ref = {}
    for which, (src, orient, rht, bm, rnd) in specs.items():
        p, sf, g, _ = ora.quantize(src, orient, rht, signs, bm, rnd, seed)
        ref[which] = (p, sf, g)
        gd, gs, gg, (vr, vc) = ws_operand(ws, M, K, N, which)
        assert np.array_equal(gd, p), f"operand {which} codes"
        assert np.array_equal(gs, ora.sf_swizzle(sf, vc)), f"operand {which} scales"
        assert f32_bits(gg) == f32_bits(g), f"operand {which} tensor scale"

    for out, a, b, alpha in ((Y, capi.LIN_X_ROW, capi.LIN_W_ROW, 1.0),
                             (dX, capi.LIN_DY_ROW, capi.LIN_W_COL, 1.0 / 16 if rot else 1.0)):
        pa, sa, ga = ref[a]
        pb, sb, gb = ref[b]
        r, bound = ora.gemm(pa, sa, pb, sb, alpha * float(ga) * float(gb))
        got = out.float().cpu().numpy().astype(np.float64)
        assert (np.abs(got - r) <= TOL * bound + BF16_REL * np.abs(r) + 1e-30).all()


def test_dgrad_rotation_estimates_product(ora):
    """Under the rotation dgrad still estimates dY W (the 1/16 undoes H H^T)."""
    X, W, dY = syn.linear_small_inputs(3)
    M, K = X.shape
    N = W.shape[0]
    ws = torch.empty(capi.linear_workspace_bytes(M, K, N), dtype=torch.uint8, device=DEV)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=DEV)
    signs = syn.rht_signs(2)
    capi.nvfp4_linear_fprop_ex(to_dev_bf16(X), to_dev_bf16(W), Y, signs, ws, capi.BLOCK_1X16, 1)
    capi.nvfp4_linear_dgrad_ex(to_dev_bf16(dY), dX, 5, signs, ws, capi.BLOCK_1X16, 1)
    torch.cuda.synchronize()
    exact = syn.bf16_bits_to_f32(dY).astype(np.float64) @ syn.bf16_bits_to_f32(W)
    got = dX.float().cpu().numpy()
    assert np.linalg.norm(got - exact) / np.linalg.norm(exact) < 0.3


def test_invalid_options_rejected():
    capi.load()
    M = K = N = 128
    ws = torch.empty(capi.linear_workspace_bytes(M, K, N), dtype=torch.uint8, device=DEV)
    x = torch.zeros((M, K), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((N, K), dtype=torch.bfloat16, device=DEV)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(capi.NVFP4Error):
        capi.nvfp4_linear_fprop_ex(x, w, y, syn.rht_signs(0), ws, capi.BLOCK_16X16, 1)
    with pytest.raises(capi.NVFP4Error):
        capi.nvfp4_linear_fprop_ex(x, w, y, syn.rht_signs(0), ws, 7, 0)
