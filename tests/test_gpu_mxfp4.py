"""GPU parity of MXFP4, the comparison format (nvfp4_mx_quantize, nvfp4_mx_gemm),
against the oracle: codes and E8M0 scales byte for byte, the block-scaled GEMM
within the fp32 bound, and the end-to-end product (MXFP4 errs more than NVFP4 on
data with outliers: one power-of-two scale per 32 elements is blunter)."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, to_dev_bf16, to_dev_u8, u8
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu
TOL = 1e-4


def mx_quantize_gpu(x_bits):
    rows, cols = x_bits.shape
    packed = torch.full((rows * cols // 2,), 0xA5, dtype=torch.uint8, device=DEV)
    sf = torch.full((capi.mx_scale_bytes(rows, cols),), 0xA5, dtype=torch.uint8, device=DEV)
    capi.nvfp4_mx_quantize(to_dev_bf16(x_bits), packed, sf)
    torch.cuda.synchronize()
    return packed, sf


@pytest.mark.parametrize("rows,cols,kind", [(128, 256, "normal"), (300, 96, "outliers"),
                                            (64, 4096, "student"), (17, 32, "zeros"),
                                            (256, 640, "tiny")])
def test_mx_quantize_parity(ora, rows, cols, kind):
    if kind == "normal":
        x = syn.normal_bf16((rows, cols), 1)
    elif kind == "outliers":
        x = syn.normal_bf16((rows, cols), 2, outlier_prob=0.02)
    elif kind == "student":
        x = syn.student_t_bf16((rows, cols), 3)
    elif kind == "zeros":
        x = np.zeros((rows, cols), np.uint16)
        x[3, 5] = syn.f32_to_bf16_bits(np.array([-2.5], np.float32))[0]
    else:
        x = syn.normal_bf16((rows, cols), 4, std=1e-30)
    packed, sf = mx_quantize_gpu(x)
    p, s = ora.mx_quantize(x)
    assert np.array_equal(u8(packed).reshape(rows, cols // 2), p)
    assert np.array_equal(u8(sf), ora.mx_sf_swizzle(s, cols))


@pytest.mark.parametrize("M,N,K", [(128, 256, 128), (256, 512, 1024), (200, 136, 384),
                                   (128, 256, 2048), (640, 520, 1152)])
def test_mx_gemm_parity(ora, M, N, K):
    rng = np.random.default_rng(M + N + K)
    A = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    B = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sA = rng.integers(117, 138, (M, K // 32), dtype=np.uint8)
    sB = rng.integers(117, 138, (N, K // 32), dtype=np.uint8)
    D = torch.empty((M, N), dtype=torch.float32, device=DEV)
    D16 = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
    capi.nvfp4_mx_gemm(to_dev_u8(A), to_dev_u8(ora.mx_sf_swizzle(sA, K)), to_dev_u8(B),
                       to_dev_u8(ora.mx_sf_swizzle(sB, K)), 0.5, M, N, K, D_bf16=D16, D_f32=D)
    torch.cuda.synchronize()
    ref, bound = ora.mx_gemm(A, sA, B, sB, 0.5)
    got = D.cpu().numpy().astype(np.float64)
    assert (np.abs(got - ref) <= TOL * bound + 1e-30).all()
    assert torch.equal(D16, D.to(torch.bfloat16))


def test_mx_blunter_than_nvfp4(ora):
    M, N, K = 256, 256, 1024
    X = syn.normal_bf16((M, K), 7, outlier_prob=0.01)
    W = syn.normal_bf16((N, K), 8, std=0.02, outlier_prob=0.01)
    exact = syn.bf16_bits_to_f32(X).astype(np.float64) @ syn.bf16_bits_to_f32(W).astype(np.float64).T
    px, sx = mx_quantize_gpu(X)
    pw, sw = mx_quantize_gpu(W)
    D = torch.empty((M, N), dtype=torch.float32, device=DEV)
    capi.nvfp4_mx_gemm(px, sx, pw, sw, 1.0, M, N, K, D_f32=D)
    torch.cuda.synchronize()
    mx_err = np.linalg.norm(D.cpu().numpy() - exact) / np.linalg.norm(exact)
    ref, _ = ora.mx_gemm(*ora.mx_quantize(X), *ora.mx_quantize(W), 1.0)
    assert np.allclose(D.cpu().numpy(), ref, rtol=0, atol=1e-4 * np.abs(ref).max())
    qx, sfx, gx, _ = ora.quantize(X, 0, False, None, 0, 0)
    qw, sfw, gw, _ = ora.quantize(W, 0, False, None, 0, 0)
    nv, _ = ora.gemm(qx, sfx, qw, sfw, float(gx) * float(gw))
    nv_err = np.linalg.norm(nv - exact) / np.linalg.norm(exact)
    assert mx_err > nv_err
