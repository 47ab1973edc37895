"""GPU parity of the block-scaled FP4 GEMM (nvfp4_gemm) against the oracle's fp64
GEMM over the same dequantized operands.  The fp32 output (before the bf16
rounding) must satisfy |D - D_ref| <= 1e-4 * sum_k |a_mk b_nk| per element; the
bf16 output must be the round-to-nearest-even of that fp32 value."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, to_dev_u8
from nvfp4_bit_quantized_amax_b200 import capi
from nvfp4_bit_quantized_amax_b200 import synthetic as syn

pytestmark = pytest.mark.gpu
TOL = 1e-4


def random_operand(ora, rows, K, rng, sf_lo=0x20, sf_hi=0x58):
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    sf = rng.integers(sf_lo, sf_hi, size=(rows, K // 16), dtype=np.uint8)
    return codes, sf, ora.sf_swizzle(sf, K)


def run_gemm(A, sfA_sw, B, sfB_sw, M, N, K, alpha=1.0, ga=None, gb=None):
    D32 = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
    D16 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    sa = torch.tensor([ga], dtype=torch.float32, device=DEV) if ga is not None else None
    sb = torch.tensor([gb], dtype=torch.float32, device=DEV) if gb is not None else None
    capi.nvfp4_gemm(to_dev_u8(A), to_dev_u8(sfA_sw), to_dev_u8(B), to_dev_u8(sfB_sw), alpha, M,
                    N, K, D_bf16=D16, D_f32=D32, scale_a=sa, scale_b=sb, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return D32, D16


def check(D32, D16, ref, bound, what):
    d = D32.cpu().numpy().astype(np.float64)
    err = np.abs(d - ref)
    lim = TOL * bound + 1e-30
    bad = np.nonzero(err > lim)
    assert bad[0].size == 0, (f"{what}: {bad[0].size} outputs off, first ({bad[0][0]},{bad[1][0]}) "
                              f"got {d[bad][0]} ref {ref[bad][0]}")
    assert torch.equal(D32.to(torch.bfloat16).view(torch.int16), D16.view(torch.int16)), what


@pytest.mark.parametrize("M,N,K", [
    (128, 256, 256),      # one tile, one k-tile
    (128, 256, 64),       # one MMA
    (256, 512, 1024),     # several tiles, k-tiles > stages
    (200, 136, 320),      # ragged M, N; partial last k-tile
    (256, 256, 768),      # odd number of 256-deep k-tiles (last stage half empty)
    (128, 512, 1344),     # K % 256 == 64: k-tile slabs loaded one by one
    (384, 1024, 4096),
    (1, 8, 128),          # degenerate tiny output
])
def test_gemm_random_operands(ora, M, N, K):
    rng = np.random.default_rng(M * 7 + N * 3 + K)
    A, sA, sA_sw = random_operand(ora, M, K, rng)
    B, sB, sB_sw = random_operand(ora, N, K, rng)
    D32, D16 = run_gemm(A, sA_sw, B, sB_sw, M, N, K)
    ref, bound = ora.gemm(A, sA, B, sB, 1.0)
    check(D32, D16, ref, bound, f"{M}x{N}x{K}")


def test_gemm_integer_special_case_exact(ora):
    """All block scales 1.0: the fp32 result is exact (|D| < 2^24 quarter units)."""
    rng = np.random.default_rng(1)
    M, N, K = 256, 512, 4096
    A = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    B = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sA = np.full((M, K // 16), 0x38, np.uint8)
    sB = np.full((N, K // 16), 0x38, np.uint8)
    D32, _ = run_gemm(A, ora.sf_swizzle(sA, K), B, ora.sf_swizzle(sB, K), M, N, K)
    ref, _ = ora.gemm(A, sA, B, sB, 1.0)
    assert np.array_equal(D32.cpu().numpy().astype(np.float64), ref)


def test_gemm_alpha_and_tensor_scales(ora):
    rng = np.random.default_rng(2)
    M, N, K = 128, 256, 512
    A, sA, sA_sw = random_operand(ora, M, K, rng)
    B, sB, sB_sw = random_operand(ora, N, K, rng)
    ga, gb, alpha = np.float32(0.0123), np.float32(3.5e-4), np.float32(1.0 / 16.0)
    D32, D16 = run_gemm(A, sA_sw, B, sB_sw, M, N, K, alpha=float(alpha), ga=float(ga), gb=float(gb))
    ref, bound = ora.gemm(A, sA, B, sB, float(alpha) * float(ga) * float(gb))
    check(D32, D16, ref, bound, "scaled")


def test_gemm_full_range_scales(ora):
    """Scale codes over the whole finite E4M3 range, including subnormals and 448."""
    rng = np.random.default_rng(3)
    M, N, K = 256, 256, 2048
    A, sA, sA_sw = random_operand(ora, M, K, rng, 0x00, 0x7F)
    B, sB, sB_sw = random_operand(ora, N, K, rng, 0x00, 0x7F)
    D32, D16 = run_gemm(A, sA_sw, B, sB_sw, M, N, K)
    ref, bound = ora.gemm(A, sA, B, sB, 1.0)
    check(D32, D16, ref, bound, "full range")


def sampled_gemm_check(ora, M, N, K, seed, nsamp=2048):
    rng = np.random.default_rng(seed)
    A, sA, sA_sw = random_operand(ora, M, K, rng)
    B, sB, sB_sw = random_operand(ora, N, K, rng)
    D32, D16 = run_gemm(A, sA_sw, B, sB_sw, M, N, K)
    mi = rng.integers(0, M, nsamp)
    ni = rng.integers(0, N, nsamp)
    # always include the corners of the output
    mi[:4] = [0, 0, M - 1, M - 1]
    ni[:4] = [0, N - 1, 0, N - 1]
    ref, bound = ora.gemm_pairs(A, sA, B, sB, 1.0, mi, ni)
    got = D32[torch.from_numpy(mi).to(DEV), torch.from_numpy(ni).to(DEV)].cpu().numpy()
    err = np.abs(got.astype(np.float64) - ref)
    assert (err <= TOL * bound + 1e-30).all(), f"{M}x{N}x{K}: max err/bound {np.max(err / bound)}"
    assert not torch.isnan(D32).any()
    assert torch.equal(D32.to(torch.bfloat16).view(torch.int16), D16.view(torch.int16))


@pytest.mark.parametrize("n", syn.GEMM_SQUARE)
def test_gemm_square_sweep_sampled(ora, n):
    sampled_gemm_check(ora, n, n, n, seed=n)


@pytest.mark.parametrize("M,N,K", [
    (2432, 2688, 25600),   # smaller operand > 32 MB: bands of 8 tile rows, last band 2 rows (one half tile)
    (640, 2304, 1024),     # M < N, small operands: M fastest, ragged last tile row
    (2304, 640, 1024),     # M >= N: N fastest, ragged last tile column
])
def test_gemm_tile_orders_sampled(ora, M, N, K):
    """Every tile of the 2-SM kernel is computed once in each of its tile orders."""
    sampled_gemm_check(ora, M, N, K, seed=M + 3 * N, nsamp=4096)


@pytest.mark.parametrize("N,K", syn.GEMM_SKINNY_WGRAD)
def test_gemm_skinny_wgrad_sampled(ora, N, K):
    """wgrad shapes: output N x K, reduction over 32768 tokens."""
    sampled_gemm_check(ora, N, K, 32768, seed=N + K, nsamp=512)
