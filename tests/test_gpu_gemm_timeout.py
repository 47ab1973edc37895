"""Failure path of the GEMM's bounded waits, made to happen without a fault.

nvfp4_gemm_wait_limit bounds every pipeline wait by a caller-given number of clock
cycles.  With a bound of one cycle the waits run out in normal operation: the
kernel must record NVFP4_ERR_TIMEOUT in the status word, wait for the copies and
MMAs it already issued, free its tensor memory and return, leaving the context
usable.  The same GEMM right after it, with the default bound, must then match the
oracle.  Both kernels are covered: one SM per 128-row tile (M <= 128) and the
two-SM pair (M > 128)."""
import numpy as np
import pytest
import torch

from gpu_util import DEV, to_dev_u8
from nvfp4_bit_quantized_amax_b200 import capi

pytestmark = pytest.mark.gpu
TOL = 1e-4
ERR_TIMEOUT = -6


def operand(ora, rows, K, rng):
    codes = rng.integers(0, 256, size=(rows, K // 2), dtype=np.uint8)
    sf = rng.integers(0x20, 0x58, size=(rows, K // 16), dtype=np.uint8)
    return codes, sf, ora.sf_swizzle(sf, K)


@pytest.mark.parametrize("M,N,K", [(128, 256, 8192), (512, 512, 8192)])
def test_wait_runs_out_then_gemm_recovers(ora, M, N, K):
    rng = np.random.default_rng(M + N + K)
    A, sA, sA_sw = operand(ora, M, K, rng)
    B, sB, sB_sw = operand(ora, N, K, rng)
    dA, dsA, dB, dsB = to_dev_u8(A), to_dev_u8(sA_sw), to_dev_u8(B), to_dev_u8(sB_sw)

    # 32 k-tiles per output tile: the epilogue's wait for the accumulator alone
    # lasts microseconds, far past a one-cycle bound
    for _ in range(2):
        status = torch.zeros(1, dtype=torch.int32, device=DEV)
        D = torch.zeros((M, N), dtype=torch.bfloat16, device=DEV)
        capi.nvfp4_gemm_wait_limit(dA, dsA, dB, dsB, 1.0, M, N, K, 1, D_bf16=D, status=status)
        torch.cuda.synchronize()  # the kernel returned
        assert status.item() == ERR_TIMEOUT

    # the context is intact: the default bound gives the right product
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    D32 = torch.full((M, N), float("nan"), dtype=torch.float32, device=DEV)
    D16 = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    capi.nvfp4_gemm_wait_limit(dA, dsA, dB, dsB, 1.0, M, N, K, 0, D_bf16=D16, D_f32=D32,
                               status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    mi = rng.integers(0, M, 2048)
    ni = rng.integers(0, N, 2048)
    ref, bound = ora.gemm_pairs(A, sA, B, sB, 1.0, mi, ni)
    got = D32.cpu().numpy().astype(np.float64)[mi, ni]
    assert (np.abs(got - ref) <= TOL * bound + 1e-30).all()
    assert torch.equal(D32.to(torch.bfloat16).view(torch.int16), D16.view(torch.int16))

    # and the plain entry point agrees with it bit for bit
    D16b = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device=DEV)
    capi.nvfp4_gemm(dA, dsA, dB, dsB, 1.0, M, N, K, D_bf16=D16b, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert torch.equal(D16b.view(torch.int16), D16.view(torch.int16))


def test_wait_limit_rejects_negative_bound():
    z = torch.zeros(64, dtype=torch.uint8, device=DEV)
    D = torch.zeros((128, 8), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(capi.NVFP4Error):
        capi.nvfp4_gemm_wait_limit(z, z, z, z, 1.0, 128, 8, 64, -1, D_bf16=D)
