"""Pins of the oracle's quantizer, transform, scale layout and GEMM against closed
forms, constructed exact cases, invariants the pages state (16x16 forward/backward
consistency, analytic undoing of the RHT in the wgrad product) and library
routines (numpy matmul).  CPU only; small sizes."""
import numpy as np
import pytest
import scipy.linalg
import torch

from nvfp4_bit_quantized_amax_b200 import synthetic as syn

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


@pytest.fixture(scope="module")
def tables(ora):
    e2 = np.array([ora.e2m1_decode(c) for c in range(16)])
    e4 = np.array([ora.e4m3_decode(c) for c in range(256)])
    return e2, e4


def unpack(packed):
    lo = packed & 0x0F
    hi = packed >> 4
    out = np.empty((packed.shape[0], packed.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = lo
    out[:, 1::2] = hi
    return out


def dequant(packed, sf, g, tables):
    e2, e4 = tables
    codes = unpack(packed)
    return e2[codes] * np.repeat(e4[sf], 16, axis=1) * float(g)


def test_input_rounding_matches_torch():
    a = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 37
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert (syn.f32_to_bf16_bits(a) == ref).all()


def test_tensor_scale_closed_form(ora):
    x = syn.normal_bf16((64, 64), 3)
    amax = ora.tensor_amax(x)
    assert amax == np.abs(syn.bf16_bits_to_f32(x)).max()
    assert ora.tensor_scale(amax) == np.float32(amax) / np.float32(6 * 448)


def test_zero_tensor(ora):
    x = np.zeros((32, 64), np.uint16)
    x[1, ::3] = 0x8000  # negative zeros keep their sign bit in the code
    packed, sf, g, amax = ora.quantize(x)
    assert amax == 0 and g == 0 and (sf == 0).all()
    codes = unpack(packed)
    assert ((codes == 0) | (codes == 8)).all()
    assert (codes[1, ::3] == 8).all() and codes[0].max() == 0


def test_block_holding_tensor_max_gets_max_scale(ora):
    x = syn.normal_bf16((128, 256), 9, outlier_prob=0.01)
    packed, sf, g, amax = ora.quantize(x)
    xf = syn.bf16_bits_to_f32(x)
    r, c = np.unravel_index(np.argmax(np.abs(xf)), xf.shape)
    assert sf[r, c // 16] == 0x7E  # t = 448
    assert unpack(packed)[r, c] & 7 == 7  # +-6


def test_exact_power_of_two_construction(ora, tables):
    """Blocks built from E2M1 grid values times a per-block power of two, each block
    holding a +-6: the codes must reproduce the grid values and the scale code of a
    block 2^-j below the tensor max is 1.75*2^(8-j), i.e. ((15-j) << 3) | 6."""
    rng = np.random.default_rng(4)
    rows, cols = 48, 160
    kmax = 3
    j = rng.integers(0, 12, size=(rows, cols // 16))
    j[0, 0] = 0
    vals = rng.choice(np.concatenate([GRID, -GRID]), size=(rows, cols))
    vals[:, ::16] = 6.0 * rng.choice([-1.0, 1.0], size=(rows, cols // 16))
    x = vals * np.repeat(2.0 ** (kmax - j), 16, axis=1)
    xb = syn.f32_to_bf16_bits(x.astype(np.float32))
    assert (syn.bf16_bits_to_f32(xb) == x).all()
    packed, sf, g, amax = ora.quantize(xb)
    assert amax == 6.0 * 2 ** kmax
    assert (sf == (((15 - j) << 3) | 6)).all()
    e2, _ = tables
    assert (e2[unpack(packed)] == vals).all()


def test_single_nonzero_blocks(ora, tables):
    """A block with one nonzero c: its scale decodes to within E4M3 rounding of
    448 c / amax, the nonzero lands on +-6 (|v| in [5.6, 6.4]) and the rest on 0."""
    e2, e4 = tables
    rng = np.random.default_rng(8)
    rows, cols = 64, 64
    x = np.zeros((rows, cols), np.float32)
    pos = rng.integers(0, 16, size=(rows, cols // 16))
    mag = np.exp(rng.uniform(np.log(0.05), np.log(40.0), size=(rows, cols // 16)))
    for r in range(rows):
        for b in range(cols // 16):
            x[r, 16 * b + pos[r, b]] = mag[r, b] * (1 if (r + b) % 2 else -1)
    xb = syn.f32_to_bf16_bits(x)
    xf = syn.bf16_bits_to_f32(xb)
    packed, sf, g, amax = ora.quantize(xb)
    codes = unpack(packed)
    for r in range(rows):
        for b in range(cols // 16):
            c = abs(xf[r, 16 * b + pos[r, b]])
            target = 448.0 * c / amax
            assert abs(e4[sf[r, b]] / target - 1) <= 2 ** -4 + 1e-6
            blk = codes[r, 16 * b:16 * b + 16]
            assert blk[pos[r, b]] & 7 == 7
            assert np.all(np.delete(blk & 7, pos[r, b]) == 0)


@pytest.mark.parametrize("gen", ["normal", "t3", "laplace"])
def test_rne_error_bound(ora, tables, gen):
    e2, e4 = tables
    x = {"normal": syn.normal_bf16, "t3": syn.student_t_bf16,
         "laplace": syn.laplace_bf16}[gen]((64, 256), 1)
    packed, sf, g, amax = ora.quantize(x)
    xf = syn.bf16_bits_to_f32(x).astype(np.float64)
    d = np.repeat(e4[sf], 16, axis=1) * float(g)
    q = e2[unpack(packed)]
    v = np.where(d > 0, xf / np.where(d > 0, d, 1), 0)
    a = np.minimum(np.abs(v), 6.0)
    half = np.where(a < 2, 0.25, np.where(a < 4, 0.5, 1.0))
    err = np.abs(np.sign(v) * a - q)
    assert (err <= half * (1 + 1e-5)).all()
    # the block scale never sits more than one E4M3 step below the block max
    assert (np.abs(v) <= 6.0 * (1 + 2 ** -3)).all()


def test_16x16_forward_backward_consistency(ora, tables):
    """16x16 weight blocks give the same quantized weight whether it is read along
    K (fprop) or along N (dgrad)."""
    W = syn.normal_bf16((96, 160), 2, std=0.02)
    p_row, sf_row, g_row, _ = ora.quantize(W, orient=0, block_mode=1)
    p_col, sf_col, g_col, _ = ora.quantize(W, orient=1, block_mode=1)
    assert g_row == g_col
    assert (unpack(p_row) == unpack(p_col).T).all()
    for t in range(0, 96, 16):
        assert (sf_row[t:t + 16] == sf_row[t]).all()
    assert np.array_equal(dequant(p_row, sf_row, g_row, tables).T,
                          dequant(p_col, sf_col, g_col, tables))
    # and it is a genuinely different quantization from 1x16 strips
    p_1d, _, _, _ = ora.quantize(W, orient=0, block_mode=0)
    assert (p_1d != p_row).any()


def test_colwise_rht_amax_and_reconstruction(ora, tables):
    x = syn.normal_bf16((128, 48), 6, outlier_prob=0.01)
    s = syn.rht_signs(1)
    y = ora.rht(x, 0, s)  # 16-chunks down the rows
    H = scipy.linalg.hadamard(16).astype(np.float64)
    xf = syn.bf16_bits_to_f32(x).astype(np.float64)
    ref = np.einsum("jic,i,ik->jkc", xf.reshape(8, 16, 48), s.astype(np.float64), H)
    assert np.array_equal(y.reshape(8, 16, 48), ref.astype(np.float32))
    amax = ora.tensor_amax(x, orient=1, rht_on=True, signs=s)
    assert amax == np.abs(y).max()
    packed, sf, g, _ = ora.quantize(x, orient=1, rht_on=True, signs=s)
    deq = dequant(packed, sf, g, tables)  # [48, 128] = RHT(x)^T, quantized
    blk_max = np.repeat(np.abs(y.T).reshape(48, 8, 16).max(axis=2), 16, axis=1)
    assert (np.abs(deq - y.T) <= blk_max * (1.0 / 6.0) * (1 + 2 ** -3) + 1e-30).all()


def test_rht_undone_analytically_fp64(ora):
    """(dY^T D H)(X^T D H)^T / 16 == dY^T X: the rotation cancels in the wgrad product."""
    rng = np.random.default_rng(0)
    M, N, K = 64, 24, 40
    dY = rng.standard_normal((M, N)).astype(np.float32).astype(np.float64)
    X = rng.standard_normal((M, K)).astype(np.float32).astype(np.float64)
    s = syn.rht_signs(5)

    def rot(A):  # along M, chunk by chunk, with the oracle's fp64 transform
        out = np.empty_like(A)
        for c in range(A.shape[1]):
            for j in range(M // 16):
                out[16 * j:16 * j + 16, c] = ora.rht16(A[16 * j:16 * j + 16, c], s)[0]
        return out

    lhs = rot(dY).T @ rot(X) / 16.0
    rhs = dY.T @ X
    assert (np.abs(lhs - rhs) <= 1e-12 * (np.abs(dY).T @ np.abs(X))).all()


def test_rht_wgrad_quantized_close_to_exact(ora, tables):
    M, N, K = 256, 64, 64
    X = syn.normal_bf16((M, K), 1, outlier_prob=0.01)
    dY = syn.normal_bf16((M, N), 2, outlier_prob=0.01)
    s = syn.rht_signs(3)
    pa, sa, ga, _ = ora.quantize(dY, orient=1, rht_on=True, signs=s, rounding=1, seed=9)
    pb, sb, gb, _ = ora.quantize(X, orient=1, rht_on=True, signs=s)
    got = dequant(pa, sa, ga, tables) @ dequant(pb, sb, gb, tables).T / 16.0
    exact = syn.bf16_bits_to_f32(dY).astype(np.float64).T @ syn.bf16_bits_to_f32(X)
    rel = np.linalg.norm(got - exact) / np.linalg.norm(exact)
    # without the rotation the same quantizer gives an error of the same order;
    # the rotation is undone (no 16x error) and only quantization noise remains
    qa, ta, ha, _ = ora.quantize(dY, orient=1, rounding=1, seed=9)
    qb, tb, hb, _ = ora.quantize(X, orient=1)
    plain = dequant(qa, ta, ha, tables) @ dequant(qb, tb, hb, tables).T
    rel_plain = np.linalg.norm(plain - exact) / np.linalg.norm(exact)
    assert rel < 0.3 and rel < 1.5 * rel_plain


def test_sf_layout_independent_construction(ora):
    """Scale atoms: 32 lines of 16 bytes; line l carries rows l, l+32, l+64, l+96,
    4 blocks each.  Built here with numpy reshapes rather than the offset formula."""
    rng = np.random.default_rng(1)
    vrows, vcols = 300, 16 * 10  # ragged: pads rows to 384, blocks 10 -> 12
    sf = rng.integers(1, 255, size=(vrows, vcols // 16), dtype=np.uint8)
    got = ora.sf_swizzle(sf, vcols)
    padded = np.zeros((384, 12), np.uint8)
    padded[:vrows, :10] = sf
    atoms = padded.reshape(3, 128, 3, 4).transpose(0, 2, 1, 3)  # [rowblk, katom, 128, 4]
    atoms = atoms.reshape(3, 3, 4, 32, 4).transpose(0, 1, 3, 2, 4)  # [.., line, i, kb]
    assert np.array_equal(got, atoms.reshape(-1))
    assert ora.sf_bytes(vrows, vcols) == 384 * 12


def test_gemm_integer_special_case(ora):
    """All block scales 1.0 (E4M3 0x38): 2*E2M1 values are integers in [-12, 12] and
    the GEMM must equal an exact integer matrix product divided by 4."""
    rng = np.random.default_rng(3)
    M, N, K = 40, 24, 512
    ca = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    cb = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    A = (ca[:, 0::2] | (ca[:, 1::2] << 4)).astype(np.uint8)
    B = (cb[:, 0::2] | (cb[:, 1::2] << 4)).astype(np.uint8)
    one = np.full((M, K // 16), 0x38, np.uint8)
    D, bound = ora.gemm(A, one, B, np.full((N, K // 16), 0x38, np.uint8), alpha=1.0)
    ia = np.rint(2 * np.array([ora.e2m1_decode(c) for c in range(16)])).astype(np.int64)
    ref = (ia[ca] @ ia[cb].T).astype(np.float64) / 4.0
    assert np.array_equal(D, ref)


def test_gemm_matches_numpy_and_pairs(ora, tables):
    rng = np.random.default_rng(4)
    M, N, K = 33, 47, 256
    A = rng.integers(0, 256, size=(M, K // 2), dtype=np.uint8)
    B = rng.integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = rng.integers(0, 0x7F, size=(M, K // 16), dtype=np.uint8)
    sb = rng.integers(0, 0x7F, size=(N, K // 16), dtype=np.uint8)
    alpha = 0.37
    D, bound = ora.gemm(A, sa, B, sb, alpha)
    da, db = dequant(A, sa, 1.0, tables), dequant(B, sb, 1.0, tables)
    ref = alpha * (da @ db.T)
    assert (np.abs(D - ref) <= 1e-12 * bound + 1e-300).all()
    assert np.allclose(bound, alpha * (np.abs(da) @ np.abs(db).T))
    mi = rng.integers(0, M, 50)
    ni = rng.integers(0, N, 50)
    out, bnd = ora.gemm_pairs(A, sa, B, sb, alpha, mi, ni)
    assert np.array_equal(out, D[mi, ni]) and np.array_equal(bnd, bound[mi, ni])


# ---- R14: RHT along the row of the quantized view (dgrad operands rotated along N) ----
def test_row_rht_equals_column_rht_of_transpose(ora):
    """The rotation along a view row is the same whether the view is x (orient 0) or
    the transpose of x^T (orient 1, pinned above): same amax, codes and scales (RNE;
    SR draws differ by stream)."""
    x = syn.normal_bf16((48, 64), 21, outlier_prob=0.02)
    s = syn.rht_signs(3)
    xt = np.ascontiguousarray(x.T)
    for bm in (0, 1):
        p0, sf0, g0, a0 = ora.quantize(x, 0, True, s, bm, 0)
        p1, sf1, g1, a1 = ora.quantize(xt, 1, True, s, bm, 0)
        assert a0 == a1 and g0 == g1
        assert np.array_equal(p0, p1) and np.array_equal(sf0, sf1)


def test_row_rht_dense_product(ora):
    """The standalone transform along the contiguous axis is the dense product
    x_chunk . diag(s) . H16 of every 16-chunk of every row, rounded once to fp32: a
    mistake that moves outputs to other columns, drops the signs or uses the wrong
    chunk fails here, not only in the maximum."""
    x = syn.normal_bf16((40, 96), 23, outlier_prob=0.02)
    s = syn.rht_signs(7)
    y = ora.rht(x, 1, s)
    H = scipy.linalg.hadamard(16).astype(np.float64)
    xf = syn.bf16_bits_to_f32(x).astype(np.float64)
    ref = np.einsum("rji,i,ik->rjk", xf.reshape(40, 6, 16), s.astype(np.float64), H)
    assert np.array_equal(y.reshape(40, 6, 16), ref.astype(np.float32))
    # one nonzero input picks out one signed row of H in its own chunk, nothing else
    e = np.zeros((2, 32), dtype=np.uint16)
    e[1, 16 + 5] = 0x3F80  # 1.0
    ye = ora.rht(e, 1, s)
    assert (ye[0] == 0).all() and (ye[1, :16] == 0).all()
    assert np.array_equal(ye[1, 16:], (s[5] * H[5]).astype(np.float32))


def test_rht_exact_zero_is_positive_zero(ora):
    """Reading R7: the transform is the fp32 rounding of the exact sum, and an exact
    sum of zero is the real number 0, stored as +0 whatever the input signs (zero
    inputs, -0 inputs, negative rotation signs, or nonzero inputs that cancel)."""
    s = np.array([-1, 1] * 8, dtype=np.int8)
    x = np.zeros((4, 16), np.uint16)
    x[1, :] = 0x8000                       # -0 everywhere
    x[2, 0], x[2, 1] = 0x3F80, 0x3F80      # 1, 1 with signs -1, +1: cancels in half the outputs
    x[3, 8] = 0xC000                       # one -2, the rest +0
    y = ora.rht(x, 1, s)
    H = scipy.linalg.hadamard(16).astype(np.float64)
    exact = (syn.bf16_bits_to_f32(x).astype(np.float64) * s) @ H
    assert np.array_equal(y, exact.astype(np.float32))
    zero = exact == 0
    assert zero.any() and (y.view(np.uint32)[zero] == 0).all()   # +0, never -0


def test_row_rht_amax_is_max_of_standalone_rht(ora):
    x = syn.normal_bf16((32, 96), 22)
    s = syn.rht_signs(4)
    y = ora.rht(x, 1, s)                  # 16-chunks along the contiguous columns
    _, _, _, amax = ora.quantize(x, 0, True, s, 0, 0)
    assert amax == np.float32(np.abs(y).max())


def test_dgrad_rotation_identity_fp64():
    """(dY D H)(W^T D H)^T = 16 dY W on unquantized data: the rotation along N cancels
    in dgrad with alpha 1/16."""
    rng = np.random.default_rng(7)
    M, N, K = 8, 32, 12
    dY = rng.standard_normal((M, N))
    W = rng.standard_normal((N, K))
    s = syn.rht_signs(6).astype(np.float64)
    H = np.array([[(-1.0) ** bin(i & j).count("1") for j in range(16)] for i in range(16)])
    R = np.kron(np.eye(N // 16), np.diag(s) @ H)      # block-diagonal rotation along N
    lhs = (dY @ R) @ (W.T @ R).T / 16.0
    assert np.allclose(lhs, dY @ W, rtol=1e-12, atol=1e-12)
