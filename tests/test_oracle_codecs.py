"""Pins of the oracle's codecs, RNG and Hadamard matrix against facts fixed outside
the oracle: the pages' format statements, exhaustive enumeration, an independent
library conversion (torch float8_e4m3fn), published Philox known answers, and
scipy's Hadamard construction.  CPU only."""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden



# ---- E2M1 ---------------------------------------------------------------------------
def test_e2m1_value_set_matches_golden(ora):
    table = {int(c): float(v) for c, v in (r.split() for r in read_golden("e2m1_values.txt"))}
    assert len(table) == 16
    for code, val in table.items():
        got = ora.e2m1_decode(code)
        assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), code
    mags = sorted({abs(v) for v in table.values()})
    assert mags == [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


@pytest.mark.parametrize("v,expected", [
    (0.25, 0.0), (0.75, 1.0), (1.25, 1.0), (1.75, 2.0), (2.5, 2.0), (3.5, 4.0), (5.0, 4.0),
    (0.2499, 0.0), (0.2501, 0.5), (5.0001, 6.0), (6.0, 6.0), (7.0, 6.0), (1e30, 6.0),
])
def test_e2m1_rne_ties_and_saturation(ora, v, expected):
    for s in (1.0, -1.0):
        code = ora.e2m1_encode_rne(s * v)
        assert ora.e2m1_decode(code) == s * expected
        assert (code >> 3) == (1 if s < 0 else 0)


def test_e2m1_rne_brute_force_neighbourhoods(ora):
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    for lo, hi in zip(grid[:-1], grid[1:]):
        mid = np.float32((lo + hi) / 2)
        below = np.nextafter(mid, np.float32(-1))
        above = np.nextafter(mid, np.float32(100))
        assert ora.e2m1_decode(ora.e2m1_encode_rne(below)) == lo
        assert ora.e2m1_decode(ora.e2m1_encode_rne(above)) == hi
        # grid points are fixed points
        assert ora.e2m1_decode(ora.e2m1_encode_rne(lo)) == lo


def test_e2m1_sign_of_zero(ora):
    assert ora.e2m1_encode_rne(-0.1) == 0x8
    assert ora.e2m1_encode_rne(-0.0) == 0x8
    assert ora.e2m1_encode_rne(0.1) == 0x0


# ---- E4M3 ---------------------------------------------------------------------------
def test_e4m3_enumerate_all_codes_against_torch(ora):
    ref = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn)
    ref = ref.to(torch.float64).numpy()
    got = np.array([ora.e4m3_decode(c) for c in range(256)])
    nan = np.isnan(ref)
    assert (np.isnan(got) == nan).all()
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert (got[~nan] == ref[~nan]).all()
    finite = got[:0x7F]
    assert finite.max() == 448.0 and finite[0x7E] == 448.0
    assert (np.diff(finite) > 0).all()  # monotone in the code
    assert finite[1] == 2.0 ** -9 and finite[8] == 2.0 ** -6


def test_e4m3_encode_roundtrip_and_torch_rne(ora):
    for c in range(0x7F):
        assert ora.e4m3_encode(ora.e4m3_decode(c)) == c
    rng = np.random.default_rng(5)
    # random magnitudes across the whole range incl. subnormals, plus exact midpoints
    t = np.concatenate([
        np.exp(rng.uniform(np.log(1e-4), np.log(464.0), 20000)).astype(np.float32),
        np.array([(ora.e4m3_decode(c) + ora.e4m3_decode(c + 1)) / 2 for c in range(0x7E)],
                 dtype=np.float32),
    ])
    ref = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([ora.e4m3_encode(v) for v in t], dtype=np.uint8)
    assert (got == ref).all()


def test_e4m3_saturates(ora):
    for t in (448.0, 449.0, 464.0, 480.0, 1e6, float("inf")):
        assert ora.e4m3_encode(t) == 0x7E


# ---- Philox -------------------------------------------------------------------------
def test_philox_known_answers(ora):
    rows = read_golden("philox4x32_10_kat.txt")
    assert len(rows) == 3
    for r in rows:
        lhs, rhs = r.split(":")
        w = [int(h, 16) for h in lhs.split()]
        expect = [int(h, 16) for h in rhs.split()]
        assert list(ora.philox4x32_10(w[:4], w[4:6])) == expect


def test_sr_draw_layout(ora):
    """Each Philox block serves 8 consecutive elements; the words pair elements
    (0,2), (1,3), (4,6), (5,7), the first of a pair taking bytes 2:0 of its word,
    the second bytes 3:1; together the 8 draws use every bit of the block once."""
    seed = 0x0123456789ABCDEF
    for blk in (0, 1, 12345, (1 << 33) + 7):
        words = [int(w) for w in ora.philox4x32_10([blk & 0xFFFFFFFF, blk >> 32, 1, 0],
                                                   [seed & 0xFFFFFFFF, seed >> 32])]
        pair_word = {0: 0, 2: 0, 1: 1, 3: 1, 4: 2, 6: 2, 5: 3, 7: 3}
        used = [0, 0, 0, 0]
        for j in range(8):
            w = words[pair_word[j]]
            second = j in (2, 3, 6, 7)
            b = [(w >> (8 * k)) & 0xFF for k in range(4)]
            expect = (b[3] << 8 | b[1]) if second else (b[2] << 8 | b[0])
            assert ora.sr_draw16(seed, 1, blk * 8 + j) == expect
            used[pair_word[j]] |= (0xFF00FF00 if second else 0x00FF00FF)
        assert used == [0xFFFFFFFF] * 4


# ---- stochastic rounding ------------------------------------------------------------
@pytest.mark.parametrize("v", [0.1, 0.3, 0.6, 0.9, 1.2, 1.7, 2.2, 2.9, 3.3, 4.7, 5.9, -1.3,
                               -0.05, 0.123456])
def test_sr_unbiased_1e6(ora, v):
    n = 1_000_000
    codes = ora.e2m1_sr_array(np.full(n, v, dtype=np.float32), seed=7, stream=0)
    table = np.array([ora.e2m1_decode(c) for c in range(16)])
    vals = table[codes]
    grid = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    a = abs(np.float32(v))
    lo = max(g for g in grid if g <= a)
    hi = min(g for g in grid if g > a)
    assert set(np.unique(np.abs(vals))) <= {lo, hi}
    p = (a - lo) / (hi - lo)
    sigma = math.sqrt(p * (1 - p)) * (hi - lo)
    assert abs(vals.mean() - float(np.float32(v))) < 4 * sigma / math.sqrt(n) + 1e-12


def _f32(bits):
    return float(np.array([bits], dtype=np.uint32).view(np.float32)[0])


@pytest.mark.parametrize("v", [_f32(0x3F800000 + 12345), _f32(0x3F800000 + (0xFF00 << 6) + 63),
                               _f32(0x3F000000 + 2 * 777777), _f32(0x40800000 + (0x1234 << 6) + 9),
                               _f32(0x3A000000 + 4321), 0.1, 0.3, 2.9, 5.99, -1.3, -0.05, 1e-20])
def test_sr_exact_round_up_count(ora, v):
    """Every one of the 65536 draws, for values whose p * 2^16 is not an integer:
    the number of draws that round up is the one integer n with
    p * 2^16 - 1 < n <= p * 2^16 (the probability is within 2^-16 of p and never
    above it), and they are the n largest draws."""
    from fractions import Fraction
    grid = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3),
            Fraction(4), Fraction(6)]
    a = Fraction(abs(float(np.float32(v))))
    c = max(i for i in range(8) if grid[i] <= a)
    p = (a - grid[c]) / (grid[c + 1] - grid[c])
    codes = np.array([ora.e2m1_encode_sr(v, r) for r in range(65536)])
    sign = 8 if v < 0 else 0
    assert set(np.unique(codes)) <= {sign | c, sign | (c + 1)}
    up = codes == (sign | (c + 1))
    n = int(up.sum())
    assert p * 65536 - 1 < n <= p * 65536
    assert up[65536 - n:].all() and not up[:65536 - n].any()


def test_sr_grid_points_fixed_and_saturation(ora):
    for g in [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0, 7.5, 100.0]:
        codes = ora.e2m1_sr_array(np.full(4096, g, dtype=np.float32), seed=3, stream=0)
        assert (codes == ora.e2m1_encode_rne(min(g, 6.0))).all()


def test_sr_reproducible_and_stream_separated(ora):
    v = np.random.default_rng(1).uniform(-6, 6, 50000).astype(np.float32)
    a = ora.e2m1_sr_array(v, seed=11, stream=0)
    assert (a == ora.e2m1_sr_array(v, seed=11, stream=0)).all()
    assert (a != ora.e2m1_sr_array(v, seed=12, stream=0)).mean() > 0.1
    assert (a != ora.e2m1_sr_array(v, seed=11, stream=1)).mean() > 0.1


# ---- Hadamard -----------------------------------------------------------------------
def test_hadamard_sylvester(ora):
    import scipy.linalg
    H = ora.hadamard16()
    assert (H == scipy.linalg.hadamard(16)).all()
    assert (H @ H.T == 16 * np.eye(16, dtype=np.int64)).all()


def test_rht16_matches_dense_product(ora):
    import scipy.linalg
    H = scipy.linalg.hadamard(16).astype(np.float64)
    rng = np.random.default_rng(2)
    for _ in range(200):
        x = rng.standard_normal(16).astype(np.float32).astype(np.float64)
        s = (rng.integers(0, 2, 16) * 2 - 1).astype(np.int8)
        y, rc = ora.rht16(x, s)
        assert rc == 0
        assert np.array_equal(y, (x * s) @ H)
    # outside the exact-summation domain the oracle says so
    x = np.zeros(16)
    x[0], x[1] = 1.0, 2.0 ** -60
    assert ora.rht16(x, np.ones(16, np.int8))[1] == -1


def test_format_facts(ora):
    facts = dict(r.split() for r in read_golden("format_facts.txt"))
    bits = 4 + 8 / int(facts["block_elems"])
    assert bits == float(facts["nvfp4_bits_per_elem"])
    assert round(int(facts["bf16_bits_per_elem"]) / bits, 2) == float(facts["shrink_vs_bf16"])
    assert 4 + 8 / int(facts["mxfp4_block_elems"]) == float(facts["mxfp4_bits_per_elem"])
    # storage of the oracle's own layout at a 128-multiple shape: codes + scales
    R, Cc = 256, 512
    assert (R * Cc // 2 + ora.sf_bytes(R, Cc)) * 8 / (R * Cc) == bits
