"""ctypes binding of liboracle.so (test infrastructure; see nvfp4_oracle.h).

Arrays are numpy; bf16 tensors are passed as their uint16 bit patterns.
"""
import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        i64, u64, u32, f32, f64, vp, ci = (C.c_int64, C.c_uint64, C.c_uint32, C.c_float,
                                           C.c_double, C.c_void_p, C.c_int)
        sig = {
            "ora_e2m1_decode": (f64, [C.c_uint]),
            "ora_e2m1_encode_rne": (C.c_uint, [f32]),
            "ora_e4m3_decode": (f64, [C.c_uint]),
            "ora_e4m3_encode_rne_sat": (C.c_uint, [f32]),
            "ora_bf16_to_f32": (f32, [C.c_uint16]),
            "ora_philox4x32_10": (None, [vp, vp, vp]),
            "ora_sr_draw16": (C.c_uint, [u64, u32, u64]),
            "ora_e2m1_encode_sr": (C.c_uint, [f32, C.c_uint]),
            "ora_e2m1_sr_array": (None, [vp, i64, u64, u32, u64, vp]),
            "ora_hadamard16": (ci, [ci, ci]),
            "ora_rht16": (ci, [vp, vp, vp]),
            "ora_rht": (ci, [vp, i64, i64, ci, vp, vp]),
            "ora_tensor_amax": (ci, [vp, i64, i64, ci, ci, vp, vp, ci]),
            "ora_tensor_scale": (f32, [f32]),
            "ora_quantize_rows": (ci, [vp, i64, i64, ci, ci, vp, ci, ci, u64, f32, i64, i64,
                                       vp, vp, ci]),
            "ora_sf_bytes": (i64, [i64, i64]),
            "ora_sf_offset": (i64, [i64, i64, i64]),
            "ora_sf_swizzle": (None, [vp, i64, i64, vp]),
            "ora_gemm_pairs": (None, [vp, vp, vp, vp, i64, f64, i64, vp, vp, vp, vp, ci]),
            "ora_gemm": (None, [vp, vp, vp, vp, i64, i64, i64, f64, vp, vp, ci]),
            "ora_e8m0_decode": (f64, [C.c_uint]),
            "ora_mx_scale_code": (C.c_uint, [f64]),
            "ora_mx_quantize_rows": (ci, [vp, i64, i64, vp, vp]),
            "ora_mx_gemm": (None, [vp, vp, vp, vp, i64, i64, i64, f64, vp, vp, ci]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p)


def _signs(signs):
    s = np.ascontiguousarray(np.asarray(signs if signs is not None else np.ones(16), dtype=np.int8))
    assert s.shape == (16,)
    return s


# ---- codecs ----------------------------------------------------------------
def e2m1_decode(code):
    return lib().ora_e2m1_decode(int(code))


def e2m1_encode_rne(v):
    return lib().ora_e2m1_encode_rne(float(v))


def e4m3_decode(code):
    return lib().ora_e4m3_decode(int(code))


def e4m3_encode(t):
    return lib().ora_e4m3_encode_rne_sat(float(t))


def bf16_to_f32(bits):
    return lib().ora_bf16_to_f32(int(bits))


def philox4x32_10(ctr, key):
    c = np.ascontiguousarray(np.asarray(ctr, dtype=np.uint32))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint32))
    out = np.zeros(4, dtype=np.uint32)
    lib().ora_philox4x32_10(_p(c), _p(k), _p(out))
    return out


def sr_draw16(seed, stream, idx):
    return lib().ora_sr_draw16(int(seed), int(stream), int(idx))


def e2m1_encode_sr(v, r16):
    return lib().ora_e2m1_encode_sr(float(v), int(r16))


def e2m1_sr_array(v, seed, stream, idx0=0):
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.zeros(v.shape, dtype=np.uint8)
    lib().ora_e2m1_sr_array(_p(v), v.size, int(seed), int(stream), int(idx0), _p(out))
    return out


# ---- Hadamard ----------------------------------------------------------------
def hadamard16():
    L = lib()
    return np.array([[L.ora_hadamard16(i, j) for j in range(16)] for i in range(16)],
                    dtype=np.int64)


def rht16(x, signs):
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float64))
    y = np.zeros(16, dtype=np.float64)
    rc = lib().ora_rht16(_p(x), _p(_signs(signs)), _p(y))
    return y, rc


def rht(x_bits, axis, signs):
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    y = np.zeros(x.shape, dtype=np.float32)
    rc = lib().ora_rht(_p(x), x.shape[0], x.shape[1], int(axis), _p(_signs(signs)), _p(y))
    if rc == -2:
        raise ValueError("length along the transform axis must be a multiple of 16")
    if rc != 0:
        raise ArithmeticError("RHT input chunk spans more than 41 binades (outside exact domain)")
    return y


# ---- quantizer ---------------------------------------------------------------
def tensor_amax(x_bits, orient=0, rht_on=False, signs=None, nthreads=0):
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    out = np.zeros(1, dtype=np.float32)
    rc = lib().ora_tensor_amax(_p(x), x.shape[0], x.shape[1], int(orient), int(bool(rht_on)),
                               _p(_signs(signs)), _p(out), int(nthreads))
    if rc == -2:
        raise ValueError("bad shape")
    if rc != 0:
        raise ArithmeticError("RHT input chunk outside exact domain")
    return np.float32(out[0])


def tensor_scale(amax):
    return np.float32(lib().ora_tensor_scale(float(amax)))


def quantize_rows(x_bits, orient, rht_on, signs, block_mode, rounding, seed, amax, r0, r1,
                  nthreads=0):
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, cols = x.shape
    vcols = rows if orient else cols
    packed = np.zeros((r1 - r0, vcols // 2), dtype=np.uint8)
    sf = np.zeros((r1 - r0, vcols // 16), dtype=np.uint8)
    rc = lib().ora_quantize_rows(_p(x), rows, cols, int(orient), int(bool(rht_on)),
                                 _p(_signs(signs)), int(block_mode), int(rounding), int(seed),
                                 float(amax), int(r0), int(r1), _p(packed), _p(sf),
                                 int(nthreads))
    if rc == -2:
        raise ValueError("bad shape")
    if rc == -3:
        raise ArithmeticError("non-finite tensor amax")
    if rc != 0:
        raise ArithmeticError("RHT input chunk outside exact domain")
    return packed, sf


def quantize(x_bits, orient=0, rht_on=False, signs=None, block_mode=0, rounding=0, seed=0,
             nthreads=0):
    """Whole-tensor quantization: returns (packed, sf_logical, g, amax)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    amax = tensor_amax(x, orient, rht_on, signs, nthreads)
    vrows = x.shape[1] if orient else x.shape[0]
    packed, sf = quantize_rows(x, orient, rht_on, signs, block_mode, rounding, seed, amax, 0,
                               vrows, nthreads)
    return packed, sf, tensor_scale(amax), amax


# ---- scale layout ----------------------------------------------------------------
def sf_bytes(vrows, vcols):
    return lib().ora_sf_bytes(int(vrows), int(vcols))


def sf_offset(r, kb, vcols):
    return lib().ora_sf_offset(int(r), int(kb), int(vcols))


def sf_swizzle(sf_logical, vcols):
    sf = np.ascontiguousarray(sf_logical, dtype=np.uint8)
    vrows = sf.shape[0]
    out = np.zeros(sf_bytes(vrows, vcols), dtype=np.uint8)
    lib().ora_sf_swizzle(_p(sf), vrows, int(vcols), _p(out))
    return out


# ---- GEMM --------------------------------------------------------------------------
def gemm_pairs(A, sfA, B, sfB, alpha, m_idx, n_idx, nthreads=0):
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sfA = np.ascontiguousarray(sfA, dtype=np.uint8)
    sfB = np.ascontiguousarray(sfB, dtype=np.uint8)
    K = A.shape[1] * 2
    assert B.shape[1] * 2 == K and sfA.shape[1] * 16 == K and sfB.shape[1] * 16 == K
    mi = np.ascontiguousarray(m_idx, dtype=np.int64)
    ni = np.ascontiguousarray(n_idx, dtype=np.int64)
    out = np.zeros(mi.shape[0], dtype=np.float64)
    bound = np.zeros(mi.shape[0], dtype=np.float64)
    lib().ora_gemm_pairs(_p(A), _p(sfA), _p(B), _p(sfB), K, float(alpha), mi.shape[0], _p(mi),
                         _p(ni), _p(out), _p(bound), int(nthreads))
    return out, bound


def gemm(A, sfA, B, sfB, alpha, nthreads=0):
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sfA = np.ascontiguousarray(sfA, dtype=np.uint8)
    sfB = np.ascontiguousarray(sfB, dtype=np.uint8)
    M, N, K = A.shape[0], B.shape[0], A.shape[1] * 2
    D = np.zeros((M, N), dtype=np.float64)
    bound = np.zeros((M, N), dtype=np.float64)
    lib().ora_gemm(_p(A), _p(sfA), _p(B), _p(sfB), M, N, K, float(alpha), _p(D), _p(bound),
                   int(nthreads))
    return D, bound


def num_threads_default():
    return os.cpu_count() or 1


# ---- MXFP4 (the comparison format; reading R15) ------------------------------------
def e8m0_decode(code):
    return lib().ora_e8m0_decode(int(code))


def mx_scale_code(amax_b):
    return lib().ora_mx_scale_code(float(amax_b))


def mx_quantize(x_bits):
    """Row orientation, 1x32 E8M0 blocks, RNE: returns (packed, sf_logical)."""
    x = np.ascontiguousarray(x_bits, dtype=np.uint16)
    rows, cols = x.shape
    packed = np.zeros((rows, cols // 2), dtype=np.uint8)
    sf = np.zeros((rows, cols // 32), dtype=np.uint8)
    rc = lib().ora_mx_quantize_rows(_p(x), rows, cols, _p(packed), _p(sf))
    if rc != 0:
        raise ValueError(f"ora_mx_quantize_rows failed: {rc}")
    return packed, sf


def mx_sf_swizzle(sf_logical, vcols):
    """The block-scaled MMA's atom layout over 32-element blocks."""
    return sf_swizzle(sf_logical, vcols // 2)


def mx_gemm(A, sfA, B, sfB, alpha, nthreads=0):
    A = np.ascontiguousarray(A, dtype=np.uint8)
    B = np.ascontiguousarray(B, dtype=np.uint8)
    sfA = np.ascontiguousarray(sfA, dtype=np.uint8)
    sfB = np.ascontiguousarray(sfB, dtype=np.uint8)
    M, N, K = A.shape[0], B.shape[0], A.shape[1] * 2
    D = np.zeros((M, N), dtype=np.float64)
    bound = np.zeros((M, N), dtype=np.float64)
    lib().ora_mx_gemm(_p(A), _p(sfA), _p(B), _p(sfB), M, N, K, float(alpha), _p(D), _p(bound),
                      int(nthreads))
    return D, bound
