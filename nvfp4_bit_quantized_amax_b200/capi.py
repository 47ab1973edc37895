"""Thin Python binding of libnvfp4.so (C ABI in include/nvfp4.h).

Argument marshalling only: torch tensors give device pointers and the current
CUDA stream; every step of the computation runs in the library's kernels.  The
library must be present (built by `python -m nvfp4_bit_quantized_amax_b200.build`
or `__graft_entry__.build()`); there is no CPU fallback and `load()` raises if it
is missing.
"""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libnvfp4.so")

OK, ERR_ARG, ERR_SHAPE, ERR_ALIGN, ERR_CUDA, ERR_NONFINITE, ERR_TIMEOUT, ERR_WORKSPACE, \
    ERR_DEVICE, ERR_INDEX, ERR_RHT_RANGE = 0, -1, -2, -3, -4, -5, -6, -7, -8, -9, -10
BLOCK_1X16, BLOCK_16X16 = 0, 1
ROUND_RNE, ROUND_SR = 0, 1
LIN_X_ROW, LIN_X_COL, LIN_W_ROW, LIN_W_COL, LIN_DY_ROW, LIN_DY_COL = range(6)

# Every symbol include/nvfp4.h declares.
EXPORTS = (
    "nvfp4_packed_bytes", "nvfp4_scale_bytes", "nvfp4_quantize_workspace_bytes",
    "nvfp4_quantize", "nvfp4_quantize_2d", "nvfp4_rht", "nvfp4_gemm",
    "nvfp4_linear_workspace_bytes", "nvfp4_linear_fprop", "nvfp4_linear_dgrad",
    "nvfp4_linear_wgrad", "nvfp4_linear_operand", "nvfp4_read_status",
    "nvfp4_status_string", "nvfp4_version", "nvfp4_quantize_noalloc",
    "nvfp4_moe_workspace_bytes", "nvfp4_moe_expert_workspace", "nvfp4_moe_linear_fprop",
    "nvfp4_moe_linear_dgrad", "nvfp4_moe_linear_wgrad", "nvfp4_moe_gather", "nvfp4_moe_combine",
    "nvfp4_linear_fprop_ex", "nvfp4_linear_dgrad_ex",
    "nvfp4_mx_scale_bytes", "nvfp4_mx_quantize", "nvfp4_mx_gemm",
    "nvfp4_moe_grouped_workspace_bytes", "nvfp4_moe_grouped_operand", "nvfp4_moe_grouped_fprop",
    "nvfp4_moe_grouped_dgrad", "nvfp4_moe_grouped_wgrad", "nvfp4_gemm_wait_limit",
    "nvfp4_moe_grouped_fprop_gather",
)


class NVFP4Error(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__(f"{fn} failed: {status} ({status_string(status)})")


class Tensor(C.Structure):
    """nvfp4_tensor: one quantized operand (device pointers)."""
    _fields_ = [("data", C.c_void_p), ("scales", C.c_void_p), ("tensor_scale", C.c_void_p),
                ("rows", C.c_int64), ("cols", C.c_int64)]


class LinearOpts(C.Structure):
    """nvfp4_linear_opts: weight block mode, RHT on the dgrad operands."""
    _fields_ = [("weight_block_mode", C.c_int), ("dgrad_rht", C.c_int)]


class QuantizeOpts(C.Structure):
    _fields_ = [("block_mode", C.c_int), ("row_rounding", C.c_int), ("col_rounding", C.c_int),
                ("seed", C.c_uint64), ("col_rht", C.c_int), ("rht_signs", C.c_void_p)]


_lib = None


def load(path: str = LIB_PATH):
    """Load libnvfp4.so once; raises if it is missing (no fallback path exists)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libnvfp4.so not found at {path}; build it with "
                           "`python -m nvfp4_bit_quantized_amax_b200.build`")
    L = C.CDLL(path)
    i64, u64, vp, ci, sz, f32 = C.c_int64, C.c_uint64, C.c_void_p, C.c_int, C.c_size_t, C.c_float
    sig = {
        "nvfp4_packed_bytes": (sz, [i64, i64]),
        "nvfp4_scale_bytes": (sz, [i64, i64]),
        "nvfp4_quantize_workspace_bytes": (sz, []),
        "nvfp4_quantize": (ci, [vp, i64, i64, ci, ci, u64, vp, vp, vp, vp, vp]),
        "nvfp4_quantize_2d": (ci, [vp, i64, i64, C.POINTER(QuantizeOpts), C.POINTER(Tensor),
                                   C.POINTER(Tensor), vp, vp]),
        "nvfp4_rht": (ci, [vp, i64, i64, ci, vp, ci, vp, vp]),
        "nvfp4_gemm": (ci, [vp, vp, vp, vp, vp, vp, f32, i64, i64, i64, vp, vp, vp, vp]),
        "nvfp4_gemm_wait_limit": (ci, [vp, vp, vp, vp, vp, vp, f32, i64, i64, i64, vp, vp, vp,
                                       C.c_longlong, vp]),
        "nvfp4_linear_workspace_bytes": (sz, [i64, i64, i64]),
        "nvfp4_linear_fprop": (ci, [vp, vp, vp, i64, i64, i64, vp, vp, sz, vp]),
        "nvfp4_linear_dgrad": (ci, [vp, vp, i64, i64, i64, u64, vp, vp, sz, vp]),
        "nvfp4_linear_wgrad": (ci, [vp, vp, i64, i64, i64, u64, vp, vp, sz, vp]),
        "nvfp4_linear_operand": (ci, [vp, i64, i64, i64, ci, C.POINTER(Tensor)]),
        "nvfp4_read_status": (ci, [vp, C.POINTER(ci), vp]),
        "nvfp4_status_string": (C.c_char_p, [ci]),
        "nvfp4_version": (ci, []),
        "nvfp4_quantize_noalloc": (ci, [vp, i64, i64, ci, ci, u64, vp, vp, vp, vp]),
        "nvfp4_moe_workspace_bytes": (sz, [vp, ci, i64, i64]),
        "nvfp4_moe_expert_workspace": (ci, [vp, vp, ci, i64, i64, ci, C.POINTER(vp),
                                            C.POINTER(sz)]),
        "nvfp4_moe_linear_fprop": (ci, [vp, vp, vp, vp, ci, i64, i64, vp, vp, sz, vp]),
        "nvfp4_moe_linear_dgrad": (ci, [vp, vp, vp, ci, i64, i64, u64, vp, vp, sz, vp]),
        "nvfp4_moe_linear_wgrad": (ci, [vp, vp, ci, i64, i64, u64, vp, vp, sz, vp]),
        "nvfp4_moe_gather": (ci, [vp, vp, i64, i64, vp, vp]),
        "nvfp4_moe_combine": (ci, [vp, vp, i64, ci, i64, vp, vp]),
        "nvfp4_linear_fprop_ex": (ci, [vp, vp, vp, i64, i64, i64, vp, C.POINTER(LinearOpts), vp, sz, vp]),
        "nvfp4_linear_dgrad_ex": (ci, [vp, vp, i64, i64, i64, u64, vp, C.POINTER(LinearOpts), vp, sz, vp]),
        "nvfp4_mx_scale_bytes": (sz, [i64, i64]),
        "nvfp4_mx_quantize": (ci, [vp, i64, i64, vp, vp, vp]),
        "nvfp4_mx_gemm": (ci, [vp, vp, vp, vp, f32, i64, i64, i64, vp, vp, vp, vp]),
        "nvfp4_moe_grouped_workspace_bytes": (sz, [vp, ci, i64, i64]),
        "nvfp4_moe_grouped_operand": (ci, [vp, vp, ci, i64, i64, ci, C.POINTER(Tensor)]),
        "nvfp4_moe_grouped_fprop": (ci, [vp, vp, vp, vp, ci, i64, i64, vp, vp, sz, vp]),
        "nvfp4_moe_grouped_fprop_gather": (ci, [vp, vp, i64, vp, vp, vp, ci, i64, i64, vp, vp, sz, vp]),
        "nvfp4_moe_grouped_dgrad": (ci, [vp, vp, vp, ci, i64, i64, u64, vp, vp, sz, vp]),
        "nvfp4_moe_grouped_wgrad": (ci, [vp, vp, ci, i64, i64, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def status_string(status: int) -> str:
    return load().nvfp4_status_string(int(status)).decode()


def _check(fn, rc):
    if rc != OK:
        raise NVFP4Error(fn, rc)


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _signs(signs):
    import numpy as np
    s = np.ascontiguousarray(np.asarray(signs, dtype=np.int8))
    if s.shape != (16,):
        raise ValueError("rht signs must be 16 entries of +1/-1")
    return s, s.ctypes.data_as(C.c_void_p)


# ---- sizes -------------------------------------------------------------------------
def packed_bytes(rows, cols):
    return load().nvfp4_packed_bytes(rows, cols)


def scale_bytes(rows, cols):
    return load().nvfp4_scale_bytes(rows, cols)


def quantize_workspace_bytes():
    return load().nvfp4_quantize_workspace_bytes()


def linear_workspace_bytes(M, K, N):
    return load().nvfp4_linear_workspace_bytes(M, K, N)


# ---- entry points (torch tensors in, torch tensors written) -------------------------
def nvfp4_quantize(x, block_mode, rounding, seed, packed, scales, tensor_scale, workspace,
                   stream=None):
    rows, cols = x.shape
    _check("nvfp4_quantize", load().nvfp4_quantize(
        _ptr(x), rows, cols, block_mode, rounding, seed, _ptr(packed), _ptr(scales),
        _ptr(tensor_scale), _ptr(workspace), _stream(stream)))


def nvfp4_quantize_noalloc(x, block_mode, rounding, seed, packed, scales, tensor_scale,
                           stream=None):
    """nvfp4_quantize without a workspace (scratch in the library's static array)."""
    rows, cols = x.shape
    _check("nvfp4_quantize_noalloc", load().nvfp4_quantize_noalloc(
        _ptr(x), rows, cols, block_mode, rounding, seed, _ptr(packed), _ptr(scales),
        _ptr(tensor_scale), _stream(stream)))


def make_tensor(data, scales, tensor_scale):
    return Tensor(data.data_ptr(), scales.data_ptr(), tensor_scale.data_ptr(), 0, 0)


def nvfp4_quantize_2d(x, block_mode, row_rounding, col_rounding, seed, col_rht, rht_signs,
                      row_out, col_out, workspace, stream=None):
    """row_out / col_out: (data, scales, tensor_scale) torch tensors or None."""
    rows, cols = x.shape
    keep = None
    sp = None
    if col_rht:
        keep, sp = _signs(rht_signs)
    opts = QuantizeOpts(block_mode, row_rounding, col_rounding, seed, int(bool(col_rht)), sp)
    r = make_tensor(*row_out) if row_out is not None else None
    c = make_tensor(*col_out) if col_out is not None else None
    _check("nvfp4_quantize_2d", load().nvfp4_quantize_2d(
        _ptr(x), rows, cols, C.byref(opts), C.byref(r) if r is not None else None,
        C.byref(c) if c is not None else None, _ptr(workspace), _stream(stream)))
    del keep


def nvfp4_rht(x, signs, n, y, axis=1, stream=None):
    rows, cols = x.shape
    keep, sp = _signs(signs)
    _check("nvfp4_rht", load().nvfp4_rht(_ptr(x), rows, cols, axis, sp, n, _ptr(y),
                                         _stream(stream)))
    del keep


def nvfp4_gemm(A, sfA, B, sfB, alpha, M, N, K, D_bf16=None, D_f32=None, scale_a=None,
               scale_b=None, status=None, stream=None):
    _check("nvfp4_gemm", load().nvfp4_gemm(
        _ptr(A), _ptr(sfA), _ptr(B), _ptr(sfB), _ptr(scale_a), _ptr(scale_b), float(alpha), M, N,
        K, _ptr(D_bf16), _ptr(D_f32), _ptr(status), _stream(stream)))


def nvfp4_gemm_wait_limit(A, sfA, B, sfB, alpha, M, N, K, wait_cycles, D_bf16=None, D_f32=None,
                          scale_a=None, scale_b=None, status=None, stream=None):
    """nvfp4_gemm with the pipeline waits bounded by `wait_cycles` clock cycles (a
    testing hook of the timeout path; 0 selects the default bound)."""
    _check("nvfp4_gemm_wait_limit", load().nvfp4_gemm_wait_limit(
        _ptr(A), _ptr(sfA), _ptr(B), _ptr(sfB), _ptr(scale_a), _ptr(scale_b), float(alpha), M, N,
        K, _ptr(D_bf16), _ptr(D_f32), _ptr(status), int(wait_cycles), _stream(stream)))


def nvfp4_linear_fprop(X, W, Y, rht_signs, ws, stream=None):
    M, K = X.shape
    N = W.shape[0]
    keep, sp = _signs(rht_signs)
    _check("nvfp4_linear_fprop", load().nvfp4_linear_fprop(
        _ptr(X), _ptr(W), _ptr(Y), M, K, N, sp, _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    del keep


def nvfp4_linear_dgrad(dY, dX, seed, rht_signs, ws, stream=None):
    M, N = dY.shape
    K = dX.shape[1]
    keep, sp = _signs(rht_signs)
    _check("nvfp4_linear_dgrad", load().nvfp4_linear_dgrad(
        _ptr(dY), _ptr(dX), M, K, N, seed, sp, _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    del keep


def nvfp4_linear_wgrad(dY, dW, M, seed, rht_signs, ws, stream=None):
    N, K = dW.shape
    keep, sp = _signs(rht_signs)
    _check("nvfp4_linear_wgrad", load().nvfp4_linear_wgrad(
        _ptr(dY), _ptr(dW), M, K, N, seed, sp, _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    del keep


def nvfp4_linear_fprop_ex(X, W, Y, rht_signs, ws, weight_block_mode=1, dgrad_rht=0, stream=None):
    M, K = X.shape
    N = W.shape[0]
    keep, sp = _signs(rht_signs)
    o = LinearOpts(weight_block_mode, dgrad_rht)
    _check("nvfp4_linear_fprop_ex", load().nvfp4_linear_fprop_ex(
        _ptr(X), _ptr(W), _ptr(Y), M, K, N, sp, C.byref(o), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def nvfp4_linear_dgrad_ex(dY, dX, seed, rht_signs, ws, weight_block_mode=1, dgrad_rht=0, stream=None):
    M, N = dY.shape
    K = dX.shape[1]
    keep, sp = _signs(rht_signs)
    o = LinearOpts(weight_block_mode, dgrad_rht)
    _check("nvfp4_linear_dgrad_ex", load().nvfp4_linear_dgrad_ex(
        _ptr(dY), _ptr(dX), M, K, N, seed, sp, C.byref(o), _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep


def mx_scale_bytes(rows, cols):
    return load().nvfp4_mx_scale_bytes(rows, cols)


def nvfp4_mx_quantize(x, packed, scales, stream=None):
    rows, cols = x.shape
    _check("nvfp4_mx_quantize", load().nvfp4_mx_quantize(_ptr(x), rows, cols, _ptr(packed),
                                                         _ptr(scales), _stream(stream)))


def nvfp4_mx_gemm(A, sfA, B, sfB, alpha, M, N, K, D_bf16=None, D_f32=None, status=None,
                  stream=None):
    _check("nvfp4_mx_gemm", load().nvfp4_mx_gemm(
        _ptr(A), _ptr(sfA), _ptr(B), _ptr(sfB), float(alpha), M, N, K, _ptr(D_bf16),
        _ptr(D_f32), _ptr(status), _stream(stream)))


def nvfp4_linear_operand(ws, M, K, N, which):
    t = Tensor()
    _check("nvfp4_linear_operand", load().nvfp4_linear_operand(
        C.c_void_p(ws.data_ptr()), M, K, N, which, C.byref(t)))
    return t


# ---- mixture of experts -----------------------------------------------------------
def _rows(group_rows):
    import numpy as np
    g = np.ascontiguousarray(np.asarray(group_rows, dtype=np.int64))
    return g, g.ctypes.data_as(C.c_void_p)


def moe_workspace_bytes(group_rows, K, N):
    g, gp = _rows(group_rows)
    return load().nvfp4_moe_workspace_bytes(gp, len(g), K, N)


def nvfp4_moe_expert_workspace(ws, group_rows, K, N, expert):
    g, gp = _rows(group_rows)
    p, n = C.c_void_p(), C.c_size_t()
    _check("nvfp4_moe_expert_workspace", load().nvfp4_moe_expert_workspace(
        C.c_void_p(ws.data_ptr()), gp, len(g), K, N, expert, C.byref(p), C.byref(n)))
    return p.value, n.value


def nvfp4_moe_linear_fprop(X_perm, W, Y_perm, group_rows, rht_signs, ws, stream=None):
    g, gp = _rows(group_rows)
    E, N, K = W.shape
    keep, sp = _signs(rht_signs)
    _check("nvfp4_moe_linear_fprop", load().nvfp4_moe_linear_fprop(
        _ptr(X_perm), _ptr(W), _ptr(Y_perm), gp, E, K, N, sp, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep, g


def nvfp4_moe_linear_dgrad(dY_perm, dX_perm, group_rows, seed, rht_signs, ws, stream=None):
    g, gp = _rows(group_rows)
    K = dX_perm.shape[1]
    N = dY_perm.shape[1]
    keep, sp = _signs(rht_signs)
    _check("nvfp4_moe_linear_dgrad", load().nvfp4_moe_linear_dgrad(
        _ptr(dY_perm), _ptr(dX_perm), gp, len(g), K, N, seed, sp, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep, g


def nvfp4_moe_linear_wgrad(dW, group_rows, seed, rht_signs, ws, stream=None):
    g, gp = _rows(group_rows)
    E, N, K = dW.shape
    keep, sp = _signs(rht_signs)
    _check("nvfp4_moe_linear_wgrad", load().nvfp4_moe_linear_wgrad(
        _ptr(dW), gp, E, K, N, seed, sp, _ptr(ws), ws.numel() * ws.element_size(),
        _stream(stream)))
    del keep, g


def moe_grouped_workspace_bytes(group_rows, K, N):
    g, gp = _rows(group_rows)
    return load().nvfp4_moe_grouped_workspace_bytes(gp, len(g), K, N)


def nvfp4_moe_grouped_operand(ws, group_rows, K, N, which):
    g, gp = _rows(group_rows)
    t = Tensor()
    _check("nvfp4_moe_grouped_operand", load().nvfp4_moe_grouped_operand(
        C.c_void_p(ws.data_ptr()), gp, len(g), K, N, which, C.byref(t)))
    return t


def nvfp4_moe_grouped_fprop(X_perm, W, Y_perm, group_rows, rht_signs, ws, stream=None):
    g, gp = _rows(group_rows)
    E, N, K = W.shape
    keep, sp = _signs(rht_signs)
    _check("nvfp4_moe_grouped_fprop", load().nvfp4_moe_grouped_fprop(
        _ptr(X_perm), _ptr(W), _ptr(Y_perm), gp, E, K, N, sp, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep, g


def nvfp4_moe_grouped_fprop_gather(X_tok, row_src, W, Y_perm, group_rows, rht_signs, ws, stream=None):
    """Grouped fprop reading X's rows through row_src (the gather fused in)."""
    g, gp = _rows(group_rows)
    E, N, K = W.shape
    keep, sp = _signs(rht_signs)
    _check("nvfp4_moe_grouped_fprop_gather", load().nvfp4_moe_grouped_fprop_gather(
        _ptr(X_tok), _ptr(row_src), X_tok.shape[0], _ptr(W), _ptr(Y_perm), gp, E, K, N, sp, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep, g


def nvfp4_moe_grouped_dgrad(dY_perm, dX_perm, group_rows, seed, rht_signs, ws, stream=None):
    g, gp = _rows(group_rows)
    K = dX_perm.shape[1]
    N = dY_perm.shape[1]
    keep, sp = _signs(rht_signs)
    _check("nvfp4_moe_grouped_dgrad", load().nvfp4_moe_grouped_dgrad(
        _ptr(dY_perm), _ptr(dX_perm), gp, len(g), K, N, seed, sp, _ptr(ws),
        ws.numel() * ws.element_size(), _stream(stream)))
    del keep, g


def nvfp4_moe_grouped_wgrad(dW, group_rows, ws, stream=None):
    g, gp = _rows(group_rows)
    E, N, K = dW.shape
    _check("nvfp4_moe_grouped_wgrad", load().nvfp4_moe_grouped_wgrad(
        _ptr(dW), gp, E, K, N, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)))
    del g


def nvfp4_moe_gather(src, row_src, dst, stream=None):
    rows, cols = dst.shape
    _check("nvfp4_moe_gather", load().nvfp4_moe_gather(_ptr(src), _ptr(row_src), rows, cols,
                                                       _ptr(dst), _stream(stream)))


def nvfp4_moe_combine(src, slots, dst, stream=None):
    tokens, topk = slots.shape
    cols = dst.shape[1]
    _check("nvfp4_moe_combine", load().nvfp4_moe_combine(_ptr(src), _ptr(slots), tokens, topk,
                                                         cols, _ptr(dst), _stream(stream)))


def nvfp4_read_status(workspace, stream=None):
    v = C.c_int(0)
    _check("nvfp4_read_status", load().nvfp4_read_status(_ptr(workspace), C.byref(v),
                                                         _stream(stream)))
    return v.value
