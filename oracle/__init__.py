"""ctypes shim over the plain-C NVFP4 oracle (oracle/nvfp4_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg may use this module; the product (the CUDA
library and its binding) never imports it.  Arrays are numpy; bf16 tensors
are passed as their uint16 bit patterns.  The oracle's arithmetic lives in
the C file; this module only marshals arguments.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        L = _lib
        i64, f32, f64, i32 = ctypes.c_int64, ctypes.c_float, ctypes.c_double, ctypes.c_int
        vp = ctypes.c_void_p
        L.oracle_e2m1_value.restype = f64
        L.oracle_e2m1_value.argtypes = [i32]
        L.oracle_e4m3_value.restype = f64
        L.oracle_e4m3_value.argtypes = [i32]
        L.oracle_e2m1_encode.restype = i32
        L.oracle_e2m1_encode.argtypes = [f64, f64]
        L.oracle_e4m3_round_quotient.restype = i32
        L.oracle_e4m3_round_quotient.argtypes = [f64, f64]
        L.oracle_effective_scale.restype = f32
        L.oracle_effective_scale.argtypes = [f32, i32]
        L.oracle_float_to_bf16.restype = ctypes.c_uint16
        L.oracle_float_to_bf16.argtypes = [f32]
        L.oracle_floats_to_bf16.argtypes = [vp, i64, vp]
        L.oracle_global_scale.argtypes = [vp, i64, vp]
        L.oracle_max_rule_code.argtypes = [vp, f32]
        L.oracle_scale_search_max.argtypes = [vp, i64, i64, f32, vp]
        L.oracle_four_over_six_code.argtypes = [vp, f32]
        L.oracle_gemm_nvfp4.argtypes = [vp, vp, f32, vp, vp, f32, i64, i64, i64, vp, vp]
        L.oracle_fake_quant_static.argtypes = [vp, i64, i64, f32, vp, vp, vp]
        L.oracle_abs_histogram.argtypes = [vp, i64, vp]
        L.oracle_quantile_magnitude.argtypes = [vp, f64, vp]
        L.oracle_static_scale.restype = f32
        L.oracle_static_scale.argtypes = [f64]
        L.oracle_quant_error.restype = f64
        L.oracle_quant_error.argtypes = [vp, i64, i64, f32]
        L.oracle_scale_search_four_over_six.argtypes = [vp, i64, i64, f32, vp]
        L.oracle_block_mse.restype = f64
        L.oracle_block_mse.argtypes = [vp, f32, i32]
        L.oracle_block_lh.restype = f64
        L.oracle_block_lh.argtypes = [vp, f32, i32, vp]
        L.oracle_block_objectives.argtypes = [vp, f32, vp, vp]
        L.oracle_scale_search_mse.argtypes = [vp, i64, i64, f32, vp, vp, vp]
        L.oracle_scale_search_lh.argtypes = [vp, i64, i64, f32, vp, vp, vp, vp]
        L.oracle_scale_search_sampled.argtypes = [vp, i64, f32, vp, vp, vp, i64, vp, vp]
        L.oracle_gram_accumulate.argtypes = [vp, i64, i64, vp]
        L.oracle_gram_accumulate_grouped.argtypes = [vp, vp, i64, i64, vp]
        L.oracle_quantize_pack.argtypes = [vp, i64, i64, f32, vp, vp]
        L.oracle_dequantize.argtypes = [vp, vp, f32, i64, i64, vp]
        L.oracle_fake_quant.argtypes = [vp, i64, i64, vp, vp, vp, vp]
        L.oracle_max_threads.restype = i32
        L.oracle_gram_full.argtypes = [vp, i64, i64, vp]
        L.oracle_gptq_factor.argtypes = [vp, i64, f64, vp]
        L.oracle_gptq_rows.argtypes = [vp, i64, f32, vp, vp, vp, i64, vp, vp]
        L.oracle_gptq.argtypes = [vp, i64, i64, f32, vp, vp, f64, vp]
    return _lib


class OracleError(RuntimeError):
    pass


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    a = np.ascontiguousarray(a)
    if a.dtype != np.uint16:
        raise TypeError("bf16 data must be passed as uint16 bit patterns")
    return a


def _check(st):
    if st != 0:
        raise OracleError("oracle status %d" % st)


def max_threads():
    return lib().oracle_max_threads()


# ------------------------------------------------------------ scalar helpers
def e2m1_value(code):
    return lib().oracle_e2m1_value(int(code))


def e4m3_value(code):
    return lib().oracle_e4m3_value(int(code))


def e2m1_encode(x, s):
    return lib().oracle_e2m1_encode(float(x), float(s))


def e4m3_round_quotient(num, den):
    return lib().oracle_e4m3_round_quotient(float(num), float(den))


def effective_scale(s_g, code):
    return lib().oracle_effective_scale(float(s_g), int(code))


def float_to_bf16(f):
    return lib().oracle_float_to_bf16(float(f))


def floats_to_bf16(a):
    """bf16 bit patterns (uint16) of an fp32 array, rounded by the oracle."""
    a = np.ascontiguousarray(a, np.float32)
    out = np.empty(a.shape, np.uint16)
    lib().oracle_floats_to_bf16(_ptr(a), a.size, _ptr(out))
    return out


# ------------------------------------------------------------ tensor ops
def global_scale(x_u16):
    x = _u16(x_u16)
    out = ctypes.c_float()
    _check(lib().oracle_global_scale(_ptr(x), x.size, ctypes.byref(out)))
    return np.float32(out.value)


def scale_search_max(w_u16, s_g):
    w = _u16(w_u16)
    R, C = w.shape
    codes = np.zeros((R, C // 16), np.uint8)
    _check(lib().oracle_scale_search_max(_ptr(w), R, C, float(s_g), _ptr(codes)))
    return codes


def scale_search_four_over_six(w_u16, s_g):
    w = _u16(w_u16)
    R, C = w.shape
    codes = np.zeros((R, C // 16), np.uint8)
    _check(lib().oracle_scale_search_four_over_six(_ptr(w), R, C, float(s_g), _ptr(codes)))
    return codes


def block_mse(blk_u16, s_g, code):
    b = _u16(blk_u16).reshape(16)
    return lib().oracle_block_mse(_ptr(b), ctypes.c_float(float(s_g)), int(code))


def four_over_six_code(blk_u16, s_g):
    b = _u16(blk_u16).reshape(16)
    return lib().oracle_four_over_six_code(_ptr(b), ctypes.c_float(float(s_g)))


def gemm_nvfp4(a_packed, a_codes, a_sg, b_packed, b_codes, b_sg):
    """Y = dequant(A) dequant(B)^T in fp64 (exact products), and the sum of
    the terms' magnitudes; A [M, K], B [N, K] as packed codes [*, K/2] and
    block codes [*, K/16]."""
    ap = np.ascontiguousarray(a_packed, np.uint8)
    ac = np.ascontiguousarray(a_codes, np.uint8)
    bp = np.ascontiguousarray(b_packed, np.uint8)
    bc = np.ascontiguousarray(b_codes, np.uint8)
    M, N, K = ap.shape[0], bp.shape[0], ap.shape[1] * 2
    Y = np.zeros((M, N), np.float64)
    A = np.zeros((M, N), np.float64)
    _check(lib().oracle_gemm_nvfp4(_ptr(ap), _ptr(ac), float(a_sg), _ptr(bp), _ptr(bc),
                                   float(b_sg), M, N, K, _ptr(Y), _ptr(A)))
    return Y, A


def scale_search_mse(w_u16, s_g, runner_up=False):
    """(codes, best objectives[, runner-up objectives]) of every block."""
    w = _u16(w_u16)
    R, C = w.shape
    codes = np.zeros((R, C // 16), np.uint8)
    best = np.zeros((R, C // 16), np.float64)
    second = np.zeros((R, C // 16), np.float64) if runner_up else None
    _check(lib().oracle_scale_search_mse(_ptr(w), R, C, float(s_g), _ptr(codes), _ptr(best),
                                         _ptr(second)))
    return (codes, best, second) if runner_up else (codes, best)


def scale_search_lh(w_u16, s_g, H, runner_up=False):
    """(codes, best objectives[, runner-up objectives]) of every block."""
    w = _u16(w_u16)
    R, C = w.shape
    H = np.ascontiguousarray(H, dtype=np.float64).reshape(C // 16, 16, 16)
    codes = np.zeros((R, C // 16), np.uint8)
    best = np.zeros((R, C // 16), np.float64)
    second = np.zeros((R, C // 16), np.float64) if runner_up else None
    _check(lib().oracle_scale_search_lh(_ptr(w), R, C, float(s_g), _ptr(H), _ptr(codes),
                                        _ptr(best), _ptr(second)))
    return (codes, best, second) if runner_up else (codes, best)


def scale_search_sampled(w_u16, s_g, H, rows, blocks):
    """Search only the blocks (rows[i], blocks[i]); H=None selects MSE."""
    w = _u16(w_u16)
    C = w.shape[-1]
    rows = np.ascontiguousarray(rows, np.int64)
    blocks = np.ascontiguousarray(blocks, np.int64)
    if H is not None:
        H = np.ascontiguousarray(H, dtype=np.float64).reshape(C // 16, 16, 16)
    codes = np.zeros(rows.size, np.uint8)
    best = np.zeros(rows.size, np.float64)
    _check(lib().oracle_scale_search_sampled(_ptr(w), C, float(s_g), _ptr(H), _ptr(rows),
                                             _ptr(blocks), rows.size, _ptr(codes), _ptr(best)))
    return codes, best


def block_objectives(blk_u16, s_g, Hb=None):
    """All 126 objectives of one 16-element block (index c-1)."""
    b = _u16(blk_u16).reshape(16)
    out = np.zeros(126, np.float64)
    if Hb is not None:
        Hb = np.ascontiguousarray(Hb, dtype=np.float64).reshape(16, 16)
    lib().oracle_block_objectives(_ptr(b), float(s_g), _ptr(Hb), _ptr(out))
    return out


def max_rule_code(blk_u16, s_g):
    b = _u16(blk_u16).reshape(16)
    return lib().oracle_max_rule_code(_ptr(b), ctypes.c_float(float(s_g)))


def gram(x_u16, H=None):
    x = _u16(x_u16)
    N, C = x.shape
    if H is None:
        H = np.zeros((C // 16, 16, 16), np.float64)
    else:
        H = np.ascontiguousarray(H, np.float64).copy()
    _check(lib().oracle_gram_accumulate(_ptr(x), N, C, _ptr(H)))
    return H


def gram_grouped(x_u16, offsets, G):
    x = _u16(x_u16)
    C = x.shape[-1]
    offsets = np.ascontiguousarray(offsets, np.int64)
    H = np.zeros((G, C // 16, 16, 16), np.float64)
    _check(lib().oracle_gram_accumulate_grouped(_ptr(x), _ptr(offsets), G, C, _ptr(H)))
    return H


def quantize_pack(w_u16, s_g, codes):
    w = _u16(w_u16)
    R, C = w.shape
    codes = np.ascontiguousarray(codes, np.uint8)
    packed = np.zeros((R, C // 2), np.uint8)
    _check(lib().oracle_quantize_pack(_ptr(w), R, C, float(s_g), _ptr(codes), _ptr(packed)))
    return packed


def dequantize(packed, codes, s_g):
    packed = np.ascontiguousarray(packed, np.uint8)
    codes = np.ascontiguousarray(codes, np.uint8)
    R, C = packed.shape[0], packed.shape[1] * 2
    out = np.zeros((R, C), np.uint16)
    _check(lib().oracle_dequantize(_ptr(packed), _ptr(codes), float(s_g), R, C, _ptr(out)))
    return out


def fake_quant_static(x_u16, s_g, want_packed=True):
    x = _u16(x_u16)
    R, C = x.shape
    out = np.zeros((R, C), np.uint16)
    packed = np.zeros((R, C // 2), np.uint8) if want_packed else None
    codes = np.zeros((R, C // 16), np.uint8) if want_packed else None
    _check(lib().oracle_fake_quant_static(_ptr(x), R, C, float(s_g), _ptr(out), _ptr(packed),
                                          _ptr(codes)))
    return out, packed, codes


def abs_histogram(x_u16, hist=None):
    x = _u16(x_u16).reshape(-1)
    if hist is None:
        hist = np.zeros(32768, np.uint64)
    lib().oracle_abs_histogram(_ptr(x), x.size, _ptr(hist))
    return hist


def quantile_magnitude(hist, p):
    m = ctypes.c_double()
    h = np.ascontiguousarray(hist, np.uint64)
    _check(lib().oracle_quantile_magnitude(_ptr(h), float(p), ctypes.byref(m)))
    return m.value


def static_scale(clip):
    return np.float32(lib().oracle_static_scale(float(clip)))


def quant_error(x_u16, s_g):
    x = _u16(x_u16)
    R, C = x.shape
    return lib().oracle_quant_error(_ptr(x), R, C, float(s_g))


def fake_quant(x_u16, want_packed=True):
    x = _u16(x_u16)
    R, C = x.shape
    out = np.zeros((R, C), np.uint16)
    packed = np.zeros((R, C // 2), np.uint8) if want_packed else None
    codes = np.zeros((R, C // 16), np.uint8) if want_packed else None
    s_g = ctypes.c_float()
    _check(lib().oracle_fake_quant(_ptr(x), R, C, _ptr(out), _ptr(packed), _ptr(codes),
                                   ctypes.byref(s_g)))
    return out, packed, codes, np.float32(s_g.value)


# ------------------------------------------------------------ full Gram, GPTQ
def gram_full(x_u16, H=None):
    """H += X^T X over all channels (fp64 [C, C])."""
    x = _u16(x_u16)
    N, C = x.shape
    if H is None:
        H = np.zeros((C, C), np.float64)
    H = np.ascontiguousarray(H, np.float64)
    _check(lib().oracle_gram_full(_ptr(x), N, C, _ptr(H)))
    return H


def gptq_factor(H, damp=0.01):
    """Upper Cholesky factor U of (H + damp mean(diag H) I)^-1."""
    H = np.ascontiguousarray(H, np.float64)
    C = H.shape[0]
    U = np.zeros((C, C), np.float64)
    _check(lib().oracle_gptq_factor(_ptr(H), C, float(damp), _ptr(U)))
    return U


def gptq_rows(w_u16, s_g, codes, U, rows):
    """GPTQ codes of the listed rows: (packed [n, C/2], value at rounding [n, C])."""
    w = _u16(w_u16)
    C = w.shape[1]
    codes = np.ascontiguousarray(codes, np.uint8)
    U = np.ascontiguousarray(U, np.float64)
    rows = np.ascontiguousarray(rows, np.int64)
    packed = np.zeros((rows.size, C // 2), np.uint8)
    wq = np.zeros((rows.size, C), np.float64)
    _check(lib().oracle_gptq_rows(_ptr(w), C, float(s_g), _ptr(codes), _ptr(U), _ptr(rows),
                                  rows.size, _ptr(packed), _ptr(wq)))
    return packed, wq


def gptq(w_u16, s_g, codes, H, damp=0.01):
    """Packed GPTQ codes of W [R, C] at the given block codes."""
    w = _u16(w_u16)
    R, C = w.shape
    codes = np.ascontiguousarray(codes, np.uint8)
    H = np.ascontiguousarray(H, np.float64)
    packed = np.zeros((R, C // 2), np.uint8)
    _check(lib().oracle_gptq(_ptr(w), R, C, float(s_g), _ptr(codes), _ptr(H), float(damp),
                             _ptr(packed)))
    return packed
