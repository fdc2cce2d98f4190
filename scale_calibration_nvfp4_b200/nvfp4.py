"""Thin ctypes binding of libnvfp4.so (see include/nvfp4.h).

Argument marshalling only: every function checks dtype, device, shape and
contiguity of the torch tensors it is given, passes their device pointers and
torch's current CUDA stream to the C entry point of the same name, and raises
``NVFP4Error`` on a non-OK status.  All computation happens in the library's
CUDA kernels; there is no CPU or PyTorch fallback.  If the library is missing
the first call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

STATUS = {
    0: "NVFP4_OK", 1: "NVFP4_ERR_INVALID_ARG", 2: "NVFP4_ERR_SHAPE", 3: "NVFP4_ERR_MISALIGNED",
    4: "NVFP4_ERR_NONFINITE", 5: "NVFP4_ERR_CUDA", 6: "NVFP4_ERR_NOT_IMPLEMENTED",
    7: "NVFP4_ERR_TOO_LARGE", 8: "NVFP4_ERR_DEVICE_TIMEOUT", 9: "NVFP4_ERR_NOT_POSITIVE_DEFINITE",
    10: "NVFP4_ERR_DEVICE_UNDRAINED",
}

# C entry points and their argument types (mirrors include/nvfp4.h)
_vp, _i64 = ctypes.c_void_p, ctypes.c_int64
SIGNATURES = {
    "nvfp4_global_scale": [_vp, _i64, _i64, _vp, _vp],
    "nvfp4_hessian_accumulate": [_vp, _i64, _i64, _vp, _vp],
    "nvfp4_hessian_accumulate_noalloc": [_vp, _i64, _i64, _vp, _vp],
    "nvfp4_hessian_accumulate_grouped": [_vp, _vp, _i64, _i64, _i64, _vp, _vp],
    "nvfp4_scale_search_max": [_vp, _i64, _i64, _i64, _vp, _vp, _vp],
    "nvfp4_scale_search_four_over_six": [_vp, _i64, _i64, _i64, _vp, _vp, _vp],
    "nvfp4_scale_search_mse": [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp],
    "nvfp4_scale_search_local_hessian": [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp],
    "nvfp4_quantize_pack": [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp],
    "nvfp4_dequantize": [_vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp],
    "nvfp4_fake_quant": [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp],
    "nvfp4_get_device_status": [_vp, _vp],
    "nvfp4_search_evaluations": [_vp, ctypes.c_int, _vp],
    "nvfp4_search_rescores": [_vp, ctypes.c_int, _vp],
    "nvfp4_self_test_device_timeout": [_vp],
    "nvfp4_self_test_mma": [_vp, _vp, _vp, _vp, _i64, _vp],
    "nvfp4_gemm": [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp],
    "nvfp4_abs_histogram": [_vp, _i64, _vp, _vp],
    "nvfp4_static_scale_from_histogram": [_vp, ctypes.c_double, _vp, _vp],
    "nvfp4_fake_quant_static": [_vp, _i64, _i64, _vp, _vp, _vp, _vp, _vp],
    "nvfp4_quant_error": [_vp, _i64, _i64, _vp, _vp, _vp],
    "nvfp4_hessian_full_accumulate": [_vp, _i64, _i64, _vp, _vp],
    "nvfp4_gptq": [_vp, _i64, _i64, _i64, _vp, _vp, _vp, ctypes.c_double, _vp, _vp],
}


class NVFP4Error(RuntimeError):
    def __init__(self, fn, status):
        self.status = status
        super().__init__("%s failed: %s" % (fn, STATUS.get(status, str(status))))


_lib = None


def lib():
    """Load libnvfp4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libnvfp4.so not found at %s; build it with "
                               "`python -m scale_calibration_nvfp4_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, args in SIGNATURES.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.nvfp4_status_string.argtypes = [ctypes.c_int]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        L.nvfp4_shutdown.argtypes = []
        L.nvfp4_shutdown.restype = None
        _lib = L
    return _lib


def _call(name, *args):
    st = getattr(lib(), name)(*args)
    if st != 0:
        raise NVFP4Error(name, st)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, dtype, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


def _weight_shape(w):
    if w.dim() == 2:
        return 1, w.shape[0], w.shape[1]
    if w.dim() == 3:
        return w.shape[0], w.shape[1], w.shape[2]
    raise ValueError("weights must be [R, C] or [batch, R, C]")


# --------------------------------------------------------------- entry points
def global_scale(x, batch=1, out=None, stream=None):
    """FP32 tensor scale(s) of ``x`` (bf16); ``batch`` equal slices."""
    _need(x, torch.bfloat16, "x")
    n = x.numel()
    if n % batch:
        raise ValueError("numel not divisible by batch")
    if out is None:
        out = torch.empty(batch, dtype=torch.float32, device=x.device)
    _need(out, torch.float32, "out")
    _call("nvfp4_global_scale", _p(x), batch, n // batch, _p(out), _stream(stream))
    return out


def hessian_accumulate(x, H, stream=None):
    """H[C/16,16,16] += block-diagonal Gram of x[N, C] (in place)."""
    _need(x, torch.bfloat16, "x")
    _need(H, torch.float32, "H")
    N, C = x.shape
    if H.numel() != (C // 16) * 256:
        raise ValueError("H must hold C/16 x 16 x 16 floats")
    _call("nvfp4_hessian_accumulate", _p(x), N, C, _p(H), _stream(stream))
    return H


def hessian_full_accumulate(x, H, stream=None):
    """H[C, C] += x^T x over all channels (in place, tensor cores)."""
    _need(x, torch.bfloat16, "x")
    _need(H, torch.float32, "H")
    N, C = x.shape
    if H.numel() != C * C:
        raise ValueError("H must hold C x C floats")
    _call("nvfp4_hessian_full_accumulate", _p(x), N, C, _p(H), _stream(stream))
    return H


def hessian_accumulate_noalloc(x, H, stream=None):
    """As hessian_accumulate, for callers that may not allocate device memory:
    the library keeps the partial sums in its own fixed 16 MiB device array
    (C <= 262,144).  Calls that overlap on the GPU share that array and race;
    make the first call on a device outside stream capture."""
    _need(x, torch.bfloat16, "x")
    _need(H, torch.float32, "H")
    N, C = x.shape
    if H.numel() != (C // 16) * 256:
        raise ValueError("H must hold C/16 x 16 x 16 floats")
    _call("nvfp4_hessian_accumulate_noalloc", _p(x), N, C, _p(H), _stream(stream))
    return H


def hessian_accumulate_grouped(x, offsets, H, stream=None):
    """H[g] += Gram of rows offsets[g]..offsets[g+1] of x (offsets: CUDA int64 [G+1])."""
    _need(x, torch.bfloat16, "x")
    _need(offsets, torch.int64, "offsets")
    _need(H, torch.float32, "H")
    N, C = x.shape
    G = offsets.numel() - 1
    if H.numel() != G * (C // 16) * 256:
        raise ValueError("H must hold G x C/16 x 16 x 16 floats")
    _call("nvfp4_hessian_accumulate_grouped", _p(x), _p(offsets), G, N, C, _p(H),
          _stream(stream))
    return H


def _codes_out(w, out):
    B, R, C = _weight_shape(w)
    shape = (R, C // 16) if w.dim() == 2 else (B, R, C // 16)
    if out is None:
        out = torch.empty(shape, dtype=torch.uint8, device=w.device)
    _need(out, torch.uint8, "scale_codes")
    return out


def _obj_out(w, want):
    if not want:
        return None
    B, R, C = _weight_shape(w)
    shape = (R, C // 16) if w.dim() == 2 else (B, R, C // 16)
    return torch.empty(shape, dtype=torch.float32, device=w.device)


def scale_search_max(w, s_g, out=None, stream=None):
    _need(w, torch.bfloat16, "w")
    _need(s_g, torch.float32, "s_g")
    B, R, C = _weight_shape(w)
    out = _codes_out(w, out)
    _call("nvfp4_scale_search_max", _p(w), B, R, C, _p(s_g), _p(out), _stream(stream))
    return out


def scale_search_four_over_six(w, s_g, out=None, stream=None):
    _need(w, torch.bfloat16, "w")
    _need(s_g, torch.float32, "s_g")
    B, R, C = _weight_shape(w)
    out = _codes_out(w, out)
    _call("nvfp4_scale_search_four_over_six", _p(w), B, R, C, _p(s_g), _p(out), _stream(stream))
    return out


def scale_search_mse(w, s_g, out=None, return_objective=False, stream=None):
    _need(w, torch.bfloat16, "w")
    _need(s_g, torch.float32, "s_g")
    B, R, C = _weight_shape(w)
    out = _codes_out(w, out)
    obj = _obj_out(w, return_objective)
    _call("nvfp4_scale_search_mse", _p(w), B, R, C, _p(s_g), _p(out), _p(obj),
          _stream(stream))
    return (out, obj) if return_objective else out


def scale_search_local_hessian(w, s_g, H, out=None, return_objective=False, stream=None):
    _need(w, torch.bfloat16, "w")
    _need(s_g, torch.float32, "s_g")
    _need(H, torch.float32, "H")
    B, R, C = _weight_shape(w)
    if H.numel() != B * (C // 16) * 256:
        raise ValueError("H must hold batch x C/16 x 16 x 16 floats")
    out = _codes_out(w, out)
    obj = _obj_out(w, return_objective)
    _call("nvfp4_scale_search_local_hessian", _p(w), B, R, C, _p(s_g), _p(H), _p(out), _p(obj),
          _stream(stream))
    return (out, obj) if return_objective else out


def quantize_pack(w, s_g, scale_codes, out=None, stream=None):
    _need(w, torch.bfloat16, "w")
    _need(s_g, torch.float32, "s_g")
    _need(scale_codes, torch.uint8, "scale_codes")
    B, R, C = _weight_shape(w)
    shape = (R, C // 2) if w.dim() == 2 else (B, R, C // 2)
    if out is None:
        out = torch.empty(shape, dtype=torch.uint8, device=w.device)
    _need(out, torch.uint8, "packed")
    _call("nvfp4_quantize_pack", _p(w), B, R, C, _p(s_g), _p(scale_codes), _p(out),
          _stream(stream))
    return out


def gptq(w, s_g, scale_codes, H, damp=0.01, out=None, stream=None):
    """Packed GPTQ codes of w ([R, C] or [batch, R, C]) at the given block
    codes, with the full Hessian(s) H ([C, C] or [batch, C, C], float32)."""
    _need(w, torch.bfloat16, "w")
    _need(s_g, torch.float32, "s_g")
    _need(scale_codes, torch.uint8, "scale_codes")
    _need(H, torch.float32, "H")
    B, R, C = _weight_shape(w)
    if H.numel() != B * C * C:
        raise ValueError("H must hold batch x C x C floats")
    shape = (R, C // 2) if w.dim() == 2 else (B, R, C // 2)
    if out is None:
        out = torch.empty(shape, dtype=torch.uint8, device=w.device)
    _need(out, torch.uint8, "packed")
    _call("nvfp4_gptq", _p(w), B, R, C, _p(s_g), _p(scale_codes), _p(H), float(damp), _p(out),
          _stream(stream))
    return out


def dequantize(packed, scale_codes, s_g, out=None, stream=None):
    _need(packed, torch.uint8, "packed")
    _need(scale_codes, torch.uint8, "scale_codes")
    _need(s_g, torch.float32, "s_g")
    if packed.dim() == 2:
        B, R, C = 1, packed.shape[0], packed.shape[1] * 2
        shape = (R, C)
    else:
        B, R, C = packed.shape[0], packed.shape[1], packed.shape[2] * 2
        shape = (B, R, C)
    if out is None:
        out = torch.empty(shape, dtype=torch.bfloat16, device=packed.device)
    _need(out, torch.bfloat16, "out")
    _call("nvfp4_dequantize", _p(packed), _p(scale_codes), _p(s_g), B, R, C, _p(out),
          _stream(stream))
    return out


def fake_quant(x, want_packed=False, out=None, stream=None):
    """Dynamic W4A4 fake-quant of x[rows, C]: (out, packed|None, codes|None, s_g)."""
    _need(x, torch.bfloat16, "x")
    rows, C = x.shape
    if out is None:
        out = torch.empty_like(x)
    _need(out, torch.bfloat16, "out")
    packed = torch.empty(rows, C // 2, dtype=torch.uint8, device=x.device) if want_packed else None
    codes = torch.empty(rows, C // 16, dtype=torch.uint8, device=x.device) if want_packed else None
    s_g = torch.empty(1, dtype=torch.float32, device=x.device)
    _call("nvfp4_fake_quant", _p(x), rows, C, _p(out), _p(packed), _p(codes), _p(s_g),
          _stream(stream))
    return out, packed, codes, s_g


def get_device_status(stream=None):
    """Synchronise the stream and return (and clear) the device-side status name."""
    st = ctypes.c_int(0)
    _call("nvfp4_get_device_status", _stream(stream), ctypes.byref(st))
    return STATUS.get(st.value, str(st.value))


def search_evaluations(reset=False, stream=None):
    """(MSE, Local-Hessian) counts of (block, candidate) objective evaluations
    made by the scale searches on the current device since the last reset;
    synchronises the stream."""
    out = (ctypes.c_uint64 * 2)()
    _call("nvfp4_search_evaluations", _stream(stream), int(bool(reset)), out)
    return int(out[0]), int(out[1])


def search_rescores(reset=False, stream=None):
    """Rows sent to the fp64 re-score since the last reset: (MSE over the
    best two, MSE over all 126, Local-Hessian over the best two, Local-Hessian
    over all 126); synchronises the stream.  A reset zeroes every search
    statistic, the evaluation counts included."""
    out = (ctypes.c_uint64 * 4)()
    _call("nvfp4_search_rescores", _stream(stream), int(bool(reset)), out)
    return tuple(int(v) for v in out)


def gemm(a_packed, a_codes, a_sg, b_packed, b_codes, b_sg, out=None, stream=None):
    """out[M, N] (bf16) = A B^T for NVFP4 operands A [M, K] and B [N, K] given
    as packed codes [*, K/2], block codes [*, K/16] and tensor scales [1]."""
    for t, n in ((a_packed, "a_packed"), (a_codes, "a_codes"), (b_packed, "b_packed"),
                 (b_codes, "b_codes")):
        _need(t, torch.uint8, n)
    _need(a_sg, torch.float32, "a_sg")
    _need(b_sg, torch.float32, "b_sg")
    M, N, K = a_packed.shape[0], b_packed.shape[0], a_packed.shape[1] * 2
    if b_packed.shape[1] * 2 != K or a_codes.shape != (M, K // 16) or b_codes.shape != (N, K // 16):
        raise ValueError("operand shapes do not match")
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=a_packed.device)
    _need(out, torch.bfloat16, "out")
    _call("nvfp4_gemm", _p(a_packed), _p(a_codes), _p(a_sg), _p(b_packed), _p(b_codes), _p(b_sg),
          M, N, K, _p(out), _stream(stream))
    return out


def abs_histogram(x, hist=None, stream=None):
    """hist[32768] (uint64, CUDA) += counts of |x| by bf16 magnitude pattern."""
    _need(x, torch.bfloat16, "x")
    if hist is None:
        hist = torch.zeros(32768, dtype=torch.int64, device=x.device)
    if hist.dtype != torch.int64 or hist.numel() != 32768 or not hist.is_cuda:
        raise ValueError("hist must be a CUDA int64 tensor of 32768 counts")
    _call("nvfp4_abs_histogram", _p(x), x.numel(), _p(hist), _stream(stream))
    return hist


def static_scale_from_histogram(hist, p, out=None, stream=None):
    """Static tensor scale fl32(m / 2688) from the p-quantile m of the counts."""
    if out is None:
        out = torch.empty(1, dtype=torch.float32, device=hist.device)
    _call("nvfp4_static_scale_from_histogram", _p(hist), float(p), _p(out), _stream(stream))
    return out


def fake_quant_static(x, s_g, want_packed=False, stream=None):
    """Fake-quant of x [rows, C] at the given tensor scale; returns
    (out, packed, codes) (packed/codes None unless want_packed)."""
    _need(x, torch.bfloat16, "x")
    _need(s_g, torch.float32, "s_g")
    rows, C = x.shape
    out = torch.empty_like(x)
    packed = torch.empty(rows, C // 2, dtype=torch.uint8, device=x.device) if want_packed else None
    codes = torch.empty(rows, C // 16, dtype=torch.uint8, device=x.device) if want_packed else None
    _call("nvfp4_fake_quant_static", _p(x), rows, C, _p(s_g), _p(out),
          _p(packed) if packed is not None else None, _p(codes) if codes is not None else None,
          _stream(stream))
    return out, packed, codes


def quant_error(x, s_g, out=None, stream=None):
    """sum (x - fake_quant_static(x, s_g))^2 in fp64, as a CUDA float64 [1]."""
    _need(x, torch.bfloat16, "x")
    _need(s_g, torch.float32, "s_g")
    rows, C = x.shape
    if out is None:
        out = torch.empty(1, dtype=torch.float64, device=x.device)
    _call("nvfp4_quant_error", _p(x), rows, C, _p(s_g), _p(out), _stream(stream))
    return out


def self_test_device_timeout(stream=None):
    """Enqueue the diagnostic wait that times out (about one second); the
    next get_device_status() reports NVFP4_ERR_DEVICE_TIMEOUT."""
    _call("nvfp4_self_test_device_timeout", _stream(stream))


def self_test_mma(a, b, c, stream=None):
    """d = a b + c per tile through the screen's tensor-core instruction:
    a [n, 16, 16] and b [n, 16, 8] float16, c [n, 16, 8] float32 (CUDA)."""
    _need(a, torch.float16, "a")
    _need(b, torch.float16, "b")
    _need(c, torch.float32, "c")
    n = a.shape[0]
    if a.shape != (n, 16, 16) or b.shape != (n, 16, 8) or c.shape != (n, 16, 8):
        raise ValueError("a [n,16,16], b [n,16,8], c [n,16,8]")
    d = torch.empty_like(c)
    _call("nvfp4_self_test_mma", _p(a), _p(b), _p(c), _p(d), n, _stream(stream))
    return d


def status_string(code):
    return lib().nvfp4_status_string(int(code)).decode()


def shutdown():
    lib().nvfp4_shutdown()
