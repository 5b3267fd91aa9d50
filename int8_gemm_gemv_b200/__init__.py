"""Python binding of libbsq (include/bsq.h): same names, argument marshalling
only.  Every step of every call runs in libbsq's CUDA kernels; there is no
Python or CPU fallback, and importing a function whose library is missing
raises.

Tensor arguments are CUDA tensors (any dtype of the right width: BF16 data
may be torch.bfloat16 or int16; E4M3/E2M1 data uint8), or raw integer device
addresses.  ``stream`` is a torch.cuda.Stream, a raw cudaStream_t integer, or
None for torch's current stream.  A non-OK status raises BsqError.
"""
from __future__ import annotations

import ctypes
import os

__all__ = [
    "BsqError", "BSQ_OK", "BSQ_ERR_INVALID_ARG", "BSQ_ERR_MISALIGNED", "BSQ_ERR_UNSUPPORTED",
    "BSQ_ERR_CUDA", "BSQ_FP8_PER_ROW", "BSQ_FP8_BLOCK_SCALED", "BSQ_FP8_SINGLE_SCALE", "BSQ_BF16",
    "BSQ_NVFP4", "quantize_bf16_to_nvfp4", "quantize_bf16_to_nvfp4_devscale", "w4a4_gemm",
    "w4a4_gemm_devscale", "fp8_gemv_rowscale", "fp8_gemv_blockscaled",
    "quant_rowwise_fp8",
    "quant_blockfp8", "requant_w_nvfp4_int8", "quant_act_int8_per32", "int8_blockscaled_gemm",
    "int8_w4a8_prefill", "int8_w4a8_prefill_noalloc", "requant_blockfp8_to_rowwise", "fp8_gemm_rowscale", "bsq_amax_bf16",
    "status_string", "debug_launch_count", "debug_take_timeouts", "library_path", "lib",
]

BSQ_OK, BSQ_ERR_INVALID_ARG, BSQ_ERR_MISALIGNED, BSQ_ERR_UNSUPPORTED, BSQ_ERR_CUDA = range(5)
BSQ_FP8_PER_ROW, BSQ_FP8_BLOCK_SCALED, BSQ_FP8_SINGLE_SCALE, BSQ_BF16, BSQ_NVFP4 = range(5)

_HERE = os.path.dirname(os.path.abspath(__file__))


def library_path() -> str:
    return os.path.join(_HERE, "libbsq.so")


class BsqError(RuntimeError):
    def __init__(self, status: int, fn: str, detail: str | None = None):
        self.status = status
        msg = f"{fn}: {status_string(status)}"
        super().__init__(msg + (f" ({detail})" if detail else ""))


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float

_SIGS = {
    "quantize_bf16_to_nvfp4": [_P, _P, _P, _F, _I, _I, _P],
    "quantize_bf16_to_nvfp4_devscale": [_P, _P, _P, _P, _P, _I, _I, _P],
    "w4a4_gemm": [_P, _P, _P, _P, _P, _F, _F, _I, _I, _I, _P],
    "w4a4_gemm_devscale": [_P, _P, _P, _P, _P, _F, _P, _I, _I, _I, _P],
    "fp8_gemv_rowscale": [_P, _P, _P, _P, _I, _I, _I, _P],
    "fp8_gemv_blockscaled": [_P, _P, _P, _P, _I, _I, _I, _P],
    "quant_rowwise_fp8": [_P, _P, _P, _I, _I, _P],
    "quant_blockfp8": [_P, _P, _P, _I, _I, _P],
    "requant_w_nvfp4_int8": [_P, _P, _F, _P, _P, _I, _I, _P],
    "quant_act_int8_per32": [_P, _P, _P, _I, _I, _P],
    "int8_blockscaled_gemm": [_P, _P, _P, _P, _P, _I, _I, _I, _P],
    "int8_blockscaled_gemm_ws": [_P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _P],
    "int8_w4a8_prefill": [_P, _P, _P, _P, _P, _P, _I, _I, _I, _P],
    "int8_w4a8_prefill_noalloc": [_P, _P, _P, _P, _I, _I, _I, _P],
    "requant_blockfp8_to_rowwise": [_I, _P, _P, _I, _I, _P, _P, ctypes.POINTER(_P), ctypes.POINTER(_P), _P],
    "fp8_gemm_rowscale": [_P, _P, _P, _P, _P, _I, _I, _I, _P],
    "bsq_amax_bf16": [_P, ctypes.c_size_t, _P, _P],
    "bsq_debug_stream_read": [_P, ctypes.c_size_t, _P, _I, _P],
}


def lib() -> ctypes.CDLL:
    """The loaded libbsq.so.  Raises when it has not been built."""
    global _lib
    if _lib is None:
        path = library_path()
        if not os.path.exists(path):
            raise ImportError(f"libbsq.so not found at {path}; build it with "
                              "`python -m int8_gemm_gemv_b200.build`")
        L = ctypes.CDLL(path)
        for name, args in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ctypes.c_int
        L.bsq_status_string.argtypes = [ctypes.c_int]
        L.bsq_status_string.restype = ctypes.c_char_p
        L.bsq_debug_launch_count.argtypes = []
        L.bsq_debug_launch_count.restype = ctypes.c_uint64
        L.bsq_debug_take_timeouts.argtypes = []
        L.bsq_debug_take_timeouts.restype = ctypes.c_uint32
        L.bsq_debug_take_cuda_error.argtypes = []
        L.bsq_debug_take_cuda_error.restype = ctypes.c_int
        L.bsq_debug_cuda_error_string.argtypes = [ctypes.c_int]
        L.bsq_debug_cuda_error_string.restype = ctypes.c_char_p
        L.int8_gemm_workspace_bytes.argtypes = []
        L.int8_gemm_workspace_bytes.restype = ctypes.c_size_t
        _lib = L
    return _lib


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda:
        raise ValueError("libbsq takes CUDA tensors (device memory)")
    if not t.is_contiguous():
        raise ValueError("libbsq takes contiguous tensors")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _call(name, *args):
    L = lib()
    st = getattr(L, name)(*args)
    if st != BSQ_OK:
        detail = None
        if st == BSQ_ERR_CUDA:
            code = L.bsq_debug_take_cuda_error()
            detail = f"cudaError {code}: {L.bsq_debug_cuda_error_string(code).decode()}"
        raise BsqError(st, name, detail)


def status_string(status: int) -> str:
    return lib().bsq_status_string(status).decode()


def debug_launch_count() -> int:
    return lib().bsq_debug_launch_count()


def debug_take_timeouts() -> int:
    return lib().bsq_debug_take_timeouts()


def quantize_bf16_to_nvfp4(inp, packed, scale, scale2, m, k, stream=None):
    _call("quantize_bf16_to_nvfp4", _ptr(inp), _ptr(packed), _ptr(scale), scale2, m, k, _stream(stream))


def quantize_bf16_to_nvfp4_devscale(inp, packed, scale, amax, scale2_out, m, k, stream=None):
    """scale2 = amax / (6 * 448) formed on the device; scale2_out may be None."""
    _call("quantize_bf16_to_nvfp4_devscale", _ptr(inp), _ptr(packed), _ptr(scale), _ptr(amax), _ptr(scale2_out),
          m, k, _stream(stream))


def w4a4_gemm_devscale(a_packed, a_scale, w_packed, w_scale, out, scaleA2, scaleB2_dev, m, n, k, stream=None):
    _call("w4a4_gemm_devscale", _ptr(a_packed), _ptr(a_scale), _ptr(w_packed), _ptr(w_scale), _ptr(out),
          scaleA2, _ptr(scaleB2_dev), m, n, k, _stream(stream))


def w4a4_gemm(a_packed, a_scale, w_packed, w_scale, out, scaleA2, scaleB2, m, n, k, stream=None):
    _call("w4a4_gemm", _ptr(a_packed), _ptr(a_scale), _ptr(w_packed), _ptr(w_scale), _ptr(out),
          scaleA2, scaleB2, m, n, k, _stream(stream))


def fp8_gemv_rowscale(inp, w, row_scale, out, m, n, k, stream=None):
    _call("fp8_gemv_rowscale", _ptr(inp), _ptr(w), _ptr(row_scale), _ptr(out), m, n, k, _stream(stream))


def fp8_gemv_blockscaled(inp, w, block_scale, out, m, n, k, stream=None):
    _call("fp8_gemv_blockscaled", _ptr(inp), _ptr(w), _ptr(block_scale), _ptr(out), m, n, k, _stream(stream))


def quant_rowwise_fp8(inp, q, scale, rows, k, stream=None):
    _call("quant_rowwise_fp8", _ptr(inp), _ptr(q), _ptr(scale), rows, k, _stream(stream))


def quant_blockfp8(inp, q, scale, n, k, stream=None):
    _call("quant_blockfp8", _ptr(inp), _ptr(q), _ptr(scale), n, k, _stream(stream))


def requant_w_nvfp4_int8(w_packed, w_e4m3, scale2, w_i8, w_scale, n, k, stream=None):
    _call("requant_w_nvfp4_int8", _ptr(w_packed), _ptr(w_e4m3), scale2, _ptr(w_i8), _ptr(w_scale), n, k,
          _stream(stream))


def quant_act_int8_per32(a, a_i8, a_scale, m, k, stream=None):
    _call("quant_act_int8_per32", _ptr(a), _ptr(a_i8), _ptr(a_scale), m, k, _stream(stream))


def int8_blockscaled_gemm(a_i8, w_i8, a_scale, w_scale, out, m, n, k, stream=None):
    _call("int8_blockscaled_gemm", _ptr(a_i8), _ptr(w_i8), _ptr(a_scale), _ptr(w_scale), _ptr(out), m, n, k,
          _stream(stream))


def int8_gemm_workspace_bytes():
    """Bytes of the workspace int8_blockscaled_gemm_ws needs on the current
    device (0 when it cannot be queried)."""
    return int(lib().int8_gemm_workspace_bytes())


def int8_blockscaled_gemm_ws(a_i8, w_i8, a_scale, w_scale, out, workspace, ws_bytes, m, n, k, stream=None):
    """int8_blockscaled_gemm with a workspace (zeroed once before first use)
    that lets a partial last round of tiles be split along K."""
    _call("int8_blockscaled_gemm_ws", _ptr(a_i8), _ptr(w_i8), _ptr(a_scale), _ptr(w_scale), _ptr(out),
          _ptr(workspace), ws_bytes, m, n, k, _stream(stream))


def int8_w4a8_prefill(a_bf16, w_i8, w_scale, a_i8_scratch, a_scale_scratch, out, m, n, k, stream=None):
    _call("int8_w4a8_prefill", _ptr(a_bf16), _ptr(w_i8), _ptr(w_scale), _ptr(a_i8_scratch),
          _ptr(a_scale_scratch), _ptr(out), m, n, k, _stream(stream))


def int8_w4a8_prefill_noalloc(a_bf16, w_i8, w_scale, out, m, n, k, stream=None):
    """int8_w4a8_prefill with the activation scratch inside the library (for
    callers that cannot allocate device memory); see include/bsq.h."""
    _call("int8_w4a8_prefill_noalloc", _ptr(a_bf16), _ptr(w_i8), _ptr(w_scale), _ptr(out), m, n, k,
          _stream(stream))


def requant_blockfp8_to_rowwise(tag, w, scale, n, k, w_out, scale_out, stream=None):
    """Returns (w_used, scale_used) as integer device addresses."""
    wu, su = _P(), _P()
    _call("requant_blockfp8_to_rowwise", tag, _ptr(w), _ptr(scale), n, k, _ptr(w_out), _ptr(scale_out),
          ctypes.byref(wu), ctypes.byref(su), _stream(stream))
    return wu.value, su.value


def fp8_gemm_rowscale(a, a_scale, w, w_scale, out, m, n, k, stream=None):
    _call("fp8_gemm_rowscale", _ptr(a), _ptr(a_scale), _ptr(w), _ptr(w_scale), _ptr(out), m, n, k,
          _stream(stream))


def bsq_amax_bf16(x, count, amax_dev, stream=None):
    _call("bsq_amax_bf16", _ptr(x), count, _ptr(amax_dev), _stream(stream))


def debug_stream_read(src, nbytes, sink, mode=0, stream=None):
    """Read-only streaming kernel over nbytes of src (the HBM floor)."""
    _call("bsq_debug_stream_read", _ptr(src), nbytes, _ptr(sink), mode, _stream(stream))
