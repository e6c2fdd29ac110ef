"""Python binding of libsq (include/sq.h): argument marshalling only.

Every function has the name of the C entry point it calls and takes torch CUDA
tensors (bf16 matrices as ``torch.bfloat16``, codes as ``torch.int8``, scales as
``torch.float32``); it checks dtypes, shapes and strides, passes raw device
pointers and the current (or given) stream, and raises ``SqError`` on a non-OK
status. All computation happens in the library's CUDA kernels; there is no
fallback of any kind: if ``libsq.so`` is missing, importing this module fails.
"""
from __future__ import annotations

import ctypes as C
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
# SQ_LIB_PATH selects another build of the same ABI (the bounds-guard build libsq_debug.so)
LIB_PATH = os.environ.get("SQ_LIB_PATH") or os.path.join(_HERE, "libsq.so")

SQ_OK, SQ_ERR_INVALID, SQ_ERR_ALIGN, SQ_ERR_CUDA, SQ_ERR_TIMEOUT, SQ_ERR_WORKSPACE, SQ_ERR_UNSUPPORTED = \
    0, -1, -2, -3, -4, -5, -6
SQ_ERR_BOUNDS = -7
SQ_PER_TENSOR, SQ_PER_CHANNEL = 0, 1
SQ_OP_SMOOTH_QUANT_WEIGHT, SQ_OP_INT8_GEMM_DEQUANT, SQ_OP_LLMINT8 = 1, 2, 3
SQ_OP_QUANT_ACT_PER_TENSOR, SQ_OP_MEAN_STD_THRESHOLD, SQ_OP_ABS_PERCENTILE = 4, 5, 6
SQ_NORM_LAYER, SQ_NORM_RMS = 0, 1

if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m w8a8_quantized_gemm_b200.build`")

_lib = C.CDLL(LIB_PATH)
_p, _i64, _i32, _f32, _sz = C.c_void_p, C.c_int64, C.c_int, C.c_float, C.c_size_t
_SIGS = {
    "sq_act_channel_absmax": ([_p, _i64, _i64, _i64, _p, _i32, _p], _i32),
    "sq_smooth_scale": ([_p, _p, _i64, _i64, _i64, _f32, _p, _p, _p], _i32),
    "sq_smooth_quant_weight": ([_p, _i64, _i64, _i64, _p, _i32, _p, _p, _p, _sz, _p], _i32),
    "sq_quant_act_per_token": ([_p, _i64, _i64, _i64, _p, _p, _p, _p], _i32),
    "sq_int8_gemm_dequant": ([_p, _p, _p, _p, _i32, _p, _p, _i64, _i64, _i64, _p, _p, _sz, _p], _i32),
    "llmint8_decomposed_linear": ([_p, _p, _p, _p, _f32, _p, _p, _i64, _i64, _i64, _p, _p, _p, _p, _sz, _p], _i32),
    "sq_smooth_quant_weight_noalloc": ([_p, _i64, _i64, _i64, _p, _i32, _p, _p, _p], _i32),
    "sq_quant_act_per_tensor": ([_p, _i64, _i64, _i64, _p, _p, _p, _p, _p, _sz, _p], _i32),
    "sq_smooth_scale_ex": ([_p, _p, _i64, _i64, _i64, _f32, _i32, _p, _p, _p], _i32),
    "sq_int8_gemm_dequant_ex": ([_p, _p, _p, _i32, _p, _p, _i32, _p, _p, _p, _i64, _i64, _i64, _p, _p, _sz, _p],
                                _i32),
    "sq_norm_smooth_quant": ([_p, _i64, _i64, _i64, _i32, _p, _p, _f32, _p, _p, _p, _p, _p], _i32),
    "sq_act_mean_std_threshold": ([_p, _i64, _i64, _i64, C.c_double, _p, _p, _p, _sz, _p], _i32),
    "llmint8_decomposed_linear_ex": ([_p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _p, _p, _p, _p, _sz, _p], _i32),
    "sq_act_abs_percentile": ([_p, _i64, _i64, _i64, C.c_double, _p, _p, _sz, _p], _i32),
    "sq_quant_act_per_token_asym": ([_p, _i64, _i64, _i64, _p, _p, _p, _p, _p], _i32),
    "sq_weight_row_sums": ([_p, _i64, _i64, _p, _p], _i32),
    "sq_workspace_size": ([_i32, _i64, _i64, _i64], _sz),
    "sq_last_error": ([], C.c_char_p),
    "sq_sync_status": ([_p], _i32),
    "sq_version": ([], C.c_char_p),
    "sq_debug_arm_fault": ([_i32, C.c_uint64], None),
    "sq_debug_gemm_plan": ([_i64, _i64, _i64, _i32, _p], _i32),
    "sq_kernel_launch_count": ([], C.c_uint64),
}
for _name, (_args, _res) in _SIGS.items():
    _fn = getattr(_lib, _name)
    _fn.argtypes = _args
    _fn.restype = _res


class SqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"status {status}: {msg}")
        self.status = status


def lib():
    """The loaded ctypes library (raw C entry points)."""
    return _lib


def sq_last_error() -> str:
    return (_lib.sq_last_error() or b"").decode()


def sq_version() -> str:
    return _lib.sq_version().decode()


def _check(st: int):
    if st != SQ_OK:
        raise SqError(st, sq_last_error())


def _torch():
    import torch
    return torch


def _stream(stream) -> Optional[int]:
    torch = _torch()
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _ptr(t, dtype=None, name="tensor", rowmajor=False):
    if t is None:
        return None
    torch = _torch()
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if rowmajor:
        if t.dim() != 2 or t.stride(1) != 1:
            raise ValueError(f"{name} must be 2-D with unit column stride")
    elif not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _ws(ws):
    if ws is None:
        return None, 0
    return _ptr(ws, None, "ws"), ws.numel() * ws.element_size()


def sq_act_channel_absmax(X, amax, accumulate: bool = False, stream=None):
    torch = _torch()
    M, K = X.shape
    _check(_lib.sq_act_channel_absmax(_ptr(X, torch.bfloat16, "X", True), M, K, X.stride(0),
                                      _ptr(amax, torch.float32, "amax"), int(bool(accumulate)), _stream(stream)))
    return amax


def sq_smooth_scale(act_amax, W, alpha: float, s, inv_s, stream=None):
    torch = _torch()
    N, K = W.shape
    _check(_lib.sq_smooth_scale(_ptr(act_amax, torch.float32, "act_amax"), _ptr(W, torch.bfloat16, "W", True), N, K,
                                W.stride(0), float(alpha), _ptr(s, torch.float32, "s"),
                                _ptr(inv_s, torch.float32, "inv_s"), _stream(stream)))
    return s, inv_s


def sq_smooth_quant_weight(W, s, gran: int, Wq, w_scale, ws=None, stream=None):
    torch = _torch()
    N, K = W.shape
    wsp, wsb = _ws(ws)
    _check(_lib.sq_smooth_quant_weight(_ptr(W, torch.bfloat16, "W", True), N, K, W.stride(0),
                                       _ptr(s, torch.float32, "s"), int(gran), _ptr(Wq, torch.int8, "Wq"),
                                       _ptr(w_scale, torch.float32, "w_scale"), wsp, wsb, _stream(stream)))
    return Wq, w_scale


def sq_smooth_quant_weight_noalloc(W, s, gran: int, Wq, w_scale, stream=None):
    """sq_smooth_quant_weight without a workspace (scratch lives in the library), for
    callers that cannot allocate device memory; calls overlapping on the GPU must not run
    concurrently."""
    torch = _torch()
    N, K = W.shape
    _check(_lib.sq_smooth_quant_weight_noalloc(_ptr(W, torch.bfloat16, "W", True), N, K, W.stride(0),
                                               _ptr(s, torch.float32, "s"), int(gran), _ptr(Wq, torch.int8, "Wq"),
                                               _ptr(w_scale, torch.float32, "w_scale"), _stream(stream)))
    return Wq, w_scale


def sq_quant_act_per_token(X, inv_s, Xq, x_scale, stream=None):
    torch = _torch()
    M, K = X.shape
    _check(_lib.sq_quant_act_per_token(_ptr(X, torch.bfloat16, "X", True), M, K, X.stride(0),
                                       _ptr(inv_s, torch.float32, "inv_s"), _ptr(Xq, torch.int8, "Xq"),
                                       _ptr(x_scale, torch.float32, "x_scale"), _stream(stream)))
    return Xq, x_scale


def sq_int8_gemm_dequant(Xq, Wq, x_scale, w_scale, w_gran: int, bias, Y, acc_out=None, ws=None, stream=None):
    torch = _torch()
    M, K = Xq.shape
    N = Wq.shape[0]
    wsp, wsb = _ws(ws)
    _check(_lib.sq_int8_gemm_dequant(_ptr(Xq, torch.int8, "Xq"), _ptr(Wq, torch.int8, "Wq"),
                                     _ptr(x_scale, torch.float32, "x_scale"), _ptr(w_scale, torch.float32, "w_scale"),
                                     int(w_gran), _ptr(bias, torch.bfloat16, "bias"), _ptr(Y, torch.bfloat16, "Y"),
                                     M, N, K, _ptr(acc_out, torch.int32, "acc_out"), wsp, wsb, _stream(stream)))
    return Y


def llmint8_decomposed_linear(X, W, Wq, w_scale, threshold: float, bias, Y, mask_out=None, n_outliers_out=None,
                              acc_out=None, ws=None, stream=None):
    """mask_out is passed as a torch.int32 tensor of ceil(K/32) words (same bits as uint32)."""
    torch = _torch()
    M, K = X.shape
    N = W.shape[0]
    wsp, wsb = _ws(ws)
    _check(_lib.llmint8_decomposed_linear(
        _ptr(X, torch.bfloat16, "X"), _ptr(W, torch.bfloat16, "W"), _ptr(Wq, torch.int8, "Wq"),
        _ptr(w_scale, torch.float32, "w_scale"), float(threshold), _ptr(bias, torch.bfloat16, "bias"),
        _ptr(Y, torch.bfloat16, "Y"), M, N, K, _ptr(mask_out, torch.int32, "mask_out"),
        _ptr(n_outliers_out, torch.int32, "n_outliers_out"), _ptr(acc_out, torch.int32, "acc_out"), wsp, wsb,
        _stream(stream)))
    return Y


# ---------------------------------------------------------------- variants
def sq_quant_act_per_tensor(X, inv_s, Xq, x_scale, clip=None, ws=None, stream=None):
    """Per-tensor activation scale: dynamic (clip None, needs ws) or the calibrated *clip."""
    torch = _torch()
    M, K = X.shape
    wsp, wsb = _ws(ws)
    _check(_lib.sq_quant_act_per_tensor(_ptr(X, torch.bfloat16, "X", True), M, K, X.stride(0),
                                        _ptr(inv_s, torch.float32, "inv_s"), _ptr(clip, torch.float32, "clip"),
                                        _ptr(Xq, torch.int8, "Xq"), _ptr(x_scale, torch.float32, "x_scale"), wsp, wsb,
                                        _stream(stream)))
    return Xq, x_scale


def sq_smooth_scale_ex(act_amax, W, alpha: float, normalize: bool, s, inv_s, stream=None):
    torch = _torch()
    N, K = W.shape
    _check(_lib.sq_smooth_scale_ex(_ptr(act_amax, torch.float32, "act_amax"), _ptr(W, torch.bfloat16, "W", True), N,
                                   K, W.stride(0), float(alpha), int(bool(normalize)), _ptr(s, torch.float32, "s"),
                                   _ptr(inv_s, torch.float32, "inv_s"), _stream(stream)))
    return s, inv_s


def sq_int8_gemm_dequant_ex(Xq, Wq, x_scale, x_gran: int, x_zero, w_scale, w_gran: int, w_rowsum, bias, Y,
                            acc_out=None, ws=None, stream=None):
    torch = _torch()
    M, K = Xq.shape
    N = Wq.shape[0]
    wsp, wsb = _ws(ws)
    _check(_lib.sq_int8_gemm_dequant_ex(
        _ptr(Xq, torch.int8, "Xq"), _ptr(Wq, torch.int8, "Wq"), _ptr(x_scale, torch.float32, "x_scale"), int(x_gran),
        _ptr(x_zero, torch.int32, "x_zero"), _ptr(w_scale, torch.float32, "w_scale"), int(w_gran),
        _ptr(w_rowsum, torch.int32, "w_rowsum"), _ptr(bias, torch.bfloat16, "bias"), _ptr(Y, torch.bfloat16, "Y"),
        M, N, K, _ptr(acc_out, torch.int32, "acc_out"), wsp, wsb, _stream(stream)))
    return Y


def sq_norm_smooth_quant(X, norm: int, gamma, beta, eps: float, inv_s, Xq, x_scale, mean_rstd=None, stream=None):
    torch = _torch()
    M, K = X.shape
    _check(_lib.sq_norm_smooth_quant(_ptr(X, torch.bfloat16, "X", True), M, K, X.stride(0), int(norm),
                                     _ptr(gamma, torch.bfloat16, "gamma"), _ptr(beta, torch.bfloat16, "beta"),
                                     float(eps), _ptr(inv_s, torch.float32, "inv_s"), _ptr(Xq, torch.int8, "Xq"),
                                     _ptr(x_scale, torch.float32, "x_scale"),
                                     _ptr(mean_rstd, torch.float32, "mean_rstd"), _stream(stream)))
    return Xq, x_scale


def sq_act_mean_std_threshold(X, k: float, threshold, mean_std=None, ws=None, stream=None):
    torch = _torch()
    M, K = X.shape
    wsp, wsb = _ws(ws)
    _check(_lib.sq_act_mean_std_threshold(_ptr(X, torch.bfloat16, "X", True), M, K, X.stride(0), float(k),
                                          _ptr(threshold, torch.float32, "threshold"),
                                          _ptr(mean_std, torch.float64, "mean_std"), wsp, wsb, _stream(stream)))
    return threshold


def llmint8_decomposed_linear_ex(X, W, Wq, w_scale, threshold, bias, Y, mask_out=None, n_outliers_out=None,
                                 acc_out=None, ws=None, stream=None):
    """llmint8_decomposed_linear with the threshold in a device fp32 [1] tensor."""
    torch = _torch()
    M, K = X.shape
    N = W.shape[0]
    wsp, wsb = _ws(ws)
    _check(_lib.llmint8_decomposed_linear_ex(
        _ptr(X, torch.bfloat16, "X"), _ptr(W, torch.bfloat16, "W"), _ptr(Wq, torch.int8, "Wq"),
        _ptr(w_scale, torch.float32, "w_scale"), _ptr(threshold, torch.float32, "threshold"),
        _ptr(bias, torch.bfloat16, "bias"), _ptr(Y, torch.bfloat16, "Y"), M, N, K,
        _ptr(mask_out, torch.int32, "mask_out"), _ptr(n_outliers_out, torch.int32, "n_outliers_out"),
        _ptr(acc_out, torch.int32, "acc_out"), wsp, wsb, _stream(stream)))
    return Y


def sq_act_abs_percentile(X, p: float, out, ws=None, stream=None):
    torch = _torch()
    M, K = X.shape
    wsp, wsb = _ws(ws)
    _check(_lib.sq_act_abs_percentile(_ptr(X, torch.bfloat16, "X", True), M, K, X.stride(0), float(p),
                                      _ptr(out, torch.float32, "out"), wsp, wsb, _stream(stream)))
    return out


def sq_quant_act_per_token_asym(X, inv_s, Xq, x_scale, x_zero, stream=None):
    torch = _torch()
    M, K = X.shape
    _check(_lib.sq_quant_act_per_token_asym(_ptr(X, torch.bfloat16, "X", True), M, K, X.stride(0),
                                            _ptr(inv_s, torch.float32, "inv_s"), _ptr(Xq, torch.int8, "Xq"),
                                            _ptr(x_scale, torch.float32, "x_scale"),
                                            _ptr(x_zero, torch.int32, "x_zero"), _stream(stream)))
    return Xq, x_scale, x_zero


def sq_weight_row_sums(Wq, rowsum, stream=None):
    torch = _torch()
    N, K = Wq.shape
    _check(_lib.sq_weight_row_sums(_ptr(Wq, torch.int8, "Wq"), N, K, _ptr(rowsum, torch.int32, "rowsum"),
                                   _stream(stream)))
    return rowsum


def sq_workspace_size(op: int, M: int, N: int, K: int) -> int:
    return int(_lib.sq_workspace_size(int(op), int(M), int(N), int(K)))


def sq_sync_status(stream=None):
    _check(_lib.sq_sync_status(_stream(stream)))


def sq_kernel_launch_count() -> int:
    return int(_lib.sq_kernel_launch_count())


def sq_debug_arm_fault(fault: int, wait_limit_ns: int = 0):
    _lib.sq_debug_arm_fault(int(fault), int(wait_limit_ns))


GEMM_PLAN_FIELDS = ("path", "swap", "bn", "whole_tiles", "split_tiles", "splits", "kb_per_split")
GEMM_PATH_CUDA_CORES, GEMM_PATH_TENSOR, GEMM_PATH_TENSOR_PAIRS = 0, 1, 2


def sq_debug_gemm_plan(M: int, N: int, K: int, outliers: bool = False) -> dict:
    """The launch plan of the GEMM for an M x N x K product (host only, no device)."""
    out = (C.c_int64 * 7)()
    _check(_lib.sq_debug_gemm_plan(int(M), int(N), int(K), 1 if outliers else 0, C.cast(out, C.c_void_p)))
    return dict(zip(GEMM_PLAN_FIELDS, (int(v) for v in out)))


def workspace(op: int, M: int, N: int, K: int, device="cuda"):
    """A uint8 torch tensor of sq_workspace_size(op, M, N, K) bytes (None if 0), zero-filled."""
    torch = _torch()
    n = sq_workspace_size(op, M, N, K)
    return torch.zeros(n, dtype=torch.uint8, device=device) if n else None
