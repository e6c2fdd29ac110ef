"""CPU oracle for the W8A8 quantized linear layer (ctypes front end of ``sq_oracle.c``).

TEST INFRASTRUCTURE: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package. The product path never
does, and this package imports nothing from it.

Arrays are numpy: bf16 tensors are uint16 bit patterns, row-major with K
contiguous. Each wrapper calls one C function of ``sq_oracle.c``; the two
compositions at the end only chain those calls in the order the pages give.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math"]

PER_TENSOR = 0
PER_CHANNEL = 1
NORM_LAYER = 0
NORM_RMS = 1


def build(force: bool = False) -> str:
    """Compile ``sq_oracle.c`` with gcc into ``liboracle.so`` (if missing or stale)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(build())
        p, i64, i32, f32 = C.c_void_p, C.c_int64, C.c_int, C.c_float
        sig = {
            "oracle_act_channel_absmax": ([p, i64, i64, i64, p, i32], None),
            "oracle_smooth_scale": ([p, p, i64, i64, i64, f32, p, p], None),
            "oracle_smooth_quant_weight": ([p, i64, i64, i64, p, i32, p, p], None),
            "oracle_quant_act_per_token": ([p, i64, i64, i64, p, p, p, p], None),
            "oracle_int8_gemm": ([p, p, i64, i64, i64, p], i64),
            "oracle_dequant": ([p, i64, i64, p, p, i32, p, p, p, p], None),
            "oracle_outlier_columns": ([p, i64, f32, p, p, p], C.c_int32),
            "oracle_outlier_product": ([p, i64, p, i64, i64, i64, p, C.c_int32, p], None),
            "oracle_quant_act_per_tensor": ([p, i64, i64, i64, p, f32, p, p], None),
            "oracle_smooth_scale_normalize": ([p, p, i64], None),
            "oracle_norm_smooth_quant": ([p, i64, i64, i64, i32, p, p, f32, p, p, p, p, p, i32], None),
            "oracle_mean_std_threshold": ([p, i64, i64, i64, C.c_double, p, p], f32),
            "oracle_abs_percentile": ([p, i64, i64, i64, C.c_double], f32),
            "oracle_quant_act_per_token_asym": ([p, i64, i64, i64, p, p, p, p], None),
            "oracle_weight_row_sums": ([p, i64, i64, p], None),
            "oracle_dequant_ex": ([p, i64, i64, p, i32, p, i32, p, p, p, p, p], None),
            "oracle_bf16_to_float": ([p, i64, p], None),
            "oracle_float_to_bf16": ([p, i64, p], None),
            "oracle_num_threads": ([], i32),
        }
        for name, (args, res) in sig.items():
            fn = getattr(_lib, name)
            fn.argtypes = args
            fn.restype = res
    return _lib


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def bf16_to_float(b) -> np.ndarray:
    b = _c(b, np.uint16)
    out = np.empty(b.shape, np.float32)
    lib().oracle_bf16_to_float(_ptr(b), b.size, _ptr(out))
    return out


def float_to_bf16(f) -> np.ndarray:
    f = _c(f, np.float32)
    out = np.empty(f.shape, np.uint16)
    lib().oracle_float_to_bf16(_ptr(f), f.size, _ptr(out))
    return out


def act_channel_absmax(X, prev: Optional[np.ndarray] = None) -> np.ndarray:
    """Column absmax of X [M,K]; with ``prev`` the running maximum max(prev, .)."""
    X = _c(X, np.uint16)
    M, K = X.shape
    amax = np.zeros(K, np.float32) if prev is None else np.array(prev, np.float32, copy=True)
    lib().oracle_act_channel_absmax(_ptr(X), M, K, K, _ptr(amax), 0 if prev is None else 1)
    return amax


def smooth_scale(act_amax, W, alpha: float, normalize: bool = False):
    """Returns (s, inv_s), fp32 [K]; ``normalize`` applies s/max(s)*127 clamped at 1e-5."""
    a = _c(act_amax, np.float32)
    W = _c(W, np.uint16)
    N, K = W.shape
    s = np.empty(K, np.float32)
    inv_s = np.empty(K, np.float32)
    lib().oracle_smooth_scale(_ptr(a), _ptr(W), N, K, K, float(alpha), _ptr(s), _ptr(inv_s))
    if normalize:
        lib().oracle_smooth_scale_normalize(_ptr(s), _ptr(inv_s), K)
    return s, inv_s


def smooth_quant_weight(W, s: Optional[np.ndarray], gran: int):
    """Returns (Wq int8 [N,K], e fp32 [N] or [1])."""
    W = _c(W, np.uint16)
    s = _c(s, np.float32)
    N, K = W.shape
    Wq = np.empty((N, K), np.int8)
    e = np.empty(N if gran == PER_CHANNEL else 1, np.float32)
    lib().oracle_smooth_quant_weight(_ptr(W), N, K, K, _ptr(s), int(gran), _ptr(Wq), _ptr(e))
    return Wq, e


def quant_act_per_token(X, inv_s: Optional[np.ndarray] = None, skip_mask: Optional[np.ndarray] = None):
    """Returns (Xq int8 [M,K], d fp32 [M])."""
    X = _c(X, np.uint16)
    inv_s = _c(inv_s, np.float32)
    skip_mask = _c(skip_mask, np.uint32)
    M, K = X.shape
    Xq = np.empty((M, K), np.int8)
    d = np.empty(M, np.float32)
    lib().oracle_quant_act_per_token(_ptr(X), M, K, K, _ptr(inv_s), _ptr(skip_mask), _ptr(Xq), _ptr(d))
    return Xq, d


def int8_gemm(Xq, Wq) -> np.ndarray:
    """acc[m,n] = sum_k Xq[m,k]*Wq[n,k] as int32 (raises if a sum leaves int32)."""
    Xq = _c(Xq, np.int8)
    Wq = _c(Wq, np.int8)
    M, K = Xq.shape
    N = Wq.shape[0]
    acc = np.empty((M, N), np.int32)
    over = lib().oracle_int8_gemm(_ptr(Xq), _ptr(Wq), M, N, K, _ptr(acc))
    if over:
        raise OverflowError(f"{over} int32 overflows in oracle_int8_gemm")
    return acc


def dequant(acc, d, e, bias=None, o=None):
    """Returns (y_ref fp64 [M,N], y_bf16 uint16 [M,N]); e of size 1 means per-tensor."""
    acc = _c(acc, np.int32)
    d = _c(d, np.float32)
    e = _c(e, np.float32)
    bias = _c(bias, np.uint16)
    o = _c(o, np.float64)
    M, N = acc.shape
    y_ref = np.empty((M, N), np.float64)
    y_bf = np.empty((M, N), np.uint16)
    if e.size not in (1, N):
        raise ValueError("e must have 1 or N entries")
    lib().oracle_dequant(_ptr(acc), M, N, _ptr(d), _ptr(e), 1 if e.size == N else 0,
                         _ptr(bias), _ptr(o), _ptr(y_ref), _ptr(y_bf))
    return y_ref, y_bf


def outlier_columns(amax, threshold: float):
    """Returns (mask uint32 [ceil(K/32)], idx int32 [count], count)."""
    a = _c(amax, np.float32)
    K = a.size
    mask = np.zeros((K + 31) // 32, np.uint32)
    idx = np.zeros(max(K, 1), np.int32)
    cnt = C.c_int32(0)
    lib().oracle_outlier_columns(_ptr(a), K, float(threshold), _ptr(mask), _ptr(idx), C.addressof(cnt))
    return mask, idx[: cnt.value].copy(), int(cnt.value)


def outlier_product(X, W, idx) -> np.ndarray:
    """o[m,n] = sum_{j in idx} X[m,j]*W[n,j] in fp64."""
    X = _c(X, np.uint16)
    W = _c(W, np.uint16)
    idx = _c(idx, np.int32)
    M, K = X.shape
    N = W.shape[0]
    o = np.empty((M, N), np.float64)
    lib().oracle_outlier_product(_ptr(X), K, _ptr(W), K, M, N, _ptr(idx), int(idx.size), _ptr(o))
    return o


# ------------------------------------------------------------------ variants
def quant_act_per_tensor(X, inv_s: Optional[np.ndarray] = None, clip: Optional[float] = None):
    """Per-tensor activation quantization: returns (Xq int8 [M,K], d fp32 [1]). ``clip``: a
    static calibration value (e.g. a percentile of |X|) used instead of the tensor's absmax."""
    X = _c(X, np.uint16)
    inv_s = _c(inv_s, np.float32)
    M, K = X.shape
    Xq = np.empty((M, K), np.int8)
    d = np.empty(1, np.float32)
    lib().oracle_quant_act_per_tensor(_ptr(X), M, K, K, _ptr(inv_s), -1.0 if clip is None else float(clip),
                                      _ptr(Xq), _ptr(d))
    return Xq, d


def norm_smooth_quant(X, norm: int, gamma, beta=None, eps: float = 1e-5, inv_s: Optional[np.ndarray] = None,
                      stats: Optional[np.ndarray] = None, with_stats: bool = False):
    """LayerNorm (NORM_LAYER) or RMSNorm (NORM_RMS) with bf16 gamma/beta, smoothing and
    per-token quantization in one pass: returns (Xq int8 [M,K], d fp32 [M], y fp32 [M,K]),
    plus the row statistics fp32 [M,2] (mean or 0, rstd) with ``with_stats``. ``stats``
    supplies the statistics instead of computing them."""
    X = _c(X, np.uint16)
    gamma = _c(gamma, np.uint16)
    beta = _c(beta, np.uint16)
    inv_s = _c(inv_s, np.float32)
    M, K = X.shape
    Xq = np.empty((M, K), np.int8)
    d = np.empty(M, np.float32)
    y = np.empty((M, K), np.float32)
    given = stats is not None
    st = np.array(stats, np.float32, copy=True).reshape(M, 2) if given else np.empty((M, 2), np.float32)
    lib().oracle_norm_smooth_quant(_ptr(X), M, K, K, int(norm), _ptr(gamma), _ptr(beta), float(eps), _ptr(inv_s),
                                   _ptr(Xq), _ptr(d), _ptr(y), _ptr(st), 1 if given else 0)
    return (Xq, d, y, st) if with_stats else (Xq, d, y)


def smooth_scale_normalize(s):
    """The normalisation step alone on given factors: returns (s', inv_s') fp32 [K]."""
    s2 = np.array(s, np.float32, copy=True)
    inv = np.empty_like(s2)
    lib().oracle_smooth_scale_normalize(_ptr(s2), _ptr(inv), s2.size)
    return s2, inv


def mean_std_threshold(X, k: float):
    """Returns (threshold fp32 = fp32(mean + k*std), mean fp64, std fp64) over all of X."""
    X = _c(X, np.uint16)
    M, K = X.shape
    mean, sd = C.c_double(0.0), C.c_double(0.0)
    t = lib().oracle_mean_std_threshold(_ptr(X), M, K, K, float(k), C.addressof(mean), C.addressof(sd))
    return np.float32(t), mean.value, sd.value


def abs_percentile(X, p: float) -> np.float32:
    """Nearest-rank p-th percentile of |X| over all elements."""
    X = _c(X, np.uint16)
    M, K = X.shape
    return np.float32(lib().oracle_abs_percentile(_ptr(X), M, K, K, float(p)))


def quant_act_per_token_asym(X, inv_s: Optional[np.ndarray] = None):
    """Asymmetric per-token quantization: returns (Xq int8 [M,K], d fp32 [M], z int32 [M])."""
    X = _c(X, np.uint16)
    inv_s = _c(inv_s, np.float32)
    M, K = X.shape
    Xq = np.empty((M, K), np.int8)
    d = np.empty(M, np.float32)
    z = np.empty(M, np.int32)
    lib().oracle_quant_act_per_token_asym(_ptr(X), M, K, K, _ptr(inv_s), _ptr(Xq), _ptr(d), _ptr(z))
    return Xq, d, z


def weight_row_sums(Wq) -> np.ndarray:
    """rs[n] = sum_k Wq[n,k] (int32)."""
    Wq = _c(Wq, np.int8)
    N, K = Wq.shape
    rs = np.empty(N, np.int32)
    lib().oracle_weight_row_sums(_ptr(Wq), N, K, _ptr(rs))
    return rs


def dequant_ex(acc, d, e, bias=None, x_zero=None, rs=None):
    """Dequantization with d per token ([M]) or per tensor ([1]), e per channel or per tensor,
    and the exact zero-point correction acc - z_m*rs_n when ``x_zero`` is given.
    Returns (y_ref fp64 [M,N], y_bf16 uint16 [M,N])."""
    acc = _c(acc, np.int32)
    d = _c(d, np.float32)
    e = _c(e, np.float32)
    bias = _c(bias, np.uint16)
    x_zero = _c(x_zero, np.int32)
    rs = _c(rs, np.int32)
    M, N = acc.shape
    if (x_zero is None) != (rs is None):
        raise ValueError("x_zero and rs go together")
    y_ref = np.empty((M, N), np.float64)
    y_bf = np.empty((M, N), np.uint16)
    if d.size not in (1, M) or e.size not in (1, N):
        raise ValueError("d must have 1 or M entries and e 1 or N")
    lib().oracle_dequant_ex(_ptr(acc), M, N, _ptr(d), 1 if d.size == M else 0,
                            _ptr(e), 1 if e.size == N else 0, _ptr(x_zero), _ptr(rs), _ptr(bias), _ptr(y_ref),
                            _ptr(y_bf))
    return y_ref, y_bf


def smoothquant_linear(X, W, bias=None, alpha: float = 0.5, gran: int = PER_CHANNEL, calib=None,
                       s=None, inv_s=None):
    """SmoothQuant W8A8 linear ("SmoothQuant量化实战" §3.2-§3.4): calibrate the activation
    channel absmax (on ``calib`` or on X), smoothing factors, smoothed weight and activation
    quantization, INT8 GEMM, dequantization. ``s``/``inv_s`` override the computed factors
    (so that later stages can be checked on the factors another implementation produced)."""
    out = {}
    if s is None:
        amax = act_channel_absmax(X if calib is None else calib)
        s, inv_s = smooth_scale(amax, W, alpha)
        out["amax"] = amax
    out["s"], out["inv_s"] = s, inv_s
    Wq, e = smooth_quant_weight(W, s, gran)
    Xq, d = quant_act_per_token(X, inv_s)
    acc = int8_gemm(Xq, Wq)
    y_ref, y_bf = dequant(acc, d, e, bias)
    out.update(Wq=Wq, e=e, Xq=Xq, d=d, acc=acc, y_ref=y_ref, y_bf16=y_bf)
    return out


def llmint8_linear(X, W, bias=None, threshold: float = 6.0, amax=None):
    """LLM.int8() decomposed linear ("LLM.int8()技术解析" §2.1, §2.2, §3.1): column absmax,
    outlier columns over the threshold, per-token int8 of the other columns with a
    per-channel int8 weight (no smoothing), INT8 GEMM, fp64 product of the outlier columns,
    summed before the single output rounding."""
    if amax is None:
        amax = act_channel_absmax(X)
    mask, idx, count = outlier_columns(amax, threshold)
    Wq, e = smooth_quant_weight(W, None, PER_CHANNEL)
    Xq, d = quant_act_per_token(X, None, mask)
    acc = int8_gemm(Xq, Wq)
    o = outlier_product(X, W, idx)
    y_ref, y_bf = dequant(acc, d, e, bias, o)
    return dict(amax=amax, mask=mask, idx=idx, count=count, Wq=Wq, e=e, Xq=Xq, d=d, acc=acc, o=o,
                y_ref=y_ref, y_bf16=y_bf)
