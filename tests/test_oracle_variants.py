"""Pins of the oracle's variant functions (per-tensor activation scale, smoothing-factor
normalisation, fused LayerNorm/RMSNorm -> smooth -> quantize, mu + k*sigma outlier
threshold, percentile calibration, asymmetric activations with the zero-point correction)
to facts fixed by the pages and by the mathematics: hand-worked examples, closed forms,
exact invariances, library special cases and brute force. The last test plants mistakes.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from w8a8_quantized_gemm_b200 import workloads as wl

U32 = 2.0 ** -24


def _bits(x):
    return wl.f32_to_bf16_bits(np.asarray(x, np.float32))


def _f32(bits):
    return wl.bf16_bits_to_f32(bits)


# --------------------------------------------------------------------------- per-tensor scale
def test_per_tensor_act_outlier_example(golden_dir):
    """SmoothQuant量化实战 §1.2: per-tensor activations with one channel at +-50 get scale
    50/127 ~ 0.39 and squeeze the [-1, 1] values into a handful of codes."""
    with open(os.path.join(golden_dir, "sq_per_tensor_outlier_example.json")) as f:
        g = json.load(f)
    rows, cols = g["shape"]
    x = np.random.default_rng(2).uniform(-1.0, 1.0, size=(rows, cols)).astype(np.float32)
    ch = g["outlier_channel"]
    x[:, ch] = np.linspace(-50.0, 50.0, rows).astype(np.float32)
    q, d = oracle.quant_act_per_tensor(_bits(x))
    assert d.shape == (1,)
    assert abs(float(d[0]) - g["printed_scale"]) <= g["printed_scale_tolerance"]
    small = np.ones_like(q, dtype=bool)
    small[:, ch] = False
    lo, hi = g["small_value_code_range"]
    assert q[small].min() >= lo and q[small].max() <= hi


def test_per_tensor_act_hand_example():
    """a = 4: r = 31.75; 1 -> 31.75 -> 32, -2 -> -63.5 -> -64 (tie to even), 0.5 -> 15.875 -> 16."""
    q, d = oracle.quant_act_per_tensor(_bits([[1.0, -2.0], [0.5, 4.0]]))
    assert d[0] == np.float32(4.0) / np.float32(127.0)
    assert q.tolist() == [[32, -64], [16, 127]]


def test_per_tensor_static_clip_saturates():
    """A calibrated clip below the tensor's absmax: codes saturate at the clamp bounds."""
    q, d = oracle.quant_act_per_tensor(_bits([[3.0, -3.0, 0.5, -1.0]]), clip=1.0)
    assert d[0] == np.float32(1.0) / np.float32(127.0)
    assert q.tolist() == [[127, -128, 64, -127]]


@pytest.mark.parametrize("seed", [0, 1])
def test_per_tensor_error_bound(seed):
    rng = np.random.default_rng(seed)
    x = _bits(rng.standard_t(3, size=(37, 200)).astype(np.float32))
    inv_s = rng.uniform(0.2, 3.0, 200).astype(np.float32)
    q, d = oracle.quant_act_per_tensor(x, inv_s)
    v = _f32(x).astype(np.float64) * inv_s.astype(np.float32).astype(np.float64)
    err = np.abs(v - q.astype(np.float64) * float(d[0]))
    assert err.max() <= float(d[0]) / 2 + 4 * U32 * np.abs(v).max()
    assert np.abs(q).max() == 127 and q.min() >= -127


# --------------------------------------------------------------------------- normalisation
def test_smooth_scale_normalisation():
    """SmoothQuant量化实战 §3.3: s / max(s) * 127, clamped below at 1e-5."""
    rng = np.random.default_rng(4)
    K = 96
    amax = rng.uniform(0.1, 30.0, K).astype(np.float32)
    amax[5] = 0.0  # clamped at 1e-8 before the power: with alpha 0.9 its factor falls below 1e-5
    W = _bits(rng.normal(0, 0.02, (64, K)).astype(np.float32))
    s0, _ = oracle.smooth_scale(amax, W, 0.9)
    s, inv_s = oracle.smooth_scale(amax, W, 0.9, normalize=True)
    j = int(np.argmax(s0))
    assert s[j] == np.float32(127.0)  # max/max is exactly 1
    assert s.max() == np.float32(127.0) and s.min() >= np.float32(1e-5)
    assert s[5] == np.float32(1e-5)
    keep = np.arange(K) != 5
    ratio = s[keep].astype(np.float64) / 127.0
    ref = s0[keep].astype(np.float64) / float(s0.max())
    assert np.all(np.abs(ratio - ref) <= 3 * U32 * ref)
    assert np.all(inv_s * s > 0.99999) and np.all(inv_s * s < 1.00001)


def test_normalised_factors_keep_the_identity():
    """X W^T = (X diag(1/s)) (W diag(s))^T holds for any positive s, the normalised one too."""
    p = wl.random_problem(24, 40, 128, seed=6, outliers=3)
    amax = oracle.act_channel_absmax(p.X)
    s, inv_s = oracle.smooth_scale(amax, p.W, 0.5, normalize=True)
    X = _f32(p.X).astype(np.float64)
    W = _f32(p.W).astype(np.float64)
    lhs = X @ W.T
    rhs = (X * inv_s.astype(np.float64)) @ (W * s.astype(np.float64)).T
    assert np.abs(lhs - rhs).max() <= 1e-5 * np.abs(X).max() * np.abs(W).max() * p.K


# --------------------------------------------------------------------------- fused norm
def _ln_ref(x, g, b, eps):
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * g + (0 if b is None else b)


@pytest.mark.parametrize("norm", [oracle.NORM_LAYER, oracle.NORM_RMS])
def test_norm_matches_fp64_library_definition(norm):
    rng = np.random.default_rng(7)
    M, K = 9, 320
    x = _bits(rng.normal(0.3, 2.0, (M, K)).astype(np.float32))
    g = _bits(rng.uniform(0.5, 1.5, K).astype(np.float32))
    b = _bits(rng.normal(0, 0.1, K).astype(np.float32))
    _, _, y = oracle.norm_smooth_quant(x, norm, g, b, 1e-5)
    X, G, B = _f32(x).astype(np.float64), _f32(g).astype(np.float64), _f32(b).astype(np.float64)
    if norm == oracle.NORM_LAYER:
        ref = _ln_ref(X, G, B, 1e-5)
    else:
        ref = X / np.sqrt((X ** 2).mean(axis=1, keepdims=True) + 1e-5) * G + B
    assert np.abs(y - ref).max() <= 16 * U32 * np.abs(ref).max()


def test_layernorm_constant_row_gives_beta():
    x = _bits(np.full((2, 64), 3.25, np.float32))
    g = _bits(np.full(64, 1.5, np.float32))
    b = _bits(np.linspace(-1, 1, 64).astype(np.float32))
    _, _, y = oracle.norm_smooth_quant(x, oracle.NORM_LAYER, g, b, 1e-5)
    assert np.array_equal(y, np.broadcast_to(_f32(b), y.shape))


@pytest.mark.parametrize("norm", [oracle.NORM_LAYER, oracle.NORM_RMS])
def test_norm_power_of_two_scale_invariance(norm):
    """With eps = 0 the statistics scale exactly by powers of two, so norm(2x) == norm(x)."""
    rng = np.random.default_rng(8)
    x = _bits(rng.normal(0, 1, (5, 256)).astype(np.float32))
    x2 = _bits(2.0 * _f32(x))
    g = _bits(rng.uniform(0.5, 2, 256).astype(np.float32))
    q1, d1, y1 = oracle.norm_smooth_quant(x, norm, g, None, 0.0)
    q2, d2, y2 = oracle.norm_smooth_quant(x2, norm, g, None, 0.0)
    assert np.array_equal(y1, y2) and np.array_equal(q1, q2) and np.array_equal(d1, d2)


def test_rmsnorm_unit_gamma_has_unit_rms():
    rng = np.random.default_rng(9)
    x = _bits(rng.normal(0, 3, (6, 512)).astype(np.float32))
    g = _bits(np.ones(512, np.float32))
    _, _, y = oracle.norm_smooth_quant(x, oracle.NORM_RMS, g, None, 0.0)
    rms = np.sqrt((y.astype(np.float64) ** 2).mean(axis=1))
    assert np.all(np.abs(rms - 1.0) <= 1e-6)


def test_norm_quant_bound_and_smoothing():
    rng = np.random.default_rng(10)
    M, K = 7, 192
    x = _bits(rng.normal(0, 1, (M, K)).astype(np.float32))
    g = _bits(rng.uniform(0.5, 1.5, K).astype(np.float32))
    inv_s = rng.uniform(0.1, 4.0, K).astype(np.float32)
    q, d, y = oracle.norm_smooth_quant(x, oracle.NORM_LAYER, g, None, 1e-5, inv_s)
    v = y.astype(np.float64) * inv_s.astype(np.float64)
    err = np.abs(v - q * d[:, None].astype(np.float64))
    assert np.all(err <= d[:, None] / 2 + 4 * U32 * np.abs(v).max(axis=1, keepdims=True))
    assert np.all(np.abs(q).max(axis=1) == 127)


# --------------------------------------------------------------------------- mu + k sigma
def test_mean_std_threshold_closed_form():
    thr, mean, sd = oracle.mean_std_threshold(_bits([[1.0, 2.0], [3.0, 4.0]]), 3.0)
    assert mean == 2.5 and abs(sd - math.sqrt(5.0 / 3.0)) <= 1e-15
    assert thr == np.float32(2.5 + 3.0 * math.sqrt(5.0 / 3.0))


def test_mean_std_threshold_matches_numpy():
    rng = np.random.default_rng(11)
    x = _bits(rng.normal(0.2, 1.5, (33, 130)).astype(np.float32))
    thr, mean, sd = oracle.mean_std_threshold(x, 6.0)
    X = _f32(x).astype(np.float64)
    assert abs(mean - X.mean()) <= 1e-12 and abs(sd - X.std(ddof=1)) <= 1e-12
    assert thr == np.float32(X.mean() + 6.0 * X.std(ddof=1))


def test_three_sigma_example_flags_the_offset_channels():
    """从自动驾驶芯片到大语言模型INT8量化训练实战解析 §2.1: randn*0.1 activations of shape
    (2, 128, 4096) with the first 10 channels offset by +50; mean + 3 std flags exactly
    those channels (their column absmax is ~50, every other one below 1)."""
    rng = np.random.default_rng(0)
    x = (rng.standard_normal((256, 4096), dtype=np.float32) * np.float32(0.1))
    x[:, :10] += np.float32(50.0)
    bits = _bits(x)
    thr, mean, sd = oracle.mean_std_threshold(bits, 3.0)
    assert 5.0 < thr < 10.0
    _, idx, cnt = oracle.outlier_columns(oracle.act_channel_absmax(bits), thr)
    assert cnt == 10 and idx.tolist() == list(range(10))
    flat = np.abs(_f32(bits))
    assert (flat > thr).mean() == pytest.approx(10 / 4096)


# --------------------------------------------------------------------------- percentile
def test_percentile_closed_forms():
    vals = np.arange(1, 257, dtype=np.float32)  # exact in bf16
    x = _bits(np.random.default_rng(1).permutation(vals).reshape(16, 16) * np.where(
        np.arange(256).reshape(16, 16) % 3 == 0, -1, 1).astype(np.float32))
    assert oracle.abs_percentile(x, 100.0) == 256.0
    assert oracle.abs_percentile(x, 99.99) == 256.0  # ceil(0.9999 * 256) = 256
    assert oracle.abs_percentile(x, 50.0) == 128.0
    assert oracle.abs_percentile(x, 0.1) == 1.0  # rank ceil(0.256) = 1
    assert oracle.abs_percentile(x, 0.0) == 1.0  # rank at least 1


@pytest.mark.parametrize("p", [99.99, 99.9, 90.0, 37.5])
def test_percentile_brute_force(p):
    rng = np.random.default_rng(int(p * 100))
    x = _bits(rng.standard_t(3, size=(41, 77)).astype(np.float32))
    v = np.sort(np.abs(_f32(x)).ravel())
    rank = max(1, math.ceil(p / 100.0 * v.size))
    assert oracle.abs_percentile(x, p) == v[rank - 1]


# --------------------------------------------------------------------------- asymmetric
def test_asym_hand_example(golden_dir):
    with open(os.path.join(golden_dir, "asym_hand_quant.json")) as f:
        g = json.load(f)
    q, d, z = oracle.quant_act_per_token_asym(_bits(g["rows"]))
    assert z.tolist() == g["zero_point"]
    assert q.tolist() == g["codes"]
    assert np.array_equal(d, np.array(g["range"], np.float32) / np.float32(255.0))


def test_asym_bound_and_exact_zero():
    rng = np.random.default_rng(12)
    x = rng.normal(0.8, 1.0, (19, 150)).astype(np.float32)
    x[:, ::7] = 0.0
    bits = _bits(x)
    inv_s = rng.uniform(0.3, 2.0, 150).astype(np.float32)
    q, d, z = oracle.quant_act_per_token_asym(bits, inv_s)
    v = _f32(bits).astype(np.float64) * inv_s.astype(np.float64)
    deq = d[:, None].astype(np.float64) * (q.astype(np.int64) - z[:, None]).astype(np.float64)
    assert np.all(np.abs(v - deq) <= d[:, None] / 2 + 4 * U32 * np.abs(v).max(axis=1, keepdims=True))
    assert np.all(q[:, ::7] == z[:, None])  # zero is represented exactly
    assert np.all(z >= -128) and np.all(z <= 127)
    assert np.all(q.min(axis=1) == -128) or np.all(z == -128)


def test_asym_gemm_correction_equals_centered_product():
    """sum_k (q - z) w computed by a plain int64 matmul of the centred codes equals the
    oracle's acc - z * rowsum (exact), and dequant_ex follows it."""
    rng = np.random.default_rng(13)
    M, N, K = 11, 23, 208
    xq = rng.integers(-128, 128, (M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, (N, K), dtype=np.int8)
    z = rng.integers(-128, 128, M).astype(np.int32)
    d = rng.uniform(1e-3, 1e-2, M).astype(np.float32)
    e = rng.uniform(1e-3, 1e-2, N).astype(np.float32)
    rs = oracle.weight_row_sums(wq)
    assert np.array_equal(rs, wq.astype(np.int64).sum(axis=1))
    acc = oracle.int8_gemm(xq, wq)
    y_ref, _ = oracle.dequant_ex(acc, d, e, None, z, rs)
    centred = (xq.astype(np.int64) - z[:, None]) @ wq.astype(np.int64).T
    ref = centred.astype(np.float64) * d[:, None].astype(np.float64) * e[None, :].astype(np.float64)
    assert np.allclose(y_ref, ref, rtol=1e-15, atol=0)


def test_per_tensor_dequant_is_the_broadcast_scale():
    rng = np.random.default_rng(14)
    acc = rng.integers(-10 ** 6, 10 ** 6, (5, 9)).astype(np.int32)
    e = rng.uniform(1e-3, 1e-2, 9).astype(np.float32)
    d1 = np.array([0.0123], np.float32)
    a = oracle.dequant_ex(acc, d1, e)
    b = oracle.dequant_ex(acc, np.repeat(d1, 5), e)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    assert np.allclose(a[0], acc * float(d1[0]) * e.astype(np.float64)[None, :], rtol=1e-15)


# --------------------------------------------------------------------------- planted mistakes
def test_variant_pins_catch_planted_mistakes():
    # 1. percentile off by one rank: the brute-force pin differs
    rng = np.random.default_rng(15)
    x = _bits(rng.normal(0, 1, (8, 64)).astype(np.float32))
    v = np.sort(np.abs(_f32(x)).ravel())
    rank = math.ceil(0.5 * v.size)
    assert oracle.abs_percentile(x, 50.0) == v[rank - 1] and v[rank - 1] != v[rank]
    # 2. biased instead of unbiased std: the closed form differs
    _, _, sd = oracle.mean_std_threshold(_bits([[1.0, 2.0], [3.0, 4.0]]), 3.0)
    assert abs(sd - math.sqrt(5.0 / 4.0)) > 1e-3
    # 3. zero point with the wrong sign: the hand example fails
    q, d, z = oracle.quant_act_per_token_asym(_bits([[-1.0, 0.0, 3.0, 0.5]]))
    assert z[0] == -64 and -z[0] != z[0]
    # 4. correction term dropped: differs from the centred product whenever z*rs != 0
    xq = np.array([[1, 2, 3]], np.int8)
    wq = np.array([[1, 1, 1]], np.int8)
    acc = oracle.int8_gemm(xq, wq)
    y0, _ = oracle.dequant_ex(acc, np.ones(1, np.float32), np.ones(1, np.float32))
    y1, _ = oracle.dequant_ex(acc, np.ones(1, np.float32), np.ones(1, np.float32), None,
                              np.array([5], np.int32), oracle.weight_row_sums(wq))
    assert y0[0, 0] == 6.0 and y1[0, 0] == 6.0 - 15.0
    # 5. LayerNorm without mean subtraction: the constant-row pin fails
    xc = _bits(np.full((1, 32), 2.0, np.float32))
    _, _, y_rms = oracle.norm_smooth_quant(xc, oracle.NORM_RMS, _bits(np.ones(32, np.float32)), None, 0.0)
    assert not np.allclose(y_rms, 0.0)


def test_norm_statistics_round_trip():
    """Statistics returned by the oracle and fed back reproduce its result; other statistics
    change it (the override is really used)."""
    rng = np.random.default_rng(16)
    x = _bits(rng.normal(0.5, 2.0, (6, 128)).astype(np.float32))
    g = _bits(rng.uniform(0.5, 1.5, 128).astype(np.float32))
    q, d, y, st = oracle.norm_smooth_quant(x, oracle.NORM_LAYER, g, None, 1e-5, with_stats=True)
    X = _f32(x).astype(np.float64)
    assert np.all(st[:, 0] == X.mean(axis=1).astype(np.float32))
    q2, d2, y2 = oracle.norm_smooth_quant(x, oracle.NORM_LAYER, g, None, 1e-5, stats=st)
    assert np.array_equal(q, q2) and np.array_equal(d, d2) and np.array_equal(y, y2)
    st3 = st.copy()
    st3[:, 1] *= np.float32(2.0)
    _, _, y3 = oracle.norm_smooth_quant(x, oracle.NORM_LAYER, g, None, 1e-5, stats=st3)
    assert np.array_equal(y3, 2.0 * y)
