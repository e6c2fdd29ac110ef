"""Pins of the CPU oracle to facts the pages and the mathematics fix.

Each test checks the oracle against something other than itself: values the
pages print (fixtures under tests/golden/, each with its citation), closed forms,
invariants, special cases that reduce to plain library routines, error bounds,
and brute force on tiny inputs. The last group plants mistakes in the oracle's
outputs (on the CPU) and checks that the pins catch them.
"""
import json
import os
import subprocess
import sys
from fractions import Fraction

import numpy as np
import pytest

import oracle
from w8a8_quantized_gemm_b200 import workloads as wl

U32 = 2.0 ** -24  # fp32 unit roundoff


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def _f32(bits):
    return wl.bf16_bits_to_f32(bits)


# --------------------------------------------------------------------------- printed values
def test_per_tensor_outlier_example(golden_dir):
    """SmoothQuant量化实战 §1.2: an outlier channel at +-50 forces scale 50/127 ~ 0.39."""
    g = _load(golden_dir, "sq_per_tensor_outlier_example.json")
    rows, cols = g["shape"]
    rng = np.random.default_rng(1)
    x = rng.uniform(-1.0, 1.0, size=(rows, cols)).astype(np.float32)
    ch = g["outlier_channel"]
    x[:, ch] = np.linspace(-50.0, 50.0, rows).astype(np.float32)
    bits = wl.f32_to_bf16_bits(x)
    assert float(np.abs(_f32(bits)).max()) == g["outlier_absmax"]
    q, e = oracle.smooth_quant_weight(bits, None, oracle.PER_TENSOR)
    assert e.shape == (1,)
    assert abs(float(e[0]) - g["printed_scale"]) <= g["printed_scale_tolerance"]
    assert e[0] == np.float32(np.float32(50.0) / np.float32(127.0))
    small = np.ones_like(q, dtype=bool)
    small[:, ch] = False
    lo, hi = g["small_value_code_range"]
    assert q[small].min() >= lo and q[small].max() <= hi
    # the outlier channel itself spans the full range
    assert q[:, ch].min() == -127 and q[:, ch].max() == 127


def test_tiny_absmax_saturates_and_just_above_does_not():
    """Degenerate rows: an absmax below 127/FLT_MAX makes the fp32 factor 127/a infinite, so
    the non-zero values saturate (127 or -128); an absmax just above keeps codes in [-127, 127]
    with both ends reached (the value at the absmax itself maps to exactly +-127)."""
    x = np.array([[1e-37, -2e-37, 0.5e-37, -1.5e-37],
                  [4.4e-37, -4.4e-37, 2.2e-37, -1.1e-37]], np.float32)
    bits = wl.f32_to_bf16_bits(x)
    xb = _f32(bits)
    a = np.abs(xb).max(axis=1)
    with np.errstate(over="ignore"):
        assert np.isinf(np.float32(127.0) / a[0]) and np.isfinite(np.float32(127.0) / a[1])
    q, d = oracle.quant_act_per_token(bits, None)
    assert list(q[0]) == [127, -128, 127, -128]
    assert q[1].max() == 127 and q[1].min() == -127 and abs(int(q[1, 2])) in (63, 64)
    assert d[0] == np.float32(a[0] / np.float32(127.0))


def test_hand_quantization(golden_dir):
    """量化基础与INT8 quantization-flow example, worked by hand (ties to even)."""
    g = _load(golden_dir, "basics_hand_quant.json")
    x = np.array(g["rows"], np.float32)
    bits = wl.f32_to_bf16_bits(x)
    assert np.array_equal(_f32(bits), x)
    q, d = oracle.quant_act_per_token(bits)
    assert np.array_equal(q, np.array(g["codes"], np.int8))
    want = [np.float32(float(Fraction(s))) for s in g["scales"]]
    assert np.array_equal(d, np.array(want, np.float32))
    # the same rows quantized as per-channel weights give the same codes and scales
    qw, e = oracle.smooth_quant_weight(bits, None, oracle.PER_CHANNEL)
    assert np.array_equal(qw, q) and np.array_equal(e, d)


def test_bf16_rounding(golden_dir):
    g = _load(golden_dir, "bf16_rounding.json")
    vals = np.array([c["value"] for c in g["cases"]], np.float32)
    out = oracle.bf16_to_float(oracle.float_to_bf16(vals))
    assert np.array_equal(out, np.array([c["expect"] for c in g["cases"]], np.float32))


# --------------------------------------------------------------------------- closed forms
def _colmax_w(W):
    return np.abs(_f32(W)).max(axis=0)


@pytest.mark.parametrize("seed", [0, 1])
def test_alpha_special_cases(seed):
    """s_j = max|X_j|^a / max|W_j|^(1-a): a=1 gives the act absmax, a=0 gives 1/wmax,
    a=0.5 gives sqrt(amax/wmax); both maxima clamped at 1e-8."""
    p = wl.random_problem(24, 40, 96, seed=seed, outliers=3)
    amax = np.abs(_f32(p.X)).max(axis=0)
    amax[5] = 0.0  # exercises the 1e-8 clamp
    wmax = _colmax_w(p.W)
    s1, i1 = oracle.smooth_scale(amax, p.W, 1.0)
    assert np.array_equal(s1, np.maximum(amax, np.float32(1e-8)))
    s0, _ = oracle.smooth_scale(amax, p.W, 0.0)
    assert np.array_equal(s0, (1.0 / np.maximum(wmax, np.float32(1e-8)).astype(np.float64)).astype(np.float32))
    sh, ih = oracle.smooth_scale(amax, p.W, 0.5)
    ref = np.sqrt(np.maximum(amax, np.float32(1e-8)).astype(np.float64) / wmax.astype(np.float64))
    assert np.all(np.abs(sh.astype(np.float64) - ref) <= np.spacing(sh).astype(np.float64))
    # inv_s is the fp32 reciprocal: within half an ulp of 1/s
    exact = 1.0 / sh.astype(np.float64)
    assert np.all(np.abs(ih.astype(np.float64) - exact) <= 0.5 * np.spacing(ih).astype(np.float64))


def test_channel_absmax_and_running_max():
    """SmoothQuant量化实战 §3.2: per-channel amax over tokens, running maximum across batches."""
    a = wl.random_problem(33, 8, 80, seed=3, outliers=4).X
    b = wl.random_problem(17, 8, 80, seed=4, outliers=1).X
    m1 = oracle.act_channel_absmax(a)
    assert np.array_equal(m1, np.abs(_f32(a)).max(axis=0))
    m2 = oracle.act_channel_absmax(b, prev=m1)
    assert np.array_equal(m2, np.abs(_f32(np.vstack([a, b]))).max(axis=0))


def _quant_bound_ok(xp, q, d):
    """|x' - q*d| <= d/2 + 4u|x'| for every element (symmetric absmax, fp32 reciprocal)."""
    xp = xp.astype(np.float64)
    dd = d.astype(np.float64)[:, None]
    err = np.abs(xp - q.astype(np.float64) * dd)
    return np.all(err <= 0.5 * dd + 4 * U32 * np.abs(xp) + 1e-300)


@pytest.mark.parametrize("shape", [(7, 33 * 16), (64, 256), (3, 4096)])
def test_quant_error_bound_and_invariants(shape):
    M, K = shape
    p = wl.random_problem(M, 8, K, seed=K, outliers=5, offset=40.0)
    amax = oracle.act_channel_absmax(p.X)
    s, inv_s = oracle.smooth_scale(amax, p.W, 0.5)
    q, d = oracle.quant_act_per_token(p.X, inv_s)
    xp = _f32(p.X) * inv_s[None, :]  # fp32 smoothed values
    assert _quant_bound_ok(xp, q, d)
    # every nonzero row reaches +-127; -128 never occurs
    assert np.all(np.abs(q.astype(np.int32)).max(axis=1) == 127)
    assert q.min() >= -127
    # d is absmax/127 of the smoothed row
    assert np.all(np.abs(d.astype(np.float64) - np.abs(xp).max(axis=1) / 127.0) <= np.spacing(d))


def test_zero_rows_and_columns():
    X = np.zeros((4, 32), np.uint16)
    X[1, 3] = wl.f32_to_bf16_bits(np.array([-2.0], np.float32))[0]
    q, d = oracle.quant_act_per_token(X)
    assert np.all(q[[0, 2, 3]] == 0) and np.all(d[[0, 2, 3]] == 0)
    assert q[1, 3] == -127 and d[1] == np.float32(2.0) / np.float32(127.0)
    qw, e = oracle.smooth_quant_weight(np.zeros((3, 32), np.uint16), None, oracle.PER_TENSOR)
    assert np.all(qw == 0) and e[0] == 0


# --------------------------------------------------------------------------- integer GEMM
def test_int8_gemm_brute_force():
    rng = np.random.default_rng(5)
    xq = rng.integers(-128, 128, size=(3, 7), dtype=np.int8)
    wq = rng.integers(-128, 128, size=(5, 7), dtype=np.int8)
    acc = oracle.int8_gemm(xq, wq)
    for m in range(3):
        for n in range(5):
            assert acc[m, n] == sum(int(xq[m, k]) * int(wq[n, k]) for k in range(7))


def test_int8_gemm_vs_exact_matmul():
    rng = np.random.default_rng(6)
    xq = rng.integers(-127, 128, size=(37, 300), dtype=np.int8)
    wq = rng.integers(-127, 128, size=(53, 300), dtype=np.int8)
    acc = oracle.int8_gemm(xq, wq)
    ref = xq.astype(np.float64) @ wq.astype(np.float64).T  # exact: |acc| < 2^53
    assert np.array_equal(acc.astype(np.float64), ref)


def test_int8_gemm_overflow_detected():
    K = 131072  # 131072 * 128 * 128 = 2^31 leaves int32
    xq = np.full((1, K), -128, np.int8)
    with pytest.raises(OverflowError):
        oracle.int8_gemm(xq, xq)
    assert oracle.int8_gemm(xq[:, :-1], xq[:, :-1])[0, 0] == (K - 1) * 128 * 128


# --------------------------------------------------------------------------- identity / chain
def _identity_residual(p, out):
    """Dequantized smoothed product vs the fp64 dense X.W^T: residual / rigorous bound."""
    x = _f32(p.X).astype(np.float64)
    w = _f32(p.W).astype(np.float64)
    inv_s, s = out["inv_s"].astype(np.float64), out["s"].astype(np.float64)
    xp = np.abs(x * inv_s[None, :])
    wp = np.abs(w * s[None, :])
    d = out["d"].astype(np.float64)
    e = out["e"].astype(np.float64)
    e = np.broadcast_to(e if e.size > 1 else e[0], (p.N,))
    bound = (xp @ (0.5 * np.ones_like(wp.T)) * e[None, :]
             + (0.5 * d[:, None]) * (np.ones_like(xp) @ wp.T)
             + 0.25 * p.K * d[:, None] * e[None, :])
    bound = bound * (1 + 1e-3) + 1e-5 * (xp @ wp.T + np.abs(x) @ np.abs(w).T) + 1e-30
    y_q = (out["Xq"].astype(np.float64) * d[:, None]) @ (out["Wq"].astype(np.float64) * e[:, None]).T
    dense = x @ w.T
    return np.abs(y_q - dense) / bound, dense


@pytest.mark.parametrize("gran", [oracle.PER_CHANNEL, oracle.PER_TENSOR])
@pytest.mark.parametrize("alpha", [0.3, 0.5, 0.7])
def test_smoothquant_identity_bound(gran, alpha):
    """SmoothQuant量化实战 §1.3: X.W = (X diag(s)^-1)(diag(s) W); after int8 quantization of
    both factors the product stays within the rigorous quantization error bound."""
    p = wl.random_problem(29, 45, 176, seed=11, outliers=4, offset=60.0, w_gran=gran, alpha=alpha)
    out = oracle.smoothquant_linear(p.X, p.W, None, alpha, gran)
    ratio, _ = _identity_residual(p, out)
    assert ratio.max() <= 1.0
    # y_ref of the oracle is exactly that dequantized product (fp64, no bias here)
    y_q = (out["acc"].astype(np.float64) * out["d"].astype(np.float64)[:, None]
           * (out["e"].astype(np.float64) if out["e"].size > 1 else out["e"][0])[None])
    assert np.allclose(out["y_ref"], y_q, rtol=1e-12, atol=0)


def test_dequant_bias_and_bf16_rounding():
    p = wl.random_problem(13, 70, 128, seed=2, outliers=2, bias=True)
    out = oracle.smoothquant_linear(p.X, p.W, p.bias, 0.5, oracle.PER_CHANNEL)
    b = _f32(p.bias).astype(np.float64)
    y_nob = out["y_ref"] - b[None, :]
    y_q = (out["acc"].astype(np.float64) * out["d"].astype(np.float64)[:, None]
           * out["e"].astype(np.float64)[None, :])
    assert np.allclose(y_nob, y_q, rtol=1e-12, atol=1e-12)
    ybf = _f32(out["y_bf16"]).astype(np.float64)
    # one bf16 rounding of a value within a few fp32 ulps of y_ref
    assert np.all(np.abs(ybf - out["y_ref"]) <= 2.0 ** -8 * np.abs(out["y_ref"]) + 1e-6 * (1 + np.abs(b)))


# --------------------------------------------------------------------------- LLM.int8
def test_outlier_mask_strict_threshold():
    amax = np.array([6.0, np.nextafter(np.float32(6.0), np.float32(7)), np.nextafter(np.float32(6.0), np.float32(0)),
                     100.0, 0.0] + [1.0] * 30 + [7.0], np.float32)
    mask, idx, count = oracle.outlier_columns(amax, 6.0)
    assert list(idx) == [1, 3, 35] and count == 3
    bits = [(int(mask[j // 32]) >> (j % 32)) & 1 for j in range(amax.size)]
    assert [j for j, b in enumerate(bits) if b] == [1, 3, 35]
    assert mask.size == 2


def test_llmint8_tiny_outliers_are_channels_0_1():
    """Config with channels 0-1 offset by +50: exactly those cross 6.0."""
    p = wl.tiny()
    out = oracle.llmint8_linear(p.X, p.W, None, p.threshold)
    assert list(out["idx"]) == [0, 1]
    assert np.all(out["Xq"][:, :2] == 0)


def test_llmint8_no_outliers_equals_plain_per_token():
    p = wl.random_problem(21, 19, 64, seed=8, outliers=0)
    out = oracle.llmint8_linear(p.X, p.W, p.bias, threshold=1e30)
    assert out["count"] == 0
    xq, d = oracle.quant_act_per_token(p.X)
    wq, e = oracle.smooth_quant_weight(p.W, None, oracle.PER_CHANNEL)
    assert np.array_equal(out["Xq"], xq) and np.array_equal(out["d"], d)
    y_ref, y_bf = oracle.dequant(oracle.int8_gemm(xq, wq), d, e, p.bias)
    assert np.array_equal(out["y_ref"], y_ref) and np.array_equal(out["y_bf16"], y_bf)


def test_llmint8_all_outliers_is_dense_product():
    p = wl.random_problem(9, 23, 48, seed=9, outliers=0)
    out = oracle.llmint8_linear(p.X, p.W, p.bias, threshold=-1.0)
    assert out["count"] == p.K and np.all(out["acc"] == 0) and np.all(out["d"] == 0)
    dense = _f32(p.X).astype(np.float64) @ _f32(p.W).astype(np.float64).T + _f32(p.bias).astype(np.float64)
    assert np.allclose(out["y_ref"], dense, rtol=1e-12, atol=1e-12)


def test_llmint8_decomposition_bound():
    """Y = int8 part over normal columns + exact 16-bit part over outlier columns, within the
    quantization error bound of the normal columns only."""
    p = wl.random_problem(31, 27, 160, seed=12, outliers=3, offset=50.0)
    out = oracle.llmint8_linear(p.X, p.W, None, 6.0)
    assert out["count"] == 3
    x = _f32(p.X).astype(np.float64)
    w = _f32(p.W).astype(np.float64)
    keep = np.ones(p.K, bool)
    keep[out["idx"]] = False
    d = out["d"].astype(np.float64)
    e = out["e"].astype(np.float64)
    xa, wa = np.abs(x[:, keep]), np.abs(w[:, keep])
    bound = (xa.sum(1)[:, None] * e[None] / 2 + d[:, None] * wa.sum(1)[None] / 2
             + 0.25 * keep.sum() * d[:, None] * e[None]) * (1 + 1e-3) + 1e-5 * (xa @ wa.T) + 1e-30
    assert np.all(np.abs(out["y_ref"] - x @ w.T) <= bound)


# --------------------------------------------------------------------------- determinism
def test_oracle_thread_count_invariance():
    code = ("import sys, hashlib; sys.path.insert(0, %r); import oracle; "
            "from w8a8_quantized_gemm_b200 import workloads as wl; p = wl.random_problem(64, 96, 256, seed=3); "
            "o = oracle.smoothquant_linear(p.X, p.W, p.bias); "
            "print(hashlib.sha256(o['Xq'].tobytes() + o['Wq'].tobytes() + o['acc'].tobytes() + o['y_bf16'].tobytes()).hexdigest())"
            % os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    outs = set()
    for t in ("1", "3"):
        env = dict(os.environ, OMP_NUM_THREADS=t)
        outs.add(subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                                check=True).stdout.strip())
    assert len(outs) == 1


# --------------------------------------------------------------------------- planted mistakes
def test_pins_catch_planted_mistakes():
    """Plant plausible mistakes in the oracle's outputs and check a pin fails for each."""
    p = wl.random_problem(29, 45, 176, seed=11, outliers=4, offset=60.0)
    good = oracle.smoothquant_linear(p.X, p.W, None, 0.5, oracle.PER_CHANNEL)
    assert _identity_residual(p, good)[0].max() <= 1.0

    # 1. activations multiplied by s instead of divided by it (inv_s replaced by s)
    bad = oracle.smoothquant_linear(p.X, p.W, None, 0.5, oracle.PER_CHANNEL, s=good["s"], inv_s=good["s"])
    assert _identity_residual(p, bad)[0].max() > 1.0

    # 2. weight left unsmoothed while the activations are divided by s
    ones = np.ones(p.K, np.float32)
    bad = oracle.smoothquant_linear(p.X, p.W, None, 0.5, oracle.PER_CHANNEL, s=ones, inv_s=good["inv_s"])
    assert _identity_residual(p, dict(bad, s=ones))[0].max() > 1.0

    # 3. transposed weight scales (scale of row n applied to row N-1-n)
    bad = dict(good, e=good["e"][::-1].copy())
    assert _identity_residual(p, bad)[0].max() > 1.0

    # 4. one dropped column in the integer sum
    acc_bad = oracle.int8_gemm(good["Xq"][:, 1:], good["Wq"][:, 1:])
    ref = good["Xq"].astype(np.float64) @ good["Wq"].astype(np.float64).T
    assert not np.array_equal(acc_bad.astype(np.float64), ref)

    # 5. >= instead of > at the threshold
    amax = np.array([6.0, 1.0], np.float32)
    assert oracle.outlier_columns(amax, 6.0)[2] == 0
