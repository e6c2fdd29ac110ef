"""Full-size workloads (the benchmark's launch configuration) checked against the oracle on
sampled rows: statistics and scales in full, codes / INT32 / bf16 outputs on a seeded
sample of token rows (and weight rows), since the oracle would take minutes on the rest.

Workloads: Llama-2-7B MLP up-projection [2048 x 4096] x [11008 x 4096]; decode sweep
M in {1,4,16,64} at 4096 x 4096; LLM.int8 sweep [4096 x 8192] x [8192 x 8192] at outlier
fractions 0, 0.1%, 1% and the untruncated heavy-tailed draw; 70B FFN [8192 x 8192] x
[28672 x 8192] with bias at alpha 0.3 / 0.5 / 0.7."""
import numpy as np
import pytest

import oracle
from w8a8_quantized_gemm_b200 import workloads as wl

from _gpu import assert_close_bf16, llmint8_gpu, smoothquant_gpu

pytestmark = pytest.mark.gpu


def _rows(M, n, seed):
    rng = np.random.default_rng(seed)
    r = np.unique(np.concatenate([[0, M - 1], rng.choice(M, min(n, M), replace=False)]))
    return np.sort(r).astype(np.int64)


def _check_smoothquant(p, n_rows=32, n_wrows=64):
    rows = _rows(p.M, n_rows, 1)
    wrows = _rows(p.N, n_wrows, 2)
    g = smoothquant_gpu(p, calib=p.calib, rows=rows, wrows=wrows)
    amax = oracle.act_channel_absmax(p.X if p.calib is None else p.calib)
    assert np.array_equal(g["amax"], amax)
    os_, _ = oracle.smooth_scale(amax, p.W, p.alpha)
    assert np.abs(g["s"].view(np.int32).astype(np.int64) - os_.view(np.int32).astype(np.int64)).max() <= 1
    # weights: sampled rows with the GPU's own factors (per-channel rows are independent)
    oWq, oe = oracle.smooth_quant_weight(p.W[wrows], g["s"], p.w_gran)
    assert np.array_equal(g["Wq"], oWq) and np.array_equal(g["e"], oe)
    # activations and outputs: sampled token rows against the full quantized weight
    Wq_full, e_full = oracle.smooth_quant_weight(p.W, g["s"], p.w_gran)
    assert np.array_equal(g["e_full"], e_full)
    xq, d = oracle.quant_act_per_token(p.X[rows], g["inv_s"])
    assert np.array_equal(g["Xq"], xq) and np.array_equal(g["d"], d)
    acc = oracle.int8_gemm(xq, Wq_full)
    assert np.array_equal(g["acc"], acc)
    y_ref, y_bf = oracle.dequant(acc, d, e_full, p.bias)
    assert np.array_equal(g["Y"], y_bf)
    assert_close_bf16(g["Y"], y_ref, p.name)


def _check_llmint8(p, n_rows=24):
    rows = _rows(p.M, n_rows, 3)
    g = llmint8_gpu(p, rows=rows)
    amax = oracle.act_channel_absmax(p.X)
    mask, idx, count = oracle.outlier_columns(amax, p.threshold)
    assert g["count"] == count and np.array_equal(g["mask"], mask)
    Wq, e = oracle.smooth_quant_weight(p.W, None, 1)
    assert np.array_equal(g["Wq"], Wq) and np.array_equal(g["e"], e)
    xq, d = oracle.quant_act_per_token(p.X[rows], None, mask)
    acc = oracle.int8_gemm(xq, Wq)
    assert np.array_equal(g["acc"], acc)
    o = oracle.outlier_product(p.X[rows], p.W, idx)
    y_ref, _ = oracle.dequant(acc, d, e, p.bias, o)
    assert_close_bf16(g["Y"], y_ref, p.name)
    return count


def test_llama7b_mlp_up_full():
    _check_smoothquant(wl.llama7b_mlp_up())


@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_decode_sweep_full(M):
    _check_smoothquant(wl.decode(M), n_rows=M, n_wrows=128)


@pytest.mark.parametrize("frac,expect", [(0.0, 0), (0.001, 8), (0.01, 82)])
def test_llmint8_sweep_full(frac, expect):
    assert _check_llmint8(wl.llmint8_sweep(frac)) == expect


def test_llmint8_literal_heavy_tail_full():
    """Untruncated 0.5*t(3): nearly every column crosses 6.0, the outlier GEMM does most of the work."""
    count = _check_llmint8(wl.llmint8_sweep(0.0, truncate=None), n_rows=8)
    assert count > 0.9 * 8192


@pytest.fixture(scope="module")
def ffn70b_inputs():
    return wl.ffn70b(0.5)


@pytest.mark.parametrize("alpha", [0.3, 0.5, 0.7])
def test_ffn70b_full(alpha, ffn70b_inputs):
    p = ffn70b_inputs
    p.alpha = alpha
    _check_smoothquant(p, n_rows=12, n_wrows=64)
