"""GPU parity of the HBM-bound kernels against the oracle: column absmax, smoothing
factors, smoothed weight quantization, per-token activation quantization.

Integer and max outputs must match bit for bit; the smoothing factor (a pow) within one
fp32 ulp. Later stages take the GPU's own factors as input on both sides."""
import numpy as np
import pytest
import torch

import oracle
from w8a8_quantized_gemm_b200 import sq
from w8a8_quantized_gemm_b200 import workloads as wl

from _gpu import dev_bf16, empty, host

pytestmark = pytest.mark.gpu

# K values chosen to hit every threads-per-row branch of the row kernel and a ragged
# column block of the column-absmax kernel (K % 256 != 0)
ROW_SHAPES = [(1, 16), (3, 48), (5, 512), (4, 528), (9, 1024), (7, 2048), (6, 4096), (3, 8192), (2, 8208),
              (2, 16384), (2, 20000), (1, 65536)]


# column blocks of 64 / 128 / 256 columns (the kernel picks by K and SM count), clusters of
# 1 to 8 CTAs along the rows (at least 64 rows each), ragged last blocks and row splits
@pytest.mark.parametrize("M,K", [(1, 16), (7, 48), (33, 272), (300, 4112), (2048, 4096), (129, 8192), (600, 8192),
                                 (520, 8208), (5000, 1024)])
def test_channel_absmax_exact(M, K):
    p = wl.random_problem(M, 8, K, seed=M + K, outliers=3, offset=50.0)
    amax = empty(K, torch.float32)
    sq.sq_act_channel_absmax(dev_bf16(p.X), amax)
    got = host(amax)
    assert np.array_equal(got, oracle.act_channel_absmax(p.X))
    # running maximum over a second batch
    q = wl.random_problem(M // 2 + 1, 8, K, seed=M + K + 1, outliers=1, offset=80.0)
    sq.sq_act_channel_absmax(dev_bf16(q.X), amax, accumulate=True)
    assert np.array_equal(host(amax), oracle.act_channel_absmax(q.X, prev=got))


def test_channel_absmax_strided():
    """Leading dimension larger than K (a column slice of a wider matrix)."""
    p = wl.random_problem(40, 8, 512, seed=3, outliers=2)
    X = dev_bf16(p.X)[:, 128:384]
    amax = empty(256, torch.float32)
    sq.sq_act_channel_absmax(X, amax)
    assert np.array_equal(host(amax), oracle.act_channel_absmax(p.X[:, 128:384]))


@pytest.mark.parametrize("alpha", [0.0, 0.3, 0.5, 0.7, 1.0])
@pytest.mark.parametrize("N,K", [(24, 96), (300, 4096), (1000, 8192), (11008, 4096)])
def test_smooth_scale_within_one_ulp(alpha, N, K):
    p = wl.random_problem(64, N, K, seed=N, outliers=4, offset=40.0)
    amax = oracle.act_channel_absmax(p.X)
    amax[3] = 0.0  # clamp path
    s, inv_s = empty(K, torch.float32), empty(K, torch.float32)
    sq.sq_smooth_scale(torch.from_numpy(amax).cuda(), dev_bf16(p.W), alpha, s, inv_s)
    gs, gi = host(s), host(inv_s)
    os_, oi = oracle.smooth_scale(amax, p.W, alpha)
    ulps = np.abs(gs.view(np.int32).astype(np.int64) - os_.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1
    # inv_s is the IEEE fp32 reciprocal of the GPU's own s
    assert np.array_equal(gi, (np.float32(1.0) / gs).astype(np.float32))


@pytest.mark.parametrize("M,K", ROW_SHAPES)
@pytest.mark.parametrize("smooth", [False, True])
def test_quant_act_per_token_exact(M, K, smooth):
    p = wl.random_problem(M, 8, K, seed=K + M, outliers=4, offset=30.0)
    inv_s = None
    if smooth:
        rng = np.random.default_rng(K)
        inv_s = rng.uniform(0.05, 4.0, K).astype(np.float32)
    Xq, d = empty((M, K), torch.int8), empty(M, torch.float32)
    sq.sq_quant_act_per_token(dev_bf16(p.X), None if inv_s is None else torch.from_numpy(inv_s).cuda(), Xq, d)
    oq, od = oracle.quant_act_per_token(p.X, inv_s)
    assert np.array_equal(host(Xq), oq)
    assert np.array_equal(host(d), od)


def test_quant_act_zero_rows_and_ties():
    X = np.zeros((5, 32), np.uint16)
    vals = np.array([127.0, 2.5, 1.5, -0.5, 0.5, -2.5], np.float32)
    X[2, :6] = wl.f32_to_bf16_bits(vals)
    Xq, d = empty((5, 32), torch.int8), empty(5, torch.float32)
    sq.sq_quant_act_per_token(dev_bf16(X), None, Xq, d)
    q = host(Xq)
    assert list(q[2, :6]) == [127, 2, 2, 0, 0, -2]
    assert np.all(q[[0, 1, 3, 4]] == 0) and np.all(host(d)[[0, 1, 3, 4]] == 0)


@pytest.mark.parametrize("K", [272, 8192])
def test_quant_act_tiny_row_absmax(K):
    """Rows of tiny magnitude: below an absmax of 127 / FLT_MAX (about 3.7e-37) the factor
    127/a overflows to infinity on both sides and every code saturates to 127 or -128 (the
    kernel's clamped branch); just above it the factor is finite and near FLT_MAX (the
    unclamped branch). Non-zero values only: 0 * inf has no code."""
    rng = np.random.default_rng(K)
    M = 4
    x = rng.uniform(0.5, 2.0, (M, K)).astype(np.float32) * np.where(rng.random((M, K)) < 0.5, -1.0, 1.0)
    x[0] *= np.float32(1e-37)     # absmax ~2e-37: 127/a = inf
    x[2] *= np.float32(2.2e-37)   # absmax ~4.4e-37: 127/a ~ 2.9e38, finite
    X = wl.f32_to_bf16_bits(x.astype(np.float32))
    Xq, d = empty((M, K), torch.int8), empty(M, torch.float32)
    sq.sq_quant_act_per_token(dev_bf16(X), None, Xq, d)
    oq, od = oracle.quant_act_per_token(X, None)
    assert np.array_equal(host(Xq), oq)
    assert np.array_equal(host(d), od)
    assert set(np.unique(oq[0]).tolist()) <= {127, -128}
    assert np.abs(oq[2].astype(np.int32)).max() == 127 and np.unique(oq[2]).size > 2


@pytest.mark.parametrize("gran", [sq.SQ_PER_CHANNEL, sq.SQ_PER_TENSOR])
@pytest.mark.parametrize("N,K", [(1, 16), (13, 528), (256, 256), (300, 4096), (64, 8208), (8, 20000)])
def test_smooth_quant_weight_exact(gran, N, K):
    p = wl.random_problem(4, N, K, seed=N * 7 + K, outliers=2)
    rng = np.random.default_rng(N)
    s = rng.uniform(0.1, 30.0, K).astype(np.float32)
    Wq = empty((N, K), torch.int8)
    e = empty(N if gran == sq.SQ_PER_CHANNEL else 1, torch.float32)
    ws = sq.workspace(sq.SQ_OP_SMOOTH_QUANT_WEIGHT, 0, N, K)
    sq.sq_smooth_quant_weight(dev_bf16(p.W), torch.from_numpy(s).cuda(), gran, Wq, e, ws)
    oq, oe = oracle.smooth_quant_weight(p.W, s, gran)
    assert np.array_equal(host(Wq), oq)
    assert np.array_equal(host(e), oe)


def test_validation_errors_do_not_launch():
    X = empty((4, 20), torch.bfloat16)  # K % 16 != 0
    with pytest.raises(sq.SqError) as ei:
        sq.sq_act_channel_absmax(X, empty(20, torch.float32))
    assert ei.value.status == sq.SQ_ERR_INVALID
    W = empty((8, 32), torch.bfloat16)
    with pytest.raises(sq.SqError) as ei:
        sq.sq_smooth_quant_weight(W, None, sq.SQ_PER_TENSOR, empty((8, 32), torch.int8), empty(1, torch.float32))
    assert ei.value.status == sq.SQ_ERR_WORKSPACE
