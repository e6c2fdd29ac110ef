"""GPU parity of the tcgen05 INT8 GEMM + dequant epilogue (and the whole SmoothQuant
path) against the oracle: the INT32 accumulator bit for bit, the bf16 output bit for bit
against the oracle's fp32 sequence and within the stated tolerance of the fp64 reference."""
import numpy as np
import pytest
import torch

import oracle
from w8a8_quantized_gemm_b200 import sq
from w8a8_quantized_gemm_b200 import workloads as wl

from _gpu import assert_close_bf16, dev_bf16, empty, host, host_bits, smoothquant_gpu

pytestmark = pytest.mark.gpu


def _gemm_direct(xq, wq, d, e, gran, bias_bits):
    M, K = xq.shape
    N = wq.shape[0]
    Y = empty((M, N), torch.bfloat16)
    acc = empty((M, N), torch.int32)
    sq.sq_int8_gemm_dequant(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(), torch.from_numpy(d).cuda(),
                            torch.from_numpy(e).cuda(), gran, None if bias_bits is None else dev_bf16(bias_bits), Y,
                            acc, sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K))
    sq.sq_sync_status()
    return host(acc), host_bits(Y)


# shapes: single tile, ragged in every dimension, K below one k-block, several tiles for the
# BN = 64 / 128 / 256 variants (the variant depends on the tile count versus the SM count)
# (128,128,4096), (257,1000,528), (3,200,1040) and (64,4096,4096) split K over int32 partials;
# up to 64 tokens swap the operands (weight rows on the 128-row MMA operand): (37,9736,256)
# fills the SMs with whole swapped tiles, (1,4096,4096) splits them, (65,296,512) does not swap;
# (2304,2120,720), (2433,1800,272) and (4100,1288,1040) run on CTA pairs (256 x 256 tiles): the
# last column tile leaves the odd CTA's half of B out of range, 2433 and 4100 leave the odd
# CTA's rows of the last row tile (nearly) empty, 4100 x 1288 takes two passes of the pairs;
# (100, 37888, 128) fills the SMs with 256-wide tiles of one 128-row tile (no pairs: the odd
# CTA would only compute padding). Up to 4 tokens take the CUDA-core product (a warp per output
# channel): (1, 8, 16) gives one CTA fewer channels than warps, (4, 3000, 4096) a channel count
# that is no multiple of the CTA's warps, (2, 520, 16384) the longest rows (several rounds of
# loads per row), (3, 2000, 12304) a last round of loads that runs past the end of the row.
# More swapped K splits: (33, 4736, 2048) on all 148 SMs (one token in the second column
# half), (48, 3000, 1024) with a ragged last weight tile, (8, 2048, 4096) in eight parts
GEMM_SHAPES = [(1, 8, 16), (16, 256, 256), (5, 24, 48), (130, 72, 144), (200, 264, 208), (128, 128, 4096),
               (257, 1000, 528), (3, 200, 1040), (64, 4096, 4096), (1024, 2048, 1024), (300, 9480, 528),
               (2304, 2120, 720), (37, 9736, 256), (1, 4096, 4096), (65, 296, 512), (2433, 1800, 272),
               (4100, 1288, 1040), (100, 37888, 128), (4, 3000, 4096), (2, 520, 16384), (3, 2000, 12304),
               (33, 4736, 2048), (48, 3000, 1024), (8, 2048, 4096)]


@pytest.mark.parametrize("M,N,K", GEMM_SHAPES)
def test_int8_gemm_random_codes(M, N, K):
    rng = np.random.default_rng(M * 31 + N * 7 + K)
    xq = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    d = rng.uniform(1e-3, 2e-2, M).astype(np.float32)
    e = rng.uniform(1e-4, 1e-3, N).astype(np.float32)
    bias = wl.f32_to_bf16_bits(rng.normal(0, 0.1, N).astype(np.float32))
    acc, y = _gemm_direct(xq, wq, d, e, sq.SQ_PER_CHANNEL, bias)
    oacc = oracle.int8_gemm(xq, wq)
    assert np.array_equal(acc, oacc)
    y_ref, y_bf = oracle.dequant(oacc, d, e, bias)
    assert np.array_equal(y, y_bf)
    assert_close_bf16(y, y_ref, f"gemm {M}x{N}x{K}")


def test_int8_gemm_extreme_codes():
    """All codes -128 x -128 at K = 65536 reaches 2^30 (the largest sum the bounds allow)."""
    M, N, K = 3, 16, 65536
    xq = np.full((M, K), -128, np.int8)
    wq = np.full((N, K), -128, np.int8)
    wq[1] = 127
    d = np.ones(M, np.float32)
    e = np.ones(1, np.float32)
    acc, _ = _gemm_direct(xq, wq, d, e, sq.SQ_PER_TENSOR, None)
    assert np.all(acc[:, 0] == K * 128 * 128) and np.all(acc[:, 1] == -K * 128 * 127)


@pytest.mark.parametrize("gran", [sq.SQ_PER_TENSOR, sq.SQ_PER_CHANNEL])
def test_tiny_config_full_path(gran):
    """X [16,256] ~N(0,0.1) with channels 0-1 +50, W [256,256] ~N(0,0.02), alpha 0.5."""
    p = wl.tiny()
    p.w_gran = gran
    g = smoothquant_gpu(p)
    o = oracle.smoothquant_linear(p.X, p.W, None, p.alpha, gran, s=g["s"], inv_s=g["inv_s"])
    assert np.array_equal(g["amax"], oracle.act_channel_absmax(p.X))
    os_, _ = oracle.smooth_scale(g["amax"], p.W, p.alpha)
    assert np.abs(g["s"].view(np.int32).astype(np.int64) - os_.view(np.int32).astype(np.int64)).max() <= 1
    for k in ("Wq", "e", "Xq", "d", "acc"):
        assert np.array_equal(g[k], o[k]), k
    assert np.array_equal(g["Y"], o["y_bf16"])
    assert_close_bf16(g["Y"], o["y_ref"], "tiny")


@pytest.mark.parametrize("M,N,K,gran", [(77, 136, 528, sq.SQ_PER_CHANNEL), (300, 520, 1040, sq.SQ_PER_TENSOR),
                                        (300, 9480, 528, sq.SQ_PER_TENSOR),
                                        (1, 4096, 4096, sq.SQ_PER_CHANNEL), (64, 1024, 4096, sq.SQ_PER_CHANNEL)])
def test_smoothquant_path_ragged(M, N, K, gran):
    p = wl.random_problem(M, N, K, seed=M + N + K, outliers=3, offset=40.0, w_gran=gran)
    g = smoothquant_gpu(p)
    o = oracle.smoothquant_linear(p.X, p.W, p.bias, p.alpha, gran, s=g["s"], inv_s=g["inv_s"])
    for k in ("Wq", "e", "Xq", "d", "acc"):
        assert np.array_equal(g[k], o[k]), k
    assert np.array_equal(g["Y"], o["y_bf16"])
    assert_close_bf16(g["Y"], o["y_ref"], p.name)


def test_split_k_workspace_reused_across_calls():
    """The split-K arrival counters return to zero, so one workspace serves call after call."""
    M, N, K = 32, 1024, 4096  # swapped operands, 8 tiles each split 16 ways
    assert sq.sq_workspace_size(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K) > 0
    rng = np.random.default_rng(11)
    ws = sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K)
    d = np.full(M, 1e-2, np.float32)
    e = np.full(N, 1e-3, np.float32)
    dd, ee = torch.from_numpy(d).cuda(), torch.from_numpy(e).cuda()
    for rep in range(3):
        xq = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
        wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
        Y = empty((M, N), torch.bfloat16)
        acc = empty((M, N), torch.int32)
        sq.sq_int8_gemm_dequant(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(), dd, ee, sq.SQ_PER_CHANNEL,
                                None, Y, acc, ws)
        sq.sq_sync_status()
        oacc = oracle.int8_gemm(xq, wq)
        assert np.array_equal(host(acc), oacc)
        assert np.array_equal(host_bits(Y), oracle.dequant(oacc, d, e)[1])
    n_t = (N + 63) // 64
    ctr = ws[-((n_t * 8 * 4 + 255) // 256 * 256):].view(torch.int32)
    assert int(ctr.abs().sum()) == 0


def test_repeated_calls_are_deterministic():
    p = wl.random_problem(300, 520, 1040, seed=5, outliers=2)
    a = smoothquant_gpu(p)
    b = smoothquant_gpu(p)
    for k in ("Xq", "Wq", "acc", "Y"):
        assert np.array_equal(a[k], b[k])
