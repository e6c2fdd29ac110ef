"""GPU parity of the LLM.int8() decomposed linear: outlier mask and count bit for bit,
INT32 accumulator of the int8 part bit for bit, bf16 output within tolerance of the
oracle's fp64 reference (the outlier part is accumulated in fp32 on the tensor cores)."""
import numpy as np
import pytest

import oracle
from w8a8_quantized_gemm_b200 import workloads as wl

from _gpu import assert_close_bf16, llmint8_gpu

pytestmark = pytest.mark.gpu


def _check(p, threshold=None):
    thr = p.threshold if threshold is None else threshold
    g = llmint8_gpu(p, threshold=thr)
    o = oracle.llmint8_linear(p.X, p.W, p.bias, thr)
    assert g["count"] == o["count"]
    assert np.array_equal(g["mask"], o["mask"])
    assert np.array_equal(g["Wq"], o["Wq"]) and np.array_equal(g["e"], o["e"])
    assert np.array_equal(g["acc"], o["acc"])
    assert_close_bf16(g["Y"], o["y_ref"], p.name)
    return g, o


def test_tiny_config_outliers_are_channels_0_1():
    g, o = _check(wl.tiny())
    assert g["count"] == 2 and list(o["idx"]) == [0, 1]


# (2433, 1800, 272) runs on CTA pairs (256 x 256 tiles; 70 outlier columns = two bf16 k-blocks);
# (2048, 7168, 1152) gives each pair three or four tiles and (384, 32768, 1152) each single CTA
# two or three (both accumulator buffers reused; nine k-blocks, so each tile's outlier
# k-blocks run after eight k-blocks of the next tile), (1152, 2304, 256) runs 128-wide tiles
@pytest.mark.parametrize("M,N,K,nout", [(5, 24, 48, 1), (130, 72, 144, 3), (200, 264, 208, 7),
                                        (257, 1000, 528, 70), (1024, 2048, 1024, 10), (64, 4096, 4096, 6),
                                        (300, 9480, 528, 5), (2433, 1800, 272, 70), (2048, 7168, 1152, 12),
                                        (384, 32768, 1152, 12), (1152, 2304, 256, 9)])
def test_random_ragged(M, N, K, nout):
    p = wl.random_problem(M, N, K, seed=M + 3 * N + K, outliers=nout, offset=25.0)
    g, _ = _check(p)
    assert g["count"] == nout


@pytest.mark.parametrize("M,N,K", [(96, 136, 272), (2433, 1800, 272)])
def test_no_outliers_is_plain_w8a8(M, N, K):
    """No outlier column: the kernel double-buffers its int32 accumulator (also on CTA pairs)."""
    p = wl.random_problem(M, N, K, seed=4, outliers=0)
    g, _ = _check(p, threshold=1e30)
    assert g["count"] == 0


def test_all_columns_outliers_is_bf16_gemm():
    p = wl.random_problem(40, 56, 80, seed=6, outliers=0)
    g, o = _check(p, threshold=-1.0)
    assert g["count"] == p.K and np.all(g["acc"] == 0)


def test_threshold_equal_is_not_outlier():
    p = wl.random_problem(16, 16, 32, seed=1, outliers=0)
    x = wl.bf16_bits_to_f32(p.X)
    x[3, 5] = 6.0
    x[0, 9] = -6.03125  # next bf16 above 6 in magnitude (ulp 2^-5 in [4, 8))
    p.X = wl.f32_to_bf16_bits(x)
    g, o = _check(p, threshold=6.0)
    assert list(o["idx"]) == [9]
