"""Host logic of the GEMM launch plan (no GPU): which path, operand roles, tile width, CTA
pairs and K split each shape gets, read through the sq_debug_gemm_plan hook, against rules
restated here from the kernel design (not from the planner's code):

- up to 4 tokens without outlier columns (K <= 16384): the CUDA-core product;
- up to 64 tokens without outlier columns: swapped operands, 32-token tiles up to 32 tokens and
  64-token tiles above;
- otherwise the widest of 256/128/64 whose 128-row tile count covers the 148 SMs;
- 256-wide tiles run on CTA pairs (256 x 256) when the pair tiles cover the 74 SM pairs and
  the 256-row tiles add no padded rows (an even number of 128-row tiles, or >= 32 of them);
- fewer tiles than half the SMs (and no outlier product) split every tile along K."""
import itertools

import numpy as np
import pytest

from w8a8_quantized_gemm_b200 import sq


SMS = 148


def plan(M, N, K, outliers=False):
    return sq.sq_debug_gemm_plan(M, N, K, outliers)


def cdiv(a, b):
    return -(-a // b)


def test_llama7b_mlp_up_runs_on_pairs():
    p = plan(2048, 11008, 4096)
    assert p["path"] == sq.GEMM_PATH_TENSOR_PAIRS and p["bn"] == 256 and p["swap"] == 0
    assert p["whole_tiles"] == (2048 // 256) * cdiv(11008, 256) and p["split_tiles"] == 0
    q = plan(2048, 11008, 4096, outliers=True)
    assert q["path"] == sq.GEMM_PATH_TENSOR_PAIRS and q["whole_tiles"] == p["whole_tiles"]


@pytest.mark.parametrize("M", [1, 2, 3, 4])
def test_few_tokens_use_the_cuda_core_product(M):
    assert plan(M, 4096, 4096)["path"] == sq.GEMM_PATH_CUDA_CORES
    # not with outlier columns, and not past the staged-activation limit
    assert plan(M, 4096, 4096, outliers=True)["path"] == sq.GEMM_PATH_TENSOR
    assert plan(M, 4096, 16400)["path"] == sq.GEMM_PATH_TENSOR


@pytest.mark.parametrize("M", [5, 16, 64])
def test_decode_swaps_and_splits_k(M):
    p = plan(M, 4096, 4096)
    assert p["path"] == sq.GEMM_PATH_TENSOR and p["swap"] == 1 and p["bn"] == (32 if M <= 32 else 64)
    tiles = 4096 // 128  # weight rows on the 128-row operand, one token column tile
    assert p["whole_tiles"] == 0 and p["split_tiles"] == tiles
    kb = 4096 // 128
    assert p["splits"] >= 2 and p["splits"] * tiles <= SMS
    assert p["splits"] * p["kb_per_split"] >= kb > (p["splits"] - 1) * p["kb_per_split"]


def test_65_tokens_do_not_swap():
    p = plan(65, 4096, 4096)
    assert p["swap"] == 0 and p["path"] == sq.GEMM_PATH_TENSOR


def test_wide_projection_of_one_row_tile_stays_on_single_ctas():
    """65..128 tokens x a vocabulary-wide N: a pair's odd CTA would only compute padding."""
    for M in (65, 100, 128):
        p = plan(M, 37888, 4096)
        assert p["path"] == sq.GEMM_PATH_TENSOR and p["bn"] == 256
        assert p["whole_tiles"] == cdiv(37888, 256)
    # two 128-row tiles: the pair adds no padding
    assert plan(256, 37888, 4096)["path"] == sq.GEMM_PATH_TENSOR_PAIRS


@pytest.mark.parametrize("M,pair", [(2304, True), (2433, True), (2176, False), (4100, True), (3968, False)])
def test_pair_padding_rule(M, pair):
    """128-row tile counts 18, 20 (even), 17 (odd, < 32), 33 (>= 32), 31 (odd, < 32)."""
    p = plan(M, 9472, 1024)
    assert (p["path"] == sq.GEMM_PATH_TENSOR_PAIRS) == pair, p


def test_outlier_products_are_never_split():
    p = plan(128, 1024, 8192, outliers=True)
    assert p["split_tiles"] == 0 and p["whole_tiles"] > 0


def test_plan_invariants_and_workspace_agree():
    rng = np.random.default_rng(0)
    shapes = [(int(m), int(n) * 8, int(k) * 16) for m, n, k in
              zip(rng.integers(1, 9000, 300), rng.integers(1, 4000, 300), rng.integers(1, 600, 300))]
    shapes += [(m, n, k) for m, n, k in itertools.product((1, 5, 64, 65, 128, 129, 256, 2048, 8192),
                                                          (8, 512, 4096, 11008, 28672), (16, 4096))]
    for (M, N, K), outliers in itertools.product(shapes, (False, True)):
        p = plan(M, N, K, outliers)
        kb = cdiv(K, 128)
        if p["path"] == sq.GEMM_PATH_CUDA_CORES:
            assert M <= 4 and not outliers
            continue
        rows, cols = (N, M) if p["swap"] else (M, N)
        assert p["swap"] == (not outliers and M <= 64)
        tile_m = 256 if p["path"] == sq.GEMM_PATH_TENSOR_PAIRS else 128
        tiles = cdiv(rows, tile_m) * cdiv(cols, p["bn"])
        assert p["whole_tiles"] + p["split_tiles"] == tiles
        if p["path"] == sq.GEMM_PATH_TENSOR_PAIRS:
            m_t = cdiv(rows, 128)
            assert p["bn"] == 256 and not p["swap"] and tiles >= SMS // 2
            assert m_t % 2 == 0 or m_t >= 32
        if p["split_tiles"]:
            assert not outliers and p["whole_tiles"] == 0 and 2 * tiles <= SMS
            assert p["splits"] * p["kb_per_split"] >= kb > (p["splits"] - 1) * p["kb_per_split"]
        else:
            assert p["splits"] == 1
        ws = sq.sq_workspace_size(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K) if not outliers else None
        if ws is not None:
            assert (ws > 0) == (p["split_tiles"] > 0)
            if p["split_tiles"]:
                # each K-split unit stores, for each of the 8 epilogue warps, a 32 x 32 int32
                # block per 32-column chunk of the warp's column half (the larger half when
                # the tile has an odd number of chunks); one arrival counter per tile and warp
                chunks = (p["bn"] // 32 + 1) // 2
                slot = 8 * chunks * 32 * 32 * 4
                assert ws >= p["split_tiles"] * p["splits"] * slot + p["split_tiles"] * 8 * 4, (M, N, K, p, ws)


def test_bad_sizes_are_rejected():
    with pytest.raises(sq.SqError) as ei:
        plan(0, 8, 16)
    assert ei.value.status == sq.SQ_ERR_INVALID
