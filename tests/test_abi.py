"""The C ABI without a GPU: the library loads, exports exactly what include/sq.h
declares, sizes workspaces, and rejects bad arguments before launching anything
(validation never touches the device, so these calls are safe on a CPU-only host)."""
import ctypes as C
import os
import re

import pytest

from w8a8_quantized_gemm_b200 import sq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    text = open(os.path.join(ROOT, "include", "sq.h")).read()
    return re.findall(r"SQ_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)


def test_header_symbols_exported():
    names = _declared()
    assert set(names) >= {"sq_act_channel_absmax", "sq_smooth_scale", "sq_smooth_quant_weight",
                          "sq_quant_act_per_token", "sq_int8_gemm_dequant", "llmint8_decomposed_linear",
                          "sq_workspace_size", "sq_last_error", "sq_sync_status"}
    lib = C.CDLL(sq.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n


def test_only_declared_symbols_exported():
    out = os.popen(f"nm -D --defined-only {sq.LIB_PATH}").read().split("\n")
    exported = {l.split()[-1] for l in out if " T " in l}
    assert exported == set(_declared())


def test_version():
    assert "sm_100a" in sq.sq_version()


def test_workspace_sizes():
    assert sq.sq_workspace_size(sq.SQ_OP_SMOOTH_QUANT_WEIGHT, 0, 100, 64) >= 4
    M, N, K = 2048, 11008, 4096
    ws = sq.sq_workspace_size(sq.SQ_OP_LLMINT8, M, N, K)
    # int8 activations + gathered bf16 outlier operands (worst case: every column)
    assert ws >= M * K + 2 * (M + N) * K
    assert sq.sq_workspace_size(99, M, N, K) == 0
    # enough output tiles to fill the GPU: whole tiles, no workspace
    assert sq.sq_workspace_size(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K) == 0
    dec = sq.sq_workspace_size(sq.SQ_OP_INT8_GEMM_DEQUANT, 64, 4096, 4096)
    assert dec >= 2 * 64 * 4096 * 4


FAKE = 1 << 20  # a 16-byte-aligned non-null address; never dereferenced on these paths


def _raw():
    return sq.lib()


@pytest.mark.parametrize("M,K,ld,code", [(0, 64, 64, sq.SQ_ERR_INVALID), (4, 20, 20, sq.SQ_ERR_INVALID),
                                         (4, 64, 32, sq.SQ_ERR_INVALID), (4, 64, 68, sq.SQ_ERR_ALIGN),
                                         (4, 65552, 65552, sq.SQ_ERR_INVALID)])
def test_absmax_validation(M, K, ld, code):
    assert _raw().sq_act_channel_absmax(FAKE, M, K, ld, FAKE, 0, None) == code
    assert sq.sq_last_error() != ""


def test_null_and_alignment_rejected():
    L = _raw()
    assert L.sq_quant_act_per_token(None, 4, 64, 64, None, FAKE, FAKE, None) == sq.SQ_ERR_INVALID
    assert L.sq_quant_act_per_token(FAKE + 8, 4, 64, 64, None, FAKE, FAKE, None) == sq.SQ_ERR_ALIGN
    assert L.sq_smooth_scale(FAKE, FAKE, 8, 64, 64, C.c_float(1.5), FAKE, FAKE + 256, None) == sq.SQ_ERR_INVALID
    assert L.sq_smooth_scale(FAKE, FAKE, 8, 64, 64, C.c_float(0.5), FAKE, FAKE, None) == sq.SQ_ERR_INVALID


def test_gemm_validation():
    L = _raw()
    # N not a multiple of 8
    assert L.sq_int8_gemm_dequant(FAKE, FAKE, FAKE, FAKE, 1, None, FAKE, 16, 12, 64, None, None, 0, None) \
        == sq.SQ_ERR_INVALID
    # bad granularity
    assert L.sq_int8_gemm_dequant(FAKE, FAKE, FAKE, FAKE, 7, None, FAKE, 16, 16, 64, None, None, 0, None) \
        == sq.SQ_ERR_INVALID
    # per-tensor weight quantization without workspace
    assert L.sq_smooth_quant_weight(FAKE, 8, 64, 64, None, 0, FAKE, FAKE, None, 0, None) == sq.SQ_ERR_WORKSPACE


def test_llmint8_validation():
    L = _raw()
    need = sq.sq_workspace_size(sq.SQ_OP_LLMINT8, 16, 16, 64)
    assert L.llmint8_decomposed_linear(FAKE, FAKE, FAKE, FAKE, C.c_float(6.0), None, FAKE, 16, 16, 64, None, None,
                                       None, FAKE, need - 1, None) == sq.SQ_ERR_WORKSPACE
    assert L.llmint8_decomposed_linear(FAKE, FAKE, FAKE, FAKE, C.c_float(float("nan")), None, FAKE, 16, 16, 64,
                                       None, None, None, FAKE, need, None) == sq.SQ_ERR_INVALID


def test_variant_workspace_sizes():
    assert sq.sq_workspace_size(sq.SQ_OP_QUANT_ACT_PER_TENSOR, 16, 0, 64) >= 4
    assert sq.sq_workspace_size(sq.SQ_OP_MEAN_STD_THRESHOLD, 4096, 0, 8192) >= 8 * 2 * 1024
    assert sq.sq_workspace_size(sq.SQ_OP_MEAN_STD_THRESHOLD, 3, 0, 64) >= 8 * 2 * 3
    assert sq.sq_workspace_size(sq.SQ_OP_ABS_PERCENTILE, 1, 0, 16) == 8 * (1 << 15)


def test_variant_validation():
    L = _raw()
    # dynamic per-tensor without workspace; clip misaligned
    assert L.sq_quant_act_per_tensor(FAKE, 4, 64, 64, None, None, FAKE, FAKE, None, 0, None) == sq.SQ_ERR_WORKSPACE
    assert L.sq_quant_act_per_tensor(FAKE, 4, 64, 64, None, FAKE + 2, FAKE, FAKE, None, 0, None) == sq.SQ_ERR_ALIGN
    # asymmetric GEMM needs per-token scales and row sums
    assert L.sq_int8_gemm_dequant_ex(FAKE, FAKE, FAKE, 0, FAKE, FAKE, 1, FAKE, None, FAKE, 16, 16, 64, None, None, 0,
                                     None) == sq.SQ_ERR_INVALID
    assert L.sq_int8_gemm_dequant_ex(FAKE, FAKE, FAKE, 1, FAKE, FAKE, 1, None, None, FAKE, 16, 16, 64, None, None, 0,
                                     None) == sq.SQ_ERR_INVALID
    assert L.sq_int8_gemm_dequant_ex(FAKE, FAKE, FAKE, 5, None, FAKE, 1, None, None, FAKE, 16, 16, 64, None, None, 0,
                                     None) == sq.SQ_ERR_INVALID
    # fused norm: K above 16384 (the longest row a row group holds), bad norm, negative eps, no gamma
    assert L.sq_norm_smooth_quant(FAKE, 4, 16400, 16400, 0, FAKE, None, C.c_float(1e-5), None, FAKE, FAKE, None,
                                  None) == sq.SQ_ERR_INVALID
    assert L.sq_norm_smooth_quant(FAKE, 4, 64, 64, 2, FAKE, None, C.c_float(1e-5), None, FAKE, FAKE, None,
                                  None) == sq.SQ_ERR_INVALID
    assert L.sq_norm_smooth_quant(FAKE, 4, 64, 64, 0, FAKE, None, C.c_float(-1.0), None, FAKE, FAKE, None,
                                  None) == sq.SQ_ERR_INVALID
    assert L.sq_norm_smooth_quant(FAKE, 4, 64, 64, 1, None, None, C.c_float(1e-5), None, FAKE, FAKE, None,
                                  None) == sq.SQ_ERR_INVALID
    # threshold and percentile: workspace, NaN k, p out of range
    need = sq.sq_workspace_size(sq.SQ_OP_MEAN_STD_THRESHOLD, 4, 0, 64)
    assert L.sq_act_mean_std_threshold(FAKE, 4, 64, 64, C.c_double(6.0), FAKE, None, FAKE, need - 8, None) \
        == sq.SQ_ERR_WORKSPACE
    assert L.sq_act_mean_std_threshold(FAKE, 4, 64, 64, C.c_double(float("nan")), FAKE, None, FAKE, need, None) \
        == sq.SQ_ERR_INVALID
    pneed = sq.sq_workspace_size(sq.SQ_OP_ABS_PERCENTILE, 4, 0, 64)
    assert L.sq_act_abs_percentile(FAKE, 4, 64, 64, C.c_double(100.5), FAKE, FAKE, pneed, None) == sq.SQ_ERR_INVALID
    assert L.sq_act_abs_percentile(FAKE, 4, 64, 64, C.c_double(50.0), FAKE, FAKE, pneed - 1, None) \
        == sq.SQ_ERR_WORKSPACE
    # asymmetric quantization and row sums: null outputs
    assert L.sq_quant_act_per_token_asym(FAKE, 4, 64, 64, None, FAKE, FAKE, None, None) == sq.SQ_ERR_INVALID
    assert L.sq_weight_row_sums(FAKE, 4, 64, None, None) == sq.SQ_ERR_INVALID
    # LLM.int8 with a device threshold: NULL threshold
    lneed = sq.sq_workspace_size(sq.SQ_OP_LLMINT8, 16, 16, 64)
    assert L.llmint8_decomposed_linear_ex(FAKE, FAKE, FAKE, FAKE, None, None, FAKE, 16, 16, 64, None, None, None,
                                          FAKE, lneed, None) == sq.SQ_ERR_INVALID


def test_debug_build_exports_the_same_symbols():
    """libsq_debug.so (bounds guards) carries the ABI of libsq.so (plus the device-link
    registration stubs that relocatable device code adds)."""
    from w8a8_quantized_gemm_b200 import build as _b
    out = os.popen(f"nm -D --defined-only {_b.LIB_DEBUG}").read().split("\n")
    exported = {l.split()[-1] for l in out if " T " in l}
    assert exported >= set(_declared())
    assert all(n in _declared() or n.startswith("__cuda") for n in exported)
