"""GPU parity of the variants against the oracle, through the C ABI: per-tensor activation
scale (dynamic and calibrated), smoothing-factor normalisation, the GEMM with a per-tensor
activation scale and with asymmetric activations, asymmetric quantization and weight row
sums, fused LayerNorm / RMSNorm + smoothing + quantization, the mean + k*std threshold
feeding LLM.int8, and the percentile of |X|.

Codes, zero points, row sums, int32 accumulators and percentiles must match bit for bit;
bf16 outputs bit for bit against the oracle's fp32 sequence and within the stated tolerance
of its fp64 reference. Values that come out of fp64 sums whose order differs between the
two sides (normalisation statistics, the threshold) are gated within one fp32 ulp and the
steps after them are checked on the GPU's values (chained), as for the smoothing factor."""
import numpy as np
import pytest
import torch

import oracle
from w8a8_quantized_gemm_b200 import sq
from w8a8_quantized_gemm_b200 import workloads as wl

from _gpu import assert_close_bf16, dev_bf16, empty, host, host_bits

pytestmark = pytest.mark.gpu

ROW_SHAPES = [(1, 16), (5, 48), (37, 528), (300, 4096), (7, 8192), (3, 16384), (2, 20000)]


def _x(M, K, seed, outliers=3, offset=40.0):
    return wl.random_problem(M, 8, K, seed=seed, outliers=outliers, offset=offset).X


def _ulps(a, b):
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)


# --------------------------------------------------------------------------- per-tensor
@pytest.mark.parametrize("M,K", ROW_SHAPES)
@pytest.mark.parametrize("smooth", [False, True])
def test_quant_act_per_tensor_dynamic(M, K, smooth):
    X = _x(M, K, M + K)
    inv_s = np.random.default_rng(K).uniform(0.2, 3.0, K).astype(np.float32) if smooth else None
    Xq, d = empty((M, K), torch.int8), empty(1, torch.float32)
    sq.sq_quant_act_per_tensor(dev_bf16(X), None if inv_s is None else torch.from_numpy(inv_s).cuda(), Xq, d,
                               ws=sq.workspace(sq.SQ_OP_QUANT_ACT_PER_TENSOR, M, 0, K))
    sq.sq_sync_status()
    oq, od = oracle.quant_act_per_tensor(X, inv_s)
    assert np.array_equal(host(d), od)
    assert np.array_equal(host(Xq), oq)


@pytest.mark.parametrize("M,K,p", [(64, 512, 99.99), (300, 4096, 99.9), (2, 20000, 90.0)])
def test_percentile_then_static_per_tensor(M, K, p):
    """Calibrated clip from the GPU percentile (exact), then the one-pass static quantization."""
    X = wl.llmint8_sweep(0.001, M=M, K=K, N=8).X
    ws = sq.workspace(sq.SQ_OP_ABS_PERCENTILE, M, 0, K)
    clip = empty(1, torch.float32)
    sq.sq_act_abs_percentile(dev_bf16(X), p, clip, ws)
    sq.sq_sync_status()
    c = float(host(clip)[0])
    assert np.float32(c) == oracle.abs_percentile(X, p)
    Xq, d = empty((M, K), torch.int8), empty(1, torch.float32)
    sq.sq_quant_act_per_tensor(dev_bf16(X), None, Xq, d, clip=clip)
    sq.sq_sync_status()
    oq, od = oracle.quant_act_per_tensor(X, None, clip=c)
    assert np.array_equal(host(d), od) and np.array_equal(host(Xq), oq)
    assert (np.abs(host(Xq).astype(np.int32)) >= 127).any()


@pytest.mark.parametrize("M,K,ld", [(1, 16, 16), (9, 48, 64), (256, 4096, 4096), (33, 1000 * 16, 16000),
                                    (40, 256, 512)])
@pytest.mark.parametrize("p", [0.0, 50.0, 99.99, 100.0])
def test_abs_percentile_exact(M, K, ld, p):
    rng = np.random.default_rng(M * 7 + K)
    full = wl.f32_to_bf16_bits(rng.standard_t(3, size=(M, ld)).astype(np.float32))
    X = dev_bf16(full)[:, :K]
    out = empty(1, torch.float32)
    sq.sq_act_abs_percentile(X, p, out, sq.workspace(sq.SQ_OP_ABS_PERCENTILE, M, 0, K))
    sq.sq_sync_status()
    assert host(out)[0] == oracle.abs_percentile(np.ascontiguousarray(full[:, :K]), p)


def test_statistics_workspaces_serve_calls_in_a_row():
    """One workspace (sized for the largest call) serves percentile and threshold calls of
    different shapes in a row, each matching the oracle: nothing a call leaves in the
    workspace changes the next call's result."""
    wsp = sq.workspace(sq.SQ_OP_ABS_PERCENTILE, 1, 0, 16)
    wms = sq.workspace(sq.SQ_OP_MEAN_STD_THRESHOLD, 4096, 0, 64)
    thr, out = empty(1, torch.float32), empty(1, torch.float32)
    for M, K, p in [(256, 4096, 99.99), (9, 48, 50.0), (2000, 1024, 0.0), (3, 16, 100.0), (256, 4096, 99.9)]:
        X = _x(M, K, M + 3 * K)
        Xt = dev_bf16(X)
        sq.sq_act_abs_percentile(Xt, p, out, wsp)
        sq.sq_act_mean_std_threshold(Xt, 6.0, thr, None, wms)
        sq.sq_sync_status()
        assert host(out)[0] == oracle.abs_percentile(X, p)
        assert _ulps(host(thr), oracle.mean_std_threshold(X, 6.0)[0]).max() <= 1


def test_smooth_scale_normalised():
    rng = np.random.default_rng(5)
    K, N = 1040, 96
    amax = rng.uniform(0.0, 40.0, K).astype(np.float32)
    amax[::97] = 0.0
    W = wl.f32_to_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    a_t, W_t = torch.from_numpy(amax).cuda(), dev_bf16(W)
    s0, i0 = empty(K, torch.float32), empty(K, torch.float32)
    s1, i1 = empty(K, torch.float32), empty(K, torch.float32)
    sq.sq_smooth_scale(a_t, W_t, 0.9, s0, i0)
    sq.sq_smooth_scale_ex(a_t, W_t, 0.9, True, s1, i1)
    sq.sq_sync_status()
    os_, _ = oracle.smooth_scale(amax, W, 0.9)
    assert _ulps(host(s0), os_).max() <= 1
    # the normalisation step, chained on the GPU's unnormalised factors: bit for bit
    ns, ni = oracle.smooth_scale_normalize(host(s0))
    assert np.array_equal(host(s1), ns) and np.array_equal(host(i1), ni)
    assert host(s1).max() == np.float32(127.0) and (host(s1) == np.float32(1e-5)).any()


# --------------------------------------------------------------------------- GEMM variants
GEMM_EX_SHAPES = [(1, 8, 16), (5, 24, 48), (64, 4096, 4096), (130, 72, 144), (300, 9480, 528), (257, 1000, 528),
                  (1024, 2048, 1024), (37, 9736, 256), (2433, 1800, 272)]


def _codes(rng, M, N, K):
    xq = rng.integers(-128, 128, size=(M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    return xq, wq


@pytest.mark.parametrize("M,N,K", GEMM_EX_SHAPES)
def test_gemm_per_tensor_activation_scale(M, N, K):
    rng = np.random.default_rng(M + 3 * N + 5 * K)
    xq, wq = _codes(rng, M, N, K)
    d = np.array([rng.uniform(1e-3, 2e-2)], np.float32)
    e = rng.uniform(1e-4, 1e-3, N).astype(np.float32)
    bias = wl.f32_to_bf16_bits(rng.normal(0, 0.1, N).astype(np.float32))
    Y, acc = empty((M, N), torch.bfloat16), empty((M, N), torch.int32)
    sq.sq_int8_gemm_dequant_ex(torch.from_numpy(xq).cuda(), torch.from_numpy(wq).cuda(), torch.from_numpy(d).cuda(),
                               sq.SQ_PER_TENSOR, None, torch.from_numpy(e).cuda(), sq.SQ_PER_CHANNEL, None,
                               dev_bf16(bias), Y, acc, sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K))
    sq.sq_sync_status()
    oacc = oracle.int8_gemm(xq, wq)
    assert np.array_equal(host(acc), oacc)
    y_ref, y_bf = oracle.dequant_ex(oacc, d, e, bias)
    assert np.array_equal(host_bits(Y), y_bf)
    assert_close_bf16(host_bits(Y), y_ref, f"per-tensor x {M}x{N}x{K}")


@pytest.mark.parametrize("M,N,K", GEMM_EX_SHAPES + [(3, 16, 65536)])
@pytest.mark.parametrize("w_gran", [sq.SQ_PER_CHANNEL, sq.SQ_PER_TENSOR])
def test_gemm_asymmetric_correction(M, N, K, w_gran):
    rng = np.random.default_rng(M + 7 * N + 11 * K + w_gran)
    xq, wq = _codes(rng, M, N, K)
    if K == 65536:  # extreme: the corrected sum needs more than 32 bits in the product term
        xq[:] = -128
        wq[:] = 127
    z = rng.integers(-128, 128, M).astype(np.int32)
    d = rng.uniform(1e-3, 2e-2, M).astype(np.float32)
    e = rng.uniform(1e-4, 1e-3, N if w_gran == sq.SQ_PER_CHANNEL else 1).astype(np.float32)
    wq_t = torch.from_numpy(wq).cuda()
    rs = empty(N, torch.int32)
    sq.sq_weight_row_sums(wq_t, rs)
    sq.sq_sync_status()
    ors = oracle.weight_row_sums(wq)
    assert np.array_equal(host(rs), ors)
    Y = empty((M, N), torch.bfloat16)
    sq.sq_int8_gemm_dequant_ex(torch.from_numpy(xq).cuda(), wq_t, torch.from_numpy(d).cuda(), sq.SQ_PER_CHANNEL,
                               torch.from_numpy(z).cuda(), torch.from_numpy(e).cuda(), w_gran, rs, None, Y, None,
                               sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K))
    sq.sq_sync_status()
    y_ref, y_bf = oracle.dequant_ex(oracle.int8_gemm(xq, wq), d, e, None, z, ors)
    assert np.array_equal(host_bits(Y), y_bf)
    assert_close_bf16(host_bits(Y), y_ref, f"asym {M}x{N}x{K}")


@pytest.mark.parametrize("M,K", ROW_SHAPES)
def test_asymmetric_quantization_exact(M, K):
    rng = np.random.default_rng(M * 3 + K)
    x = rng.normal(0.7, 1.5, (M, K)).astype(np.float32)
    x[:, ::11] = 0.0
    if M > 2:
        x[1] = 0.0            # range 0
        x[2] = np.abs(x[2])   # one-signed row
    X = wl.f32_to_bf16_bits(x)
    inv_s = rng.uniform(0.3, 2.0, K).astype(np.float32)
    Xq, d, z = empty((M, K), torch.int8), empty(M, torch.float32), empty(M, torch.int32)
    sq.sq_quant_act_per_token_asym(dev_bf16(X), torch.from_numpy(inv_s).cuda(), Xq, d, z)
    sq.sq_sync_status()
    oq, od, oz = oracle.quant_act_per_token_asym(X, inv_s)
    assert np.array_equal(host(z), oz)
    assert np.array_equal(host(d), od)
    assert np.array_equal(host(Xq), oq)


def test_asymmetric_linear_end_to_end():
    """ReLU-like (non-negative) activations through the asymmetric path: quantize, row sums,
    GEMM with the exact correction, bit for bit against the oracle chain. Against the fp64
    dense product it is more accurate than the symmetric per-token path on the same data
    (the zero point spends all 256 codes on [0, max] instead of 128)."""
    p = wl.random_problem(96, 264, 1024, seed=21, outliers=0, bias=True)
    X = wl.f32_to_bf16_bits(np.maximum(wl.bf16_bits_to_f32(p.X), 0.0))
    M, N, K = 96, 264, 1024
    X_t = dev_bf16(X)
    Wq, e = empty((N, K), torch.int8), empty(N, torch.float32)
    sq.sq_smooth_quant_weight(dev_bf16(p.W), None, sq.SQ_PER_CHANNEL, Wq, e)
    Xq, d, z = empty((M, K), torch.int8), empty(M, torch.float32), empty(M, torch.int32)
    sq.sq_quant_act_per_token_asym(X_t, None, Xq, d, z)
    rs = empty(N, torch.int32)
    sq.sq_weight_row_sums(Wq, rs)
    gws = sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K)
    Y = empty((M, N), torch.bfloat16)
    sq.sq_int8_gemm_dequant_ex(Xq, Wq, d, sq.SQ_PER_CHANNEL, z, e, sq.SQ_PER_CHANNEL, rs, dev_bf16(p.bias), Y,
                               ws=gws)
    # the symmetric per-token path on the same activations
    Xs, ds, Ys = empty((M, K), torch.int8), empty(M, torch.float32), empty((M, N), torch.bfloat16)
    sq.sq_quant_act_per_token(X_t, None, Xs, ds)
    sq.sq_int8_gemm_dequant(Xs, Wq, ds, e, sq.SQ_PER_CHANNEL, dev_bf16(p.bias), Ys, None, gws)
    sq.sq_sync_status()
    oq, od, oz = oracle.quant_act_per_token_asym(X)
    owq, oe = oracle.smooth_quant_weight(p.W, None, oracle.PER_CHANNEL)
    y_ref, y_bf = oracle.dequant_ex(oracle.int8_gemm(oq, owq), od, oe, p.bias, oz, oracle.weight_row_sums(owq))
    assert np.array_equal(host_bits(Y), y_bf)
    assert_close_bf16(host_bits(Y), y_ref, "asymmetric linear")
    dense = wl.bf16_bits_to_f32(X).astype(np.float64) @ wl.bf16_bits_to_f32(p.W).astype(np.float64).T
    dense += wl.bf16_bits_to_f32(p.bias).astype(np.float64)

    def rel(yb):
        y = wl.bf16_bits_to_f32(yb).astype(np.float64)
        return np.linalg.norm(y - dense) / np.linalg.norm(dense)

    assert rel(host_bits(Y)) < rel(host_bits(Ys)) < 5e-2


# --------------------------------------------------------------------------- fused norm
# register rows up to K = 4096, pipelined row groups beyond (ragged last chunks at 1040, 2064,
# 5008 and 12304 columns; a group with a single row at 9 x 8192 and 3 x 16384; more rows than
# row groups at 700 x 8192 and 1300 x 16384, so every ring slot is refilled several times)
NORM_SHAPES = [(1, 16), (7, 256), (33, 528), (300, 4096), (9, 8192), (3, 16384), (5, 1040), (37, 2064),
               (11, 5008), (6, 12304), (1000, 4096), (700, 8192), (1300, 16384)]


# beta without smoothing and smoothing without beta: the remaining compile-time forms of the
# pipelined row groups (both group shapes, a ragged row)
NORM_MIXED = [(M, K, beta, smooth) for (M, K) in [(9, 8192), (700, 8192), (6, 12304), (300, 4096)]
              for (beta, smooth) in [(True, False), (False, True)]]


@pytest.mark.parametrize("M,K,beta,smooth", [(M, K, b, s) for (M, K) in NORM_SHAPES for (b, s) in
                                             [(True, True), (False, False)]] + NORM_MIXED)
@pytest.mark.parametrize("norm", [sq.SQ_NORM_LAYER, sq.SQ_NORM_RMS])
def test_norm_smooth_quant(M, K, norm, beta, smooth):
    rng = np.random.default_rng(M + K + 10 * norm + 100 * beta)
    X = wl.f32_to_bf16_bits(rng.normal(0.3, 2.0, (M, K)).astype(np.float32))
    g = wl.f32_to_bf16_bits(rng.uniform(0.5, 1.5, K).astype(np.float32))
    b = wl.f32_to_bf16_bits(rng.normal(0, 0.2, K).astype(np.float32)) if beta else None
    inv_s = rng.uniform(0.2, 3.0, K).astype(np.float32) if smooth else None
    Xq, d, st = empty((M, K), torch.int8), empty(M, torch.float32), empty((M, 2), torch.float32)
    sq.sq_norm_smooth_quant(dev_bf16(X), norm, dev_bf16(g), None if b is None else dev_bf16(b), 1e-5,
                            None if inv_s is None else torch.from_numpy(inv_s).cuda(), Xq, d, st)
    sq.sq_sync_status()
    oq, od, oy, ost = oracle.norm_smooth_quant(X, norm, g, b, 1e-5, inv_s, with_stats=True)
    gst = host(st)
    # statistics: fp64 sums in another order; at most one fp32 ulp, almost always equal
    assert _ulps(gst, ost).max() <= 1
    assert (_ulps(gst, ost) != 0).sum() <= max(1, M // 100)
    # the rest, chained on the GPU's statistics: bit for bit
    cq, cd, _ = oracle.norm_smooth_quant(X, norm, g, b, 1e-5, inv_s, stats=gst)
    assert np.array_equal(host(d), cd)
    assert np.array_equal(host(Xq), cq)


@pytest.mark.parametrize("K", [4096, 8192, 16384])
@pytest.mark.parametrize("norm", [sq.SQ_NORM_LAYER, sq.SQ_NORM_RMS])
@pytest.mark.parametrize("eps", [1e-5, 0.0])
def test_norm_statistics_of_nearly_constant_rows(K, norm, eps):
    """Rows whose mean is large next to their spread, where a one-pass variance
    E[x^2] - mean^2 cancels: one repeated value, or a constant 1024 (or 3e4, or 2^100) with
    one, a few or half of the elements one bf16 step away. The statistics stay within one
    fp32 ulp of the two-pass definition (rows of one value: the variance is exactly 0, so
    rstd = 1/sqrt(eps), infinite at eps = 0 for LayerNorm), and the codes follow them."""
    rng = np.random.default_rng(K + norm)
    rows = []
    for base in (1024.0, 3.0e4, 2.0 ** 100, -7.5):
        step = float(np.spacing(np.float32(base))) * 2 ** 16  # one bf16 step at this magnitude
        for nd in (0, 1, 3, K // 2):
            x = np.full(K, base, np.float32)
            idx = rng.choice(K, nd, replace=False)
            x[idx] += rng.choice([-1.0, 1.0], nd).astype(np.float32) * np.float32(step)
            rows.append(x)
    X = wl.f32_to_bf16_bits(np.stack(rows))
    M = X.shape[0]
    g = wl.f32_to_bf16_bits(rng.uniform(0.5, 1.5, K).astype(np.float32))
    Xq, d, st = empty((M, K), torch.int8), empty(M, torch.float32), empty((M, 2), torch.float32)
    sq.sq_norm_smooth_quant(dev_bf16(X), norm, dev_bf16(g), None, eps, None, Xq, d, st)
    sq.sq_sync_status()
    _, _, _, ost = oracle.norm_smooth_quant(X, norm, g, None, eps, None, with_stats=True)
    gst = host(st)
    both_inf = np.isinf(gst) & np.isinf(ost) & (np.sign(gst) == np.sign(ost))
    assert (_ulps(gst, ost)[~both_inf] <= 1).all(), (gst, ost)
    finite = np.isfinite(gst).all(axis=1)
    cq, cd, _ = oracle.norm_smooth_quant(X, norm, g, None, eps, None, stats=gst)
    assert np.array_equal(host(d)[finite], cd[finite])
    assert np.array_equal(host(Xq)[finite], cq[finite])


# --------------------------------------------------------------------------- mu + k sigma
def test_three_sigma_example_through_llmint8():
    """从自动驾驶芯片到大语言模型INT8量化训练实战解析 §2.1 example ((2,128,4096) activations
    ~N(0,0.1) with the first 10 channels +50): the GPU mean + 3 std threshold flags exactly
    those channels, and LLM.int8 with the device threshold matches the oracle."""
    rng = np.random.default_rng(0)
    x = rng.standard_normal((256, 4096), dtype=np.float32) * np.float32(0.1)
    x[:, :10] += np.float32(50.0)
    X = wl.f32_to_bf16_bits(x)
    M, K, N = 256, 4096, 512
    W = wl.f32_to_bf16_bits(rng.normal(0, 0.02, (N, K)).astype(np.float32))
    thr, ms = empty(1, torch.float32), empty(2, torch.float64)
    X_t = dev_bf16(X)
    sq.sq_act_mean_std_threshold(X_t, 3.0, thr, ms, sq.workspace(sq.SQ_OP_MEAN_STD_THRESHOLD, M, 0, K))
    sq.sq_sync_status()
    othr, omean, osd = oracle.mean_std_threshold(X, 3.0)
    gm, gs = host(ms)
    assert abs(gm - omean) <= 1e-12 * max(1.0, abs(omean)) and abs(gs - osd) <= 1e-12 * osd
    assert _ulps(host(thr), othr).max() <= 1
    W_t = dev_bf16(W)
    Wq, e = empty((N, K), torch.int8), empty(N, torch.float32)
    sq.sq_smooth_quant_weight(W_t, None, sq.SQ_PER_CHANNEL, Wq, e)
    Y, mask, cnt = empty((M, N), torch.bfloat16), empty(K // 32, torch.int32), empty(1, torch.int32)
    acc = empty((M, N), torch.int32)
    sq.llmint8_decomposed_linear_ex(X_t, W_t, Wq, e, thr, None, Y, mask, cnt, acc,
                                    sq.workspace(sq.SQ_OP_LLMINT8, M, N, K))
    sq.sq_sync_status()
    o = oracle.llmint8_linear(X, W, None, float(host(thr)[0]))
    assert o["count"] == 10 and int(host(cnt)[0]) == 10
    assert np.array_equal(host(mask).view(np.uint32), o["mask"])
    # the int8 part bit for bit; the sum with the outlier product (fp32 on the tensor cores,
    # in an order the pages leave open) within the output tolerance of the fp64 reference
    assert np.array_equal(host(acc), o["acc"])
    assert_close_bf16(host_bits(Y), o["y_ref"], "llmint8 with mean + 3 std")


@pytest.mark.parametrize("M,K,k", [(1, 16, 6.0), (37, 528, 6.0), (4096, 8192, 6.0), (3000, 1000 * 16, 3.0)])
def test_mean_std_threshold(M, K, k):
    X = wl.llmint8_sweep(0.01, M=M, K=K, N=8).X if M * K >= 10 ** 6 else _x(M, K, M + K)
    thr, ms = empty(1, torch.float32), empty(2, torch.float64)
    sq.sq_act_mean_std_threshold(dev_bf16(X), k, thr, ms, sq.workspace(sq.SQ_OP_MEAN_STD_THRESHOLD, M, 0, K))
    sq.sq_sync_status()
    othr, omean, osd = oracle.mean_std_threshold(X, k)
    gm, gs = host(ms)
    assert abs(gm - omean) <= 1e-11 * max(1.0, abs(omean), osd)
    assert abs(gs - osd) <= 1e-11 * max(osd, 1e-300) or osd == 0.0
    assert _ulps(host(thr), othr).max() <= 1


# --------------------------------------------------------------------------- strided inputs
def test_strided_inputs_every_row_kernel():
    """Column slices of a wider matrix (leading dimension 1024 > K = 528): the row kernels
    read through ld, and every result equals the oracle's on the contiguous slice."""
    rng = np.random.default_rng(31)
    M, LD, K, off = 37, 1024, 528, 64
    full = wl.f32_to_bf16_bits(rng.normal(0.2, 1.5, (M, LD)).astype(np.float32))
    wfull = wl.f32_to_bf16_bits(rng.normal(0, 0.02, (96, LD)).astype(np.float32))
    X = dev_bf16(full)[:, off:off + K]
    W = dev_bf16(wfull)[:, off:off + K]
    Xc = np.ascontiguousarray(full[:, off:off + K])
    Wc = np.ascontiguousarray(wfull[:, off:off + K])
    inv_s = rng.uniform(0.3, 2.0, K).astype(np.float32)
    inv_t = torch.from_numpy(inv_s).cuda()
    # per-token quantization
    Xq, d = empty((M, K), torch.int8), empty(M, torch.float32)
    sq.sq_quant_act_per_token(X, inv_t, Xq, d)
    sq.sq_sync_status()
    oq, od = oracle.quant_act_per_token(Xc, inv_s)
    assert np.array_equal(host(Xq), oq) and np.array_equal(host(d), od)
    # smoothing factors and both weight granularities
    amax = torch.from_numpy(oracle.act_channel_absmax(Xc)).cuda()
    s, i = empty(K, torch.float32), empty(K, torch.float32)
    sq.sq_smooth_scale(amax, W, 0.5, s, i)
    sq.sq_sync_status()
    os_, _ = oracle.smooth_scale(host(amax), Wc, 0.5)
    assert _ulps(host(s), os_).max() <= 1
    for gran in (sq.SQ_PER_CHANNEL, sq.SQ_PER_TENSOR):
        Wq, e = empty((96, K), torch.int8), empty(96 if gran == sq.SQ_PER_CHANNEL else 1, torch.float32)
        sq.sq_smooth_quant_weight(W, s, gran, Wq, e, sq.workspace(sq.SQ_OP_SMOOTH_QUANT_WEIGHT, 0, 96, K))
        sq.sq_sync_status()
        owq, oe = oracle.smooth_quant_weight(Wc, host(s), gran)
        assert np.array_equal(host(Wq), owq) and np.array_equal(host(e), oe)
    # fused LayerNorm, asymmetric, per-tensor, mean/std
    g = wl.f32_to_bf16_bits(rng.uniform(0.5, 1.5, K).astype(np.float32))
    st = empty((M, 2), torch.float32)
    sq.sq_norm_smooth_quant(X, sq.SQ_NORM_LAYER, dev_bf16(g), None, 1e-5, inv_t, Xq, d, st)
    sq.sq_sync_status()
    cq, cd, _ = oracle.norm_smooth_quant(Xc, oracle.NORM_LAYER, g, None, 1e-5, inv_s, stats=host(st))
    assert np.array_equal(host(Xq), cq) and np.array_equal(host(d), cd)
    z = empty(M, torch.int32)
    sq.sq_quant_act_per_token_asym(X, inv_t, Xq, d, z)
    sq.sq_sync_status()
    aq, ad, az = oracle.quant_act_per_token_asym(Xc, inv_s)
    assert np.array_equal(host(Xq), aq) and np.array_equal(host(d), ad) and np.array_equal(host(z), az)
    d1 = empty(1, torch.float32)
    sq.sq_quant_act_per_tensor(X, inv_t, Xq, d1, None, sq.workspace(sq.SQ_OP_QUANT_ACT_PER_TENSOR, M, 0, K))
    sq.sq_sync_status()
    pq, pd = oracle.quant_act_per_tensor(Xc, inv_s)
    assert np.array_equal(host(Xq), pq) and np.array_equal(host(d1), pd)
    thr = empty(1, torch.float32)
    sq.sq_act_mean_std_threshold(X, 3.0, thr, None, sq.workspace(sq.SQ_OP_MEAN_STD_THRESHOLD, M, 0, K))
    sq.sq_sync_status()
    assert _ulps(host(thr), oracle.mean_std_threshold(Xc, 3.0)[0]).max() <= 1


@pytest.mark.parametrize("norm", [sq.SQ_NORM_LAYER, sq.SQ_NORM_RMS])
def test_norm_long_rows_strided(norm):
    """The pipelined row groups copy whole rows through the leading dimension: a column slice
    (K = 5008, ragged last chunks) of a matrix 8192 wide, starting 1024 columns in."""
    rng = np.random.default_rng(57 + norm)
    M, LD, K, off = 300, 8192, 5008, 1024
    full = wl.f32_to_bf16_bits(rng.normal(0.4, 1.7, (M, LD)).astype(np.float32))
    X = dev_bf16(full)[:, off:off + K]
    Xc = np.ascontiguousarray(full[:, off:off + K])
    g = wl.f32_to_bf16_bits(rng.uniform(0.5, 1.5, K).astype(np.float32))
    b = wl.f32_to_bf16_bits(rng.normal(0, 0.2, K).astype(np.float32))
    inv_s = rng.uniform(0.3, 2.0, K).astype(np.float32)
    Xq, d, st = empty((M, K), torch.int8), empty(M, torch.float32), empty((M, 2), torch.float32)
    sq.sq_norm_smooth_quant(X, norm, dev_bf16(g), dev_bf16(b), 1e-5, torch.from_numpy(inv_s).cuda(), Xq, d, st)
    sq.sq_sync_status()
    _, _, _, ost = oracle.norm_smooth_quant(Xc, norm, g, b, 1e-5, inv_s, with_stats=True)
    assert _ulps(host(st), ost).max() <= 1
    cq, cd, _ = oracle.norm_smooth_quant(Xc, norm, g, b, 1e-5, inv_s, stats=host(st))
    assert np.array_equal(host(d), cd) and np.array_equal(host(Xq), cq)
