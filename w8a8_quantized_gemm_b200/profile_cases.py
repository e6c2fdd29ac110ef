"""Small, self-contained launches of single kernels for profiler captures (ncu).

Usage: python -m w8a8_quantized_gemm_b200.profile_cases
       {gemm,decode,decode1,llm,quant,absmax,smooth,wquant,norm,asym,meanstd,percentile,rowsums,gemm_asym}

Each case makes random device inputs of one workload's shape and calls one entry point three
times (so that a capture can skip the first, cold launch):
  gemm    sq_int8_gemm_dequant, 2048 x 11008 x 4096 (Llama-2-7B MLP up-projection; CTA pairs)
  decode  sq_int8_gemm_dequant, 64 x 4096 x 4096 (decode: swapped operands, split K)
  decode1 sq_int8_gemm_dequant, 1 x 4096 x 4096 (one token: the CUDA-core product)
  llm     llmint8_decomposed_linear, 2048 x 11008 x 4096 with 4 outlier columns (CTA pairs)
  quant   sq_quant_act_per_token with smoothing, X bf16 [8192, 8192] (inputs larger than L2)
  absmax  sq_act_channel_absmax, X bf16 [8192, 8192]
  smooth  sq_smooth_scale (column maxima of W and the factors in one pass), W bf16 [28672, 8192]
  wquant  sq_smooth_quant_weight, smoothed, per channel, W bf16 [28672, 8192]
  norm    sq_norm_smooth_quant (LayerNorm with beta, smoothing), X bf16 [8192, 8192]
  asym    sq_quant_act_per_token_asym with smoothing, X bf16 [8192, 8192]
  meanstd sq_act_mean_std_threshold (k = 6), X bf16 [8192, 8192]
  percentile  sq_act_abs_percentile (99.99), X bf16 [8192, 8192]
  rowsums sq_weight_row_sums, Wq int8 [28672, 8192]
  gemm_asym  sq_int8_gemm_dequant_ex with asymmetric activations, 2048 x 11008 x 4096
"""
import sys

import torch

from w8a8_quantized_gemm_b200 import sq


def main(mode: str) -> None:
    torch.cuda.set_device(0)
    dev = "cuda"
    torch.manual_seed(0)
    if mode in ("gemm", "decode", "decode1"):
        M, N, K = {"gemm": (2048, 11008, 4096), "decode": (64, 4096, 4096), "decode1": (1, 4096, 4096)}[mode]
        Xq = torch.randint(-127, 128, (M, K), dtype=torch.int8, device=dev)
        Wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev)
        d = torch.rand(M, device=dev) * 1e-2
        e = torch.rand(N, device=dev) * 1e-3
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K)
        for _ in range(3):
            sq.sq_int8_gemm_dequant(Xq, Wq, d, e, sq.SQ_PER_CHANNEL, None, Y, None, ws)
    elif mode == "llm":
        M, N, K = 2048, 11008, 4096
        X = torch.randn(M, K, device=dev)
        X[:, :4] += 50
        X = X.to(torch.bfloat16)
        W = (torch.randn(N, K, device=dev) * 0.02).to(torch.bfloat16)
        Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        e = torch.empty(N, device=dev)
        sq.sq_smooth_quant_weight(W, None, sq.SQ_PER_CHANNEL, Wq, e)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = sq.workspace(sq.SQ_OP_LLMINT8, M, N, K)
        for _ in range(3):
            sq.llmint8_decomposed_linear(X, W, Wq, e, 6.0, None, Y, None, None, None, ws)
    elif mode in ("quant", "absmax"):
        M, K = 8192, 8192
        X = torch.randn(M, K, device=dev).to(torch.bfloat16)
        if mode == "quant":
            Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
            dd = torch.empty(M, device=dev)
            inv = torch.rand(K, device=dev) + 0.5
            for _ in range(3):
                sq.sq_quant_act_per_token(X, inv, Xq, dd)
        else:
            amax = torch.empty(K, device=dev)
            for _ in range(3):
                sq.sq_act_channel_absmax(X, amax)
    elif mode in ("norm", "asym", "meanstd", "percentile"):
        M, K = 8192, 8192
        X = (torch.randn(M, K, device=dev) * 1.5 + 0.2).to(torch.bfloat16)
        Xq = torch.empty((M, K), dtype=torch.int8, device=dev)
        dd = torch.empty(M, device=dev)
        inv = torch.rand(K, device=dev) + 0.5
        for _ in range(3):
            if mode == "norm":
                g = (torch.rand(K, device=dev) + 0.5).to(torch.bfloat16)
                b = (torch.randn(K, device=dev) * 0.1).to(torch.bfloat16)
                sq.sq_norm_smooth_quant(X, sq.SQ_NORM_LAYER, g, b, 1e-5, inv, Xq, dd)
            elif mode == "asym":
                z = torch.empty(M, dtype=torch.int32, device=dev)
                sq.sq_quant_act_per_token_asym(X, inv, Xq, dd, z)
            elif mode == "meanstd":
                thr = torch.empty(1, device=dev)
                sq.sq_act_mean_std_threshold(X, 6.0, thr, None, sq.workspace(sq.SQ_OP_MEAN_STD_THRESHOLD, M, 0, K))
            else:
                out = torch.empty(1, device=dev)
                sq.sq_act_abs_percentile(X, 99.99, out, sq.workspace(sq.SQ_OP_ABS_PERCENTILE, M, 0, K))
    elif mode in ("smooth", "wquant"):
        # the 70B-shaped weight W [28672, 8192] (470 MB): the smoothing factors (column maxima of
        # W in the same pass) or the smoothed per-channel weight quantization (470 -> 235 MB)
        N, K = 28672, 8192
        W = (torch.randn(N, K, device=dev) * 0.01).to(torch.bfloat16)
        amax = torch.rand(K, device=dev) * 10.0
        s = torch.empty(K, device=dev)
        inv = torch.empty(K, device=dev)
        sq.sq_smooth_scale(amax, W, 0.5, s, inv)
        Wq = torch.empty((N, K), dtype=torch.int8, device=dev)
        e = torch.empty(N, device=dev)
        for _ in range(3):
            if mode == "smooth":
                sq.sq_smooth_scale(amax, W, 0.5, s, inv)
            else:
                sq.sq_smooth_quant_weight(W, s, sq.SQ_PER_CHANNEL, Wq, e)
    elif mode == "rowsums":
        Wq = torch.randint(-127, 128, (28672, 8192), dtype=torch.int8, device=dev)
        rs = torch.empty(28672, dtype=torch.int32, device=dev)
        for _ in range(3):
            sq.sq_weight_row_sums(Wq, rs)
    elif mode == "gemm_asym":
        M, N, K = 2048, 11008, 4096
        Xq = torch.randint(-128, 128, (M, K), dtype=torch.int8, device=dev)
        Wq = torch.randint(-127, 128, (N, K), dtype=torch.int8, device=dev)
        d = torch.rand(M, device=dev) * 1e-2
        e = torch.rand(N, device=dev) * 1e-3
        z = torch.randint(-128, 128, (M,), dtype=torch.int32, device=dev)
        rs = torch.empty(N, dtype=torch.int32, device=dev)
        sq.sq_weight_row_sums(Wq, rs)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            sq.sq_int8_gemm_dequant_ex(Xq, Wq, d, sq.SQ_PER_CHANNEL, z, e, sq.SQ_PER_CHANNEL, rs, None, Y)
    else:
        raise SystemExit(f"unknown case {mode!r}")
    sq.sq_sync_status()
    torch.cuda.synchronize()
    print("ok", mode)


if __name__ == "__main__":
    main(sys.argv[1] if len(sys.argv) > 1 else "gemm")
