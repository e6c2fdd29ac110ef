"""sq_smooth_quant_weight_noalloc: the weight quantization for callers that cannot allocate
device memory (components inside a host engine or plugin interface that owns the device
memory plan, services that fix their footprint at start-up). Its scratch lives in a static
device array inside the library; this checks through the C ABI that two calls in a row give
exactly what sq_smooth_quant_weight gives with a caller-provided workspace, and exactly the
oracle's codes and scales.

This file is collected last on purpose, and passes both alone and after the other tests."""
import ctypes as C

import numpy as np
import pytest
import torch

import oracle
from w8a8_quantized_gemm_b200 import sq
from w8a8_quantized_gemm_b200 import workloads as wl

pytestmark = pytest.mark.gpu


def _reference(W, s, gran, N, K):
    Wq = torch.empty((N, K), dtype=torch.int8, device="cuda")
    e = torch.empty(N if gran == sq.SQ_PER_CHANNEL else 1, dtype=torch.float32, device="cuda")
    sq.sq_smooth_quant_weight(W, s, gran, Wq, e, sq.workspace(sq.SQ_OP_SMOOTH_QUANT_WEIGHT, 0, N, K))
    return Wq, e


def _noalloc_raw(W, s, gran, N, K):
    """Call the entry point through the raw C ABI (plain pointers, the current stream)."""
    Wq = torch.full((N, K), 99, dtype=torch.int8, device="cuda")
    e = torch.full((N if gran == sq.SQ_PER_CHANNEL else 1,), -1.0, dtype=torch.float32, device="cuda")
    st = sq.lib().sq_smooth_quant_weight_noalloc(
        C.c_void_p(W.data_ptr()), N, K, W.stride(0), C.c_void_p(s.data_ptr()), gran, C.c_void_p(Wq.data_ptr()),
        C.c_void_p(e.data_ptr()), C.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == sq.SQ_OK, sq.sq_last_error()
    return Wq, e


@pytest.mark.parametrize("gran", [sq.SQ_PER_TENSOR, sq.SQ_PER_CHANNEL])
def test_noalloc_matches_workspace_version_two_calls(gran):
    N, K = 300, 528
    p = wl.random_problem(4, N, K, seed=21, outliers=2)
    rng = np.random.default_rng(3)
    s = torch.from_numpy(rng.uniform(0.2, 20.0, K).astype(np.float32)).cuda()
    W1 = torch.from_numpy(p.W.view(np.int16)).view(torch.bfloat16).cuda()
    # second call: a weight with a smaller absmax, so a stale maximum left in the shared
    # scratch by the first call would change the result
    W2 = (W1.float() * 0.25).to(torch.bfloat16)
    for W in (W1, W2):
        ref_q, ref_e = _reference(W, s, gran, N, K)
        got_q, got_e = _noalloc_raw(W, s, gran, N, K)
        torch.cuda.synchronize()
        sq.sq_sync_status()
        assert torch.equal(got_q, ref_q)  # integer codes: bit for bit
        assert torch.equal(got_e, ref_e)  # scales: bit for bit (same fp32 operations)
        # and against the oracle on the same bf16 weight and factors
        w_bits = W.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        o_q, o_e = oracle.smooth_quant_weight(w_bits, s.cpu().numpy(), gran)
        assert np.array_equal(got_q.cpu().numpy(), o_q)
        assert np.array_equal(got_e.cpu().numpy(), o_e)


def test_noalloc_rejects_bad_arguments_without_launch():
    st = sq.lib().sq_smooth_quant_weight_noalloc(None, 8, 64, 64, None, 0, None, None, None)
    assert st == sq.SQ_ERR_INVALID and "NULL" in sq.sq_last_error()
