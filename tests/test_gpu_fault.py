"""Failure path without a GPU fault: a TMA stage is withheld on purpose (test hook), the
consumer's bounded wait gives up, the kernel drains and returns, the host reads
SQ_ERR_TIMEOUT, and the next call on the same context is correct."""
import numpy as np
import pytest
import torch

import oracle
from w8a8_quantized_gemm_b200 import sq

from _gpu import empty, host

pytestmark = pytest.mark.gpu


# one CTA per tile, and CTA pairs on 256 x 256 tiles (the abort reaches the other CTA too)
@pytest.mark.parametrize("M,N,K", [(256, 512, 1024), (2433, 1800, 272)])
def test_withheld_stage_times_out_and_context_survives(M, N, K):
    rng = np.random.default_rng(0)
    xq = rng.integers(-127, 128, size=(M, K), dtype=np.int8)
    wq = rng.integers(-127, 128, size=(N, K), dtype=np.int8)
    d = np.full(M, 1e-2, np.float32)
    e = np.full(N, 1e-3, np.float32)
    args = [torch.from_numpy(a).cuda() for a in (xq, wq, d, e)]
    Y = empty((M, N), torch.bfloat16)
    acc = empty((M, N), torch.int32)
    sq.sq_sync_status()  # clean slate
    sq.sq_debug_arm_fault(1, 50_000_000)  # 50 ms per wait
    sq.sq_int8_gemm_dequant(*args, sq.SQ_PER_CHANNEL, None, Y, acc, sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K))
    with pytest.raises(sq.SqError) as ei:
        sq.sq_sync_status()
    assert ei.value.status == sq.SQ_ERR_TIMEOUT
    # the status word was cleared and the context still works (with a fresh zeroed workspace:
    # an aborted call may leave split-K arrival counters behind)
    sq.sq_int8_gemm_dequant(*args, sq.SQ_PER_CHANNEL, None, Y, acc, sq.workspace(sq.SQ_OP_INT8_GEMM_DEQUANT, M, N, K))
    sq.sq_sync_status()
    assert np.array_equal(host(acc), oracle.int8_gemm(xq, wq))
