"""The allocation-free matmul entry point (ccq_w2a16_gemm_noalloc).

It serves callers that cannot allocate device memory (host frameworks that hand a plugin only its
input and output pointers, or code that must not call cudaMalloc/cudaFree on its critical path):
the scratch lives in a fixed array inside the library.  This file is collected last so that a run
stopping at the first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

TOL = 1e-2


def _rel(y, ref):
    y = y.float().cpu().numpy().astype(np.float64)
    ref = ref.float().cpu().numpy().astype(np.float64)
    return float(np.max(np.abs(y - ref)) / max(np.max(np.abs(ref)), 1e-30))


@pytest.mark.parametrize("m,n,k", [(1, 8192, 8192), (16, 1024, 2048), (5, 272, 576), (64, 512, 1024)])
def test_noalloc_matches_workspace_entry_point_twice(m, n, k):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import extreme_bit_weight_b200 as ccq

    codes, scales, alpha, beta = synth.w2_format_random(n, k, 7000 + m)
    W = ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, n, k, codes, scales, alpha, beta)
    assert ccq.ccq_gemm_workspace_size(W, m) <= ccq.ccq_w2a16_gemm_noalloc_max_scratch()
    for call in range(2):  # two calls in a row: the shared array keeps the previous call's bytes
        x = synth.activations(m, k, 7100 + 10 * m + call).cuda()
        ref = ccq.ccq_w2a16_gemm(W, x)
        y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
        ccq.ccq_w2a16_gemm_noalloc(W, x, y)
        torch.cuda.synchronize()
        assert _rel(y, ref) <= TOL, call


def test_noalloc_rejects_shapes_beyond_the_array():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import extreme_bit_weight_b200 as ccq

    # 4096 tokens of K = 8192 need a 64 MiB activation operand: more than the fixed array
    W = ccq.CcqWeight(ccq.CCQ_FMT_W2_CCQ_G64, 256, 8192, np.zeros((256, 2048), np.uint8),
                      np.zeros((256, 128), np.float32), np.zeros(256, np.float32), np.zeros(256, np.float32))
    assert ccq.ccq_gemm_workspace_size(W, 4096) > ccq.ccq_w2a16_gemm_noalloc_max_scratch()
    x = torch.zeros((4096, 8192), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((4096, 256), dtype=torch.bfloat16, device="cuda")
    s = W.struct()
    st = ccq._lib.ccq_w2a16_gemm_noalloc(ctypes.byref(s), x.data_ptr(), 4096, y.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)
    assert st == ccq.CCQ_ERR_UNSUPPORTED
