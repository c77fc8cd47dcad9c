"""The allocation-free MISA-dagger rerank entry point.

misa_rerank_noalloc serves callers that cannot allocate device memory (a fixed
pool they do not own, a region where cudaMalloc is forbidden): it keeps the
candidate-score scratch in the library's own device array.  Its results must be
those of misa_rerank, which takes the same scratch as caller workspace.  Two
calls in a row check that the shared array left behind by one call does not
leak into the next.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sparse_block_b200 import workloads as W

pytestmark = pytest.mark.gpu


def _case(lib, seed, n_q, q_pos0, n_k, H, d, kp, k):
    wl = W.small_workload(f"noalloc{seed}", n_q=n_q, q_pos0=q_pos0, n_k=n_k, H=H, d=d, B=64,
                          h=8, k=k, seed=seed, generator="clustered", kp=kp)
    inp = W.generate(wl)
    Q = torch.from_numpy(inp["Q"].view(np.int16)).cuda()
    K = torch.from_numpy(inp["K"].view(np.int16)).cuda()
    w = torch.from_numpy(inp["w"]).cuda()
    _, hl = lib.misa_pool_keys(K, 64)
    heads, _ = lib.misa_route_heads(Q, w, hl, q_pos0, n_k, 64, 8)
    logits = lib.misa_score_tokens(Q, w, heads, K, q_pos0)
    cand = lib.misa_topk(logits, q_pos0, n_k, kp)
    return Q, K, w, cand


def test_rerank_noalloc_matches_rerank_on_two_calls_in_a_row():
    from long_context_sparse_block_b200 import _lib as lib
    so = lib._lib
    cases = [(3, 64, 900, 1000, 64, 128, 512, 128), (4, 40, 2000, 2100, 64, 128, 1024, 256)]
    for seed, n_q, q_pos0, n_k, H, d, kp, k in cases:
        Q, K, w, cand = _case(lib, seed, n_q, q_pos0, n_k, H, d, kp, k)
        ref = lib.misa_rerank(Q, w, K, cand, q_pos0, k)            # caller workspace
        out = torch.full((n_q, k), -7, dtype=torch.int32, device="cuda")
        st = so.misa_rerank_noalloc(
            ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(w.data_ptr()),
            ctypes.c_void_p(K.data_ptr()), None, lib.MISA_K_BF16,
            ctypes.c_void_p(cand.data_ptr()), kp, n_q, q_pos0, n_k, H, d, k,
            ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == lib.MISA_OK, lib.misa_status_string(st)
        torch.cuda.synchronize()
        assert lib.misa_last_device_status() == lib.MISA_OK
        # integer token indices: the tolerance is exact equality
        assert torch.equal(out, ref)


def test_rerank_noalloc_rejects_work_beyond_its_scratch():
    from long_context_sparse_block_b200 import _lib as lib
    so = lib._lib
    p = ctypes.c_void_p(16 * 1024)          # validation runs before any launch
    # 600 queries x 8192 candidates = 4915200 scores > 4194304
    st = so.misa_rerank_noalloc(p, p, p, None, 0, p, 8192, 600, 0, 1000, 64, 128, 16, p, None)
    assert st == lib.MISA_ERR_WORKSPACE
