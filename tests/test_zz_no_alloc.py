"""The allocation-free MISA-dagger rerank entry point.

misa_rerank_noalloc serves callers that cannot allocate device memory (a fixed
pool they do not own, a region where cudaMalloc is forbidden): it keeps the
candidate-score scratch in the library's own device array.  Its results must be
those of misa_rerank, which takes the same scratch as caller workspace.  The
calls run back to back with different shapes (the first fills the whole array,
the later ones use smaller, differently pitched parts of it), so each result is
checked to be independent of what the previous call left in the array.  This
file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from long_context_sparse_block_b200 import workloads as W

pytestmark = pytest.mark.gpu

NOALLOC_MAX_SCORES = 4194304     # n_q * kp limit of the library's array


def _case(lib, seed, n_q, q_pos0, n_k, H, d, kp, k, fp8=False):
    wl = W.small_workload(f"noalloc{seed}", n_q=n_q, q_pos0=q_pos0, n_k=n_k, H=H, d=d, B=64,
                          h=8, k=k, seed=seed, generator="clustered", kp=kp)
    inp = W.generate(wl, fp8_keys=fp8)
    Q = torch.from_numpy(inp["Q"].view(np.int16)).cuda()
    K = torch.from_numpy(inp["K"].view(np.int16)).cuda()
    w = torch.from_numpy(inp["w"]).cuda()
    _, hl = lib.misa_pool_keys(K, 64)
    heads, _ = lib.misa_route_heads(Q, w, hl, q_pos0, n_k, 64, 8)
    logits = lib.misa_score_tokens(Q, w, heads, K, q_pos0)
    cand = lib.misa_topk(logits, q_pos0, n_k, kp)
    if fp8:
        K8 = torch.from_numpy(inp["K8"]).cuda()
        ks = torch.from_numpy(inp["k_scale"]).cuda()
        return Q, K8, ks, w, cand
    return Q, K, None, w, cand


def _raw_call(lib, Q, K, ks, w, cand, q_pos0, k, out):
    n_q, H, d = Q.shape
    kdtype = lib.MISA_K_FP8E4M3 if ks is not None else lib.MISA_K_BF16
    return lib._lib.misa_rerank_noalloc(
        ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(w.data_ptr()),
        ctypes.c_void_p(K.data_ptr()), None if ks is None else ctypes.c_void_p(ks.data_ptr()),
        kdtype, ctypes.c_void_p(cand.data_ptr()), cand.shape[1], n_q, q_pos0, K.shape[0], H, d, k,
        ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_rerank_noalloc_matches_rerank_on_calls_in_a_row():
    from long_context_sparse_block_b200 import _lib as lib
    cases = [
        # seed, n_q, q_pos0, n_k, H, d, kp, k, fp8, through the Python wrapper
        (6, 512, 8192, 8704, 64, 128, 8192, 2048, False, False),   # exactly the array's size
        (3, 64, 900, 1000, 64, 128, 512, 128, True, True),         # FP8 keys
        (4, 40, 2000, 2100, 64, 128, 1024, 256, False, False),
    ]
    assert cases[0][1] * cases[0][6] == NOALLOC_MAX_SCORES
    for seed, n_q, q_pos0, n_k, H, d, kp, k, fp8, wrapper in cases:
        Q, K, ks, w, cand = _case(lib, seed, n_q, q_pos0, n_k, H, d, kp, k, fp8=fp8)
        ref = lib.misa_rerank(Q, w, K, cand, q_pos0, k, k_scale=ks)     # caller workspace
        if wrapper:
            out = lib.misa_rerank_noalloc(Q, w, K, cand, q_pos0, k, k_scale=ks)
        else:
            out = torch.full((n_q, k), -7, dtype=torch.int32, device="cuda")
            st = _raw_call(lib, Q, K, ks, w, cand, q_pos0, k, out)
            assert st == lib.MISA_OK, lib.misa_status_string(st)
        torch.cuda.synchronize()
        assert lib.misa_last_device_status() == lib.MISA_OK
        # integer token indices: the tolerance is exact equality
        assert torch.equal(out, ref), f"case seed={seed}"


def test_rerank_noalloc_rejects_work_beyond_its_scratch():
    # real device buffers sized for the refused call: the size check returns
    # before any launch, and if it ever did not, nothing would read past them
    from long_context_sparse_block_b200 import _lib as lib
    n_q, kp, n_k, H, d, k = 600, 8192, 1000, 64, 128, 16
    assert n_q * kp > NOALLOC_MAX_SCORES
    Q = torch.zeros((n_q, H, d), dtype=torch.int16, device="cuda")
    K = torch.zeros((n_k, d), dtype=torch.int16, device="cuda")
    w = torch.zeros((n_q, H), dtype=torch.float32, device="cuda")
    cand = torch.full((n_q, kp), -1, dtype=torch.int32, device="cuda")
    out = torch.full((n_q, k), -7, dtype=torch.int32, device="cuda")
    st = _raw_call(lib, Q, K, None, w, cand, 0, k, out)
    assert st == lib.MISA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert lib.misa_last_device_status() == lib.MISA_OK
    assert bool((out == -7).all())      # nothing was written
