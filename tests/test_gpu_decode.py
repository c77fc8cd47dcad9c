"""Decode-shaped use of the indexer on a growing key cache: the pooled keys are
updated incrementally (only the block a new key lands in, or every block when a
new block starts) and must equal a full pooling bit for bit; one decode query
at the newest position is then routed, scored and selected and checked against
the oracle."""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_block_b200 import workloads as W
from tests.gpu_helpers import check_heads, dev, inputs_to_device, recall

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_block_b200 import _lib
    return _lib


@pytest.mark.parametrize("fp8", [False, True])
def test_incremental_pooling_equals_full(lib, fp8):
    n_max, d, B, n0 = 1400, 128, 128, 1000
    wl = W.small_workload("dec", n_q=1, q_pos0=n_max - 1, n_k=n_max, H=8, d=d, B=B, h=2, k=16,
                          seed=41, generator="clustered")
    inp = W.generate(wl, fp8_keys=fp8)
    g = inputs_to_device(inp, fp8=fp8)
    K = g["K8"] if fp8 else g["K"]
    ks = g.get("k_scale")
    m_cap = -(-n_max // B)
    kbar = torch.zeros((m_cap, d), dtype=torch.float32, device="cuda")
    hl_buf = torch.zeros(2 * m_cap * d, dtype=torch.int16, device="cuda")
    M = -(-n0 // B)
    lib.misa_pool_keys_range(K, B, 0, M, kbar=kbar, kbar_hl=hl_buf[:2 * M * d].view(2, M, d),
                             k_scale=ks, n_k=n0)
    for n_k in range(n0 + 1, n_max + 1):
        M_new = -(-n_k // B)
        hl = hl_buf[:2 * M_new * d].view(2, M_new, d)
        if M_new != M:   # a new block: the lo plane moves, pool every block
            lib.misa_pool_keys_range(K, B, 0, M_new, kbar=kbar, kbar_hl=hl, k_scale=ks, n_k=n_k)
        else:            # the new key only changes the last block
            lib.misa_pool_keys_range(K, B, M_new - 1, M_new, kbar=kbar, kbar_hl=hl, k_scale=ks,
                                     n_k=n_k)
        M = M_new
        if n_k % 37 == 0 or n_k == n_max:
            ref_kbar, ref_hl = lib.misa_pool_keys(K[:n_k], B, k_scale=None if ks is None else ks[:n_k])
            assert torch.equal(kbar[:M], ref_kbar)
            assert torch.equal(hl, ref_hl)


def test_decode_step_matches_oracle(lib):
    # one new query at the end of a 20000-key cache: pool the last block, route,
    # score, select (the unfused sequence: four launches)
    n_k, H, d, B, h, k = 20000, 64, 128, 128, 8, 256
    wl = W.small_workload("dec1", n_q=1, q_pos0=n_k - 1, n_k=n_k, H=H, d=d, B=B, h=h, k=k,
                          seed=42, generator="clustered")
    inp = W.generate(wl)
    Qd, Kd, wd = oracle.decode_inputs(inp)
    g = inputs_to_device(inp)
    M = -(-n_k // B)
    kbar, hl = lib.misa_pool_keys(g["K"][:n_k - 1], B)          # the cache before the new key
    hl_new = torch.empty((2, M, d), dtype=torch.int16, device="cuda")
    kbar_new = torch.empty((M, d), dtype=torch.float32, device="cuda")
    if M == hl.shape[1]:
        hl_new.copy_(hl)
        kbar_new.copy_(kbar)
        lib.misa_pool_keys_range(g["K"], B, M - 1, M, kbar=kbar_new, kbar_hl=hl_new)
    else:
        lib.misa_pool_keys_range(g["K"], B, 0, M, kbar=kbar_new, kbar_hl=hl_new)
    heads, r = lib.misa_route_heads(g["Q"], g["w"], hl_new, n_k - 1, n_k, B, h, want_r=True)
    logits = lib.misa_score_tokens(g["Q"], g["w"], heads, g["K"], n_k - 1)
    idx = lib.misa_topk(logits, n_k - 1, n_k, k).cpu().numpy()
    kb = oracle.pool_keys(Kd, B)
    r_o, h_o = oracle.route(Qd, wd, kb, n_k - 1, n_k, B, h)
    check_heads(heads.cpu().numpy(), r_o, h_o, h, r_gpu=r.cpu().numpy())
    lg = logits.cpu().numpy()
    assert np.array_equal(idx, oracle.topk(lg, n_k - 1, n_k, k))
    if np.array_equal(heads.cpu().numpy(), h_o):
        ref = oracle.score(Qd, wd, h_o, Kd, n_k - 1)
        assert recall(idx, oracle.topk(ref, n_k - 1, n_k, k)) >= 0.999
