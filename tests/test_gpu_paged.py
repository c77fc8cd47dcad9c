"""The indexer over a paged key cache (the integration boundary: vLLM keeps the
index keys in pages and the integration issue times the indexer with that cache
handling included).

A paged cache is built from seeded contiguous keys: each logical block of
page_size keys goes to a random page of a larger pool, and every pool row that
holds no key of the sequence (unused pages, the tail of the last page) is
filled with +inf (bf16) or NaN (e4m3) codes, so a read through a wrong table
entry shows up in the results.  Every paged entry point must equal its
contiguous counterpart on the keys gathered in logical order bit for bit, and
the oracle on those gathered keys within the usual tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_block_b200 import workloads as W
from tests.gpu_helpers import assert_logits_close, dev, inputs_to_device, logit_magnitude, recall

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_block_b200 import _lib
    return _lib


def make_paged(lib, K, ps, seed, k_scale=None, spare=3):
    """Spread the rows of K ([n_k, d] device codes) over pages of `ps` rows in a
    pool with `spare` extra pages; returns the PagedKeys cache."""
    n_k, d = K.shape
    n_blocks = -(-n_k // ps)
    n_pages = n_blocks + spare
    rng = np.random.default_rng(seed)
    table = rng.permutation(n_pages)[:n_blocks].astype(np.int32)
    fp8 = K.dtype == torch.uint8
    fill = 0x7F if fp8 else 0x7F80                         # e4m3 NaN / bf16 +inf
    pages = torch.full((n_pages, ps, d), fill, dtype=K.dtype, device=K.device)
    flat = torch.zeros((n_blocks * ps, d), dtype=K.dtype, device=K.device)
    flat[:n_k] = K
    bt = torch.from_numpy(table).to(K.device)
    pages[bt.long()] = flat.view(n_blocks, ps, d)
    tail = n_blocks * ps - n_k
    if tail:
        pages[int(table[-1]), ps - tail:] = fill
    scale = None
    if k_scale is not None:
        scale = torch.full((n_pages, ps), float("nan"), dtype=torch.float32, device=K.device)
        sflat = torch.zeros(n_blocks * ps, dtype=torch.float32, device=K.device)
        sflat[:n_k] = k_scale
        scale[bt.long()] = sflat.view(n_blocks, ps)
    return lib.PagedKeys(pages, bt, n_k, k_scale=scale)


def _setup(lib, n_q, q_pos0, n_k, H, d, B, h, k, seed, fp8=False, kp=0):
    wl = W.small_workload(f"paged{seed}", n_q=n_q, q_pos0=q_pos0, n_k=n_k, H=H, d=d, B=B, h=h,
                          k=k, seed=seed, generator="clustered", kp=kp)
    inp = W.generate(wl, fp8_keys=fp8)
    g = inputs_to_device(inp, fp8=fp8)
    return wl, inp, g


@pytest.mark.parametrize("ps,fp8", [(16, False), (32, False), (64, False), (128, False),
                                    (64, True), (16, True)])
def test_paged_pool_route_score_equal_contiguous(lib, ps, fp8):
    n_q, q_pos0, n_k, H, d, B, h = 150, 900, 1100, 64, 128, 64, 8   # n_k not a multiple of ps
    wl, inp, g = _setup(lib, n_q, q_pos0, n_k, H, d, B, h, 64, seed=ps + fp8, fp8=fp8)
    K = g["K8"] if fp8 else g["K"]
    ks = g.get("k_scale")
    pk = make_paged(lib, K, ps, seed=ps, k_scale=ks)
    kb, hl = lib.misa_pool_keys(K, B, k_scale=ks)
    kb_p, hl_p = lib.misa_pool_keys(pk, B)
    assert torch.equal(kb, kb_p) and torch.equal(hl, hl_p)
    heads, _ = lib.misa_route_heads(g["Q"], g["w"], hl_p, q_pos0, n_k, B, h)
    lg = lib.misa_score_tokens(g["Q"], g["w"], heads, K, q_pos0, k_scale=ks)
    lg_p = lib.misa_score_tokens(g["Q"], g["w"], heads, pk, q_pos0)
    assert lib.misa_last_device_status() == lib.MISA_OK
    causal = np.arange(n_k)[None, :] <= (q_pos0 + np.arange(n_q))[:, None]
    a, b = lg.cpu().numpy(), lg_p.cpu().numpy()
    assert np.array_equal(a[causal], b[causal])
    # and the oracle on the keys in logical order
    Qd, Kd, wd = oracle.decode_inputs(inp, fp8_keys=fp8)
    hs = heads.cpu().numpy()
    ref = oracle.score(Qd, wd, hs, Kd, q_pos0)
    for t in range(0, n_q, 7):
        mag = logit_magnitude(Qd, wd, Kd, hs, t, q_pos0)
        assert_logits_close(b[t], ref[t, :q_pos0 + t + 1], mag, what=f"paged row {t}")


@pytest.mark.parametrize("ps,fp8,k", [(64, False, 512), (128, False, 2048), (16, False, 300),
                                      (64, True, 1024)])
def test_paged_score_topk_equals_contiguous(lib, ps, fp8, k):
    # the fused path (sampled thresholds, select pass, finish) through pages
    n_q, q_pos0, n_k, H, d, B, h = 200, 12000, 14000, 64, 128, 128, 8
    wl, inp, g = _setup(lib, n_q, q_pos0, n_k, H, d, B, h, k, seed=100 + ps, fp8=fp8)
    K = g["K8"] if fp8 else g["K"]
    ks = g.get("k_scale")
    pk = make_paged(lib, K, ps, seed=7 * ps, k_scale=ks)
    _, hl = lib.misa_pool_keys(pk, B)
    heads, _ = lib.misa_route_heads(g["Q"], g["w"], hl, q_pos0, n_k, B, h)
    want = lib.misa_score_topk(g["Q"], g["w"], heads, K, q_pos0, k, k_scale=ks)
    got = lib.misa_score_topk(g["Q"], g["w"], heads, pk, q_pos0, k)
    assert lib.misa_last_device_status() == lib.MISA_OK
    assert torch.equal(got, want)
    # the unfused sequence through pages, and the oracle's selection of its logits
    lg = lib.misa_score_tokens(g["Q"], g["w"], heads, pk, q_pos0)
    unf = lib.misa_topk(lg, q_pos0, n_k, k)
    assert torch.equal(unf, got)
    lg_np = lg.cpu().numpy()
    got = got.cpu().numpy()
    for t in (0, n_q // 2, n_q - 1):
        assert np.array_equal(got[t], oracle.topk(lg_np[t:t + 1], q_pos0 + t, n_k, k)[0])


@pytest.mark.parametrize("ps,fp8", [(64, False), (32, True)])
def test_paged_rerank_equals_contiguous(lib, ps, fp8):
    n_q, q_pos0, n_k, H, d, B, h, kp, k = 40, 500, 600, 64, 128, 64, 4, 256, 64
    wl, inp, g = _setup(lib, n_q, q_pos0, n_k, H, d, B, h, k, seed=200 + ps, fp8=fp8, kp=kp)
    K = g["K8"] if fp8 else g["K"]
    ks = g.get("k_scale")
    pk = make_paged(lib, K, ps, seed=ps + 1, k_scale=ks)
    _, hl = lib.misa_pool_keys(pk, B)
    heads, _ = lib.misa_route_heads(g["Q"], g["w"], hl, q_pos0, n_k, B, h)
    logits = lib.misa_score_tokens(g["Q"], g["w"], heads, pk, q_pos0)
    cand = lib.misa_topk(logits, q_pos0, n_k, kp)
    idx, full = lib.misa_rerank(g["Q"], g["w"], K, cand, q_pos0, k, k_scale=ks, want_full=True)
    idx_p, full_p = lib.misa_rerank(g["Q"], g["w"], pk, cand, q_pos0, k, want_full=True)
    assert lib.misa_last_device_status() == lib.MISA_OK
    assert torch.equal(idx, idx_p) and torch.equal(full, full_p)
    Qd, Kd, wd = oracle.decode_inputs(inp, fp8_keys=fp8)
    c = cand.cpu().numpy()
    ref_idx = oracle.rerank(Qd, wd, Kd, c, q_pos0, k)
    fp = full_p.cpu().numpy()
    assert np.array_equal(idx_p.cpu().numpy(), oracle.select_candidates(fp, c, q_pos0, n_k, k))
    assert recall(idx_p.cpu().numpy(), ref_idx) >= 0.999


def test_paged_bad_table_entry_is_reported(lib):
    # a page id outside the pool: reported as a contract violation and read as
    # page 0 (no access leaves the pool)
    n_q, q_pos0, n_k, H, d, B, h = 20, 300, 400, 16, 64, 64, 4
    wl, inp, g = _setup(lib, n_q, q_pos0, n_k, H, d, B, h, 16, seed=301)
    pk = make_paged(lib, g["K"], 64, seed=302)
    bad = pk.block_table.clone()
    bad[2] = pk.n_pages + 5
    pkb = lib.PagedKeys(pk.pages, bad, n_k)
    lib.misa_pool_keys(pkb, B)
    assert lib.misa_last_device_status() == lib.MISA_ERR_DEVICE
    heads = torch.zeros((n_q, h), dtype=torch.int32, device="cuda") + torch.arange(h, device="cuda",
                                                                                   dtype=torch.int32)
    lib.misa_score_tokens(g["Q"], g["w"], heads, pkb, q_pos0)
    assert lib.misa_last_device_status() == lib.MISA_ERR_DEVICE
    lib.misa_score_tokens(g["Q"], g["w"], heads, pk, q_pos0)
    assert lib.misa_last_device_status() == lib.MISA_OK


def test_paged_decode_step_matches_oracle(lib):
    # one new query at the end of a paged 20000-key cache: re-pool its block,
    # route, score and select through the pages
    n_k, H, d, B, h, k, ps = 20000, 64, 128, 128, 8, 256, 64
    wl, inp, g = _setup(lib, 1, n_k - 1, n_k, H, d, B, h, k, seed=303)
    pk = make_paged(lib, g["K"], ps, seed=304)
    Qd, Kd, wd = oracle.decode_inputs(inp)
    M = -(-n_k // B)
    kbar = torch.empty((M, d), dtype=torch.float32, device="cuda")
    hl = torch.empty((2, M, d), dtype=torch.int16, device="cuda")
    lib.misa_pool_keys_range(pk, B, 0, M, kbar=kbar, kbar_hl=hl)
    heads, _ = lib.misa_route_heads(g["Q"], g["w"], hl, n_k - 1, n_k, B, h)
    logits = lib.misa_score_tokens(g["Q"], g["w"], heads, pk, n_k - 1)
    idx = lib.misa_topk(logits, n_k - 1, n_k, k).cpu().numpy()
    assert lib.misa_last_device_status() == lib.MISA_OK
    lg = logits.cpu().numpy()
    assert np.array_equal(idx, oracle.topk(lg, n_k - 1, n_k, k))
    hs = heads.cpu().numpy()
    ref = oracle.score(Qd, wd, hs, Kd, n_k - 1)
    mag = logit_magnitude(Qd, wd, Kd, hs, 0, n_k - 1)
    assert_logits_close(lg[0], ref[0], mag, what="paged decode")
    assert recall(idx, oracle.topk(ref, n_k - 1, n_k, k)) >= 0.999
