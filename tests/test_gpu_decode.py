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


# ------------------------------------------------------------------ batched decode

def _decode_batch(lens, H, d, B, h, k, ps, seed, fp8=False):
    """One new query per sequence at the end of its own keys; all keys in one
    page pool (pages of ps keys in a seeded random order, unused rows +inf, or
    NaN codes and scales for e4m3 pages).  Returns (seqs, Q, w, pages, bts,
    scales)."""
    seqs = []
    for b, n in enumerate(lens):
        wl = W.small_workload(f"dec{seed}_{b}", n_q=1, q_pos0=n - 1, n_k=n, H=H, d=d, B=B, h=h,
                              k=k, seed=seed + b, generator="clustered")
        seqs.append(W.generate(wl, fp8_keys=fp8))
    nb = [-(-n // ps) for n in lens]
    max_blocks = max(nb)
    table, n_pages = W.page_table(sum(nb) * ps, ps, seed=seed)
    code, fill = (np.uint8, 0x7F) if fp8 else (np.uint16, 0x7F80)
    pages = np.full((n_pages, ps, d), fill, dtype=code)
    scales = np.full((n_pages, ps), np.nan, dtype=np.float32) if fp8 else None
    bts = np.full((len(lens), max_blocks), -1, dtype=np.int32)
    o = 0
    for b, n in enumerate(lens):
        flat = np.full((nb[b] * ps, d), fill, dtype=code)
        flat[:n] = seqs[b]["K8" if fp8 else "K"]
        bts[b, :nb[b]] = table[o:o + nb[b]]
        pages[table[o:o + nb[b]]] = flat.reshape(nb[b], ps, d)
        if fp8:
            sflat = np.full(nb[b] * ps, np.nan, dtype=np.float32)
            sflat[:n] = seqs[b]["k_scale"]
            scales[table[o:o + nb[b]]] = sflat.reshape(nb[b], ps)
        o += nb[b]
    Q = np.concatenate([s["Q"] for s in seqs])
    w = np.concatenate([s["w"] for s in seqs])
    return seqs, Q, w, pages, bts, scales


@pytest.mark.parametrize("H,d,h,ps,fp8", [(64, 128, 8, 64, False), (64, 128, 64, 32, False),
                                          (32, 64, 4, 128, False), (64, 128, 8, 64, True),
                                          (16, 32, 16, 16, True)])
def test_batched_decode_matches_oracle(lib, H, d, h, ps, fp8):
    lens = [1, 100, 128, 3000, 7777, 20000]
    B, k = 128, 256
    seqs, Qn, wn, pages_n, bts_n, sc_n = _decode_batch(lens, H, d, B, h, k, ps, seed=500 + h,
                                                       fp8=fp8)
    Q, w, pages, bts = dev(Qn), dev(wn), dev(pages_n), dev(bts_n)
    ks = dev(sc_n) if fp8 else None
    seq_lens = dev(np.array(lens, dtype=np.int32))
    M_max = -(-bts_n.shape[1] * ps // B)
    _, hl = lib.misa_decode_pool_keys(pages, bts, seq_lens, B, M_max, M_max, k_scale=ks)
    dense = h == H
    heads, r = lib.misa_decode_route_heads(Q, w, hl, seq_lens, B, h, want_r=True)
    idx, logits = lib.misa_decode_score_topk(Q, w, None if dense else heads, pages, bts, seq_lens,
                                             k, h=h, k_scale=ks)
    assert lib.misa_last_device_status() == lib.MISA_OK
    hl_np, heads_np, r_np = hl.cpu().numpy(), heads.cpu().numpy(), r.cpu().numpy()
    idx_np, lg_np = idx.cpu().numpy(), logits.cpu().numpy()
    for b, n in enumerate(lens):
        g = inputs_to_device(seqs[b], fp8=fp8)
        Kb, ksb = (g["K8"], g["k_scale"]) if fp8 else (g["K"], None)
        M = -(-n // B)
        # pooling and routing equal the single-sequence calls bit for bit
        _, hl1 = lib.misa_pool_keys(Kb, B, k_scale=ksb)
        hl1 = hl1.cpu().numpy()
        assert np.array_equal(hl_np[b, 0, :M], hl1[0]) and np.array_equal(hl_np[b, 1, :M], hl1[1])
        heads1, r1 = lib.misa_route_heads(g["Q"], g["w"], dev(hl1.view(np.int16)), n - 1, n, B, h,
                                          want_r=True)
        assert np.array_equal(r_np[b], r1.cpu().numpy()[0])
        assert np.array_equal(heads_np[b], heads1.cpu().numpy()[0])
        # against the oracle
        Qd, Kd, wd = oracle.decode_inputs(seqs[b], fp8_keys=fp8)
        kb = oracle.pool_keys(Kd, B)
        r_o, h_o = oracle.route(Qd, wd, kb, n - 1, n, B, h)
        check_heads(heads_np[b:b + 1], r_o, h_o, h, r_gpu=r_np[b:b + 1])
        hs = heads_np[b:b + 1] if not dense else np.arange(H, dtype=np.int32)[None, :]
        ref = oracle.score(Qd, wd, hs, Kd, n - 1)[0]
        mag = (np.abs(wd[0, hs[0]])[:, None] * np.maximum(Qd[0, hs[0]] @ Kd.T, 0)).sum(0)
        row = lg_np[b, :n]
        assert np.all(np.abs(row.astype(np.float64) - ref) <= 2e-3 * mag + 1e-5), f"seq {b}"
        assert np.array_equal(idx_np[b], oracle.topk(row[None, :], n - 1, n, k)[0])
        assert recall(idx_np[b:b + 1], oracle.topk(ref[None, :], n - 1, n, k)) >= 0.999
        # and the prefill scoring kernel on the same query gives the same logits
        lg1 = lib.misa_score_tokens(g["Q"], g["w"], None if dense else dev(heads_np[b:b + 1]),
                                    Kb, n - 1, k_scale=ksb, h=h).cpu().numpy()[0, :n]
        assert np.array_equal(lg1, row), f"seq {b}: decode and prefill logits differ"


def test_batched_decode_appends_keys_incrementally(lib):
    # keys appended one at a time to three sequences: re-pooling only each
    # sequence's last block keeps the pooled keys equal to pooling from scratch
    H, d, B, h, k, ps = 16, 64, 32, 4, 32, 16
    lens0 = [31, 64, 200]
    steps = 40
    full = [n + steps for n in lens0]
    seqs, Qn, wn, pages_n, bts_n, _ = _decode_batch(full, H, d, B, h, k, ps, seed=600)
    pages, bts = dev(pages_n), dev(bts_n)
    M_max = -(-bts_n.shape[1] * ps // B)
    lens = np.array(lens0, dtype=np.int32)
    _, hl = lib.misa_decode_pool_keys(pages, bts, dev(lens), B, M_max, M_max)
    for i in range(steps):
        lens = lens + 1
        lib.misa_decode_pool_keys(pages, bts, dev(lens), B, M_max, 1, kbar_hl=hl)
    _, ref = lib.misa_decode_pool_keys(pages, bts, dev(lens), B, M_max, M_max)
    assert lib.misa_last_device_status() == lib.MISA_OK
    for b, n in enumerate(lens.tolist()):
        M = -(-n // B)
        assert torch.equal(hl[b, :, :M], ref[b, :, :M])
