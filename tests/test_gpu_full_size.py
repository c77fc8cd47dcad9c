"""GPU parity at the workloads' full sizes: sampled query rows that the oracle
computes one by one (the first and last query, the query whose head-0 row was
planted as needle keys, and seeded random rows) on the unfused sequence, and
every row of the fused scoring + top-k — the benchmark's launch configuration —
bit-exact against that sequence."""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_block_b200 import workloads as W
from tests.gpu_helpers import assert_logits_close, check_heads, inputs_to_device, recall

pytestmark = pytest.mark.gpu

N_RANDOM = 12


def _rows(wl):
    rng = np.random.default_rng(77)
    rows = {0, wl.n_q - 1, wl.n_q // 2} | set(rng.choice(wl.n_q, N_RANDOM, replace=False).tolist())
    return sorted(rows)


@pytest.mark.parametrize("name", ["chunk_128k", "chunk_128k_h4", "dsv32_32k", "glm5_64k"])
def test_full_size_sampled_rows(name):
    from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer
    wl = W.WORKLOADS[name]
    inp = W.generate(wl)
    rows = _rows(wl)
    g = inputs_to_device(inp)
    ix = MisaIndexer(IndexerShape(wl.n_q, wl.q_pos0, wl.n_k, wl.H, wl.d, wl.B, wl.h, wl.k,
                                  sub_chunk=1024))
    dumps = {}

    def grab(c0, c1, lg):
        for t in rows:
            if c0 <= t < c1:
                dumps[t] = lg[t - c0].cpu().numpy()

    idx = ix.run(g["Q"], g["K"], g["w"], on_subchunk=grab).cpu().numpy()
    heads = ix.heads.cpu().numpy()
    from long_context_sparse_block_b200 import _lib
    assert _lib.misa_last_device_status() == 0
    Kd = oracle.bf16_to_f64(inp["K"])
    kbar = oracle.pool_keys(Kd, wl.B)
    sel = np.array(rows)
    Qd = oracle.bf16_to_f64(inp["Q"][sel])
    wd = inp["w"][sel].astype(np.float64)
    matched = 0
    for i, t in enumerate(rows):
        pos = wl.q_pos0 + t
        r_o, h_o = oracle.route(Qd[i:i + 1], wd[i:i + 1], kbar, pos, wl.n_k, wl.B, wl.h)
        check_heads(heads[t:t + 1], r_o, h_o, wl.h)
        lg_gpu = dumps[t]
        # top-k is bit-exact on the GPU's own logits
        assert np.array_equal(idx[t], oracle.topk(lg_gpu[None, :], pos, wl.n_k, wl.k)[0])
        if not np.array_equal(heads[t], h_o[0]):
            continue
        matched += 1
        ref = oracle.score(Qd[i:i + 1], wd[i:i + 1], h_o, Kd, pos)[0]
        hs = h_o[0]
        mag = (np.abs(wd[i, hs])[:, None] * np.maximum(Qd[i, hs] @ Kd[:pos + 1].T, 0)).sum(0)
        assert_logits_close(lg_gpu, ref[:pos + 1], mag, what=f"{name} row {t}")
        assert recall(idx[t:t + 1], oracle.topk(ref[None, :], pos, wl.n_k, wl.k)) >= 0.999
    assert matched >= len(rows) - 2


@pytest.mark.parametrize("fp8", [False, True])
def test_full_size_dagger_sampled_rows(fp8):
    # MISA-dagger on the 8192 x 131072 chunk (k' = 8192 -> k = 2048); fp8=True
    # stores the keys as e4m3 with a per-token scale for every stage (pool,
    # route, score, rerank).  Per sampled row: the routed heads against the
    # oracle's, the routed logits against the oracle's where the heads agree,
    # the coarse candidates bit-exact against the oracle's top-k' of the GPU's
    # own logits, the all-head scores of those candidates against the oracle's,
    # and the final selection bit-exact against the oracle's rule on the GPU's
    # own scores (the launch configuration of the benchmark's MISA-dagger run).
    from long_context_sparse_block_b200 import _lib
    from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer
    wl = W.WORKLOADS["dagger_128k"]
    inp = W.generate(wl, fp8_keys=fp8)
    rows = _rows(wl)
    g = inputs_to_device(inp, fp8=fp8)
    ix = MisaIndexer(IndexerShape(wl.n_q, wl.q_pos0, wl.n_k, wl.H, wl.d, wl.B, wl.h, wl.k,
                                  kp=wl.kp, sub_chunk=1024))
    K = g["K8"] if fp8 else g["K"]
    ksc = g.get("k_scale")
    dumps = {}

    def grab(c0, c1, lg):
        for t in rows:
            if c0 <= t < c1:
                dumps[t] = lg[t - c0].cpu().numpy()

    fin = ix.run(g["Q"], K, g["w"], k_scale=ksc, on_subchunk=grab).cpu().numpy()
    cand = ix.sel.cpu().numpy()
    heads = ix.heads.cpu().numpy()
    # the fused coarse pass (the product path) selects the same candidates
    fused = ix.run(g["Q"], K, g["w"], k_scale=ksc).cpu().numpy()
    assert np.array_equal(ix.sel.cpu().numpy(), cand)
    assert np.array_equal(fused, fin)
    assert _lib.misa_last_device_status() == 0
    Kd = oracle.e4m3_keys_to_f64(inp["K8"], inp["k_scale"]) if fp8 else oracle.bf16_to_f64(inp["K"])
    kbar = oracle.pool_keys(Kd, wl.B)
    sel = np.array(rows)
    Qd = oracle.bf16_to_f64(inp["Q"][sel])
    wd = inp["w"][sel].astype(np.float64)
    matched = 0
    for i, t in enumerate(rows):
        pos = wl.q_pos0 + t
        r_o, h_o = oracle.route(Qd[i:i + 1], wd[i:i + 1], kbar, pos, wl.n_k, wl.B, wl.h)
        check_heads(heads[t:t + 1], r_o, h_o, wl.h)
        lg_gpu = dumps[t]
        # coarse stage: bit-exact on the GPU's own routed logits
        assert np.array_equal(cand[t], oracle.topk(lg_gpu[None, :], pos, wl.n_k, wl.kp)[0])
        if np.array_equal(heads[t], h_o[0]):
            matched += 1
            ref_lg = oracle.score(Qd[i:i + 1], wd[i:i + 1], h_o, Kd, pos)[0]
            hs = h_o[0]
            mag = (np.abs(wd[i, hs])[:, None] * np.maximum(Qd[i, hs] @ Kd[:pos + 1].T, 0)).sum(0)
            assert_logits_close(lg_gpu, ref_lg[:pos + 1], mag, what=f"dagger row {t}")
        # fine stage: the GPU's all-head scores of this row's candidates (the
        # kernel scores each candidate the same way whatever the batch)
        idx1, full1 = _lib.misa_rerank(g["Q"][t:t + 1], g["w"][t:t + 1], K,
                                        ix.sel[t:t + 1].contiguous(), pos, wl.k, k_scale=ksc,
                                        want_full=True)
        idx1, full1 = idx1.cpu().numpy(), full1.cpu().numpy()
        assert np.array_equal(idx1[0], fin[t])
        assert np.array_equal(fin[t], oracle.select_candidates(full1, cand[t:t + 1], pos,
                                                               wl.n_k, wl.k)[0])
        ref_idx, ref_full = oracle.rerank(Qd[i:i + 1], wd[i:i + 1], Kd, cand[t:t + 1], pos, wl.k,
                                          want_logits=True)
        valid = cand[t] >= 0
        dots = Qd[i] @ Kd[cand[t, valid]].T
        mag = (np.abs(wd[i])[:, None] * np.maximum(dots, 0.0)).sum(axis=0)
        assert np.all(np.abs(full1[0, valid] - ref_full[0, valid]) <= 2e-3 * mag + 1e-5)
        assert recall(fin[t:t + 1], ref_idx) >= 0.999
        assert np.all(np.diff(fin[t][fin[t] >= 0]) > 0)
    assert matched >= len(rows) - 2


@pytest.mark.parametrize("name,sub", [("chunk_128k", 8192), ("chunk_128k_h4", 8192),
                                      ("dsv32_32k", 4096), ("glm5_64k", 8192)])
def test_full_size_fused_equals_unfused(name, sub):
    # the product path (misa_score_topk per sub-chunk) against scoring every
    # logit and selecting from them, on every row; prefill chunks whose first
    # sub-chunk starts before the 4096-key sample takes the unfused sequence there
    from long_context_sparse_block_b200 import _lib
    from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer
    wl = W.WORKLOADS[name]
    inp = W.generate(wl)
    g = inputs_to_device(inp)
    shape = IndexerShape(wl.n_q, wl.q_pos0, wl.n_k, wl.H, wl.d, wl.B, wl.h, wl.k, sub_chunk=sub)
    ix = MisaIndexer(shape)
    fused = ix.run(g["Q"], g["K"], g["w"]).clone()
    unfused = ix.run(g["Q"], g["K"], g["w"], on_subchunk=lambda c0, c1, lg: None)
    assert _lib.misa_last_device_status() == 0
    assert torch.equal(fused, unfused)
    flags = ix.ws_sel[:4].view(torch.int32).item()   # any row repaired in the last sub-chunk
    print(f"{name}: {wl.n_q} rows equal; last sub-chunk repaired rows: {flags != 0}")


def test_full_size_fp8_queries_and_keys_sampled_rows():
    # the 8192 x 131072 chunk scored with e4m3 queries and keys (kind::f8f6f4)
    # for the heads the bf16 router picked; sampled rows against the oracle on
    # the dequantised operands, and the top-k bit-exact on the GPU's logits
    from long_context_sparse_block_b200 import _lib
    wl = W.WORKLOADS["chunk_128k"]
    inp = W.generate(wl, fp8_keys=True, fp8_queries=True)
    rows = _rows(wl)
    g = inputs_to_device(inp, fp8=True)
    _, hl = _lib.misa_pool_keys(g["K"], wl.B, want_kbar=False)
    heads, _ = _lib.misa_route_heads(g["Q"], g["w"], hl, wl.q_pos0, wl.n_k, wl.B, wl.h)
    Q8 = torch.from_numpy(inp["Q8"]).cuda()
    qs = torch.from_numpy(inp["q_scale"]).cuda()
    lg = _lib.misa_score_tokens_fp8(Q8, qs, g["w"], heads, g["K8"], g["k_scale"], wl.q_pos0,
                                    h=wl.h)
    idx = _lib.misa_topk(lg, wl.q_pos0, wl.n_k, wl.k).cpu().numpy()
    assert _lib.misa_last_device_status() == 0
    heads = heads.cpu().numpy()
    Kd = oracle.e4m3_keys_to_f64(inp["K8"], inp["k_scale"])
    sel = np.array(rows)
    Qd = oracle.e4m3_keys_to_f64(inp["Q8"][sel].reshape(-1, wl.d),
                                 inp["q_scale"][sel].reshape(-1)).reshape(len(rows), wl.H, wl.d)
    wd = inp["w"][sel].astype(np.float64)
    worst, rec = 0.0, []
    for i, t in enumerate(rows):
        pos = wl.q_pos0 + t
        row = lg[t].cpu().numpy()
        hs = heads[t:t + 1]
        ref = oracle.score(Qd[i:i + 1], wd[i:i + 1], hs, Kd, pos)[0]
        mag = (np.abs(wd[i, hs[0]])[:, None] * np.maximum(Qd[i, hs[0]] @ Kd[:pos + 1].T, 0)).sum(0)
        assert_logits_close(row, ref[:pos + 1], mag, what=f"fp8 q+k row {t}")
        worst = max(worst, float(np.max(np.abs(row[:pos + 1] - ref[:pos + 1]) / (mag + 1e-30))))
        assert np.array_equal(idx[t], oracle.topk(row[None, :], pos, wl.n_k, wl.k)[0])
        # the e4m3 MMA's accumulation order and width are not documented: the set
        # may differ from the fp64 one at near-ties of the k-th logit
        rec.append(recall(idx[t:t + 1], oracle.topk(ref[None, :], pos, wl.n_k, wl.k)))
        assert rec[-1] >= 0.99
    print(f"fp8 q+k chunk: max |gpu - oracle| / sum|w ReLU(q.k)| = {worst:.3e}; "
          f"min recall vs fp64 top-k = {min(rec):.4f}")


@pytest.mark.parametrize("ps", [64])
def test_full_size_paged_chunk(ps):
    # the 8192 x 131072 chunk with its keys in a paged cache (pages of `ps` keys
    # spread over a larger pool in a random order): the indices of every row
    # equal those of the contiguous cache bit for bit, and sampled rows of the
    # paged scoring pass match the oracle on the keys in logical order
    from long_context_sparse_block_b200 import _lib
    from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer
    from tests.test_gpu_paged import make_paged
    wl = W.WORKLOADS["chunk_128k"]
    inp = W.generate(wl)
    rows = _rows(wl)
    g = inputs_to_device(inp)
    pk = make_paged(_lib, g["K"], ps, seed=ps)
    shape = IndexerShape(wl.n_q, wl.q_pos0, wl.n_k, wl.H, wl.d, wl.B, wl.h, wl.k)
    ix = MisaIndexer(shape)
    want = ix.run(g["Q"], g["K"], g["w"]).clone()
    got = ix.run(g["Q"], pk, g["w"]).clone()
    assert _lib.misa_last_device_status() == 0
    assert torch.equal(got, want)
    dumps = {}

    def grab(c0, c1, lg):
        for t in rows:
            if c0 <= t < c1:
                dumps[t] = lg[t - c0].cpu().numpy()

    ix2 = MisaIndexer(IndexerShape(wl.n_q, wl.q_pos0, wl.n_k, wl.H, wl.d, wl.B, wl.h, wl.k,
                                   sub_chunk=1024))
    unf = ix2.run(g["Q"], pk, g["w"], on_subchunk=grab).cpu().numpy()
    assert np.array_equal(unf, got.cpu().numpy())
    heads = ix2.heads.cpu().numpy()
    Kd = oracle.bf16_to_f64(inp["K"])
    sel = np.array(rows)
    Qd = oracle.bf16_to_f64(inp["Q"][sel])
    wd = inp["w"][sel].astype(np.float64)
    for i, t in enumerate(rows):
        pos = wl.q_pos0 + t
        hs = heads[t:t + 1]
        lg_gpu = dumps[t]
        assert np.array_equal(unf[t], oracle.topk(lg_gpu[None, :], pos, wl.n_k, wl.k)[0])
        ref = oracle.score(Qd[i:i + 1], wd[i:i + 1], hs, Kd, pos)[0]
        mag = (np.abs(wd[i, hs[0]])[:, None] * np.maximum(Qd[i, hs[0]] @ Kd[:pos + 1].T, 0)).sum(0)
        assert_logits_close(lg_gpu, ref[:pos + 1], mag, what=f"paged row {t}")
