"""GPU parity of the fused routed scoring + top-k call (misa_score_topk).

Its result is defined as that of misa_score_tokens followed by misa_topk, both
parity-tested against the oracle elsewhere, so every case here is bit-exact
against that pair on the same device inputs, and a few rows are also checked
against the oracle's selection.  The repair flags the call leaves at the head of
its workspace show which rows took the exact fallback; the constructed cases
force the fallback on purpose (threshold too low: every logit equal; threshold
too high: the sampled blocks score far above the rest).
"""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_block_b200 import workloads as W
from tests.gpu_helpers import dev, inputs_to_device

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_block_b200 import _lib
    return _lib


def _inputs(n_q, q_pos0, n_k, H, d, B, h, k, seed, fp8=False):
    wl = W.small_workload(f"fused{seed}", n_q=n_q, q_pos0=q_pos0, n_k=n_k, H=H, d=d, B=B, h=h,
                          k=k, seed=seed, generator="clustered")
    inp = W.generate(wl, fp8_keys=fp8)
    return wl, inp, inputs_to_device(inp, fp8=fp8)


def _heads(lib, g, wl, fp8):
    Kdev = g["K8"] if fp8 else g["K"]
    _, hl = lib.misa_pool_keys(Kdev, wl.B, k_scale=g.get("k_scale"))
    heads, _ = lib.misa_route_heads(g["Q"], g["w"], hl, wl.q_pos0, wl.n_k, wl.B, wl.h)
    return heads


def _fused(lib, Q, w, heads, K, q_pos0, k, k_scale=None, h=None):
    n_q, n_k = Q.shape[0], K.shape[0]
    nbytes = lib.misa_workspace_size("score_topk", n_q, n_k, k, 0)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    ws.fill_(0xA5)    # stale contents must not matter
    idx = lib.misa_score_topk(Q, w, heads, K, q_pos0, k, k_scale=k_scale, h=h, ws=ws)
    flags = ws[:4 * (n_q + 1)].view(torch.int32).cpu().numpy() if nbytes else None
    return idx.cpu().numpy(), flags


def _unfused(lib, Q, w, heads, K, q_pos0, k, k_scale=None, h=None):
    lg = lib.misa_score_tokens(Q, w, heads, K, q_pos0, k_scale=k_scale, h=h)
    return lib.misa_topk(lg, q_pos0, K.shape[0], k).cpu().numpy(), lg


FUSED_CASES = [
    # n_q, q_pos0, n_k, H, d, B, h, k, fp8
    (300, 16000, 20000, 64, 128, 128, 8, 512, False),
    (257, 9000, 12000, 64, 128, 128, 4, 2048, False),
    (200, 12000, 14000, 32, 64, 64, 16, 256, True),
    (129, 20000, 24000, 64, 128, 128, 32, 1024, False),
    (100, 6000, 7000, 64, 128, 128, 8, 8192, False),     # k above most rows' prefix
    (64, 4095, 4200, 16, 32, 32, 4, 1, False),            # smallest fused prefix, k = 1
    # 2^17 < n_k < 2^18: more than four mask units per finish thread, and the
    # 16-bit list positions of large k cross three 65536-key boundaries
    (24, 200000, 200100, 64, 128, 128, 8, 2048, False),
    (24, 200000, 200100, 64, 128, 128, 8, 6000, False),
]


@pytest.mark.parametrize("n_q,q_pos0,n_k,H,d,B,h,k,fp8", FUSED_CASES)
def test_score_topk_equals_score_then_topk(lib, n_q, q_pos0, n_k, H, d, B, h, k, fp8):
    wl, inp, g = _inputs(n_q, q_pos0, n_k, H, d, B, h, k, seed=n_q + k, fp8=fp8)
    heads = _heads(lib, g, wl, fp8)
    Kdev, ksc = (g["K8"], g["k_scale"]) if fp8 else (g["K"], None)
    got, flags = _fused(lib, g["Q"], g["w"], heads, Kdev, q_pos0, k, k_scale=ksc)
    want, lg = _unfused(lib, g["Q"], g["w"], heads, Kdev, q_pos0, k, k_scale=ksc)
    assert np.array_equal(got, want)
    rows = np.linspace(0, n_q - 1, 5).astype(int)
    lg_np = lg.cpu().numpy()
    for t in rows:
        one = oracle.topk(lg_np[t:t + 1], q_pos0 + t, n_k, k)
        assert np.array_equal(got[t], one[0])
    assert flags is not None
    assert flags[0] == int(flags[1:].any())
    print(f"rows repaired: {int(flags[1:].sum())} of {n_q}")


def test_score_topk_dense_heads(lib):
    # heads = NULL with h = H: the dense indexer through the fused call
    n_q, q_pos0, n_k, H, d, k = 96, 8000, 9000, 64, 128, 300
    _, _, g = _inputs(n_q, q_pos0, n_k, H, d, 128, H, k, seed=5)
    got, _ = _fused(lib, g["Q"], g["w"], None, g["K"], q_pos0, k, h=H)
    want, _ = _unfused(lib, g["Q"], g["w"], None, g["K"], q_pos0, k, h=H)
    assert np.array_equal(got, want)


@pytest.mark.parametrize("q_pos0,h", [(3000, 8), (9000, 2), (9000, 128)])
def test_score_topk_unfused_shapes(lib, q_pos0, h):
    # prefix shorter than the sample, or h without a select kernel: the call
    # runs the unfused sequence and must give the same result
    n_q, n_k, H, d, k = 80, q_pos0 + 500, 128 if h == 128 else 64, 128, 200
    wl, _, g = _inputs(n_q, q_pos0, n_k, H, d, 128, h, k, seed=q_pos0 + h)
    heads = _heads(lib, g, wl, False)
    got, flags = _fused(lib, g["Q"], g["w"], heads, g["K"], q_pos0, k)
    want, _ = _unfused(lib, g["Q"], g["w"], heads, g["K"], q_pos0, k)
    assert np.array_equal(got, want)


def test_score_topk_repairs_ties_everywhere(lib):
    # every key equal: every visible logit of a row ties, far more than the
    # candidate list holds, so every row takes the exact fallback
    n_q, q_pos0, n_k, H, d, k = 40, 12000, 12100, 64, 128, 512
    wl, inp, g = _inputs(n_q, q_pos0, n_k, H, d, 128, 8, k, seed=21)
    K = g["K"][:1].expand(n_k, d).contiguous()
    heads = _heads(lib, {**g, "K": K}, wl, False)
    got, flags = _fused(lib, g["Q"], g["w"], heads, K, q_pos0, k)
    want, _ = _unfused(lib, g["Q"], g["w"], heads, K, q_pos0, k)
    assert np.array_equal(got, want)
    assert flags[0] == 1 and flags[1:].all()


def test_score_topk_repairs_unrepresentative_sample(lib):
    # the sampled blocks (32 blocks of 128 keys evenly spaced over 0..q_pos0)
    # hold the only keys that score high, each a different amount, so the
    # thresholds keep ~1.6 k * 4096 / visible of them: fewer than k
    n_q, q_pos0, n_k, H, d, k, h = 48, 14000, 14100, 64, 128, 1024, 8
    rng = np.random.default_rng(22)
    Q = (1.0 + 0.3 * rng.standard_normal((n_q, H, d))) / np.sqrt(d)
    K = 0.01 * rng.standard_normal((n_k, d)) / np.sqrt(d)
    span, nb = q_pos0 + 1, 32
    for b in range(nb):
        start = (span - 128) * b // (nb - 1)
        K[start:start + 128] = rng.uniform(2.0, 4.0, size=(128, 1)) / np.sqrt(d)
    w = np.full((n_q, H), 1.0 / H, dtype=np.float32)
    Qg, Kg, wg = dev(W.bf16_bits(Q)), dev(W.bf16_bits(K)), dev(w)
    B = 128
    _, hl = lib.misa_pool_keys(Kg, B)
    heads, _ = lib.misa_route_heads(Qg, wg, hl, q_pos0, n_k, B, h)
    got, flags = _fused(lib, Qg, wg, heads, Kg, q_pos0, k)
    want, _ = _unfused(lib, Qg, wg, heads, Kg, q_pos0, k)
    assert np.array_equal(got, want)
    assert flags[0] == 1 and flags[1:].all()


def test_score_topk_bursts_of_kept_logits(lib):
    # runs of 64 consecutive high-scoring keys: their 32-key words keep more
    # logits than a word's dense slot holds, so the rest go through the row
    n_q, q_pos0, n_k, H, d, k, h = 64, 10000, 10100, 64, 128, 256, 8
    rng = np.random.default_rng(23)
    Q = (1.0 + 0.3 * rng.standard_normal((n_q, H, d))) / np.sqrt(d)
    K = 0.5 * rng.standard_normal((n_k, d)) / np.sqrt(d)
    for start in (1000, 5003, 9990):
        K[start:start + 64] = rng.uniform(2.0, 3.0, size=(64, 1)) / np.sqrt(d)
    w = np.full((n_q, H), 1.0 / H, dtype=np.float32)
    Qg, Kg, wg = dev(W.bf16_bits(Q)), dev(W.bf16_bits(K)), dev(w)
    _, hl = lib.misa_pool_keys(Kg, 128)
    heads, _ = lib.misa_route_heads(Qg, wg, hl, q_pos0, n_k, 128, h)
    got, flags = _fused(lib, Qg, wg, heads, Kg, q_pos0, k)
    want, _ = _unfused(lib, Qg, wg, heads, Kg, q_pos0, k)
    assert np.array_equal(got, want)
    assert flags[0] == int(flags[1:].any())
    for t in range(n_q):   # every burst key visible to row t is selected
        vis = q_pos0 + t + 1
        burst = [s for st in (1000, 5003, 9990) for s in range(st, st + 64) if s < vis]
        assert set(burst) <= set(got[t].tolist())
    print(f"rows repaired: {int(flags[1:].sum())} of {n_q}")


@pytest.mark.parametrize("kp", [0, 1024])
def test_indexer_host_pipeline_equals_device_run(lib, kp):
    # run_host (copies of one query piece overlapping the indexing of another)
    # gives what run gives on device-resident inputs
    from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer
    n_q, q_pos0, n_k, H, d, B, h, k = 600, 20000, 24000, 64, 128, 128, 8, 256
    wl, inp, g = _inputs(n_q, q_pos0, n_k, H, d, B, h, k, seed=31)
    shape = IndexerShape(n_q, q_pos0, n_k, H, d, B, h, k, kp=kp, sub_chunk=256)
    want = MisaIndexer(shape).run(g["Q"], g["K"], g["w"]).cpu().numpy()
    ix = MisaIndexer(shape)
    Qh = torch.from_numpy(np.ascontiguousarray(inp["Q"]).view(np.int16)).pin_memory()
    Kh = torch.from_numpy(np.ascontiguousarray(inp["K"]).view(np.int16)).pin_memory()
    wh = torch.from_numpy(inp["w"]).pin_memory()
    for pieces in (None, 1, 3, 4):
        out = ix.run_host(Qh, Kh, wh, pieces=pieces)
        torch.cuda.current_stream().synchronize()
        assert np.array_equal(out.numpy(), want)


def test_score_topk_long_kept_lists(lib):
    # the sampled blocks hold the only small keys, so the threshold sits low and
    # every other visible key is kept: ~5.7k kept logits per row, near the top of
    # what the finish kernel's list holds; every row must still come out exact
    # without the repair path
    n_q, q_pos0, n_k, H, d, k, h = 64, 8999, 9100, 64, 128, 1024, 8
    rng = np.random.default_rng(24)
    Q = (1.0 + 0.3 * rng.standard_normal((n_q, H, d))) / np.sqrt(d)
    K = (1.0 + 0.5 * rng.standard_normal((n_k, d))) / np.sqrt(d)
    span, nb = q_pos0 + 1, 32
    for b in range(nb):
        start = (span - 128) * b // (nb - 1)
        K[start:start + 128] *= 0.01
    w = np.full((n_q, H), 1.0 / H, dtype=np.float32)
    Qg, Kg, wg = dev(W.bf16_bits(Q)), dev(W.bf16_bits(K)), dev(w)
    _, hl = lib.misa_pool_keys(Kg, 128)
    heads, _ = lib.misa_route_heads(Qg, wg, hl, q_pos0, n_k, 128, h)
    got, flags = _fused(lib, Qg, wg, heads, Kg, q_pos0, k)
    want, _ = _unfused(lib, Qg, wg, heads, Kg, q_pos0, k)
    assert np.array_equal(got, want)
    assert flags[0] == 0 and not flags[1:].any()    # no repair: the list held them


def test_e4m3_key_decode_is_exact(lib):
    # every e4m3 code (the NaN codes included) decodes to the bf16 code of its value
    codes = np.tile(np.arange(256, dtype=np.uint8), 3).reshape(6, 128)
    got = lib.misa_keys_e4m3_to_bf16(dev(codes)).cpu().numpy().view(np.uint16)
    want = oracle.e4m3_keys_to_f64(codes, np.ones(6, dtype=np.float32))
    assert np.array_equal(oracle.bf16_to_f64(got), want, equal_nan=True)


@pytest.mark.parametrize("n_q,q_pos0,n_k,k", [(200, 12000, 14000, 256),   # fused
                                              (129, 20000, 24000, 2048),  # fused
                                              (64, 1000, 1100, 64)])      # unfused shape
def test_score_topk_decoded_fp8_keys_equal_e4m3_keys(lib, n_q, q_pos0, n_k, k):
    # e4m3 keys decoded once and scored as scaled bf16 keys (what the indexer does
    # for every query piece) select what the e4m3 keys themselves select
    wl, inp, g = _inputs(n_q, q_pos0, n_k, 64, 128, 128, 8, k, seed=n_k + k, fp8=True)
    heads = _heads(lib, g, wl, True)
    Kd = lib.misa_keys_e4m3_to_bf16(g["K8"])
    got, flags = _fused(lib, g["Q"], g["w"], heads, Kd, q_pos0, k, k_scale=g["k_scale"])
    want, _ = _fused(lib, g["Q"], g["w"], heads, g["K8"], q_pos0, k, k_scale=g["k_scale"])
    assert np.array_equal(got, want)
    lg = lib.misa_score_tokens(g["Q"], g["w"], heads, g["K8"], q_pos0, k_scale=g["k_scale"])
    lg_np = lg.cpu().numpy()
    for t in (0, n_q // 2, n_q - 1):
        assert np.array_equal(got[t], oracle.topk(lg_np[t:t + 1], q_pos0 + t, n_k, k)[0])


def test_indexer_fp8_pieces_equal_whole_chunk(lib):
    # the indexer decodes the e4m3 keys once per chunk; every piece schedule of the
    # host pipeline and sub-chunking gives the whole-chunk result
    from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer
    n_q, q_pos0, n_k, H, d, B, h, k = 300, 9000, 9300, 64, 128, 128, 8, 512
    wl, inp, g = _inputs(n_q, q_pos0, n_k, H, d, B, h, k, seed=61, fp8=True)
    shape = IndexerShape(n_q, q_pos0, n_k, H, d, B, h, k)
    want = MisaIndexer(shape).run(g["Q"], g["K8"], g["w"], k_scale=g["k_scale"]).cpu().numpy()
    lg = lib.misa_score_tokens(g["Q"], g["w"], _heads(lib, g, wl, True), g["K8"], q_pos0,
                               k_scale=g["k_scale"]).cpu().numpy()
    assert np.array_equal(want[7], oracle.topk(lg[7:8], q_pos0 + 7, n_k, k)[0])
    sub = MisaIndexer(IndexerShape(n_q, q_pos0, n_k, H, d, B, h, k, sub_chunk=128))
    assert np.array_equal(sub.run(g["Q"], g["K8"], g["w"], k_scale=g["k_scale"]).cpu().numpy(),
                          want)
    Qh, K8h, wh, ksh = (t.cpu().pin_memory() for t in (g["Q"], g["K8"], g["w"], g["k_scale"]))
    for pieces in (None, 3, [100, 50, 150]):
        out = MisaIndexer(shape).run_host(Qh, K8h, wh, k_scale_h=ksh, pieces=pieces)
        torch.cuda.current_stream().synchronize()
        assert np.array_equal(out.numpy(), want)
