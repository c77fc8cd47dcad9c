"""GPU parity: every stage of the CUDA path against the fp64 oracle, through the
C ABI, on seeded inputs that span several tiles and ragged tails."""
import numpy as np
import pytest
import torch

import oracle
from long_context_sparse_block_b200 import workloads as W
from tests.gpu_helpers import (assert_logits_close, check_heads, dev, inputs_to_device,
                               logit_magnitude, recall)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    from long_context_sparse_block_b200 import _lib
    return _lib


def _wl(n_q, q_pos0, n_k, H, d, B, h, k, seed, gen="clustered", kp=0):
    return W.small_workload(f"case{seed}", n_q=n_q, q_pos0=q_pos0, n_k=n_k, H=H, d=d, B=B, h=h,
                            k=k, seed=seed, generator=gen, kp=kp)


# ------------------------------------------------------------------ pooling

@pytest.mark.parametrize("n_k,d,B,fp8", [(1024, 32, 64, False), (1000, 128, 128, False),
                                         (777, 64, 48, False), (1000, 128, 128, True),
                                         (300, 32, 1, False)])
def test_pool_matches_oracle(lib, n_k, d, B, fp8):
    inp = W.generate(_wl(1, n_k - 1, n_k, 4, d, B, 1, 1, seed=n_k + d), fp8_keys=fp8)
    Kd = oracle.e4m3_keys_to_f64(inp["K8"], inp["k_scale"]) if fp8 else oracle.bf16_to_f64(inp["K"])
    ref = oracle.pool_keys(Kd, B)
    Kdev = dev(inp["K8"]) if fp8 else dev(inp["K"])
    kbar, hl = lib.misa_pool_keys(Kdev, B, k_scale=dev(inp["k_scale"]) if fp8 else None)
    kbar = kbar.cpu().numpy().astype(np.float64)
    tol = 1e-6 * np.abs(Kd).max() + 1e-9
    assert np.max(np.abs(kbar - ref)) <= tol
    hl = hl.cpu().numpy().view(np.uint16)
    hi = oracle.bf16_to_f64(hl[0])
    lo = oracle.bf16_to_f64(hl[1])
    assert np.array_equal(W.bf16_bits(kbar), hl[0])                    # hi = bf16(kbar)
    assert np.all(np.abs(hi + lo - kbar) <= 2.0 ** -16 * np.abs(kbar) + 1e-30)


@pytest.mark.parametrize("d,B,page_size", [(128, 128, 0), (64, 64, 16), (32, 128, 128),
                                           (128, 128, 16)])
def test_pool_stream_equals_per_block_and_oracle(lib, d, B, page_size):
    # 301+ blocks (the last one partial): the full pooling takes the streaming
    # kernel (bulk-copy stages, one CTA per SM), ranges of 100 blocks the per-block
    # kernel; both sum in the same order, so they agree bit for bit, and both
    # match the oracle; through pages (runs inside pages) the same bits again
    n_k = 300 * B + 57
    inp = W.generate(_wl(1, n_k - 1, n_k, 4, d, B, 1, 1, seed=n_k + d))
    Kdev = dev(inp["K"])
    kbar, hl = lib.misa_pool_keys(Kdev, B)
    M = kbar.shape[0]
    kb2 = torch.empty_like(kbar)
    hl2 = torch.empty_like(hl)
    for m0 in range(0, M, 100):
        lib.misa_pool_keys_range(Kdev, B, m0, min(M, m0 + 100), kbar=kb2, kbar_hl=hl2)
    assert torch.equal(kbar, kb2) and torch.equal(hl, hl2)
    Kd = oracle.bf16_to_f64(inp["K"])
    ref = oracle.pool_keys(Kd, B)
    assert np.max(np.abs(kbar.cpu().numpy().astype(np.float64) - ref)) <= 1e-6 * np.abs(Kd).max() + 1e-9
    if page_size:
        n_blocks = -(-n_k // page_size)
        table = torch.from_numpy(np.random.default_rng(d + B).permutation(n_blocks + 2)[:n_blocks]
                                 .astype(np.int32)).cuda()
        pages = torch.zeros(((n_blocks + 2) * page_size, d), dtype=Kdev.dtype, device="cuda")
        flat = torch.zeros((n_blocks * page_size, d), dtype=Kdev.dtype, device="cuda")
        flat[:n_k] = Kdev
        pages.view(n_blocks + 2, page_size, d)[table.long()] = flat.view(n_blocks, page_size, d)
        pk = lib.PagedKeys(pages.view(n_blocks + 2, page_size, d), table, n_k)
        kb3, hl3 = lib.misa_pool_keys(pk, B)
        assert torch.equal(kbar, kb3) and torch.equal(hl, hl3)
    assert lib.misa_last_device_status() == lib.MISA_OK


# ------------------------------------------------------------------ router

@pytest.mark.parametrize("n_q,q_pos0,n_k,H,d,B,h,gen", [
    (1024, 0, 1024, 8, 32, 64, 2, "gaussian"),
    (300, 700, 1000, 64, 128, 128, 8, "clustered"),
    (250, 0, 300, 32, 64, 32, 4, "clustered"),
    (129, 40, 400, 16, 128, 16, 16, "gaussian"),
])
def test_route_matches_oracle(lib, n_q, q_pos0, n_k, H, d, B, h, gen):
    wl = _wl(n_q, q_pos0, n_k, H, d, B, h, 8, seed=n_q + H, gen=gen)
    inp = W.generate(wl)
    Qd, Kd, wd = oracle.decode_inputs(inp)
    kbar = oracle.pool_keys(Kd, B)
    r_ora, heads_ora = oracle.route(Qd, wd, kbar, q_pos0, n_k, B, h)
    g = inputs_to_device(inp)
    _, hl = lib.misa_pool_keys(g["K"], B)
    heads, r = lib.misa_route_heads(g["Q"], g["w"], hl, q_pos0, n_k, B, h, want_r=True)
    heads, r = heads.cpu().numpy(), r.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(r - r_ora) <= 2e-3 * np.abs(r_ora) + 1e-5)
    r32 = r.astype(np.float32)
    exempt = check_heads(heads, r_ora, heads_ora, h, r_gpu=r32)
    no_block = sum(1 for t in range(n_q) if (q_pos0 + t + 1) // B == 0)
    print(f"near-tie rows: {exempt} of {n_q} ({no_block} see no complete block)")
    assert np.all(np.diff(heads, axis=1) > 0)                           # ascending, distinct


def test_route_two_tile_units_equal_single_tiles(lib):
    # 309 row tiles of 128 (query, head) rows: the whole call contracts two row
    # tiles per pooled-key tile (the last unit holds one); slices of at most 100
    # row tiles take one tile per unit.  Each row's arithmetic is the same, so r
    # and the heads agree bit for bit, and they match the oracle.
    n_q, H, d, B, h = 618, 64, 128, 128, 8
    n_k = 9000
    q_pos0 = n_k - n_q
    wl = _wl(n_q, q_pos0, n_k, H, d, B, h, 8, seed=4242)
    inp = W.generate(wl)
    g = inputs_to_device(inp)
    _, hl = lib.misa_pool_keys(g["K"], B)
    heads, r = lib.misa_route_heads(g["Q"], g["w"], hl, q_pos0, n_k, B, h, want_r=True)
    heads2 = torch.empty_like(heads)
    r2 = torch.empty_like(r)
    step = 100 * 128 // H  # queries in 100 row tiles
    for c0 in range(0, n_q, step):
        c1 = min(n_q, c0 + step)
        hh, rr = lib.misa_route_heads(g["Q"][c0:c1], g["w"][c0:c1], hl, q_pos0 + c0, n_k, B, h,
                                      want_r=True)
        heads2[c0:c1] = hh
        r2[c0:c1] = rr
    assert torch.equal(r, r2) and torch.equal(heads, heads2)
    Qd, Kd, wd = oracle.decode_inputs(inp)
    r_ora, heads_ora = oracle.route(Qd, wd, oracle.pool_keys(Kd, B), q_pos0, n_k, B, h)
    r = r.cpu().numpy().astype(np.float64)
    assert np.all(np.abs(r - r_ora) <= 2e-3 * np.abs(r_ora) + 1e-5)
    check_heads(heads.cpu().numpy(), r_ora, heads_ora, h, r_gpu=r.astype(np.float32))


# ------------------------------------------------------------------ scoring

SCORE_CASES = [
    # n_q, q_pos0, n_k, H, d, h, dense
    (1024, 0, 1024, 8, 32, 2, False),
    (70, 300, 517, 64, 128, 8, False),
    (100, 0, 100, 64, 128, 4, False),
    (300, 50, 400, 16, 64, 1, False),
    (257, 3, 300, 8, 32, 2, False),
    (40, 1000, 1100, 32, 128, 16, False),
    (9, 200, 250, 64, 128, 64, True),
    (33, 90, 200, 8, 64, 8, True),
    (5, 130, 140, 128, 128, 128, False),
]


@pytest.mark.parametrize("n_q,q_pos0,n_k,H,d,h,dense", SCORE_CASES)
def test_score_matches_oracle(lib, n_q, q_pos0, n_k, H, d, h, dense):
    wl = _wl(n_q, q_pos0, n_k, H, d, 64, h, 8, seed=7 * n_q + h)
    inp = W.generate(wl)
    Qd, Kd, wd = oracle.decode_inputs(inp)
    rng = np.random.default_rng(n_q)
    if dense:
        heads = np.tile(np.arange(H, dtype=np.int32), (n_q, 1))
    else:
        heads = np.sort(np.stack([rng.choice(H, size=h, replace=False) for _ in range(n_q)]),
                        axis=1).astype(np.int32)
    ref = oracle.score(Qd, wd, heads, Kd, q_pos0)
    g = inputs_to_device(inp)
    ld = (n_k + 3) // 4 * 4 + 4            # a padded row pitch
    logits = torch.full((n_q, ld), float("nan"), device="cuda")
    lib.misa_score_tokens(g["Q"], g["w"], None if dense else dev(heads), g["K"], q_pos0,
                          logits=logits, h=h)
    assert lib.misa_last_device_status() == 0
    out = logits.cpu().numpy()
    for t in range(n_q):
        pos = q_pos0 + t
        mag = logit_magnitude(Qd, wd, Kd, heads, t, q_pos0)
        assert_logits_close(out[t], ref[t, :pos + 1], mag, what=f"row {t}")
        n4 = (n_k + 3) // 4 * 4
        tail = out[t, pos + 1:n4]
        assert np.all(np.isnan(tail) | np.isneginf(tail))
        assert np.all(np.isnan(out[t, n4:]))                # never past n_k rounded up to 4


@pytest.mark.parametrize("n_q,q_pos0,n_k,H,d,h", [(70, 300, 517, 64, 128, 8), (257, 3, 300, 8, 32, 2),
                                                  (40, 1000, 1100, 32, 64, 16),
                                                  (9, 200, 250, 64, 128, 64),
                                                  (100, 0, 100, 64, 128, 4)])
def test_score_fp8_keys_matches_oracle(lib, n_q, q_pos0, n_k, H, d, h):
    # keys stored as e4m3 with a per-token fp32 scale, decoded in the kernel
    wl = _wl(n_q, q_pos0, n_k, H, d, 64, h, 8, seed=11 * n_q + h)
    inp = W.generate(wl, fp8_keys=True)
    Qd, Kd, wd = oracle.decode_inputs(inp, fp8_keys=True)
    rng = np.random.default_rng(n_q + 1)
    heads = np.sort(np.stack([rng.choice(H, size=h, replace=False) for _ in range(n_q)]),
                    axis=1).astype(np.int32)
    ref = oracle.score(Qd, wd, heads, Kd, q_pos0)
    g = inputs_to_device(inp, fp8=True)
    logits = torch.full((n_q, (n_k + 3) // 4 * 4), float("nan"), device="cuda")
    lib.misa_score_tokens(g["Q"], g["w"], dev(heads), g["K8"], q_pos0, k_scale=g["k_scale"],
                          logits=logits, h=h)
    assert lib.misa_last_device_status() == 0
    out = logits.cpu().numpy()
    for t in range(n_q):
        pos = q_pos0 + t
        mag = logit_magnitude(Qd, wd, Kd, heads, t, q_pos0)
        assert_logits_close(out[t], ref[t, :pos + 1], mag, what=f"fp8 row {t}")


FP8_QK_CASES = [
    (70, 300, 517, 64, 128, 8, False),
    (40, 1000, 1100, 32, 64, 16, False),
    (9, 200, 250, 64, 128, 64, False),
    (100, 0, 100, 64, 128, 4, False),
    (257, 3, 300, 8, 64, 2, False),
    (50, 10, 300, 16, 128, 1, False),
    (33, 90, 200, 8, 64, 8, True),
    (5, 130, 140, 128, 128, 128, True),
]


@pytest.mark.parametrize("n_q,q_pos0,n_k,H,d,h,dense", FP8_QK_CASES)
def test_score_fp8_queries_and_keys_matches_oracle(lib, n_q, q_pos0, n_k, H, d, h, dense):
    # queries and keys both e4m3 (a scale per (query, head) row and per key),
    # multiplied as e4m3 on the tensor cores
    wl = _wl(n_q, q_pos0, n_k, H, d, 64, h, 8, seed=13 * n_q + h)
    inp = W.generate(wl, fp8_keys=True, fp8_queries=True)
    Qd, Kd, wd = oracle.decode_inputs(inp, fp8_keys=True, fp8_queries=True)
    rng = np.random.default_rng(n_q + 2)
    if dense:
        heads = np.tile(np.arange(H, dtype=np.int32), (n_q, 1))
    else:
        heads = np.sort(np.stack([rng.choice(H, size=h, replace=False) for _ in range(n_q)]),
                        axis=1).astype(np.int32)
    ref = oracle.score(Qd, wd, heads, Kd, q_pos0)
    ld = (n_k + 3) // 4 * 4 + 4
    logits = torch.full((n_q, ld), float("nan"), device="cuda")
    lib.misa_score_tokens_fp8(dev(inp["Q8"]), dev(inp["q_scale"]), dev(inp["w"]),
                              None if dense else dev(heads), dev(inp["K8"]), dev(inp["k_scale"]),
                              q_pos0, logits=logits, h=h)
    assert lib.misa_last_device_status() == 0
    out = logits.cpu().numpy()
    n4 = (n_k + 3) // 4 * 4
    for t in range(n_q):
        pos = q_pos0 + t
        mag = logit_magnitude(Qd, wd, Kd, heads, t, q_pos0)
        assert_logits_close(out[t], ref[t, :pos + 1], mag, what=f"fp8 q+k row {t}")
        tail = out[t, pos + 1:n4]
        assert np.all(np.isnan(tail) | np.isneginf(tail))
        assert np.all(np.isnan(out[t, n4:]))
    # top-k on those logits: bit-exact against the oracle's selection of them
    k = min(64, n_k)
    idx = lib.misa_topk(logits[:, :n_k], q_pos0, n_k, k)
    assert np.array_equal(idx.cpu().numpy(), oracle.topk(out[:, :n_k], q_pos0, n_k, k))


def test_fp8_queries_and_keys_exact_arithmetic_is_bitwise(lib):
    # small-integer e4m3 codes with power-of-two scales and weights: every
    # product and sum is exact, so the logits and the top-k match exactly
    n_q, q_pos0, n_k, H, d, h, k = 150, 200, 520, 8, 128, 4, 40
    rng = np.random.default_rng(21)
    Q8 = W.e4m3_encode(rng.integers(-3, 4, size=(n_q, H, d)).astype(np.float64))
    K8 = W.e4m3_encode(rng.integers(-3, 4, size=(n_k, d)).astype(np.float64))
    q_scale = np.ldexp(1.0, rng.integers(-3, 2, size=(n_q, H))).astype(np.float32)
    k_scale = np.ldexp(1.0, rng.integers(-3, 2, size=n_k)).astype(np.float32)
    sign = np.where(rng.integers(0, 4, size=(n_q, H)) == 0, -1.0, 1.0)
    w = (sign * np.ldexp(1.0, rng.integers(-3, 2, size=(n_q, H)))).astype(np.float32)
    heads = np.sort(np.stack([rng.choice(H, size=h, replace=False) for _ in range(n_q)]),
                    axis=1).astype(np.int32)
    inp = {"Q8": Q8, "q_scale": q_scale, "K8": K8, "k_scale": k_scale, "w": w}
    Qd, Kd, wd = oracle.decode_inputs(inp, fp8_keys=True, fp8_queries=True)
    ref = oracle.score(Qd, wd, heads, Kd, q_pos0)
    logits = lib.misa_score_tokens_fp8(dev(Q8), dev(q_scale), dev(w), dev(heads), dev(K8),
                                       dev(k_scale), q_pos0)
    idx = lib.misa_topk(logits, q_pos0, n_k, k)
    assert lib.misa_last_device_status() == 0
    out = logits.cpu().numpy().astype(np.float64)
    for t in range(n_q):
        assert np.array_equal(out[t, :q_pos0 + t + 1], ref[t, :q_pos0 + t + 1])
    assert np.array_equal(idx.cpu().numpy(), oracle.topk(ref, q_pos0, n_k, k))


def test_exact_arithmetic_is_bitwise(lib):
    # small integers and power-of-two weights: every product and sum is exact in
    # fp32, so pool, router scores, heads, logits and top-k must match exactly.
    n_q, q_pos0, n_k, H, d, B, h, k = 200, 300, 600, 8, 64, 64, 2, 40
    inp = W.exact_arithmetic_inputs(n_q, q_pos0, n_k, H, d, seed=5)
    Qd, Kd, wd = oracle.decode_inputs(inp)
    kbar = oracle.pool_keys(Kd, B)
    r_ora, heads_ora = oracle.route(Qd, wd, kbar, q_pos0, n_k, B, h)
    ref = oracle.score(Qd, wd, heads_ora, Kd, q_pos0)
    idx_ora = oracle.topk(ref, q_pos0, n_k, k)
    g = inputs_to_device(inp)
    kb, hl = lib.misa_pool_keys(g["K"], B)
    heads, r = lib.misa_route_heads(g["Q"], g["w"], hl, q_pos0, n_k, B, h, want_r=True)
    logits = lib.misa_score_tokens(g["Q"], g["w"], heads, g["K"], q_pos0)
    idx = lib.misa_topk(logits, q_pos0, n_k, k)
    full = n_k // B                       # the partial last block's mean is not exact
    assert np.array_equal(kb.cpu().numpy().astype(np.float64)[:full], kbar[:full])
    assert np.array_equal(r.cpu().numpy().astype(np.float64), r_ora)
    assert np.array_equal(heads.cpu().numpy(), heads_ora)
    out = logits.cpu().numpy().astype(np.float64)
    for t in range(n_q):
        assert np.array_equal(out[t, :q_pos0 + t + 1], ref[t, :q_pos0 + t + 1])
    assert np.array_equal(idx.cpu().numpy(), idx_ora)


# ------------------------------------------------------------------ top-k

def test_topk_on_routed_logits(lib):
    wl = W.WORKLOADS["tiny_1k"]
    inp = W.generate(wl)
    Qd, Kd, wd = oracle.decode_inputs(inp)
    g = inputs_to_device(inp)
    _, hl = lib.misa_pool_keys(g["K"], wl.B)
    heads, _ = lib.misa_route_heads(g["Q"], g["w"], hl, wl.q_pos0, wl.n_k, wl.B, wl.h)
    logits = lib.misa_score_tokens(g["Q"], g["w"], heads, g["K"], wl.q_pos0)
    idx = lib.misa_topk(logits, wl.q_pos0, wl.n_k, wl.k).cpu().numpy()
    lg = logits.cpu().numpy()
    assert np.array_equal(idx, oracle.topk(lg, wl.q_pos0, wl.n_k, wl.k))      # bit-exact
    ref = oracle.score(Qd, wd, heads.cpu().numpy(), Kd, wl.q_pos0)
    assert recall(idx, oracle.topk(ref, wl.q_pos0, wl.n_k, wl.k)) >= 0.999


def _adversarial_rows(n, rng):
    rows = []
    rows.append(np.full(n, 0.25, dtype=np.float32))                           # all equal
    z = np.zeros(n, dtype=np.float32)
    z[1::2] = -0.0
    z[rng.choice(n, 20, replace=False)] = 1.0
    rows.append(z)                                                            # +-0 ties
    rows.append((rng.integers(-3, 4, size=n) / 4.0).astype(np.float32))      # few levels
    rows.append(rng.standard_normal(n).astype(np.float32))
    rows.append(np.concatenate([np.full(n - 100, 3.0), rng.standard_normal(100)]).astype(np.float32))
    big = rng.standard_normal(n).astype(np.float32)
    big[::7] = np.float32(1e30)
    rows.append(big)
    rows.append(-np.abs(rng.standard_normal(n)).astype(np.float32) - 1.0)    # all negative
    # consecutive floats, descending with the position: the k-th key is the floor
    # of its radix bin whenever 16 | n - k, so the select stops there with the
    # threshold one ulp below it, a value the row also holds (and must not take)
    rows.append((np.uint32(0x3FC00000) + (n - 1 - np.arange(n)).astype(np.uint32)).view(np.float32))
    return np.stack(rows)


@pytest.mark.parametrize("k", [1, 7, 64, 2048, 4096, 8192, 12288, 16384])
def test_topk_adversarial_rows(lib, k):
    rng = np.random.default_rng(k)
    n = 40000
    rows = _adversarial_rows(n, rng)
    n_q = rows.shape[0]
    q_pos0 = n - n_q                      # every row sees n - n_q + t + 1 tokens
    ld = n + 4
    buf = np.full((n_q, ld), np.nan, dtype=np.float32)
    buf[:, :n] = rows
    for t in range(n_q):
        buf[t, q_pos0 + t + 1:] = np.nan  # never read
    gpu = lib.misa_topk(dev(buf), q_pos0, n, k).cpu().numpy()
    assert np.array_equal(gpu, oracle.topk(buf, q_pos0, n, k))


def test_topk_fewer_tokens_than_k(lib):
    n_q, n_k, k = 50, 60, 16
    rng = np.random.default_rng(1)
    buf = rng.standard_normal((n_q, n_k)).astype(np.float32)
    gpu = lib.misa_topk(dev(buf), 0, n_k, k).cpu().numpy()
    ref = oracle.topk(buf, 0, n_k, k)
    assert np.array_equal(gpu, ref)
    assert gpu[0, 0] == 0 and np.all(gpu[0, 1:] == -1)


# ------------------------------------------------------------------ MISA-dagger rerank

@pytest.mark.parametrize("fp8,H,d,kp,k", [(False, 64, 128, 256, 64), (True, 64, 128, 256, 64),
                                          (False, 8, 32, 100, 30), (False, 32, 64, 384, 128),
                                          (False, 64, 128, 256, 256), (True, 16, 64, 128, 128)])
def test_rerank_matches_oracle(lib, fp8, H, d, kp, k):
    # k == kp (the last two cases): every valid candidate is kept
    n_q, q_pos0, n_k, B, h = 40, 500, 600, 64, 4 if H > 8 else 2
    wl = _wl(n_q, q_pos0, n_k, H, d, B, h, k, seed=kp + H, kp=kp)
    inp = W.generate(wl, fp8_keys=fp8)
    Qd, Kd, wd = oracle.decode_inputs(inp, fp8_keys=fp8)
    g = inputs_to_device(inp, fp8=fp8)
    Kdev = g["K8"] if fp8 else g["K"]
    ksc = g.get("k_scale")
    _, hl = lib.misa_pool_keys(Kdev, B, k_scale=ksc)
    heads, _ = lib.misa_route_heads(g["Q"], g["w"], hl, q_pos0, n_k, B, h)
    logits = lib.misa_score_tokens(g["Q"], g["w"], heads, g["K"], q_pos0)
    cand = lib.misa_topk(logits, q_pos0, n_k, kp)
    idx, full = lib.misa_rerank(g["Q"], g["w"], Kdev, cand, q_pos0, k, k_scale=ksc, want_full=True)
    cand, idx, full = cand.cpu().numpy(), idx.cpu().numpy(), full.cpu().numpy()
    # selection: bit-exact against the oracle's rule on the GPU's own scores
    assert np.array_equal(idx, oracle.select_candidates(full, cand, q_pos0, n_k, k))
    # scores: within tolerance of the fp64 all-head scores
    ref_idx, ref_full = oracle.rerank(Qd, wd, Kd, cand, q_pos0, k, want_logits=True)
    for t in range(n_q):
        valid = cand[t] >= 0
        c = cand[t, valid]
        dots = Qd[t] @ Kd[c].T
        mag = (np.abs(wd[t])[:, None] * np.maximum(dots, 0.0)).sum(axis=0)
        assert np.all(np.abs(full[t, valid] - ref_full[t, valid]) <= 2e-3 * mag + 1e-5)
        assert np.all(np.isneginf(full[t, ~valid]))
    assert recall(idx, ref_idx) >= 0.999


def test_rerank_whole_prefix_is_dense_topk(lib):
    # MISA-dagger with every prefix token as a candidate selects the dense top-k
    n_q, q_pos0, n_k, H, d, k = 24, 200, 240, 64, 128, 32
    inp = W.generate(_wl(n_q, q_pos0, n_k, H, d, 64, 8, k, seed=11))
    Qd, Kd, wd = oracle.decode_inputs(inp)
    g = inputs_to_device(inp)
    kp = n_k
    cand = np.full((n_q, kp), -1, dtype=np.int32)
    for t in range(n_q):
        cand[t, :q_pos0 + t + 1] = np.arange(q_pos0 + t + 1)
    idx, full = lib.misa_rerank(g["Q"], g["w"], g["K"], dev(cand), q_pos0, k, want_full=True)
    idx, full = idx.cpu().numpy(), full.cpu().numpy()
    # bit-exact against the oracle's rule on the GPU's own scores
    assert np.array_equal(idx, oracle.select_candidates(full, cand, q_pos0, n_k, k))
    # and the GPU's scores of the whole prefix, selected with the plain token
    # top-k, give the same tokens
    rows = np.full((n_q, n_k), -np.inf, dtype=np.float32)
    for t in range(n_q):
        rows[t, :q_pos0 + t + 1] = full[t, :q_pos0 + t + 1]
    assert np.array_equal(idx, oracle.topk(rows, q_pos0, n_k, k))
    dense_ref = oracle.topk(oracle.dense_logits(Qd, wd, Kd, q_pos0), q_pos0, n_k, k)
    assert recall(idx, dense_ref) >= 0.999


def _rerank_case(lib, seed, n_q=40, q_pos0=500, n_k=600, H=64, d=128, kp=256, k=64):
    inp = W.generate(_wl(n_q, q_pos0, n_k, H, d, 64, 8, k, seed=seed, kp=kp))
    g = inputs_to_device(inp)
    _, hl = lib.misa_pool_keys(g["K"], 64)
    heads, _ = lib.misa_route_heads(g["Q"], g["w"], hl, q_pos0, n_k, 64, 8)
    logits = lib.misa_score_tokens(g["Q"], g["w"], heads, g["K"], q_pos0)
    cand = lib.misa_topk(logits, q_pos0, n_k, kp)
    return g, cand


@pytest.mark.parametrize("k", [64, 256])
def test_rerank_any_candidate_order(lib, k):
    # candidates in a shuffled order (the -1 padding spread through the row,
    # some rows reversed): ties still go to the lower token and the tokens come
    # out ascending, equal to the selection from the ascending candidates
    n_q, q_pos0, n_k, kp = 40, 150, 600, 256     # rows 0..105 see fewer than kp tokens
    g, cand = _rerank_case(lib, seed=91, n_q=n_q, q_pos0=q_pos0, n_k=n_k, kp=kp, k=k)
    want, full_sorted = lib.misa_rerank(g["Q"], g["w"], g["K"], cand, q_pos0, k, want_full=True)
    rng = np.random.default_rng(92)
    c = cand.cpu().numpy()
    shuf = np.stack([c[t, ::-1] if t % 3 == 0 else c[t, rng.permutation(kp)] for t in range(n_q)])
    shuf = np.ascontiguousarray(shuf)
    got, full = lib.misa_rerank(g["Q"], g["w"], g["K"], dev(shuf), q_pos0, k, want_full=True)
    assert lib.misa_last_device_status() == lib.MISA_OK
    got, full = got.cpu().numpy(), full.cpu().numpy()
    assert np.array_equal(got, oracle.select_candidates(full, shuf, q_pos0, n_k, k))
    assert np.array_equal(got, want.cpu().numpy())
    # a candidate's score does not depend on where it sits in the row
    fs = full_sorted.cpu().numpy()
    for t in range(n_q):
        by_tok = dict(zip(c[t].tolist(), fs[t].tolist()))
        for tok, v in zip(shuf[t].tolist(), full[t].tolist()):
            assert v == by_tok[tok] or (tok < 0 and v == -np.inf)


def test_rerank_ties_in_any_order(lib):
    # every candidate of a row scores the same (identical keys): the k lowest
    # tokens are kept whatever the candidate order
    n_q, q_pos0, n_k, H, d, kp, k = 16, 900, 1000, 64, 128, 300, 100
    inp = W.generate(_wl(n_q, q_pos0, n_k, H, d, 64, 8, k, seed=93, kp=kp))
    g = inputs_to_device(inp)
    K = g["K"][:1].expand(n_k, d).contiguous()
    rng = np.random.default_rng(94)
    cand = np.stack([rng.choice(q_pos0 + t + 1, size=kp, replace=False)
                     for t in range(n_q)]).astype(np.int32)
    got, full = lib.misa_rerank(g["Q"], g["w"], K, dev(cand), q_pos0, k, want_full=True)
    assert lib.misa_last_device_status() == lib.MISA_OK
    got, full = got.cpu().numpy(), full.cpu().numpy()
    for t in range(n_q):
        assert np.all(full[t] == full[t, 0])
        assert np.array_equal(got[t], np.sort(cand[t])[:k])
    assert np.array_equal(got, oracle.select_candidates(full, cand, q_pos0, n_k, k))


def test_rerank_reports_repeated_candidates(lib):
    # a token listed twice breaks the contract: the kernel reports it in the
    # device status (all candidates kept, so the repeat is among the kept)
    g, cand = _rerank_case(lib, seed=95, kp=128, k=128)
    c = cand.cpu().numpy().copy()
    c[3, 7] = c[3, 11]
    lib.misa_rerank(g["Q"], g["w"], g["K"], dev(c), 500, 128)
    assert lib.misa_last_device_status() == lib.MISA_ERR_DEVICE
    lib.misa_rerank(g["Q"], g["w"], g["K"], cand, 500, 128)
    assert lib.misa_last_device_status() == lib.MISA_OK


# ------------------------------------------------------------------ whole path

def test_pipeline_tiny_matches_oracle():
    from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer
    wl = W.WORKLOADS["tiny_1k"]
    inp = W.generate(wl)
    Qd, Kd, wd = oracle.decode_inputs(inp)
    kbar = oracle.pool_keys(Kd, wl.B)
    r_ora, heads_ora = oracle.route(Qd, wd, kbar, wl.q_pos0, wl.n_k, wl.B, wl.h)
    ref = oracle.score(Qd, wd, heads_ora, Kd, wl.q_pos0)
    idx_ora = oracle.topk(ref, wl.q_pos0, wl.n_k, wl.k)
    g = inputs_to_device(inp)
    ix = MisaIndexer(IndexerShape(wl.n_q, wl.q_pos0, wl.n_k, wl.H, wl.d, wl.B, wl.h, wl.k))
    idx = ix.run(g["Q"], g["K"], g["w"]).cpu().numpy()
    heads = ix.heads.cpu().numpy()
    check_heads(heads, r_ora, heads_ora, wl.h)
    same = np.all(heads == heads_ora, axis=1)
    lg = ix.logits.cpu().numpy()
    assert np.array_equal(idx, oracle.topk(lg, wl.q_pos0, wl.n_k, wl.k))
    assert recall(idx[same], idx_ora[same]) >= 0.999
    assert lib_status_ok()


def lib_status_ok():
    from long_context_sparse_block_b200 import _lib
    return _lib.misa_last_device_status() == 0
