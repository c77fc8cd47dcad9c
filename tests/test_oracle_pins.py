"""Pins for the CPU oracle, against things other than itself.

Each test checks the oracle against a hand-derived worked example, a closed form,
a library routine, brute-force enumeration, or a structural invariant that the
MISA pages state ("MISA: Mixture of Indexer Sparse Attention"; abstract and
technical summary):
  * with every head routed the routed scorer is the dense DSA indexer;
  * MISA-dagger with a candidate set holding the whole prefix is the dense top-k;
  * with blocks of one key, the pooled keys are the keys;
  * nothing after position pos(t) reaches query t.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from long_context_sparse_block_b200 import workloads as wlmod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_case(seed, n_q=9, q_pos0=3, n_k=12, H=4, d=5, scale=1.0):
    rng = np.random.default_rng(seed)
    Q = rng.standard_normal((n_q, H, d)) * scale
    K = rng.standard_normal((n_k, d))
    w = rng.standard_normal((n_q, H))
    return Q, K, w, q_pos0


# ---------------------------------------------------------------- storage formats

def test_bf16_decode_known_codes():
    assert oracle.bf16_value(0x3F80) == 1.0
    assert oracle.bf16_value(0xC000) == -2.0
    assert oracle.bf16_value(0x3F81) == 1.0 + 2.0 ** -7
    assert oracle.bf16_value(0x0000) == 0.0
    assert math.copysign(1.0, oracle.bf16_value(0x8000)) == -1.0
    assert math.isinf(oracle.bf16_value(0x7F80))
    assert oracle.bf16_value(0x0080) == 2.0 ** -126          # smallest normal


def test_bf16_round_to_nearest_even():
    # 1 + 2^-8 is halfway between 1 and 1 + 2^-7: ties go to the even code 0x3F80
    assert wlmod.bf16_bits(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3*2^-8 is halfway between 0x3F81 and 0x3F82: even is 0x3F82
    assert wlmod.bf16_bits(1.0 + 3 * 2.0 ** -8) == 0x3F82
    assert wlmod.bf16_bits(1.0 + 2.0 ** -8 + 2.0 ** -20) == 0x3F81
    codes = np.arange(0x0080, 0x7F80, 7, dtype=np.uint16)
    vals = oracle.bf16_to_f64(codes)
    assert np.array_equal(wlmod.bf16_bits(vals), codes)
    assert np.array_equal(wlmod.bf16_bits(-vals), codes | 0x8000)


def test_e4m3_decode_ocp_table():
    # OCP 8-bit floating point spec, E4M3: bias 7, max normal S.1111.110 = 448,
    # min normal 2^-6, subnormals m * 2^-9, NaN S.1111.111, no infinities.
    assert oracle.e4m3_value(0x7E) == 448.0
    assert oracle.e4m3_value(0xFE) == -448.0
    assert oracle.e4m3_value(0x08) == 2.0 ** -6
    assert oracle.e4m3_value(0x01) == 2.0 ** -9
    assert oracle.e4m3_value(0x07) == 7 * 2.0 ** -9
    assert oracle.e4m3_value(0x38) == 1.0
    assert oracle.e4m3_value(0x39) == 1.125
    assert oracle.e4m3_value(0xB8) == -1.0
    assert oracle.e4m3_value(0x00) == 0.0
    assert math.isnan(oracle.e4m3_value(0x7F))
    assert math.isnan(oracle.e4m3_value(0xFF))


def test_e4m3_encoder_and_decoder_agree_on_every_code():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)], dtype=np.uint8)
    vals = np.array([oracle.e4m3_value(int(c)) for c in codes])
    assert np.array_equal(wlmod.e4m3_encode(vals), codes)
    # ties to even: halfway between 1.0 (0x38) and 1.125 (0x39) goes to 0x38
    assert wlmod.e4m3_encode(1.0625) == 0x38
    assert wlmod.e4m3_encode(1.1875) == 0x3A
    assert wlmod.e4m3_encode(1000.0) == 0x7E            # saturates


def test_e4m3_keys_dequantise_per_token():
    codes = np.array([[0x38, 0xB8], [0x7E, 0x01]], dtype=np.uint8)
    scale = np.array([0.5, 2.0], dtype=np.float32)
    K = oracle.e4m3_keys_to_f64(codes, scale)
    assert np.array_equal(K, [[0.5, -0.5], [896.0, 2.0 ** -8]])


def test_e4m3_queries_quantise_per_query_head_row():
    # each (query, head) row gets its own scale amax/448 (1 for a zero row); the
    # row maximum maps to the largest code, and decoding through the oracle
    # recovers every value within half an e4m3 step
    rng = np.random.default_rng(3)
    Q = rng.standard_normal((3, 2, 16)) * np.array([1.0, 1e-3])[None, :, None]
    Q[2, 1] = 0.0
    codes, scale = wlmod.e4m3_quantize_queries(Q)
    assert codes.shape == (3, 2, 16) and scale.shape == (3, 2)
    assert scale[2, 1] == 1.0 and not codes[2, 1].any()
    for t in range(3):
        for j in range(2):
            if not Q[t, j].any():
                continue
            assert scale[t, j] == np.float32(np.abs(Q[t, j]).max() / 448.0)
            assert (codes[t, j] & 0x7F).max() == 0x7E
    inp = {"Q8": codes, "q_scale": scale, "K": np.zeros((1, 16), np.uint16),
           "w": np.zeros((3, 2), np.float32)}
    Qd, _, _ = oracle.decode_inputs(inp, fp8_queries=True)
    y = Q / scale.astype(np.float64)[..., None]
    step = np.where(np.abs(y) >= 2.0 ** -6, 2.0 ** (np.floor(np.log2(np.maximum(np.abs(y), 1e-300))) - 3),
                    2.0 ** -9)
    assert np.all(np.abs(Qd / scale.astype(np.float64)[..., None] - y) <= step / 2 + 1e-12)


# ---------------------------------------------------------------- worked example

def test_worked_example_every_stage():
    g = json.load(open(os.path.join(GOLDEN, "worked_example_4x4.json")))
    s = g["shape"]
    K = np.array(g["K"], dtype=np.float64)
    Q = np.tile(np.array(g["Q_every_query"], dtype=np.float64), (s["n_q"], 1, 1))
    w = np.tile(np.array(g["w_every_query"]), (s["n_q"], 1))
    kbar = oracle.pool_keys(K, s["B"])
    assert np.array_equal(kbar, g["kbar"])
    r, heads = oracle.route(Q, w, kbar, s["q_pos0"], s["n_k"], s["B"], s["h"])
    assert np.array_equal(r, g["r"])
    assert np.array_equal(heads, g["heads"])
    lg = oracle.score(Q, w, heads, K, s["q_pos0"])
    for t, row in enumerate(g["logits_causal"]):
        assert np.array_equal(lg[t, :t + 1], row)
        assert np.all(np.isneginf(lg[t, t + 1:]))
    assert np.array_equal(oracle.topk(lg, s["q_pos0"], s["n_k"], s["k"]), g["topk"])
    dense = oracle.dense_logits(Q, w, K, s["q_pos0"])
    assert np.array_equal(dense[3], g["dense_logits_t3"])
    assert np.array_equal(oracle.topk(dense[3:4], 3, s["n_k"], 2)[0], g["dense_topk_t3"])
    dg = g["dagger_t3"]
    idx = oracle.rerank(Q[3:4], w[3:4], K, np.array([dg["cand"]]), 3, dg["k"])
    assert np.array_equal(idx[0], dg["idx"])


# ---------------------------------------------------------------- pooling

def test_pool_blocks_of_one_are_the_keys():
    _, K, _, _ = _rand_case(1, n_k=37)
    assert np.array_equal(oracle.pool_keys(K, 1), K)


def test_pool_arithmetic_sequence_closed_form():
    n_k, d, B = 23, 3, 5                       # ragged last block of 3 rows
    s = np.arange(n_k, dtype=np.float64)
    K = np.stack([s, 2 * s + 1, -s], axis=1)
    kbar = oracle.pool_keys(K, B)
    for m in range(kbar.shape[0]):
        n_m = min(B, n_k - m * B)
        mid = m * B + (n_m - 1) / 2.0          # mean of an arithmetic run
        assert np.array_equal(kbar[m], [mid, 2 * mid + 1, -mid])


# ---------------------------------------------------------------- router

@pytest.mark.parametrize("B", [1, 3, 4])
def test_route_constant_keys_closed_form(B):
    rng = np.random.default_rng(5)
    n_q, H, d, n_k, q_pos0, h = 11, 5, 4, 14, 2, 2
    v = np.array([0.5, -1.0, 2.0, 0.25])
    K = np.tile(v, (n_k, 1))
    Q = rng.integers(-3, 4, size=(n_q, H, d)).astype(np.float64)
    w = rng.integers(-2, 3, size=(n_q, H)).astype(np.float64) / 4.0
    kbar = oracle.pool_keys(K, B)
    r, heads = oracle.route(Q, w, kbar, q_pos0, n_k, B, h)
    for t in range(n_q):
        pos = q_pos0 + t
        nC = min((pos + 1) // B, n_k // B)
        assert oracle.causal_blocks(pos, n_k, B) == nC
        expect = nC * w[t] * np.maximum(Q[t] @ v, 0.0)   # integer-valued products: exact
        assert np.array_equal(r[t], expect)


def test_route_complete_blocks_boundary():
    # pos = B-2: the first block is not complete yet; pos = B-1: it is.
    B, d, H = 4, 2, 3
    K = np.ones((8, d))
    Q = np.ones((2, H, d))
    w = np.array([[1.0, 2.0, 3.0], [1.0, 2.0, 3.0]])
    kbar = oracle.pool_keys(K, B)
    r, heads = oracle.route(Q, w, kbar, B - 2, 8, B, 2)
    assert np.array_equal(r[0], [0, 0, 0])           # nothing complete: all zero
    assert np.array_equal(heads[0], [0, 1])          # ties to the lower head index
    assert np.array_equal(r[1], [2.0, 4.0, 6.0])     # one block, q.kbar = 2
    assert np.array_equal(heads[1], [1, 2])


def test_route_negative_weight_ranks_last():
    K = np.ones((4, 2))
    Q = np.ones((1, 3, 2))
    w = np.array([[-1.0, 0.5, 0.25]])
    kbar = oracle.pool_keys(K, 2)
    r, heads = oracle.route(Q, w, kbar, 3, 4, 2, 2)
    assert np.array_equal(r[0], [-4.0, 2.0, 1.0])
    assert np.array_equal(heads[0], [1, 2])


def _dominates(vals, i, j):
    return vals[i] > vals[j] or (vals[i] == vals[j] and i < j)


def _brute_force_best_subset(vals, size):
    """The unique subset whose every member ranks before every non-member."""
    n = len(vals)
    winners = []
    for S in itertools.combinations(range(n), size):
        rest = [j for j in range(n) if j not in S]
        if all(_dominates(vals, i, j) for i in S for j in rest):
            winners.append(list(S))
    assert len(winners) == 1
    return winners[0]


@pytest.mark.parametrize("seed", range(6))
def test_top_h_matches_brute_force(seed):
    rng = np.random.default_rng(100 + seed)
    n_q, H, d, n_k, B, h = 6, 6, 3, 12, 2, 3
    # small-integer inputs make ties frequent
    Q = rng.integers(-1, 2, size=(n_q, H, d)).astype(np.float64)
    K = rng.integers(-1, 2, size=(n_k, d)).astype(np.float64)
    w = rng.integers(-1, 3, size=(n_q, H)).astype(np.float64)
    kbar = oracle.pool_keys(K, B)
    r, heads = oracle.route(Q, w, kbar, 4, n_k, B, h)
    for t in range(n_q):
        assert list(heads[t]) == _brute_force_best_subset(list(r[t]), h)


# ---------------------------------------------------------------- scoring

def test_score_basis_keys_closed_form():
    # K rows are unit vectors e_{s mod d}, so q . k_s = q[s mod d].
    n_q, H, d, n_k, q_pos0 = 3, 4, 3, 7, 2
    K = np.zeros((n_k, d))
    K[np.arange(n_k), np.arange(n_k) % d] = 1.0
    rng = np.random.default_rng(7)
    Q = rng.integers(-4, 5, size=(n_q, H, d)).astype(np.float64)
    w = np.array([[1.0, -0.5, 2.0, 0.25]] * n_q)
    heads = np.array([[0, 2], [1, 3], [2, 3]], dtype=np.int32)
    lg = oracle.score(Q, w, heads, K, q_pos0)
    for t in range(n_q):
        for s in range(n_k):
            if s > q_pos0 + t:
                assert lg[t, s] == -np.inf
            else:
                expect = sum(w[t, j] * max(Q[t, j, s % d], 0.0) for j in heads[t])
                assert lg[t, s] == expect


@pytest.mark.parametrize("seed", range(3))
def test_all_heads_routed_is_the_dense_indexer(seed):
    Q, K, w, q_pos0 = _rand_case(seed, n_q=7, n_k=15, H=5)
    kbar = oracle.pool_keys(K, 3)
    r, heads = oracle.route(Q, w, kbar, q_pos0, K.shape[0], 3, Q.shape[1])
    assert np.array_equal(heads, np.tile(np.arange(5), (7, 1)))
    routed = oracle.score(Q, w, heads, K, q_pos0)
    dense = oracle.dense_logits(Q, w, K, q_pos0)
    assert np.array_equal(routed, dense)          # bit-for-bit in fp64


# ---------------------------------------------------------------- top-k

def _library_topk(row, n, k):
    order = np.lexsort((np.arange(n), -row[:n]))   # stable: value desc, index asc
    sel = np.sort(order[:k])
    out = -np.ones(k, dtype=np.int64)
    out[:len(sel)] = sel
    return out


@pytest.mark.parametrize("seed", range(4))
def test_topk_equals_library_sort(seed):
    rng = np.random.default_rng(seed)
    n_q, n_k, q_pos0, k = 6, 300, 100, 37
    lg = rng.integers(-20, 20, size=(n_q, n_k)).astype(np.float64) / 8.0  # heavy ties
    idx = oracle.topk(lg, q_pos0, n_k, k)
    for t in range(n_q):
        assert np.array_equal(idx[t], _library_topk(lg[t], q_pos0 + t + 1, k))


@pytest.mark.parametrize("seed", range(5))
def test_topk_matches_brute_force(seed):
    rng = np.random.default_rng(50 + seed)
    vals = rng.integers(-2, 3, size=9).astype(np.float64)
    k = 4
    idx = oracle.topk(vals[None, :], 8, 9, k)[0]
    assert list(idx) == _brute_force_best_subset(list(vals), k)


def test_topk_edge_rows():
    neg0 = np.array([[0.0, -0.0, 0.0, -0.0, 1.0]])
    assert list(oracle.topk(neg0, 4, 5, 3)[0]) == [0, 1, 4]      # -0.0 ties +0.0
    f32 = neg0.astype(np.float32)
    assert list(oracle.topk(f32, 4, 5, 3)[0]) == [0, 1, 4]
    same = np.full((1, 10), 0.5)
    assert list(oracle.topk(same, 9, 10, 4)[0]) == [0, 1, 2, 3]
    short = np.array([[3.0, 1.0, 2.0, 9.0]])
    assert list(oracle.topk(short, 2, 4, 5)[0]) == [0, 1, 2, -1, -1]  # pos 2: 3 tokens
    assert list(oracle.topk(short, 3, 4, 0)[0]) == []


# ---------------------------------------------------------------- MISA-dagger

@pytest.mark.parametrize("seed", range(3))
def test_dagger_with_whole_prefix_is_dense_topk(seed):
    Q, K, w, q_pos0 = _rand_case(seed, n_q=8, n_k=20, H=6, d=4, q_pos0=5)
    n_k, B, h, k = K.shape[0], 4, 2, 5
    kbar = oracle.pool_keys(K, B)
    _, heads = oracle.route(Q, w, kbar, q_pos0, n_k, B, h)
    lg = oracle.score(Q, w, heads, K, q_pos0)
    kp = n_k                                        # >= pos(t)+1 for every query
    cand = oracle.topk(lg, q_pos0, n_k, kp)
    idx = oracle.rerank(Q, w, K, cand, q_pos0, k)
    dense = oracle.dense_logits(Q, w, K, q_pos0)
    assert np.array_equal(idx, oracle.topk(dense, q_pos0, n_k, k))


def test_rerank_ignores_padding_and_out_of_range():
    Q, K, w, _ = _rand_case(3, n_q=1, n_k=10, H=3, d=4)
    pos = 6
    cand = np.array([[4, -1, 9, 2, 7, 0]], dtype=np.int32)     # 9 and 7 are > pos
    idx, full = oracle.rerank(Q, w, K, cand, pos, 5, want_logits=True)
    dense = oracle.dense_logits(Q, w, K, pos)[0]
    valid = [4, 2, 0]
    assert np.all(np.isneginf(full[0, [1, 2, 4]]))
    assert np.array_equal(full[0, [0, 3, 5]], dense[valid])
    assert list(idx[0]) == sorted(valid) + [-1, -1]


# ---------------------------------------------------------------- causality

def test_no_future_input_reaches_a_query():
    Q, K, w, q_pos0 = _rand_case(11, n_q=6, n_k=16, H=4, d=3, q_pos0=4)
    n_k, B, h, k = 16, 2, 2, 3

    def run(Q, K, w):
        kbar = oracle.pool_keys(K, B)
        r, heads = oracle.route(Q, w, kbar, q_pos0, n_k, B, h)
        lg = oracle.score(Q, w, heads, K, q_pos0)
        return r, heads, lg, oracle.topk(lg, q_pos0, n_k, k)

    base = run(Q, K, w)
    rng = np.random.default_rng(0)
    for t in range(6):
        pos = q_pos0 + t
        K2, Q2, w2 = K.copy(), Q.copy(), w.copy()
        K2[pos + 1:] = rng.standard_normal(K2[pos + 1:].shape) * 10
        Q2[t + 1:] = rng.standard_normal(Q2[t + 1:].shape)
        w2[t + 1:] = -w2[t + 1:]
        pert = run(Q2, K2, w2)
        assert np.array_equal(pert[0][t], base[0][t])
        assert np.array_equal(pert[1][t], base[1][t])
        assert np.array_equal(pert[2][t, :pos + 1], base[2][t, :pos + 1])
        assert np.array_equal(pert[3][t], base[3][t])


# ---------------------------------------------------------------- cost model

def test_cost_counters_match_the_complexity_model():
    # per query: router H_I*d*|C(t)| and scoring h*d*(pos+1) multiply-adds,
    # i.e. O(H_I M + h L) (technical summary, Metodologia).
    Q, K, w, q_pos0 = _rand_case(2, n_q=9, n_k=30, H=6, d=4, q_pos0=21)
    n_k, B, h = 30, 4, 2
    kbar = oracle.pool_keys(K, B)
    cr, cs, cd = oracle._Counter(), oracle._Counter(), oracle._Counter()
    _, heads = oracle.route(Q, w, kbar, q_pos0, n_k, B, h, counter=cr)
    lg = oracle.score(Q, w, heads, K, q_pos0, counter=cs)
    pos = q_pos0 + np.arange(9)
    assert cr.v.value == sum(6 * 4 * min((p + 1) // B, n_k // B) for p in pos)
    assert cs.v.value == sum(h * 4 * (p + 1) for p in pos)
    cand = oracle.topk(lg, q_pos0, n_k, 7)
    oracle.rerank(Q, w, K, cand, q_pos0, 3, counter=cd)
    assert cd.v.value == 9 * 7 * 6 * 4


# ---------------------------------------------------------------- generators

def test_generators_are_seeded_and_shaped():
    wl = wlmod.small_workload("t", n_q=40, q_pos0=200, n_k=240, H=8, d=32, B=16, h=2, k=8,
                              seed=4, generator="clustered", n_needles=4)
    a = wlmod.generate(wl, fp8_keys=True)
    b = wlmod.generate(wl, fp8_keys=True)
    for key in ("Q", "K", "w", "K8", "k_scale", "needles"):
        assert np.array_equal(a[key], b[key])
    assert a["Q"].shape == (40, 8, 32) and a["Q"].dtype == np.uint16
    assert a["K"].shape == (240, 32) and a["w"].shape == (40, 8)
    # needles are the last query's head-0 row, below its position
    assert np.all(a["needles"] < 200 + 39)
    for s in a["needles"]:
        assert np.array_equal(a["K"][s], a["Q"][-1, 0])
    # w in the clustered recipe holds bf16 values
    assert np.array_equal(wlmod.bf16_values(wlmod.bf16_bits(a["w"].astype(np.float64))), a["w"])
    # fp8 keys: dequantised rows are within e4m3 precision of the bf16 rows
    Kd = oracle.e4m3_keys_to_f64(a["K8"], a["k_scale"])
    Kb = oracle.bf16_to_f64(a["K"])
    amax = np.abs(Kb).max(axis=1, keepdims=True)
    assert np.all(np.abs(Kd - Kb) <= amax * 2.0 ** -4 + 1e-12)


def test_workload_pair_counts():
    # causal (query, key) pairs of the four shapes, sum over t of pos(t)+1
    W = wlmod.WORKLOADS
    assert W["tiny_1k"].causal_pairs() == 524_800
    assert W["dsv32_32k"].causal_pairs() == 536_887_296
    assert W["glm5_64k"].causal_pairs() == 2_147_516_416
    assert W["chunk_128k"].causal_pairs() == 1_040_191_488
    assert W["chunk_128k"].M == 1024


# ---------------------------------------------------------------- candidate selection

@pytest.mark.parametrize("seed", range(4))
def test_select_candidates_matches_brute_force(seed):
    rng = np.random.default_rng(300 + seed)
    pos, n_k, k = 11, 14, 3
    cand = np.array([[0, 2, 3, 5, 6, 9, 11, -1, 13]], dtype=np.int32)   # 13 > pos: ignored
    vals = rng.integers(-2, 3, size=(1, 9)).astype(np.float32)
    vals[0, 4] = -np.inf                                                 # absent
    idx = oracle.select_candidates(vals, cand, pos, n_k, k)[0]
    valid = [i for i in range(9) if 0 <= cand[0, i] <= pos and vals[0, i] != -np.inf]
    best = _brute_force_best_subset([float(vals[0, i]) for i in valid], k)
    assert list(idx) == sorted(int(cand[0, valid[b]]) for b in best)


def test_select_candidates_agrees_with_rerank_on_exact_scores():
    rng = np.random.default_rng(9)
    n_q, H, d, n_k, pos0 = 4, 3, 4, 20, 12
    Q = rng.integers(-2, 3, size=(n_q, H, d)).astype(np.float64)
    K = rng.integers(-2, 3, size=(n_k, d)).astype(np.float64)
    w = rng.integers(-2, 3, size=(n_q, H)).astype(np.float64) / 2.0
    cand = np.sort(rng.choice(13, size=(n_q, 8), replace=True), axis=1).astype(np.int32)
    for t in range(n_q):                                    # distinct, ascending
        cand[t] = np.sort(rng.choice(pos0 + t + 1, size=8, replace=False))
    idx, full = oracle.rerank(Q, w, K, cand, pos0, 5, want_logits=True)
    sel = oracle.select_candidates(full.astype(np.float32), cand, pos0, n_k, 5)
    assert np.array_equal(sel, idx)      # integer-valued scores: exact in fp32


# ---------------------------------------------------------------- homogeneity

@pytest.mark.parametrize("seed", range(3))
def test_positive_scaling_of_keys_weights_and_queries(seed):
    # ReLU is positively homogeneous and the scores are linear in w: scaling K,
    # Q or w by a power of two c > 0 scales every router score and logit by c
    # (exactly) and changes no selection; c < 0 on the keys flips which dot
    # products the ReLU keeps, so the logits are NOT -c times the originals
    Q, K, w, q_pos0 = _rand_case(seed, n_q=6, q_pos0=9, n_k=15, H=6, d=4)
    B, h, k = 3, 3, 5
    n_k = K.shape[0]
    kbar = oracle.pool_keys(K, B)
    r, heads = oracle.route(Q, w, kbar, q_pos0, n_k, B, h)
    lg = oracle.score(Q, w, heads, K, q_pos0)
    sel = oracle.topk(lg, q_pos0, n_k, k)
    for c in (0.25, 4.0):
        for which in ("K", "Q", "w"):
            Q2, K2, w2 = (Q * c if which == "Q" else Q), (K * c if which == "K" else K), \
                (w * c if which == "w" else w)
            r2, heads2 = oracle.route(Q2, w2, oracle.pool_keys(K2, B), q_pos0, n_k, B, h)
            assert np.array_equal(r2, r * c) and np.array_equal(heads2, heads)
            lg2 = oracle.score(Q2, w2, heads, K2, q_pos0)
            fin = np.isfinite(lg)
            assert np.array_equal(lg2[fin], lg[fin] * c)
            assert np.array_equal(oracle.topk(lg2, q_pos0, n_k, k), sel)
    lg_neg = oracle.score(Q, w, heads, -K, q_pos0)
    fin = np.isfinite(lg)
    assert not np.allclose(lg_neg[fin], -lg[fin])


def test_scores_are_linear_in_the_head_weights():
    Q, K, w, q_pos0 = _rand_case(11, n_q=5, q_pos0=6, n_k=12, H=4, d=3)
    heads = np.tile(np.array([0, 2, 3], dtype=np.int32), (5, 1))
    rng = np.random.default_rng(12)
    w2 = rng.standard_normal(w.shape)
    a = oracle.score(Q, w, heads, K, q_pos0)
    b = oracle.score(Q, w2, heads, K, q_pos0)
    ab = oracle.score(Q, w + w2, heads, K, q_pos0)
    fin = np.isfinite(a)
    assert np.allclose(ab[fin], a[fin] + b[fin], rtol=1e-12, atol=1e-12)
