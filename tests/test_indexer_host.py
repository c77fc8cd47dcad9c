"""Host orchestration of the chunk pipeline (no GPU): the calls MisaIndexer.run
makes into the library, recorded by a stand-in for the binding — which stages
run, on which query rows, at which positions, with which buffers."""
import pytest
import torch

from long_context_sparse_block_b200 import indexer as ixmod
from long_context_sparse_block_b200.indexer import IndexerShape, MisaIndexer


class _Recorder:
    """Stands in for the binding: records (name, arguments) of every call."""

    def __init__(self):
        self.calls = []

    def misa_workspace_size(self, op, n_q, n_k, k, kp):
        return 64

    def __getattr__(self, name):
        if not name.startswith("misa_"):
            raise AttributeError(name)

        def call(*args, **kw):
            self.calls.append((name, args, kw))
        return call

    def named(self, name):
        return [(a, kw) for n, a, kw in self.calls if n == name]


@pytest.fixture
def fake(monkeypatch):
    rec = _Recorder()
    monkeypatch.setattr(ixmod, "_lib", rec)
    return rec


def _inputs(s):
    Q = torch.zeros((s.n_q, s.H, s.d), dtype=torch.int16)
    K = torch.zeros((s.n_k, s.d), dtype=torch.int16)
    w = torch.zeros((s.n_q, s.H), dtype=torch.float32)
    return Q, K, w


def _rows(t, base):
    """The row range [r0, r1) of `base` that the view `t` covers."""
    per = base.stride(0) * base.element_size()
    r0 = (t.data_ptr() - base.data_ptr()) // per
    return r0, r0 + t.shape[0]


def test_fused_path_covers_every_query_once(fake):
    s = IndexerShape(n_q=1000, q_pos0=5000, n_k=6000, H=8, d=64, B=64, h=2, k=32, sub_chunk=384)
    ix = MisaIndexer(s, device="cpu")
    Q, K, w = _inputs(s)
    out = ix.run(Q, K, w)
    assert out is ix.sel
    assert len(fake.named("misa_pool_keys")) == 1
    assert len(fake.named("misa_route_heads")) == 1
    (ra, rkw), = fake.named("misa_route_heads")
    assert ra[3:7] == (s.q_pos0, s.n_k, s.B, s.h) and rkw["heads"] is ix.heads
    calls = fake.named("misa_score_topk")
    assert len(calls) == 3                                      # 384 + 384 + 232 rows
    covered = []
    for a, kw in calls:
        r0, r1 = _rows(a[0], Q)
        assert _rows(a[1], w) == (r0, r1) and _rows(a[2], ix.heads) == (r0, r1)
        assert a[4] == s.q_pos0 + r0                            # position of the first row
        assert a[5] == s.k and kw["h"] == s.h
        assert _rows(kw["idx"], ix.sel) == (r0, r1)
        assert kw["logits"].shape[0] == r1 - r0 and kw["ws"] is ix.ws_sel
        covered.append((r0, r1))
    assert covered == [(0, 384), (384, 768), (768, 1000)]
    assert not fake.named("misa_rerank") and not fake.named("misa_score_tokens")


def test_dagger_reranks_each_subchunk_into_the_final_buffer(fake):
    s = IndexerShape(n_q=300, q_pos0=9000, n_k=9300, H=16, d=128, B=128, h=4, k=16, kp=64,
                     sub_chunk=128)
    ix = MisaIndexer(s, device="cpu")
    Q, K, w = _inputs(s)
    out = ix.run(Q, K, w)
    assert out is ix.final and ix.final.shape == (300, 16) and ix.sel.shape == (300, 64)
    sel_calls = fake.named("misa_score_topk")
    rr = fake.named("misa_rerank")
    assert len(sel_calls) == len(rr) == 3
    for (a, kw), (b, kw2) in zip(sel_calls, rr):
        r0, r1 = _rows(a[0], Q)
        assert a[5] == s.kp                                     # coarse stage keeps k'
        assert _rows(b[3], ix.sel) == (r0, r1)                  # candidates of the same rows
        assert b[4] == s.q_pos0 + r0 and b[5] == s.k
        assert _rows(kw2["idx"], ix.final) == (r0, r1) and kw2["ws"] is ix.ws


def test_dense_mode_skips_pool_and_route(fake):
    s = IndexerShape(n_q=64, q_pos0=100, n_k=164, H=8, d=64, B=64, h=8, k=8, dense=True)
    ix = MisaIndexer(s, device="cpu")
    Q, K, w = _inputs(s)
    ix.run(Q, K, w)
    assert not fake.named("misa_pool_keys") and not fake.named("misa_route_heads")
    (a, kw), = fake.named("misa_score_topk")
    assert a[2] is None and kw["h"] == 8


def test_unfused_sequence_hands_each_subchunk_to_the_callback(fake):
    s = IndexerShape(n_q=500, q_pos0=0, n_k=500, H=8, d=32, B=64, h=2, k=8, sub_chunk=200)
    ix = MisaIndexer(s, device="cpu")
    Q, K, w = _inputs(s)
    seen = []
    ix.run(Q, K, w, on_subchunk=lambda c0, c1, lg: seen.append((c0, c1, lg.shape[0])))
    assert seen == [(0, 200, 200), (200, 400, 200), (400, 500, 100)]
    sc = fake.named("misa_score_tokens")
    tk = fake.named("misa_topk")
    assert len(sc) == len(tk) == 3
    for (a, kw), (b, kw2), (c0, c1, _) in zip(sc, tk, seen):
        assert _rows(a[0], Q) == (c0, c1) and a[4] == s.q_pos0 + c0
        assert b[1] == s.q_pos0 + c0 and b[2] == s.n_k and b[3] == s.k
        assert _rows(kw2["idx"], ix.sel) == (c0, c1)
    assert not fake.named("misa_score_topk")


def test_piece_schedules_cover_the_queries_once():
    from long_context_sparse_block_b200.indexer import _bounds_of, ramp_pieces
    for n in (1, 7, 100, 1000, 8192, 12345):
        for pieces in (1, 3, 4, 8, ramp_pieces(n), [n // 2, n], [5, 0, 3]):
            b = _bounds_of(n, pieces)
            assert b[0][0] == 0 and b[-1][1] == n
            assert all(c1 > c0 for c0, c1 in b)
            assert all(b[i][1] == b[i + 1][0] for i in range(len(b) - 1))
    r = ramp_pieces(8192)
    assert r == [384, 896, 1536, 2304, 2560, 512]
    assert ramp_pieces(10) == [10]
