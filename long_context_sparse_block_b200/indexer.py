"""The MISA indexer pipeline over one prefill chunk, through the C ABI.

    pool -> route (top-h) -> for each query sub-chunk: fused score + top-k
                                                       [(top-k') -> rerank]

("MISA: Mixture of Indexer Sparse Attention", technical summary: Metodologia
steps 1-2 and Variante Hierarquica.)  Buffers are allocated once, with torch,
when the indexer is built; `run` only launches the library's kernels on the
current stream.  Scoring and selection run as one fused call (misa_score_topk),
which keeps only the logits above per-row sampled thresholds; the logits buffer
is its scratch.  Queries can be scored in sub-chunks to bound that buffer.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib


@dataclass
class IndexerShape:
    n_q: int
    q_pos0: int
    n_k: int
    H: int
    d: int
    B: int
    h: int          # routed heads (h == H with dense=True: the DSA indexer)
    k: int
    kp: int = 0     # MISA-dagger candidate count (0: plain MISA)
    dense: bool = False
    sub_chunk: int = 8192

    @property
    def M(self) -> int:
        return -(-self.n_k // self.B)


def _piece_bounds(n: int, pieces: int):
    """Query ranges of run_host: with three or more pieces the first and the last
    are half the even share (the first copy-in and the last copy-out are the
    only copies that nothing overlaps), the rest split what remains evenly."""
    pieces = max(1, min(pieces, n))
    if pieces < 3:
        step = -(-n // pieces)
        return [(c0, min(n, c0 + step)) for c0 in range(0, n, step)]
    edge = max(1, n // (2 * pieces))
    mid = n - 2 * edge
    cuts = [0, edge] + [edge + mid * i // (pieces - 2) for i in range(1, pieces - 2)] + [n - edge, n]
    return [(a, b) for a, b in zip(cuts, cuts[1:]) if b > a]


def ramp_pieces(n: int):
    """A piece schedule that starts small and grows: 3/64, 7/64, 12/64, 18/64
    and 20/64 of the queries, then a last piece of 4/64 (384, 896, 1536, 2304,
    2560 and 512 of 8192).  The first copy-in that nothing overlaps is short;
    each later piece arrives while the one before it is indexed (indexing a
    query takes about as long as copying it, plus a fixed cost per piece, so
    the pieces grow); the last piece's indexing and copy-out are short.  Chosen
    by measurement among nearby schedules on the 8192-query chunk."""
    parts = (3, 7, 12, 18, 20)
    sizes = [n * p // 64 for p in parts]
    if min(sizes) < 1:
        return [n]
    return sizes + [n - sum(sizes)]


def _bounds_of(n: int, pieces):
    """Query ranges of run_host for a piece count or for explicit piece sizes."""
    if isinstance(pieces, int):
        return _piece_bounds(n, pieces)
    out, c0 = [], 0
    for size in pieces:
        if size > 0 and c0 < n:
            out.append((c0, min(n, c0 + size)))
            c0 += size
    if c0 < n:
        out.append((c0, n))
    return out


class MisaIndexer:
    def __init__(self, shape: IndexerShape, device="cuda"):
        s = self.shape = shape
        dev = torch.device(device)
        self.sub = min(s.sub_chunk, s.n_q)
        self.kbar_hl = torch.empty((2, s.M, s.d), dtype=torch.int16, device=dev)
        self.heads = torch.empty((s.n_q, s.h), dtype=torch.int32, device=dev)
        ld = (s.n_k + 3) // 4 * 4   # 16-byte rows
        self.logits = torch.empty((self.sub, ld), dtype=torch.float32, device=dev)[:, :s.n_k]
        sel = s.kp if s.kp else s.k
        self.sel = torch.empty((s.n_q, sel), dtype=torch.int32, device=dev)
        nbytes = _lib.misa_workspace_size("score_topk", self.sub, s.n_k, sel, 0)
        self.ws_sel = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        if s.kp:
            self.final = torch.empty((s.n_q, s.k), dtype=torch.int32, device=dev)
            nbytes = _lib.misa_workspace_size("rerank", self.sub, s.n_k, s.k, s.kp)
            self.ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device=dev)
        else:
            self.final = self.sel

    def _scoring_keys(self, K, k_scale):
        """The keys the fused scoring reads: e4m3 keys decoded to bf16 codes once
        per chunk (scored with their scales), so that every query sub-chunk or
        piece does not decode them again; bf16 keys as they are."""
        if (k_scale is None or not isinstance(K, torch.Tensor)
                or K.dtype not in (torch.uint8, torch.float8_e4m3fn)):
            return K  # bf16 keys, or a paged cache (decoded inside the fused call)
        kd = getattr(self, "_kdec", None)
        if kd is None or kd.shape != K.shape or kd.device != K.device:
            kd = self._kdec = torch.empty(K.shape, dtype=torch.int16, device=K.device)
        return _lib.misa_keys_e4m3_to_bf16(K, out=kd)

    def _select(self, c0, c1, Q, K, w, k_scale, Ks=None):
        """Scoring, top-k (and the MISA-dagger rerank) of queries c0..c1-1 whose
        heads are routed; Q and w hold the whole chunk's rows.  Ks: the keys the
        scoring reads (K decoded, from _scoring_keys); the rerank reads K."""
        s = self.shape
        heads = None if s.dense else self.heads[c0:c1]
        _lib.misa_score_topk(Q[c0:c1], w[c0:c1], heads, K if Ks is None else Ks, s.q_pos0 + c0,
                             self.sel.shape[1], k_scale=k_scale, h=s.h, idx=self.sel[c0:c1],
                             logits=self.logits[:c1 - c0], ws=self.ws_sel)
        if s.kp:
            _lib.misa_rerank(Q[c0:c1], w[c0:c1], K, self.sel[c0:c1], s.q_pos0 + c0, s.k,
                             k_scale=k_scale, idx=self.final[c0:c1], ws=self.ws)

    def run(self, Q, K, w, k_scale=None, on_subchunk=None):
        """Q [n_q,H,d] bf16 codes, K [n_k,d] bf16 codes (or e4m3 + k_scale), w [n_q,H] f32.
        Returns the selected token indices [n_q, k] (int32, ascending, -1 padded).
        on_subchunk(c0, c1, logits), when given, switches to the unfused sequence
        (every logit written, then the top-k) and is called after each sub-chunk
        is scored, for inspection; the logits buffer is reused by the next one."""
        s = self.shape
        if not s.dense:
            _lib.misa_pool_keys(K, s.B, k_scale=k_scale, kbar_hl=self.kbar_hl, want_kbar=False)
            _lib.misa_route_heads(Q, w, self.kbar_hl, s.q_pos0, s.n_k, s.B, s.h, heads=self.heads)
        Ks = self._scoring_keys(K, k_scale) if on_subchunk is None else K
        for c0 in range(0, s.n_q, self.sub):
            c1 = min(s.n_q, c0 + self.sub)
            if on_subchunk is None:
                self._select(c0, c1, Q, K, w, k_scale, Ks)
                continue
            lg = self.logits[:c1 - c0]
            heads = None if s.dense else self.heads[c0:c1]
            _lib.misa_score_tokens(Q[c0:c1], w[c0:c1], heads, K, s.q_pos0 + c0,
                                   k_scale=k_scale, logits=lg, h=s.h)
            on_subchunk(c0, c1, lg)
            _lib.misa_topk(lg, s.q_pos0 + c0, s.n_k, self.sel.shape[1], idx=self.sel[c0:c1])
            if s.kp:
                _lib.misa_rerank(Q[c0:c1], w[c0:c1], K, self.sel[c0:c1], s.q_pos0 + c0, s.k,
                                 k_scale=k_scale, idx=self.final[c0:c1], ws=self.ws)
        return self.final

    def run_host(self, Qh, Kh, wh, out=None, k_scale_h=None, pieces=None, timeline=None):
        """End to end from host buffers (pin them for asynchronous copies): Q, K, w
        (and FP8 key scales) as in run(); returns the selected indices in `out`, a
        pinned host int32 [n_q, k] tensor (allocated when None), complete when the
        current stream reaches this point.  The queries go in pieces on three
        streams (copy in, index, copy out) so that the copies of one piece
        overlap the indexing of another; the keys go first.  `pieces`: a list of
        piece sizes (default ramp_pieces(n_q)) or a piece count (the first and
        last pieces small, see _piece_bounds).  `timeline` (a list, diagnostic):
        receives (label, timing event) pairs recorded at the start, after each
        copy in, after each piece is indexed and after each copy out."""
        s = self.shape
        dev = self.heads.device
        if getattr(self, "_dev", None) is None:
            self._dev = (torch.empty(Qh.shape, dtype=Qh.dtype, device=dev),
                         torch.empty(Kh.shape, dtype=Kh.dtype, device=dev),
                         torch.empty(wh.shape, dtype=wh.dtype, device=dev),
                         None if k_scale_h is None else
                         torch.empty(k_scale_h.shape, dtype=k_scale_h.dtype, device=dev))
            self._streams = (torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev))
        Q, K, w, ks = self._dev
        cin, cout = self._streams
        if out is None:
            out = torch.empty(tuple(self.final.shape), dtype=torch.int32, pin_memory=True)
        compute = torch.cuda.current_stream(dev)

        def mark(label, stream):
            if timeline is not None:
                ev = torch.cuda.Event(enable_timing=True)
                ev.record(stream)
                timeline.append((label, ev))

        mark("start", compute)
        cin.wait_stream(compute)   # the device buffers are free again
        cout.wait_stream(compute)
        bounds = _bounds_of(s.n_q, ramp_pieces(s.n_q) if pieces is None else pieces)
        ev_in = []
        with torch.cuda.stream(cin):
            K.copy_(Kh, non_blocking=True)
            if ks is not None:
                ks.copy_(k_scale_h, non_blocking=True)
            ev_k = torch.cuda.Event()
            ev_k.record(cin)
            mark("keys in", cin)
            for i, (c0, c1) in enumerate(bounds):
                Q[c0:c1].copy_(Qh[c0:c1], non_blocking=True)
                w[c0:c1].copy_(wh[c0:c1], non_blocking=True)
                e = torch.cuda.Event()
                e.record(cin)
                ev_in.append(e)
                mark(f"piece {i} in", cin)
        compute.wait_event(ev_k)
        if not s.dense:
            _lib.misa_pool_keys(K, s.B, k_scale=ks, kbar_hl=self.kbar_hl, want_kbar=False)
        Ks = self._scoring_keys(K, ks)
        for i, ((c0, c1), e) in enumerate(zip(bounds, ev_in)):
            compute.wait_event(e)
            if not s.dense:
                _lib.misa_route_heads(Q[c0:c1], w[c0:c1], self.kbar_hl, s.q_pos0 + c0, s.n_k,
                                      s.B, s.h, heads=self.heads[c0:c1])
            for a0 in range(c0, c1, self.sub):
                self._select(a0, min(c1, a0 + self.sub), Q, K, w, ks, Ks)
            done = torch.cuda.Event()
            done.record(compute)
            mark(f"piece {i} indexed", compute)
            cout.wait_event(done)
            with torch.cuda.stream(cout):
                out[c0:c1].copy_(self.final[c0:c1], non_blocking=True)
            mark(f"piece {i} out", cout)
        compute.wait_stream(cout)
        return out
