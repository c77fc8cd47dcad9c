"""ctypes binding of libmisa.so — argument marshalling only.

Every function here checks tensor devices/dtypes/shapes, allocates outputs with
torch when the caller gives none, and calls the C entry point of the same name
on the current torch CUDA stream.  No step of the indexer runs in Python; when
the library is missing the import fails loudly.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmisa.so")

MISA_OK = 0
MISA_ERR_INVALID_ARG = -1
MISA_ERR_UNSUPPORTED = -2
MISA_ERR_CUDA = -3
MISA_ERR_TIMEOUT = -4
MISA_ERR_WORKSPACE = -5
MISA_ERR_DEVICE = -6
MISA_K_BF16 = 0
MISA_K_FP8E4M3 = 1
MISA_K_BF16_SCALED = 2


class MisaError(RuntimeError):
    def __init__(self, fn: str, status: int, text: str):
        super().__init__(f"{fn} -> {status} ({text})")
        self.status = status


_vp, _i64, _int, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_size_t
_SIGS = {
    "misa_pool_keys": (_int, [_vp, _vp, _int, _i64, _int, _int, _vp, _vp, _vp]),
    "misa_pool_keys_range": (_int, [_vp, _vp, _int, _i64, _int, _int, _i64, _i64, _vp, _vp, _vp]),
    "misa_route_heads": (_int, [_vp, _vp, _vp, _int, _i64, _i64, _int, _int, _int, _int, _vp, _vp,
                                _vp]),
    "misa_score_tokens": (_int, [_vp, _vp, _vp, _vp, _vp, _int, _int, _i64, _i64, _int, _int, _int,
                                 _vp, _i64, _vp]),
    "misa_score_tokens_fp8": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _int, _i64, _i64, _int, _int,
                                     _int, _vp, _i64, _vp]),
    "misa_topk": (_int, [_vp, _i64, _int, _i64, _i64, _int, _vp, _vp, _sz, _vp]),
    "misa_rerank": (_int, [_vp, _vp, _vp, _vp, _int, _vp, _int, _int, _i64, _i64, _int, _int, _int,
                           _vp, _vp, _vp, _sz, _vp]),
    "misa_rerank_noalloc": (_int, [_vp, _vp, _vp, _vp, _int, _vp, _int, _int, _i64, _i64, _int,
                                   _int, _int, _vp, _vp]),
    "misa_score_topk": (_int, [_vp, _vp, _vp, _vp, _vp, _int, _int, _i64, _i64, _int, _int, _int,
                               _int, _vp, _vp, _i64, _vp, _sz, _vp]),
    "misa_keys_e4m3_to_bf16": (_int, [_vp, _i64, _int, _vp, _vp]),
    "misa_pool_keys_paged": (_int, [_vp, _vp, _int, _vp, _int, _i64, _i64, _int, _int, _i64, _i64,
                                    _vp, _vp, _vp]),
    "misa_score_tokens_paged": (_int, [_vp, _vp, _vp, _vp, _vp, _int, _vp, _int, _i64, _int, _i64,
                                       _i64, _int, _int, _int, _vp, _i64, _vp]),
    "misa_score_topk_paged": (_int, [_vp, _vp, _vp, _vp, _vp, _int, _vp, _int, _i64, _int, _i64,
                                     _i64, _int, _int, _int, _int, _vp, _vp, _i64, _vp, _sz, _vp]),
    "misa_rerank_paged": (_int, [_vp, _vp, _vp, _vp, _int, _vp, _int, _i64, _vp, _int, _int, _i64,
                                 _i64, _int, _int, _int, _vp, _vp, _vp, _sz, _vp]),
    "misa_decode_pool_keys": (_int, [_vp, _vp, _int, _vp, _int, _int, _i64, _vp, _int, _int, _int,
                                     _i64, _i64, _vp, _vp, _vp]),
    "misa_decode_route_heads": (_int, [_vp, _vp, _vp, _i64, _vp, _int, _int, _int, _int, _int, _vp,
                                       _vp, _vp]),
    "misa_decode_score_topk": (_int, [_vp, _vp, _vp, _vp, _vp, _int, _vp, _int, _int, _i64, _vp,
                                      _int, _int, _int, _int, _int, _vp, _vp, _i64, _vp]),
    "misa_profile_start": (_int, []),
    "misa_profile_stop": (_int, [_vp, _vp, _int]),
    "misa_profile_stage_name": (ctypes.c_char_p, [_int]),
    "misa_workspace_size": (_sz, [ctypes.c_char_p, _int, _i64, _int, _int]),
    "misa_status_string": (ctypes.c_char_p, [_int]),
    "misa_last_device_status": (_int, [_vp]),
    "misa_set_wait_limit_ns": (_int, [ctypes.c_uint64]),
}


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: build it with "
                          "`python -m long_context_sparse_block_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library()


def _check(fn: str, status: int):
    if status != MISA_OK:
        raise MisaError(fn, status, _lib.misa_status_string(status).decode())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t, dtypes=None, name="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise ValueError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    return ctypes.c_void_p(t.data_ptr())


_BF16_CODES = (torch.bfloat16, torch.int16, torch.uint16)


def _need(t, n: int, name: str):
    """The kernels read or write `n` elements of `t` (which the C ABI cannot see):
    refuse a smaller tensor before anything is launched."""
    if t is not None and t.numel() < n:
        raise ValueError(f"{name} holds {t.numel()} elements, the call needs {n}")


def _need_rows(t, rows: int, cols: int, name: str):
    """A 2-D (possibly row-padded) buffer with at least `rows` rows of `cols` entries."""
    if t.dim() != 2 or t.shape[0] < rows or t.shape[1] < cols:
        raise ValueError(f"{name} has shape {tuple(t.shape)}, the call needs [>= {rows}, >= {cols}]")


def _kdtype(K):
    K = K.pages if isinstance(K, PagedKeys) else K
    return MISA_K_FP8E4M3 if K.dtype in (torch.uint8, torch.float8_e4m3fn) else MISA_K_BF16


class PagedKeys:
    """A paged key cache: `pages` [n_pages, page_size, d] (bf16 codes, or e4m3 codes
    with `k_scale` [n_pages, page_size] fp32), `block_table` int32 with at least
    ceil(n_k / page_size) entries (logical key s is row s % page_size of page
    block_table[s // page_size]), and the sequence's `n_k` logical keys.  Every
    stage call below accepts one in place of a contiguous K [n_k, d]."""

    def __init__(self, pages, block_table, n_k: int, k_scale=None):
        if pages.dim() != 3:
            raise ValueError("pages must be [n_pages, page_size, d]")
        self.pages, self.block_table, self.n_k, self.k_scale = pages, block_table, int(n_k), k_scale
        self.n_pages, self.page_size, self.d = (int(x) for x in pages.shape)
        _need(block_table, -(-self.n_k // self.page_size), "block_table")
        _need(k_scale, self.n_pages * self.page_size, "k_scale")

    @property
    def shape(self):
        """The logical [n_k, d] shape of the keys."""
        return (self.n_k, self.d)

    def paged_args(self):
        """(pages, k_scale, kdtype, block_table, page_size, n_pages) of the C calls."""
        return (_ptr(self.pages, name="pages"), _ptr(self.k_scale, (torch.float32,), "k_scale"),
                _kdtype(self.pages), _ptr(self.block_table, (torch.int32,), "block_table"),
                self.page_size, self.n_pages)


# ---------------------------------------------------------------- stage calls

def misa_pool_keys(K, B: int, k_scale=None, kbar=None, kbar_hl=None, want_kbar: bool = True):
    """K [n_k, d] bf16 codes (or e4m3 codes + k_scale), or a PagedKeys cache
    -> (kbar [M,d] f32, kbar_hl [2,M,d])."""
    n_k, d = K.shape
    M = -(-n_k // B)
    dev = K.pages.device if isinstance(K, PagedKeys) else K.device
    if kbar is None and want_kbar:
        kbar = torch.empty((M, d), dtype=torch.float32, device=dev)
    if kbar_hl is None:
        kbar_hl = torch.empty((2, M, d), dtype=torch.int16, device=dev)
    if isinstance(K, PagedKeys):
        return misa_pool_keys_range(K, B, 0, M, kbar=kbar, kbar_hl=kbar_hl)
    _need(k_scale, n_k, "k_scale")
    _need(kbar, M * d, "kbar")
    _need(kbar_hl, 2 * M * d, "kbar_hl")
    st = _lib.misa_pool_keys(_ptr(K, name="K"), _ptr(k_scale, (torch.float32,), "k_scale"),
                             _kdtype(K), n_k, d, B, _ptr(kbar, (torch.float32,), "kbar"),
                             _ptr(kbar_hl, _BF16_CODES, "kbar_hl"), _stream())
    _check("misa_pool_keys", st)
    return kbar, kbar_hl


def misa_pool_keys_range(K, B: int, m0: int, m1: int, kbar=None, kbar_hl=None, k_scale=None,
                         n_k: int | None = None):
    """Re-pool blocks m0..m1-1 of the first n_k rows of K (default all rows) into
    existing kbar [>=M, d] f32 / kbar_hl [2, M, d] buffers (M = ceil(n_k/B))."""
    if n_k is None:
        n_k = K.shape[0]
    d = K.shape[1]
    M = -(-n_k // B) if B > 0 else 0
    _need(kbar, M * d, "kbar")
    _need(kbar_hl, 2 * M * d, "kbar_hl")
    if isinstance(K, PagedKeys):
        if n_k > K.n_k:
            raise ValueError(f"n_k={n_k} exceeds the cache's {K.n_k} keys")
        st = _lib.misa_pool_keys_paged(*K.paged_args(), n_k, d, B, m0, m1,
                                       _ptr(kbar, (torch.float32,), "kbar"),
                                       _ptr(kbar_hl, _BF16_CODES, "kbar_hl"), _stream())
        _check("misa_pool_keys_paged", st)
        return kbar, kbar_hl
    _need(K, n_k * d, "K")
    _need(k_scale, n_k, "k_scale")
    st = _lib.misa_pool_keys_range(_ptr(K, name="K"), _ptr(k_scale, (torch.float32,), "k_scale"),
                                   _kdtype(K), n_k, d, B, m0, m1,
                                   _ptr(kbar, (torch.float32,), "kbar"),
                                   _ptr(kbar_hl, _BF16_CODES, "kbar_hl"), _stream())
    _check("misa_pool_keys_range", st)
    return kbar, kbar_hl


def misa_route_heads(Q, w, kbar_hl, q_pos0: int, n_k: int, B: int, h: int, heads=None,
                     want_r: bool = False):
    """Q [n_q,H,d], w [n_q,H] f32, kbar_hl [2,M,d] -> (heads [n_q,h] int32, r [n_q,H] or None)."""
    n_q, H, d = Q.shape
    if heads is None:
        heads = torch.empty((n_q, h), dtype=torch.int32, device=Q.device)
    r = torch.empty((n_q, H), dtype=torch.float32, device=Q.device) if want_r else None
    M = -(-n_k // B) if B > 0 else 0
    _need(w, n_q * H, "w")
    _need(kbar_hl, 2 * M * d, "kbar_hl")
    _need(heads, n_q * h, "heads")
    st = _lib.misa_route_heads(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"),
                               _ptr(kbar_hl, _BF16_CODES, "kbar_hl"), n_q, q_pos0, n_k, H, d, B, h,
                               _ptr(heads, (torch.int32,), "heads"), _ptr(r, (torch.float32,), "r"),
                               _stream())
    _check("misa_route_heads", st)
    return heads, r


def misa_score_tokens(Q, w, heads, K, q_pos0: int, k_scale=None, logits=None, h: int | None = None):
    """Fused routed logits [n_q, ld] f32 (heads None: all H heads, the dense indexer)."""
    n_q, H, d = Q.shape
    n_k = K.shape[0]
    if h is None:
        h = heads.shape[1] if heads is not None else H
    if logits is None:  # rows padded to 16 bytes (the kernel stores tiles by TMA)
        logits = torch.empty((n_q, (n_k + 3) // 4 * 4), dtype=torch.float32, device=Q.device)[:, :n_k]
    ld = logits.stride(0) if logits.dim() == 2 else n_k
    _need(w, n_q * H, "w")
    _need(heads, n_q * h, "heads")
    if logits.dim() == 2:
        _need_rows(logits, n_q, n_k, "logits")
    else:
        _need(logits, n_q * n_k, "logits")
    if isinstance(K, PagedKeys):
        st = _lib.misa_score_tokens_paged(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"),
                                          _ptr(heads, (torch.int32,), "heads"), *K.paged_args(),
                                          n_q, q_pos0, n_k, H, d, h,
                                          ctypes.c_void_p(logits.data_ptr()), ld, _stream())
        _check("misa_score_tokens_paged", st)
        return logits
    _need(k_scale, n_k, "k_scale")
    st = _lib.misa_score_tokens(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"),
                                _ptr(heads, (torch.int32,), "heads"), _ptr(K, name="K"),
                                _ptr(k_scale, (torch.float32,), "k_scale"), _kdtype(K), n_q, q_pos0,
                                n_k, H, d, h, ctypes.c_void_p(logits.data_ptr()), ld, _stream())
    _check("misa_score_tokens", st)
    return logits


_E4M3_CODES = (torch.uint8, torch.float8_e4m3fn)


def misa_score_tokens_fp8(Q8, q_scale, w, heads, K8, k_scale, q_pos0: int, logits=None,
                          h: int | None = None):
    """Routed logits [n_q, ld] f32 from e4m3 queries [n_q, H, d] (scales [n_q, H]) and e4m3
    keys [n_k, d] (scales [n_k]), multiplied as e4m3 on the tensor cores."""
    n_q, H, d = Q8.shape
    n_k = K8.shape[0]
    if h is None:
        h = heads.shape[1] if heads is not None else H
    if logits is None:
        logits = torch.empty((n_q, (n_k + 3) // 4 * 4), dtype=torch.float32, device=Q8.device)[:, :n_k]
    ld = logits.stride(0) if logits.dim() == 2 else n_k
    _need(q_scale, n_q * H, "q_scale")
    _need(w, n_q * H, "w")
    _need(heads, n_q * h, "heads")
    _need(k_scale, n_k, "k_scale")
    if logits.dim() == 2:
        _need_rows(logits, n_q, n_k, "logits")
    else:
        _need(logits, n_q * n_k, "logits")
    st = _lib.misa_score_tokens_fp8(_ptr(Q8, _E4M3_CODES, "Q8"), _ptr(q_scale, (torch.float32,), "q_scale"),
                                    _ptr(w, (torch.float32,), "w"), _ptr(heads, (torch.int32,), "heads"),
                                    _ptr(K8, _E4M3_CODES, "K8"), _ptr(k_scale, (torch.float32,), "k_scale"),
                                    n_q, q_pos0, n_k, H, d, h, ctypes.c_void_p(logits.data_ptr()), ld,
                                    _stream())
    _check("misa_score_tokens_fp8", st)
    return logits


def misa_topk(logits, q_pos0: int, n_k: int, k: int, idx=None, n_q: int | None = None):
    """Top-k token indices [n_q, k] int32 (ascending, -1 padded) of fp32 logits rows."""
    if n_q is None:
        n_q = logits.shape[0]
    if idx is None:
        idx = torch.empty((n_q, k), dtype=torch.int32, device=logits.device)
    _need_rows(logits, n_q, min(n_k, q_pos0 + n_q), "logits")
    _need(idx, n_q * k, "idx")
    st = _lib.misa_topk(ctypes.c_void_p(logits.data_ptr()), logits.stride(0), n_q, q_pos0, n_k, k,
                        _ptr(idx, (torch.int32,), "idx"), None, 0, _stream())
    _check("misa_topk", st)
    return idx


def misa_score_topk(Q, w, heads, K, q_pos0: int, k: int, k_scale=None, h: int | None = None,
                    idx=None, logits=None, ws=None):
    """Routed scoring and top-k in one call -> idx [n_q, k] int32 (ascending, -1 padded).

    `logits` ([n_q, >= n_k] fp32, rows 16-byte aligned) is the exact fallback's
    scratch and `ws` the fused path's workspace; both are allocated when absent."""
    n_q, H, d = Q.shape
    n_k = K.shape[0]
    if h is None:
        h = heads.shape[1] if heads is not None else H
    if idx is None:
        idx = torch.empty((n_q, k), dtype=torch.int32, device=Q.device)
    if logits is None:
        logits = torch.empty((n_q, (n_k + 3) // 4 * 4), dtype=torch.float32, device=Q.device)
    if logits.dim() != 2 or logits.stride(1) != 1 or logits.shape[0] < n_q:
        raise ValueError("logits must be a row-major [n_q, >= n_k] fp32 buffer")
    _need(w, n_q * H, "w")
    _need(heads, n_q * h, "heads")
    _need(idx, n_q * k, "idx")
    _need_rows(logits, n_q, n_k, "logits")
    ws_bytes = misa_workspace_size("score_topk", n_q, n_k, k, 0)
    if ws_bytes and (ws is None or ws.numel() * ws.element_size() < ws_bytes):
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=Q.device)
    if isinstance(K, PagedKeys):
        st = _lib.misa_score_topk_paged(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"),
                                        _ptr(heads, (torch.int32,), "heads"), *K.paged_args(), n_q,
                                        q_pos0, n_k, H, d, h, k, _ptr(idx, (torch.int32,), "idx"),
                                        ctypes.c_void_p(logits.data_ptr()), logits.stride(0),
                                        _ptr(ws, name="ws") if ws_bytes else None, ws_bytes,
                                        _stream())
        _check("misa_score_topk_paged", st)
        return idx
    _need(k_scale, n_k, "k_scale")
    # bf16 codes that come with scales are decoded e4m3 keys (misa_keys_e4m3_to_bf16)
    kd = _kdtype(K)
    if kd == MISA_K_BF16 and k_scale is not None:
        kd = MISA_K_BF16_SCALED
    st = _lib.misa_score_topk(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"),
                              _ptr(heads, (torch.int32,), "heads"), _ptr(K, name="K"),
                              _ptr(k_scale, (torch.float32,), "k_scale"), kd, n_q, q_pos0,
                              n_k, H, d, h, k, _ptr(idx, (torch.int32,), "idx"),
                              ctypes.c_void_p(logits.data_ptr()), logits.stride(0),
                              _ptr(ws, name="ws") if ws_bytes else None, ws_bytes, _stream())
    _check("misa_score_topk", st)
    return idx


def misa_keys_e4m3_to_bf16(K8, out=None):
    """e4m3 key codes [n_k, d] -> bf16 codes [n_k, d] (int16 view), exact; the
    per-token scales are not applied (score the codes with them as scaled keys)."""
    n_k, d = K8.shape
    if out is None:
        out = torch.empty((n_k, d), dtype=torch.int16, device=K8.device)
    _need(out, n_k * d, "out")
    st = _lib.misa_keys_e4m3_to_bf16(_ptr(K8, _E4M3_CODES, "K8"), n_k, d,
                                     _ptr(out, _BF16_CODES, "out"), _stream())
    _check("misa_keys_e4m3_to_bf16", st)
    return out


def misa_workspace_size(op: str, n_q: int, n_k: int, k: int, kp: int) -> int:
    return int(_lib.misa_workspace_size(op.encode(), n_q, n_k, k, kp))


def misa_rerank(Q, w, K, cand, q_pos0: int, k: int, k_scale=None, want_full: bool = False,
                idx=None, ws=None):
    """MISA-dagger: all-head rescoring of candidates [n_q, kp] -> idx [n_q, k] (and full scores)."""
    n_q, H, d = Q.shape
    n_k = K.shape[0]
    kp = cand.shape[1]
    if idx is None:
        idx = torch.empty((n_q, k), dtype=torch.int32, device=Q.device)
    full = torch.empty((n_q, kp), dtype=torch.float32, device=Q.device) if want_full else None
    _need(w, n_q * H, "w")
    _need(cand, n_q * kp, "cand")
    _need(idx, n_q * k, "idx")
    ws_bytes = 0
    if full is None:
        ws_bytes = misa_workspace_size("rerank", n_q, n_k, k, kp)
        if ws is None or ws.numel() * ws.element_size() < ws_bytes:
            ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=Q.device)
    if isinstance(K, PagedKeys):
        st = _lib.misa_rerank_paged(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"),
                                    *K.paged_args(), _ptr(cand, (torch.int32,), "cand"), kp, n_q,
                                    q_pos0, n_k, H, d, k, _ptr(idx, (torch.int32,), "idx"),
                                    _ptr(full, (torch.float32,), "full"),
                                    _ptr(ws, name="ws") if full is None else None, ws_bytes,
                                    _stream())
        _check("misa_rerank_paged", st)
        return (idx, full) if want_full else idx
    _need(k_scale, n_k, "k_scale")
    st = _lib.misa_rerank(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"), _ptr(K, name="K"),
                          _ptr(k_scale, (torch.float32,), "k_scale"), _kdtype(K),
                          _ptr(cand, (torch.int32,), "cand"), kp, n_q, q_pos0, n_k, H, d, k,
                          _ptr(idx, (torch.int32,), "idx"), _ptr(full, (torch.float32,), "full"),
                          _ptr(ws, name="ws") if full is None else None, ws_bytes, _stream())
    _check("misa_rerank", st)
    return (idx, full) if want_full else idx


def misa_rerank_noalloc(Q, w, K, cand, q_pos0: int, k: int, k_scale=None, idx=None):
    """misa_rerank without workspace: the library's own fixed scratch (at most
    4194304 candidate scores per call) stands in for it."""
    n_q, H, d = Q.shape
    kp = cand.shape[1]
    if idx is None:
        idx = torch.empty((n_q, k), dtype=torch.int32, device=Q.device)
    _need(w, n_q * H, "w")
    _need(k_scale, K.shape[0], "k_scale")
    _need(cand, n_q * kp, "cand")
    _need(idx, n_q * k, "idx")
    st = _lib.misa_rerank_noalloc(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"),
                                  _ptr(K, name="K"), _ptr(k_scale, (torch.float32,), "k_scale"),
                                  _kdtype(K), _ptr(cand, (torch.int32,), "cand"), kp, n_q, q_pos0,
                                  K.shape[0], H, d, k, _ptr(idx, (torch.int32,), "idx"), _stream())
    _check("misa_rerank_noalloc", st)
    return idx


# ---------------------------------------------------------------- decode (many sequences)

def _decode_cache(pages, block_tables, seq_lens, k_scale):
    if pages.dim() != 3 or block_tables.dim() != 2:
        raise ValueError("pages [n_pages, page_size, d] and block_tables [n_seq, max_blocks]")
    n_pages, ps, d = (int(x) for x in pages.shape)
    n_seq, max_blocks = (int(x) for x in block_tables.shape)
    _need(seq_lens, n_seq, "seq_lens")
    _need(k_scale, n_pages * ps, "k_scale")
    args = (_ptr(pages, name="pages"), _ptr(k_scale, (torch.float32,), "k_scale"), _kdtype(pages),
            _ptr(block_tables, (torch.int32,), "block_tables"), max_blocks, ps, n_pages)
    return args, n_seq, d, max_blocks * ps


def misa_decode_pool_keys(pages, block_tables, seq_lens, B: int, M_max: int, n_last: int,
                          kbar=None, kbar_hl=None, k_scale=None, want_kbar: bool = False):
    """Re-pool the last n_last blocks of every sequence into per-sequence pooled
    keys kbar [n_seq, M_max, d] f32 (optional) and kbar_hl [n_seq, 2, M_max, d]."""
    args, n_seq, d, _ = _decode_cache(pages, block_tables, seq_lens, k_scale)
    if kbar is None and want_kbar:
        kbar = torch.empty((n_seq, M_max, d), dtype=torch.float32, device=pages.device)
    if kbar_hl is None:
        kbar_hl = torch.empty((n_seq, 2, M_max, d), dtype=torch.int16, device=pages.device)
    _need(kbar, n_seq * M_max * d, "kbar")
    _need(kbar_hl, n_seq * 2 * M_max * d, "kbar_hl")
    st = _lib.misa_decode_pool_keys(*args, _ptr(seq_lens, (torch.int32,), "seq_lens"), n_seq, d, B,
                                    M_max, n_last, _ptr(kbar, (torch.float32,), "kbar"),
                                    _ptr(kbar_hl, _BF16_CODES, "kbar_hl"), _stream())
    _check("misa_decode_pool_keys", st)
    return kbar, kbar_hl


def misa_decode_route_heads(Q, w, kbar_hl, seq_lens, B: int, h: int, heads=None,
                            want_r: bool = False):
    """Q [n_seq, H, d], w [n_seq, H], kbar_hl [n_seq, 2, M_max, d] -> (heads [n_seq, h], r)."""
    n_seq, H, d = Q.shape
    M_max = int(kbar_hl.shape[-2])
    if heads is None:
        heads = torch.empty((n_seq, h), dtype=torch.int32, device=Q.device)
    r = torch.empty((n_seq, H), dtype=torch.float32, device=Q.device) if want_r else None
    _need(w, n_seq * H, "w")
    _need(kbar_hl, n_seq * 2 * M_max * d, "kbar_hl")
    _need(seq_lens, n_seq, "seq_lens")
    _need(heads, n_seq * h, "heads")
    st = _lib.misa_decode_route_heads(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"),
                                      _ptr(kbar_hl, _BF16_CODES, "kbar_hl"), M_max,
                                      _ptr(seq_lens, (torch.int32,), "seq_lens"), n_seq, H, d, B, h,
                                      _ptr(heads, (torch.int32,), "heads"),
                                      _ptr(r, (torch.float32,), "r"), _stream())
    _check("misa_decode_route_heads", st)
    return heads, r


def misa_decode_score_topk(Q, w, heads, pages, block_tables, seq_lens, k: int, k_scale=None,
                           h: int | None = None, idx=None, logits=None):
    """Per sequence b: the top-k keys (ascending, -1 padded) of its new query's
    routed logits over its seq_lens[b] keys -> (idx [n_seq, k], logits [n_seq, ld])."""
    n_seq, H, d = Q.shape
    args, n_seq2, d2, max_len = _decode_cache(pages, block_tables, seq_lens, k_scale)
    if n_seq2 != n_seq or d2 != d:
        raise ValueError("block_tables / pages do not match Q")
    if h is None:
        h = heads.shape[1] if heads is not None else H
    if idx is None:
        idx = torch.empty((n_seq, k), dtype=torch.int32, device=Q.device)
    if logits is None:
        logits = torch.empty((n_seq, max_len), dtype=torch.float32, device=Q.device)
    _need(w, n_seq * H, "w")
    _need(heads, n_seq * h, "heads")
    _need(idx, n_seq * k, "idx")
    _need_rows(logits, n_seq, max_len, "logits")
    st = _lib.misa_decode_score_topk(_ptr(Q, _BF16_CODES, "Q"), _ptr(w, (torch.float32,), "w"),
                                     _ptr(heads, (torch.int32,), "heads"), *args,
                                     _ptr(seq_lens, (torch.int32,), "seq_lens"), n_seq, H, d, h, k,
                                     _ptr(idx, (torch.int32,), "idx"),
                                     ctypes.c_void_p(logits.data_ptr()), logits.stride(0), _stream())
    _check("misa_decode_score_topk", st)
    return idx, logits


def misa_profile_start() -> None:
    _check("misa_profile_start", _lib.misa_profile_start())


def misa_profile_stop() -> dict:
    """Per-stage device milliseconds (summed) and launch counts of the fused
    calls made since misa_profile_start()."""
    n = 16
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_int * n)()
    _check("misa_profile_stop", _lib.misa_profile_stop(ms, cnt, n))
    out = {}
    for i in range(n):
        name = _lib.misa_profile_stage_name(i)
        if name is None:
            break
        out[name.decode()] = (ms[i], cnt[i])
    return out


def misa_last_device_status() -> int:
    return int(_lib.misa_last_device_status(_stream()))


def misa_set_wait_limit_ns(ns: int) -> None:
    _check("misa_set_wait_limit_ns", _lib.misa_set_wait_limit_ns(ns))


def misa_status_string(status: int) -> str:
    return _lib.misa_status_string(status).decode()
