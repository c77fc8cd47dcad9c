"""CPU oracle for the MISA token indexer — TEST INFRASTRUCTURE ONLY.

Only the tests, the smoke check and the benchmark's CPU-baseline leg may import
this package; the product path never does.  It wraps `misa_oracle.c` (plain C,
fp64, single-threaded, written from the method's definitions) with ctypes and
shares no code with the CUDA library.

Parity status per function (what pins each one is listed in the tests):
  pool_keys, route, score, dense_logits, topk, topk_f32, rerank,
  select_candidates — pinned by
  closed forms, brute force on tiny inputs, library-routine reductions and the
  structural invariants of the method.  The router's aggregate (a sum over
  complete causal blocks of w * ReLU(q . kbar)) is a reading of a step the pages
  describe only as "aggregate"; it is pinned against that reading, not against
  the authors' code, which is not available.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "misa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "_build", "libmisa_oracle.so")
_lock = threading.Lock()
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_F = ctypes.POINTER(ctypes.c_float)
_I32 = ctypes.POINTER(ctypes.c_int32)
_I64 = ctypes.POINTER(ctypes.c_int64)
_U16 = ctypes.POINTER(ctypes.c_uint16)
_U8 = ctypes.POINTER(ctypes.c_uint8)
_i64 = ctypes.c_int64
_int = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (no fast-math, no FMA contraction)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if force or not os.path.exists(_LIB_PATH) or \
            os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            sig = {
                "oracle_bf16_to_double": (ctypes.c_double, [ctypes.c_uint16]),
                "oracle_e4m3_to_double": (ctypes.c_double, [ctypes.c_uint8]),
                "oracle_decode_bf16": (None, [_U16, _i64, _D]),
                "oracle_decode_e4m3_keys": (None, [_U8, _F, _i64, _int, _D]),
                "oracle_pool_keys": (None, [_D, _i64, _int, _int, _D]),
                "oracle_causal_blocks": (_i64, [_i64, _i64, _int]),
                "oracle_route": (None, [_D, _D, _D, _int, _i64, _i64, _int, _int, _int, _int,
                                        _D, _I32, _I64]),
                "oracle_score": (None, [_D, _D, _I32, _D, _int, _i64, _i64, _int, _int, _int,
                                        _D, _i64, _I64]),
                "oracle_dense_logits": (None, [_D, _D, _D, _int, _i64, _i64, _int, _int, _D,
                                               _i64]),
                "oracle_topk": (None, [_D, _i64, _int, _i64, _i64, _int, _I32]),
                "oracle_topk_f32": (None, [_F, _i64, _int, _i64, _i64, _int, _I32]),
                "oracle_rerank": (None, [_D, _D, _D, _I32, _int, _int, _i64, _i64, _int, _int,
                                         _int, _I32, _D, _I64]),
                "oracle_select_candidates_f32": (None, [_F, _I32, _int, _int, _i64, _i64, _int,
                                                        _I32]),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _p(a, ptype):
    return a.ctypes.data_as(ptype) if a is not None else None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


class _Counter:
    def __init__(self):
        self.v = ctypes.c_int64(0)

    def ptr(self):
        return ctypes.pointer(self.v)


# ---- storage decoding --------------------------------------------------------

def bf16_to_f64(codes) -> np.ndarray:
    codes = _c(codes, np.uint16)
    out = np.empty(codes.shape, dtype=np.float64)
    _load().oracle_decode_bf16(_p(codes, _U16), codes.size, _p(out, _D))
    return out


def e4m3_keys_to_f64(codes, scale) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scale = _c(scale, np.float32)
    n_k, d = codes.shape
    out = np.empty((n_k, d), dtype=np.float64)
    _load().oracle_decode_e4m3_keys(_p(codes, _U8), _p(scale, _F), n_k, d, _p(out, _D))
    return out


def e4m3_value(code: int) -> float:
    return _load().oracle_e4m3_to_double(code)


def bf16_value(code: int) -> float:
    return _load().oracle_bf16_to_double(code)


# ---- method stages (fp64 arrays in, fp64 / int32 out) ------------------------

def pool_keys(K: np.ndarray, B: int) -> np.ndarray:
    K = _c(K, np.float64)
    n_k, d = K.shape
    out = np.empty((-(-n_k // B), d), dtype=np.float64)
    _load().oracle_pool_keys(_p(K, _D), n_k, d, B, _p(out, _D))
    return out


def causal_blocks(pos: int, n_k: int, B: int) -> int:
    return _load().oracle_causal_blocks(pos, n_k, B)


def route(Q, w, kbar, q_pos0: int, n_k: int, B: int, h: int, counter=None):
    """Q [n_q,H,d] f64, w [n_q,H], kbar [M,d] -> (r [n_q,H] f64, heads [n_q,h] int32)."""
    Q = _c(Q, np.float64)
    w = _c(w, np.float64)
    kbar = _c(kbar, np.float64)
    n_q, H, d = Q.shape
    r = np.empty((n_q, H), dtype=np.float64)
    heads = np.empty((n_q, h), dtype=np.int32)
    _load().oracle_route(_p(Q, _D), _p(w, _D), _p(kbar, _D), n_q, q_pos0, n_k, H, d, B, h,
                         _p(r, _D), _p(heads, _I32), counter.ptr() if counter else None)
    return r, heads


def score(Q, w, heads, K, q_pos0: int, counter=None) -> np.ndarray:
    """Routed logits [n_q, n_k] (fp64, -inf beyond the causal limit)."""
    Q = _c(Q, np.float64)
    w = _c(w, np.float64)
    K = _c(K, np.float64)
    heads = _c(heads, np.int32)
    n_q, H, d = Q.shape
    n_k = K.shape[0]
    h = heads.shape[1]
    out = np.empty((n_q, n_k), dtype=np.float64)
    _load().oracle_score(_p(Q, _D), _p(w, _D), _p(heads, _I32), _p(K, _D), n_q, q_pos0, n_k,
                         H, d, h, _p(out, _D), n_k, counter.ptr() if counter else None)
    return out


def dense_logits(Q, w, K, q_pos0: int) -> np.ndarray:
    Q = _c(Q, np.float64)
    w = _c(w, np.float64)
    K = _c(K, np.float64)
    n_q, H, d = Q.shape
    n_k = K.shape[0]
    out = np.empty((n_q, n_k), dtype=np.float64)
    _load().oracle_dense_logits(_p(Q, _D), _p(w, _D), _p(K, _D), n_q, q_pos0, n_k, H, d,
                                _p(out, _D), n_k)
    return out


def topk(logits, q_pos0: int, n_k: int, k: int) -> np.ndarray:
    """Top-k token indices [n_q, k] (ascending, -1 padded) from fp64 or fp32 rows."""
    n_q, ld = logits.shape
    idx = np.empty((n_q, k), dtype=np.int32)
    if logits.dtype == np.float32:
        lg = _c(logits, np.float32)
        _load().oracle_topk_f32(_p(lg, _F), ld, n_q, q_pos0, n_k, k, _p(idx, _I32))
    else:
        lg = _c(logits, np.float64)
        _load().oracle_topk(_p(lg, _D), ld, n_q, q_pos0, n_k, k, _p(idx, _I32))
    return idx


def rerank(Q, w, K, cand, q_pos0: int, k: int, counter=None, want_logits: bool = False):
    Q = _c(Q, np.float64)
    w = _c(w, np.float64)
    K = _c(K, np.float64)
    cand = _c(cand, np.int32)
    n_q, H, d = Q.shape
    n_k = K.shape[0]
    kp = cand.shape[1]
    idx = np.empty((n_q, k), dtype=np.int32)
    full = np.empty((n_q, kp), dtype=np.float64) if want_logits else None
    _load().oracle_rerank(_p(Q, _D), _p(w, _D), _p(K, _D), _p(cand, _I32), kp, n_q, q_pos0, n_k,
                          H, d, k, _p(idx, _I32), _p(full, _D) if full is not None else None,
                          counter.ptr() if counter else None)
    return (idx, full) if want_logits else idx


def select_candidates(vals, cand, q_pos0: int, n_k: int, k: int) -> np.ndarray:
    """Top-k tokens among candidate scores [n_q, kp] (fp32) of tokens cand [n_q, kp]."""
    vals = _c(vals, np.float32)
    cand = _c(cand, np.int32)
    n_q, kp = cand.shape
    idx = np.empty((n_q, k), dtype=np.int32)
    _load().oracle_select_candidates_f32(_p(vals, _F), _p(cand, _I32), kp, n_q, q_pos0, n_k, k,
                                         _p(idx, _I32))
    return idx


# ---- whole-path helpers over stored inputs -----------------------------------

def decode_inputs(inp: dict, fp8_keys: bool = False, fp8_queries: bool = False):
    """fp64 views of the stored inputs: (Q [n_q,H,d], K [n_k,d], w [n_q,H]).
    fp8_queries: Q from its e4m3 codes times the per-(query, head) scales."""
    if fp8_queries:
        n_q, H, d = inp["Q8"].shape
        Q = e4m3_keys_to_f64(inp["Q8"].reshape(n_q * H, d),
                             inp["q_scale"].reshape(n_q * H)).reshape(n_q, H, d)
    else:
        Q = bf16_to_f64(inp["Q"])
    K = e4m3_keys_to_f64(inp["K8"], inp["k_scale"]) if fp8_keys else bf16_to_f64(inp["K"])
    w = np.asarray(inp["w"], dtype=np.float64)
    return Q, K, w


def misa_rows(Qd, Kd, wd, kbar, rows, q_pos0: int, B: int, h: int, k: int, kp: int = 0,
              want_logits: bool = True):
    """Run the whole indexer for the query rows `rows` (local indices), one row at
    a time.  Returns a dict of per-row results (r, heads, logits, idx and, when
    kp > 0, the MISA-dagger candidates and final idx)."""
    n_k = Kd.shape[0]
    out = {"r": [], "heads": [], "logits": [], "idx": [], "cand": [], "dagger": []}
    for t in rows:
        t = int(t)
        pos = q_pos0 + t
        Qt, wt = Qd[t:t + 1], wd[t:t + 1]
        r, hd = route(Qt, wt, kbar, pos, n_k, B, h)
        lg = score(Qt, wt, hd, Kd, pos)
        out["r"].append(r[0])
        out["heads"].append(hd[0])
        if want_logits:
            out["logits"].append(lg[0])
        out["idx"].append(topk(lg, pos, n_k, k)[0])
        if kp:
            cand = topk(lg, pos, n_k, kp)
            out["cand"].append(cand[0])
            out["dagger"].append(rerank(Qt, wt, Kd, cand, pos, k)[0])
    return {key: np.stack(v) if v else None for key, v in out.items()}
