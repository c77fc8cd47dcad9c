"""Seeded synthetic inputs for the MISA token indexer.

This module holds no indexer arithmetic. It draws random numbers, rounds them to
the storage formats the indexer reads (bf16 for Q, K and w; e4m3 plus a per-token
fp32 scale for the FP8 key variant), and names the workloads by what they are.
Both the CUDA path and the CPU oracle read the arrays it returns, so neither side
ever depends on the other for its inputs.

Workloads (shapes from the MISA pages: DeepSeek-V3.2 has 64 indexer heads and
GLM-5 has 32, "MISA: Mixture of Indexer Sparse Attention", Experimental Results;
the 8192 x 131072 final prefill chunk is the one in the vLLM integration issue,
"Clarification on the Figure 3 baseline ...", measurement table):

  tiny_1k          L=1024, H_I=8,  d=32,  B=64,  h=2, k=64.   Gaussian, seed 0.
  dsv32_32k        L=32768, H_I=64, d=128, B=128, h=8, k=2048. Clustered, seed 1.
  glm5_64k         L=65536, H_I=32, d=128, B=128, h=8, k=2048. Clustered, seed 2.
  chunk_128k       8192 queries at 122880..131071 vs 131072 keys, H_I=64, d=128,
                   B=128, h=8, k=2048. Clustered, seed 3.
  chunk_128k_h4    same inputs, h=4.
  dagger_128k      same inputs, h=8, coarse k'=8192 then all-head rerank to 2048.

Generator recipes:

* Gaussian (tiny_1k): K, Q ~ N(0,1)/sqrt(d); every (query, head) row of Q is
  multiplied by a lognormal(0, 0.5) gain; w ~ N(0,1)/sqrt(H_I) kept in fp32.
* Clustered (the rest): 64 centroids ~ N(0,1)/sqrt(d). Each key picks one
  centroid uniformly and adds N(0, (0.3/sqrt(d))^2) noise. Each head j owns 4
  distinct centroids; each (query, head) row picks one of its head's 4 uniformly,
  adds the same noise and is multiplied by a lognormal(0, 0.5) gain. w ~
  N(0,1)/sqrt(H_I), rounded to bf16 values. 16 "needle" keys, at distinct
  positions drawn uniformly below the last query's position, are set equal to
  that query's head-0 row.

Draw order (fixed): centroids, key components, key noise, head mixtures, query
components, query noise, gains, w, needles. All draws are fp64 and rounded once,
to nearest-even, to the storage format.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace

import numpy as np

_CHUNK_ROWS = 1 << 16


@dataclass(frozen=True)
class Workload:
    name: str
    n_q: int          # queries in the chunk
    q_pos0: int       # position of the first query
    n_k: int          # keys 0..n_k-1 (the causal prefix plus the chunk itself)
    H: int            # indexer heads H_I
    d: int            # index head dimension
    B: int            # pooling block size
    h: int            # routed heads per query
    k: int            # selected tokens per query
    generator: str    # "gaussian" or "clustered"
    seed: int
    kp: int = 0       # MISA-dagger coarse candidate count k' (0: not hierarchical)
    n_needles: int = 0
    n_centroids: int = 64
    mix_per_head: int = 4

    @property
    def M(self) -> int:
        return -(-self.n_k // self.B)

    def positions(self) -> np.ndarray:
        return self.q_pos0 + np.arange(self.n_q, dtype=np.int64)

    def causal_pairs(self) -> int:
        """Sum over queries of (pos + 1): the (query, key) pairs scored."""
        p0, n = self.q_pos0, self.n_q
        return n * (p0 + 1) + n * (n - 1) // 2


WORKLOADS = {
    "tiny_1k": Workload("tiny_1k", n_q=1024, q_pos0=0, n_k=1024, H=8, d=32, B=64,
                        h=2, k=64, generator="gaussian", seed=0),
    "dsv32_32k": Workload("dsv32_32k", n_q=32768, q_pos0=0, n_k=32768, H=64, d=128,
                          B=128, h=8, k=2048, generator="clustered", seed=1,
                          n_needles=16),
    "glm5_64k": Workload("glm5_64k", n_q=65536, q_pos0=0, n_k=65536, H=32, d=128,
                         B=128, h=8, k=2048, generator="clustered", seed=2,
                         n_needles=16),
    "chunk_128k": Workload("chunk_128k", n_q=8192, q_pos0=122880, n_k=131072, H=64,
                           d=128, B=128, h=8, k=2048, generator="clustered", seed=3,
                           n_needles=16),
}
WORKLOADS["chunk_128k_h4"] = replace(WORKLOADS["chunk_128k"], name="chunk_128k_h4", h=4)
WORKLOADS["dagger_128k"] = replace(WORKLOADS["chunk_128k"], name="dagger_128k", kp=8192)


def small_workload(name: str, n_q: int, q_pos0: int, n_k: int, H: int, d: int, B: int,
                   h: int, k: int, seed: int, generator: str = "gaussian", kp: int = 0,
                   n_needles: int = 0) -> Workload:
    """An ad-hoc workload (edge shapes for the tests)."""
    return Workload(name, n_q=n_q, q_pos0=q_pos0, n_k=n_k, H=H, d=d, B=B, h=h, k=k,
                    generator=generator, seed=seed, kp=kp, n_needles=n_needles,
                    n_centroids=64 if generator == "clustered" else 0)


# ---------------------------------------------------------------------------
# storage rounding (IEEE-754 binary16-brain "bf16" and OCP FP8 E4M3)
# ---------------------------------------------------------------------------

def bf16_bits(x) -> np.ndarray:
    """Round fp64 values to the nearest bf16 (ties to even); return the 16-bit codes.

    bf16 keeps 8 significant bits and fp32's exponent range. x = m * 2**e with
    0.5 <= |m| < 1, so rint(m * 2**8) is the significand rounded to 8 bits.
    """
    x = np.asarray(x, dtype=np.float64)
    tiny = (x != 0) & (np.abs(x) < 2.0 ** -126)
    if np.any(tiny):
        raise ValueError("value in the bf16 subnormal range; the generators never draw one")
    m, e = np.frexp(x)
    r = np.ldexp(np.rint(np.ldexp(m, 8)), e - 8)
    f = r.astype(np.float32)                      # exact: 8 significant bits
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    """The fp32 values of bf16 codes (exact)."""
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


E4M3_MAX = 448.0


def e4m3_encode(y) -> np.ndarray:
    """Round fp64 values to OCP FP8 E4M3 (nearest, ties to even, saturating at 448).

    Normal numbers carry 4 significant bits with unbiased exponents -6..8; below
    2**-6 the grid is uniform with step 2**-9. The NaN code 0x7F is never produced.
    """
    y = np.asarray(y, dtype=np.float64)
    a = np.abs(y)
    _, e = np.frexp(a)
    q_exp = np.where(a >= 2.0 ** -6, e - 4, -9)
    r = np.minimum(np.ldexp(np.rint(np.ldexp(a, -q_exp)), q_exp), E4M3_MAX)
    code = np.zeros(a.shape, dtype=np.uint8)
    sub = r < 2.0 ** -6
    code[sub] = np.ldexp(r[sub], 9).astype(np.uint8)
    nm = ~sub
    _, e2 = np.frexp(r[nm])                       # r = 1.f * 2**(e2-1)
    ex = e2 - 1
    mant = np.ldexp(r[nm], -ex) * 8 - 8
    code[nm] = ((ex + 7) << 3).astype(np.uint8) | mant.astype(np.uint8)
    code |= np.where(np.signbit(y) & (r > 0), 0x80, 0).astype(np.uint8)
    return code


def e4m3_quantize_keys(k_values: np.ndarray):
    """Per-token scale = amax|K[s,:]| / 448 (1 when the row is zero), stored fp32;
    codes = e4m3(K[s,:] / scale)."""
    k_values = np.asarray(k_values, dtype=np.float64)
    amax = np.max(np.abs(k_values), axis=1)
    scale = np.where(amax > 0, amax / E4M3_MAX, 1.0).astype(np.float32)
    codes = e4m3_encode(k_values / scale.astype(np.float64)[:, None])
    return codes, scale


def e4m3_quantize_queries(q_values: np.ndarray):
    """Per (query, head) row of [n_q, H, d]: the per-row rule of e4m3_quantize_keys.
    Returns codes [n_q, H, d] and fp32 scales [n_q, H]."""
    n_q, H, d = q_values.shape
    flat = q_values.reshape(n_q * H, d)
    codes = np.empty((n_q * H, d), dtype=np.uint8)
    scale = np.empty(n_q * H, dtype=np.float32)
    for r0 in range(0, n_q * H, _CHUNK_ROWS):
        r1 = min(n_q * H, r0 + _CHUNK_ROWS)
        codes[r0:r1], scale[r0:r1] = e4m3_quantize_keys(flat[r0:r1])
    return codes.reshape(n_q, H, d), scale.reshape(n_q, H)


# ---------------------------------------------------------------------------
# generators
# ---------------------------------------------------------------------------

def _normal_rows(rng, n_rows, n_cols, scale):
    out = np.empty((n_rows, n_cols), dtype=np.float64)
    for r0 in range(0, n_rows, _CHUNK_ROWS):
        r1 = min(n_rows, r0 + _CHUNK_ROWS)
        out[r0:r1] = rng.standard_normal((r1 - r0, n_cols)) * scale
    return out


def generate(wl: Workload, fp8_keys: bool = False, fp8_queries: bool = False) -> dict:
    """Draw the inputs of workload `wl`.

    Returns a dict with
      Q      uint16 [n_q, H, d]  bf16 codes
      K      uint16 [n_k, d]     bf16 codes
      w      float32 [n_q, H]
      needles int64 [n_needles]  positions of planted needle keys (may be empty)
      K8, k_scale                e4m3 codes [n_k, d] and fp32 [n_k] (fp8_keys only)
      Q8, q_scale                e4m3 codes [n_q, H, d] and fp32 [n_q, H] (fp8_queries only)
    """
    rng = np.random.Generator(np.random.PCG64(wl.seed))
    d, H, n_q, n_k = wl.d, wl.H, wl.n_q, wl.n_k
    sd = 1.0 / math.sqrt(d)
    needles = np.zeros(0, dtype=np.int64)
    if wl.generator == "gaussian":
        K = bf16_bits(_normal_rows(rng, n_k, d, sd))
        Qv = _normal_rows(rng, n_q * H, d, sd)
        gain = rng.lognormal(0.0, 0.5, size=n_q * H)
        Q = bf16_bits(Qv * gain[:, None]).reshape(n_q, H, d)
        del Qv
        w = (rng.standard_normal((n_q, H)) / math.sqrt(H)).astype(np.float32)
    elif wl.generator == "clustered":
        C = wl.n_centroids
        cent = rng.standard_normal((C, d)) * sd
        z = rng.integers(0, C, size=n_k)
        Kv = _normal_rows(rng, n_k, d, 0.3 * sd)
        Kv += cent[z]
        K = bf16_bits(Kv)
        del Kv
        mix = np.stack([rng.choice(C, size=wl.mix_per_head, replace=False) for _ in range(H)])
        u = rng.integers(0, wl.mix_per_head, size=(n_q, H))
        comp = mix[np.arange(H)[None, :], u].reshape(-1)
        Q = np.empty((n_q * H, d), dtype=np.uint16)
        noise = _normal_rows(rng, n_q * H, d, 0.3 * sd)
        gain = rng.lognormal(0.0, 0.5, size=n_q * H)
        for r0 in range(0, n_q * H, _CHUNK_ROWS):
            r1 = min(n_q * H, r0 + _CHUNK_ROWS)
            Q[r0:r1] = bf16_bits((cent[comp[r0:r1]] + noise[r0:r1]) * gain[r0:r1, None])
        del noise
        Q = Q.reshape(n_q, H, d)
        w = bf16_values(bf16_bits(rng.standard_normal((n_q, H)) / math.sqrt(H)))
        if wl.n_needles:
            t_star = n_q - 1
            p_star = wl.q_pos0 + t_star
            needles = np.sort(rng.choice(p_star, size=wl.n_needles, replace=False)).astype(np.int64)
            K[needles] = Q[t_star, 0]
    else:
        raise ValueError(f"unknown generator {wl.generator!r}")
    out = {"Q": np.ascontiguousarray(Q), "K": np.ascontiguousarray(K),
           "w": np.ascontiguousarray(w, dtype=np.float32), "needles": needles}
    if fp8_keys:
        out["K8"], out["k_scale"] = e4m3_quantize_keys(bf16_values(K).astype(np.float64))
    if fp8_queries:
        out["Q8"], out["q_scale"] = e4m3_quantize_queries(bf16_values(Q).astype(np.float64))
    return out


def page_table(n_k: int, page_size: int, seed: int, spare: int = 3) -> tuple:
    """A paged layout for n_k keys: pages of `page_size` rows in a pool of
    ceil(n_k / page_size) + `spare` pages, logical block b stored in page
    table[b], the pages drawn in a seeded random order.  Returns (table int32,
    n_pages).  (Storage layout only; the values stay those of the keys.)"""
    n_blocks = -(-n_k // page_size)
    n_pages = n_blocks + spare
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.permutation(n_pages)[:n_blocks].astype(np.int32), n_pages


def exact_arithmetic_inputs(n_q: int, q_pos0: int, n_k: int, H: int, d: int, seed: int,
                            qmax: int = 3, kmax: int = 3):
    """Small-integer Q and K with power-of-two w, so that every dot product, block
    mean (B a power of two), weighted sum and head-sum is exact in fp32 and fp64."""
    rng = np.random.Generator(np.random.PCG64(seed))
    Kv = rng.integers(-kmax, kmax + 1, size=(n_k, d)).astype(np.float64)
    Qv = rng.integers(-qmax, qmax + 1, size=(n_q, H, d)).astype(np.float64)
    wexp = rng.integers(-3, 2, size=(n_q, H))
    wsign = np.where(rng.integers(0, 4, size=(n_q, H)) == 0, -1.0, 1.0)
    w = (wsign * np.ldexp(1.0, wexp)).astype(np.float32)
    return {"Q": bf16_bits(Qv), "K": bf16_bits(Kv), "w": w,
            "needles": np.zeros(0, dtype=np.int64)}
