// Stage 5 — exact per-row top-k selection.
//
// For each row keep the k largest values, ties to the lower position, and
// write the kept positions in ascending order, padded with -1 ("MISA"
// technical summary, Metodologia step 2: the final top-k tokens are chosen from
// the routed scores).  Token rows are logits[t, 0 .. min(pos(t), n_k-1)] and
// the output is the token index.  Candidate rows (MISA-dagger, Variante
// Hierarquica: the final top-k among the re-scored candidates) have a kernel of
// their own at the end of this file.
//
// Values are mapped to order-preserving 32-bit keys (-0.0 folded onto +0.0,
// -inf and padding to the reserved key 0).  One CTA per row.
//
// Fast path (k <= 12288, rows of at most 131072 entries):
//   sample   32 contiguous 128-entry blocks spread over the row; the lower
//            edge of the 22-bit key bin holding the m-th largest sampled key,
//            m ~ 1.4 k * (sample / row), becomes a threshold tau (the 2m-th
//            gives a lower one, used for one re-stream if the list is short);
//   stream   ONE pass over the row from HBM with no atomics: every key >= tau
//            is appended, warp-compacted with ballots, to the warp's own region
//            of a shared-memory list (warps own interleaved 128-entry chunks);
//   check    if the list holds at least k entries it holds the whole top-k
//            (every key above the k-th largest is >= tau), including every
//            entry equal to the k-th largest key;
//   select   three radix rounds (12 + 10 + 10 bits) over the list give the
//            exact k-th key T and how many entries equal to T are kept (the
//            lowest positions); kept positions are set in a bitmap of the row
//            and a block scan over its words writes them out in ascending order.
// Fallback (sample too optimistic, list overflow, k > 12288, longer rows): a 4096-bin
// histogram pass, an ordered collection of the entries in or above the k-th
// bin (block scans keep position order), the same radix refinement, and an
// ordered selection pass — over the shared-memory list when it fits, else over
// the row in global memory.
//
// Fused top-k helpers (used by misa_score_topk with the select-mode scoring):
// a sample gather of 32 x 128 keys, a per-row threshold from the scored sample,
// and the exact selection over the logits the select pass kept (pass-mask bits,
// values in place), which flags rows it cannot finish for the exact repair.
#include <type_traits>

#include "internal.h"

namespace misa {
namespace {

constexpr int kTopkThreads = 256;
constexpr int kWarps = kTopkThreads / 32;
constexpr int kBins1 = 4096;
constexpr int kChunk = 4 * kTopkThreads;  // entries per block-wide step
constexpr int kFastMaxK = 12288;          // largest k of the fast path
constexpr int kSampleTarget = 4096;       // sampled entries per row (at most)
constexpr int kFastCap = 5120;            // list entries of the fast path (all warps)
constexpr int kCtasPerSm = 3;             // resident CTAs the fast path is sized for
constexpr double kSampleMargin = 1.4;     // list target: ~1.4 k entries above tau
constexpr int kEqMax = 1024;              // entries equal to the k-th key (fast path)

struct TopkParams {
  const float* vals;
  int64_t ld;
  int n_q;
  int64_t q_pos0;
  int64_t n_k;
  int k;
  int32_t* idx;
  int cap;               // shared-memory list capacity (entries)
  DevCtl ctl;
  const int* gate;       // nullable: row t is done unless gate[1 + t] != 0
  const int32_t* row_len;  // nullable: row t has row_len[t] visible entries (else pos(t) + 1)
};

__device__ __forceinline__ uint32_t f2key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;              // -0.0 ranks as +0.0
  if (b == 0xFF800000u) return 0u;           // -inf: absent
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct SmemCtl {
  uint32_t scan[kWarps];
  uint32_t res[4];
};

// Exclusive prefix over the block of one value per thread; `total` = block sum.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, SmemCtl& sc, uint32_t& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) sc.scan[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t s = lane < kWarps ? sc.scan[lane] : 0u;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, s, off);
      if (lane >= off) s += y;
    }
    if (lane < kWarps) sc.scan[lane] = s;
  }
  __syncthreads();
  const uint32_t before = warp > 0 ? sc.scan[warp - 1] : 0u;
  total = sc.scan[kWarps - 1];
  __syncthreads();
  return before + x - v;
}

// Finds the bin where the count from the top reaches `need` (1 <= need <= sum).
// Writes bin to sc.res[0] and the count strictly above it to sc.res[1].
template <int NB>
__device__ __forceinline__ void find_bin(const uint32_t* hist, uint32_t need, SmemCtl& sc) {
  constexpr int PER = NB / kTopkThreads;
  uint32_t loc[PER];
  uint32_t s = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    loc[i] = hist[threadIdx.x * PER + i];
    s += loc[i];
  }
  uint32_t total;
  const uint32_t excl = block_excl_scan(s, sc, total);
  uint32_t above = total - excl - s;
#pragma unroll
  for (int i = PER - 1; i >= 0; --i) {
    if (above < need && above + loc[i] >= need) {
      sc.res[0] = threadIdx.x * PER + i;
      sc.res[1] = above;
    }
    above += loc[i];
  }
  __syncthreads();
}

// Entries of one row in global memory (position = index in the row).
struct RowSrc {
  const float* row;
  int64_t n;
  bool aligned;
  __device__ __forceinline__ void load4(int64_t i0, uint32_t (&key)[4], uint32_t (&pos)[4]) const {
    if (aligned && i0 + 3 < n) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(row + i0));
      key[0] = f2key(v.x);
      key[1] = f2key(v.y);
      key[2] = f2key(v.z);
      key[3] = f2key(v.w);
    } else {
#pragma unroll
      for (int e = 0; e < 4; ++e) key[e] = (i0 + e < n) ? f2key(__ldg(row + i0 + e)) : 0u;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) pos[e] = static_cast<uint32_t>(i0 + e);
  }
};

// Entries of the shared-memory candidate list.
struct ListSrc {
  const uint32_t* keys;
  const uint32_t* poss;
  int64_t n;
  __device__ __forceinline__ void load4(int64_t i0, uint32_t (&key)[4], uint32_t (&pos)[4]) const {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool in = i0 + e < n;
      key[e] = in ? keys[i0 + e] : 0u;
      pos[e] = in ? poss[i0 + e] : 0u;
    }
  }
};

struct ListEmit {
  uint32_t* keys;
  uint32_t* poss;
  __device__ __forceinline__ void operator()(uint32_t slot, uint32_t key, uint32_t pos) const {
    keys[slot] = key;
    poss[slot] = pos;
  }
};

// Writes the position (a token index) of a kept entry to its output slot.
struct OutEmit {
  int32_t* out;           // idx row
  uint32_t k;
  __device__ __forceinline__ void operator()(uint32_t slot, uint32_t, uint32_t pos) const {
    if (slot < k) out[slot] = static_cast<int32_t>(pos);
  }
};

// One ordered pass: keeps key > T, and key == T while its rank among the
// entries equal to T (in position order) is below `need`.  Emits kept entries
// to consecutive slots in position order; stops once `stop_after` are kept.
// Returns the number kept (uniform).
template <class Src, class Emit>
__device__ uint32_t ordered_select(const Src& src, uint32_t T, uint32_t need, uint32_t stop_after,
                                   const Emit& emit, SmemCtl& sc) {
  uint32_t kept = 0, eq_seen = 0;
  for (int64_t base = 0; base < src.n; base += kChunk) {
    uint32_t key[4], pos[4];
    src.load4(base + threadIdx.x * 4, key, pos);
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      gt += key[e] > T;
      eq += (key[e] == T && key[e] != 0u);
    }
    uint32_t total;
    const uint32_t excl = block_excl_scan(gt | (eq << 16), sc, total);
    const uint32_t gt_before = excl & 0xFFFFu, eq_before = excl >> 16;
    uint32_t eq_rank = eq_seen + eq_before;
    uint32_t slot = kept + gt_before + (min(eq_rank, need) - min(eq_seen, need));
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      if (key[e] > T) {
        emit(slot++, key[e], pos[e]);
      } else if (key[e] == T && key[e] != 0u) {
        if (eq_rank < need) emit(slot++, key[e], pos[e]);
        ++eq_rank;
      }
    }
    const uint32_t gt_total = total & 0xFFFFu, eq_total = total >> 16;
    kept += gt_total + (min(eq_seen + eq_total, need) - min(eq_seen, need));
    eq_seen += eq_total;
    if (kept >= stop_after) break;
  }
  return kept;
}

// Histogram of the 10-bit digit at `shift` over entries whose key >> mshift == mval.
template <class Src>
__device__ void digit_hist(const Src& src, uint32_t mshift, uint32_t mval, uint32_t shift,
                           uint32_t* hist) {
  for (int i = threadIdx.x; i < 1024; i += kTopkThreads) hist[i] = 0u;
  __syncthreads();
  for (int64_t base = 0; base < src.n; base += kChunk) {
    uint32_t key[4], pos[4];
    src.load4(base + threadIdx.x * 4, key, pos);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (key[e] != 0u && (key[e] >> mshift) == mval) atomicAdd(&hist[(key[e] >> shift) & 1023u], 1u);
  }
  __syncthreads();
}

// Levels 2 and 3: from the level-1 bin b1 and the count above it, find the
// exact k-th key T and how many entries equal to T to keep.
template <class Src>
__device__ void refine(const Src& src, uint32_t b1, uint32_t above1, uint32_t k, uint32_t* hist,
                       SmemCtl& sc, uint32_t& T, uint32_t& need_eq) {
  uint32_t need = k - above1;
  digit_hist(src, 20, b1, 10, hist);
  find_bin<1024>(hist, need, sc);
  const uint32_t b2 = sc.res[0];
  need -= sc.res[1];
  __syncthreads();
  digit_hist(src, 10, (b1 << 10) | b2, 0, hist);
  find_bin<1024>(hist, need, sc);
  const uint32_t b3 = sc.res[0];
  need -= sc.res[1];
  __syncthreads();
  T = (b1 << 20) | (b2 << 10) | b3;
  need_eq = need;
}

// Entries of the per-warp regions of the fast-path list (flattened; slots past
// a region's count read as absent).
struct RegionSrc {
  const uint32_t* keys;
  const uint32_t* poss;
  const uint32_t* counts;  // [kWarps]
  int64_t n;               // kWarps * region
  uint32_t region;         // entries per warp region
  uint32_t inv;            // ceil(2^32 / region): x / region = umulhi(x, inv) for x < 2^16
  __device__ __forceinline__ void load4(int64_t i0, uint32_t (&key)[4], uint32_t (&pos)[4]) const {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t x = static_cast<uint32_t>(i0) + e;
      const uint32_t w = __umulhi(x, inv), j = x - w * region;
      const bool in = x < static_cast<uint32_t>(n) && j < counts[w];
      key[e] = in ? keys[x] : 0u;
      pos[e] = in ? poss[x] : 0u;
    }
  }
};

// Exact m-th largest key T among the present entries of `src` (1 <= m <=
// present); `need` = how many entries equal to T belong to the m largest.
// A radix select with the digits placed where the keys differ: every
// present key shares the bits above the highest bit in which the largest and
// the smallest present key differ, and each round histograms the next (at
// most) 12 bits below the bits already fixed, among the entries that still
// agree with the answer on them.  The lists this selects from hold a narrow
// band of values (the kept top few percent of a row), which a fixed top-bits
// digit piles onto a few bins (and their shared-memory atomics onto a few
// addresses); here they spread over up to 4096 bins.
// kWholeBin: when the bin of the m-th key holds exactly the entries still
// needed, stop there and return T = bin floor - 1 with need = 0 (every entry
// above T is taken, none equal to it) -- for callers that take the entries by
// "key > T, then `need` of key == T" and nothing else.
template <class Src, bool kWholeBin = false>
__device__ uint32_t kth_largest_spread(const Src& src, uint32_t m, uint32_t* hist, SmemCtl& sc,
                                       uint32_t& need) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int64_t base = 0; base < src.n; base += kChunk) {
    uint32_t key[4], pos[4];
    src.load4(base + threadIdx.x * 4, key, pos);
#pragma unroll
    for (int e = 0; e < 4; ++e)
      if (key[e] != 0u) {
        lo = min(lo, key[e]);
        hi = max(hi, key[e]);
      }
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    lo = min(lo, __shfl_xor_sync(0xffffffffu, lo, off));
    hi = max(hi, __shfl_xor_sync(0xffffffffu, hi, off));
  }
  if (lane == 0) {
    sc.scan[warp] = lo;
    hist[warp] = hi;
  }
  __syncthreads();
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    lo = min(lo, sc.scan[w]);
    hi = max(hi, hist[w]);
  }
  __syncthreads();
  const uint32_t diff = hi ^ lo;
  if (diff == 0u) {  // every present key equal
    need = m;
    return hi;
  }
  int hib = 31 - __clz(diff);  // bits above hib are common to every present key
  uint32_t T = hib == 31 ? 0u : (hi >> (hib + 1)) << (hib + 1);
  while (true) {
    const int lob = hib >= 11 ? hib - 11 : 0;
    const uint32_t dmask = (1u << (hib - lob + 1)) - 1u;
    for (int i = threadIdx.x; i < kBins1; i += kTopkThreads) hist[i] = 0u;
    __syncthreads();
    for (int64_t base = 0; base < src.n; base += kChunk) {
      uint32_t key[4], pos[4];
      src.load4(base + threadIdx.x * 4, key, pos);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool agree = hib == 31 || (key[e] >> (hib + 1)) == (T >> (hib + 1));
        if (key[e] != 0u && agree) atomicAdd(&hist[(key[e] >> lob) & dmask], 1u);
      }
    }
    __syncthreads();
    find_bin<kBins1>(hist, m, sc);
    T |= sc.res[0] << lob;
    m -= sc.res[1];
    const bool whole = kWholeBin && lob > 0 && T > 0u && hist[sc.res[0]] == m;
    __syncthreads();
    if (whole) {  // T is the bin floor
      need = 0u;
      return T - 1u;
    }
    if (lob == 0) break;
    hib = lob - 1;
  }
  need = m;
  return T;
}

// Ascending bitonic sort of buf[0..n) in shared memory (next power of two of n
// must fit in the buffer).
__device__ void bitonic_sort_asc(uint32_t* buf, uint32_t n) {
  uint32_t P = 1, logP = 0;
  while (P < n) {
    P <<= 1;
    ++logP;
  }
  for (uint32_t i = n + threadIdx.x; i < P; i += kTopkThreads) buf[i] = 0xFFFFFFFFu;
  __syncthreads();
  for (uint32_t ls = 1; ls <= logP; ++ls) {
    const uint32_t size = 1u << ls;
    for (int lst = static_cast<int>(ls) - 1; lst >= 0; --lst) {
      const uint32_t stride = 1u << lst;
      for (uint32_t i = threadIdx.x; i < P / 2; i += kTopkThreads) {
        const uint32_t lo = ((i >> lst) << (lst + 1)) | (i & (stride - 1)), hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const uint32_t a = buf[lo], b = buf[hi];
        if ((a > b) == asc) {
          buf[lo] = b;
          buf[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

// Emits, in ascending order, the positions whose bits are set in bitmap[0..words)
// to out slots 0.. and pads the rest of the k slots with -1.  Each thread owns a
// contiguous run of words; a block scan gives every run its first slot.
__device__ void emit_bitmap(const uint32_t* bitmap, uint32_t words, const OutEmit& out,
                            SmemCtl& sc) {
  const uint32_t per = (words + kTopkThreads - 1) / kTopkThreads;
  const uint32_t w0 = threadIdx.x * per, w1 = min(w0 + per, words);
  uint32_t c = 0;
  for (uint32_t i = w0; i < w1; ++i) c += __popc(bitmap[i]);
  uint32_t total;
  uint32_t slot = block_excl_scan(c, sc, total);
  for (uint32_t i = w0; i < w1; ++i) {
    uint32_t m = bitmap[i];
    while (m) {
      const uint32_t b = __ffs(m) - 1u;
      out(slot++, 0u, i * 32u + b);
      m &= m - 1u;
    }
  }
  for (uint32_t i = total + threadIdx.x; i < out.k; i += kTopkThreads) out.out[i] = -1;
}

// Fast path.  Returns false (and writes nothing) when the row must take the
// fallback path.  Shared memory: hist [kBins1], list keys/poss [cap] (kFastCap
// for k <= 4096, more for larger k), sel [kEqMax], counts [kWarps].
__device__ bool topk_fast(const TopkParams& p, const RowSrc& src, const OutEmit& out,
                          uint32_t* hist, uint32_t* lkeys, uint32_t* lposs, uint32_t* sel,
                          uint32_t* counts, SmemCtl& sc) {
  const uint32_t k = out.k;
  const int64_t n = src.n;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  // ---- thresholds from a sample: 32 contiguous 128-entry blocks spread over
  // the row.  tau (expected ~1.4 k entries above it) is the lower edge of the
  // 22-bit key bin holding the m-th largest sampled key; tau_retry, used when
  // the list comes out short, is the same for the 2m-th.
  uint32_t tau = 1u, tau_retry = 1u;
  if (n > p.cap) {
    constexpr int kBlocks = kSampleTarget / 128;
    const int64_t gap = (n / kBlocks) & ~static_cast<int64_t>(3);   // keeps float4 alignment
    for (int i = threadIdx.x; i < kSampleTarget / 4; i += kTopkThreads) {
      const int b = i / 32, c = i % 32;
      uint32_t key[4], pos[4];
      src.load4(b * gap + c * 4, key, pos);
#pragma unroll
      for (int e = 0; e < 4; ++e) lkeys[i * 4 + e] = key[e];
    }
    __syncthreads();
    const uint32_t sn = kSampleTarget;
    const double frac = static_cast<double>(sn) / static_cast<double>(n);
    const uint32_t m = static_cast<uint32_t>(kSampleMargin * k * frac) + 8u;
    const ListSrc ls{lkeys, lposs, static_cast<int64_t>(sn)};
    for (int i = threadIdx.x; i < kBins1; i += kTopkThreads) hist[i] = 0u;
    __syncthreads();
    for (uint32_t i = threadIdx.x; i < sn; i += kTopkThreads)
      if (lkeys[i] != 0u) atomicAdd(&hist[lkeys[i] >> 20], 1u);
    __syncthreads();
    uint32_t present;
    {
      uint32_t c = 0;
      for (int i = threadIdx.x; i < kBins1; i += kTopkThreads) c += hist[i];
      block_excl_scan(c, sc, present);
    }
    // 22-bit bin lower edges of the m-th and 2m-th largest sampled keys
    if (m <= present) {
      const uint32_t m2 = 2u * m <= present ? 2u * m : present;
      find_bin<kBins1>(hist, m, sc);
      const uint32_t b1 = sc.res[0], above1 = sc.res[1];
      __syncthreads();
      find_bin<kBins1>(hist, m2, sc);
      const uint32_t b1r = sc.res[0], above1r = sc.res[1];
      __syncthreads();
      digit_hist(ls, 20, b1, 10, hist);
      find_bin<1024>(hist, m - above1, sc);
      tau = (b1 << 20) | (sc.res[0] << 10);
      __syncthreads();
      digit_hist(ls, 20, b1r, 10, hist);
      find_bin<1024>(hist, m2 - above1r, sc);
      tau_retry = (b1r << 20) | (sc.res[0] << 10);
      if (tau == 0u) tau = 1u;
      if (tau_retry == 0u) tau_retry = 1u;
    }
    __syncthreads();
  }
  const uint32_t region = static_cast<uint32_t>(p.cap / kWarps);  // list entries per warp
  uint32_t total = 0;
  for (int attempt = 0; attempt < 2; ++attempt) {
  // ---- one pass: warp-compacted append of every key >= tau.  The test runs on
  // the float values (x >= value of tau: the same order, -0.0 == +0.0, -inf
  // never passes); only the few passing values are turned into keys.
  float tau_f;
  {
    const uint32_t b = tau & 0x80000000u ? tau & 0x7FFFFFFFu : ~tau;  // key -> float bits
    tau_f = tau <= 1u ? -3.402823466e38f : __uint_as_float(b);
  }
  uint32_t cnt = 0;  // this warp's entries (warp-uniform)
  bool overflow = false;
  uint32_t* wk = lkeys + warp * region;
  uint32_t* wp = lposs + warp * region;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int64_t nfull = src.aligned ? n / 128 : 0;   // chunks read without bounds checks
  const int64_t nchunks = (n + 127) / 128;
  constexpr int U = 8;
  auto consume = [&](const float (&x)[4], int64_t base) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool pass = x[e] >= tau_f;
      const uint32_t m = __ballot_sync(0xffffffffu, pass);
      if (m == 0u) continue;
      const uint32_t tot = __popc(m);
      if (cnt + tot > region) {
        overflow = true;
        continue;
      }
      if (pass) {
        const uint32_t slot = cnt + __popc(m & lt_mask);
        wk[slot] = f2key(x[e]);
        wp[slot] = static_cast<uint32_t>(base + lane * 4 + e);
      }
      cnt += tot;
    }
  };
  int64_t c0 = warp;
  for (; c0 + (U - 1) * kWarps < nfull; c0 += U * kWarps) {
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u)
      v[u] = __ldg(reinterpret_cast<const float4*>(src.row + (c0 + u * kWarps) * 128 + lane * 4));
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      consume(x, (c0 + u * kWarps) * 128);
    }
  }
  for (; c0 < nchunks; c0 += kWarps) {
    const int64_t i0 = c0 * 128 + lane * 4;
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = i0 + e < n ? __ldg(src.row + i0 + e) : -INFINITY;
    consume(x, c0 * 128);
  }
  if (lane == 0) counts[warp] = overflow ? 0xFFFFFFFFu : cnt;
  __syncthreads();
  total = 0;
  bool any_over = false;
#pragma unroll
  for (int w = 0; w < kWarps; ++w) {
    any_over |= counts[w] == 0xFFFFFFFFu;
    total += counts[w];
  }
  if (any_over) return false;
  if (tau <= 1u || total >= k) break;
  // short: every key >= tau is in the list but fewer than k of them; stream
  // again with the lower threshold (or give up if it is no lower)
  if (attempt == 1 || tau_retry >= tau) return false;
  tau = tau_retry;
  __syncthreads();
  }  // attempts
  const uint32_t inv = static_cast<uint32_t>((0x100000000ull + region - 1) / region);
  const RegionSrc rs{lkeys, lposs, counts, static_cast<int64_t>(kWarps) * region, region, inv};
  // ---- exact k-th key within the list
  uint32_t T = 0u, need = 0u;
  if (total > k) T = kth_largest_spread<RegionSrc, true>(rs, k, hist, sc, need);
  // ---- kept positions: key > T, and the `need` lowest positions with key == T,
  // marked in a bitmap of the row (ascending output without a sort)
  uint32_t* bitmap = hist;                       // kBins1 words = 131072 positions
  const uint32_t words = static_cast<uint32_t>((n + 31) / 32);
  uint32_t* neq = &sc.res[3];
  for (uint32_t i = threadIdx.x; i < static_cast<uint32_t>(kBins1); i += kTopkThreads) bitmap[i] = 0u;
  if (threadIdx.x == 0) *neq = 0u;
  __syncthreads();
  for (uint32_t x = threadIdx.x; x < static_cast<uint32_t>(rs.n); x += kTopkThreads) {
    const uint32_t w = __umulhi(x, inv), j = x - w * region;
    if (j >= counts[w]) continue;
    const uint32_t key = lkeys[x];
    const uint32_t pos = lposs[x];
    if (key > T) {
      atomicOr(&bitmap[pos >> 5], 1u << (pos & 31u));
    } else if (need > 0u && key == T && key != 0u) {  // (need = 0: no tie is taken)
      const uint32_t e = atomicAdd(neq, 1u);
      if (e < static_cast<uint32_t>(kEqMax)) sel[e] = pos;
    }
  }
  __syncthreads();
  const uint32_t n_eq = *neq;
  if (n_eq > static_cast<uint32_t>(kEqMax)) return false;      // massive ties: fallback
  if (n_eq > need) bitonic_sort_asc(sel, n_eq);                // lowest positions first
  for (uint32_t i = threadIdx.x; i < need; i += kTopkThreads)
    atomicOr(&bitmap[sel[i] >> 5], 1u << (sel[i] & 31u));
  __syncthreads();
  emit_bitmap(bitmap, words, out, sc);
  return true;
}

// Row t of a top-k launch (all of the block's threads).
__device__ void topk_row(const TopkParams& p, int t, uint8_t* smem_raw) {
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  SmemCtl& sc = *reinterpret_cast<SmemCtl*>(smem_raw + kBins1 * 4);
  uint32_t* lkeys = reinterpret_cast<uint32_t*>(smem_raw + kBins1 * 4 + sizeof(SmemCtl));
  uint32_t* lposs = lkeys + p.cap;
  uint32_t* sel = lposs + p.cap;             // fast path only: ties at the k-th key
  uint32_t* counts = sel + kEqMax;           // fast path only

  const uint32_t k = static_cast<uint32_t>(p.k);
  const int64_t n = p.row_len ? max(int64_t(0), min(static_cast<int64_t>(__ldg(p.row_len + t)), p.n_k))
                              : min(p.q_pos0 + t + 1, p.n_k);
  const float* row = p.vals + static_cast<int64_t>(t) * p.ld;
  const RowSrc src{row, n, (reinterpret_cast<uintptr_t>(row) & 15u) == 0u};
  const OutEmit out{p.idx + static_cast<int64_t>(t) * p.k, k};
  if (k == 0) return;
  if (k <= static_cast<uint32_t>(kFastMaxK) && n <= 32 * kBins1 &&
      topk_fast(p, src, out, hist, lkeys, lposs, sel, counts, sc))
    return;
  __syncthreads();

  // ---- fallback pass 1: histogram of key >> 20
  for (int i = threadIdx.x; i < kBins1; i += kTopkThreads) hist[i] = 0u;
  __syncthreads();
  {
    constexpr int U = 4;
    for (int64_t base = 0; base < n; base += U * kChunk) {
      uint32_t key[U][4], pos[4];
#pragma unroll
      for (int u = 0; u < U; ++u) src.load4(base + u * kChunk + threadIdx.x * 4, key[u], pos);
#pragma unroll
      for (int u = 0; u < U; ++u)
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (key[u][e] != 0u) atomicAdd(&hist[key[u][e] >> 20], 1u);
    }
  }
  __syncthreads();

  // total number of present entries
  uint32_t present;
  {
    uint32_t s = 0;
    for (int i = threadIdx.x; i < kBins1; i += kTopkThreads) s += hist[i];
    block_excl_scan(s, sc, present);
  }

  uint32_t T = 0, need_eq = 0;
  uint32_t kept;
  if (present <= k) {
    kept = ordered_select(src, 0u, 0u, k, out, sc);  // every present entry
  } else {
    find_bin<kBins1>(hist, k, sc);
    const uint32_t b1 = sc.res[0], above1 = sc.res[1];
    const uint32_t in_or_above = above1 + hist[b1];
    __syncthreads();
    if (in_or_above <= static_cast<uint32_t>(p.cap)) {
      // ordered list of the entries in or above bin b1
      const ListEmit le{lkeys, lposs};
      const uint32_t cnt = ordered_select(src, (b1 << 20) - 1u, 0u, 0xFFFFFFFFu, le, sc);
      __syncthreads();
      const ListSrc ls{lkeys, lposs, static_cast<int64_t>(cnt)};
      refine(ls, b1, above1, k, hist, sc, T, need_eq);
      kept = ordered_select(ls, T, need_eq, k, out, sc);
    } else {
      refine(src, b1, above1, k, hist, sc, T, need_eq);
      kept = ordered_select(src, T, need_eq, k, out, sc);
    }
  }
  for (uint32_t i = min(kept, k) + threadIdx.x; i < k; i += kTopkThreads) out.out[i] = -1;
}

__global__ void __launch_bounds__(kTopkThreads, kCtasPerSm)
topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  topk_row(p, blockIdx.x, smem_raw);
}

// The repair launch: only rows with gate[1 + t] != 0, a persistent grid that
// walks the row flags (nothing but the flag reads when no row is flagged).
__global__ void __launch_bounds__(kTopkThreads, kCtasPerSm)
topk_gated_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  if (p.gate[0] == 0) return;  // no row flagged
  for (int t = blockIdx.x; t < p.n_q; t += gridDim.x) {
    if (p.gate[1 + t] == 0) continue;
    topk_row(p, t, smem_raw);
    __syncthreads();  // shared memory is reused by the next flagged row
  }
}

// ---------------------------------------------------------------- fused top-k
// The scoring kernel in select mode keeps, per row, only the logits at or above
// a threshold tau; the kernels below choose tau from a scored sample of the
// row's visible keys and then take the exact top-k among the kept candidates.

constexpr double kFusedMargin = 1.4;  // ~1.4 k candidates expected above tau
constexpr int kSampleBlock = 128;     // keys per contiguous sample block

// Copies the keys of n_blocks contiguous 128-key blocks, evenly spaced over
// [0, span), into a dense sample (and their FP8 scales when given); the keys
// come from a contiguous or a paged cache.
__global__ void __launch_bounds__(256)
gather_sample_kernel(const uint8_t* __restrict__ K, const float* __restrict__ k_scale, KeyPages kpg,
                     int row_bytes, int64_t span, int n_blocks, uint8_t* __restrict__ Ks,
                     float* __restrict__ ks_scale, DevCtl ctl) {
  const int b = blockIdx.x;
  const int64_t start = n_blocks > 1 ? (span - kSampleBlock) * b / (n_blocks - 1) : 0;
  const int upr = row_bytes / 16;
  const int units = kSampleBlock * upr;
  uint4* dst = reinterpret_cast<uint4*>(Ks + static_cast<int64_t>(b) * kSampleBlock * row_bytes);
  for (int i = threadIdx.x; i < units; i += blockDim.x) {
    const int r = i / upr;
    const int64_t prow = kpg.row(start + r, ctl);
    dst[i] = __ldg(reinterpret_cast<const uint4*>(K + prow * row_bytes) + (i - r * upr));
  }
  if (k_scale)
    for (int i = threadIdx.x; i < kSampleBlock; i += blockDim.x)
      ks_scale[b * kSampleBlock + i] = __ldg(k_scale + kpg.row(start + i, ctl));
}

// Per row: tau[t] = lower edge of the 22-bit key bin holding the m-th largest
// sampled logit, m ~ 1.4 k * n_s / visible(t) (or -inf: keep every visible key).
// Also zeroes the row's repair flag gate[1 + t] and (block 0) the any-row flag
// gate[0].
constexpr int kTauPer = 16;  // sample keys held per thread: n_s <= kTauPer * kTopkThreads

__global__ void __launch_bounds__(kTopkThreads)
fused_tau_kernel(const float* __restrict__ sample, int64_t lds, int n_s, int64_t q_pos0,
                 int64_t n_k, int k, float* __restrict__ tau, int* __restrict__ gate) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  SmemCtl& sc = *reinterpret_cast<SmemCtl*>(smem_raw + kBins1 * 4);
  const int t = blockIdx.x;
  if (threadIdx.x == 0) {
    gate[1 + t] = 0;
    if (t == 0) gate[0] = 0;
  }
  const int64_t visible = min(q_pos0 + t + 1, n_k);
  const float* row = sample + static_cast<int64_t>(t) * lds;
  // the row's sampled logits as keys in registers (0 = absent or past n_s),
  // every load issued before the first is used
  uint32_t key[kTauPer];
  if ((n_s & 3) == 0 && (reinterpret_cast<uintptr_t>(row) & 15u) == 0) {
    const float4* row4 = reinterpret_cast<const float4*>(row);
    const int n4 = n_s >> 2;
    float4 v[kTauPer / 4];
#pragma unroll
    for (int j = 0; j < kTauPer / 4; ++j) {
      const int i = threadIdx.x + j * kTopkThreads;
      v[j] = i < n4 ? __ldg(row4 + i) : make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
    }
#pragma unroll
    for (int j = 0; j < kTauPer / 4; ++j) {
      key[4 * j] = f2key(v[j].x);
      key[4 * j + 1] = f2key(v[j].y);
      key[4 * j + 2] = f2key(v[j].z);
      key[4 * j + 3] = f2key(v[j].w);
    }
  } else {
    float v[kTauPer];
#pragma unroll
    for (int j = 0; j < kTauPer; ++j) {
      const int i = threadIdx.x + j * kTopkThreads;
      v[j] = i < n_s ? __ldg(row + i) : -INFINITY;
    }
#pragma unroll
    for (int j = 0; j < kTauPer; ++j) key[j] = f2key(v[j]);
  }
  for (int i = threadIdx.x; i < kBins1; i += kTopkThreads) hist[i] = 0u;
  uint32_t c = 0;
#pragma unroll
  for (int j = 0; j < kTauPer; ++j) c += key[j] != 0u;
  uint32_t present;
  block_excl_scan(c, sc, present);  // (also orders the zeroing before the counts below)
  const uint32_t m = static_cast<uint32_t>(kFusedMargin * k * static_cast<double>(n_s) /
                                           static_cast<double>(visible)) + 16u;
  float tf = -INFINITY;
  if (m <= present) {
    // the m-th largest key's 12-bit top digit, then its next 10 bits
#pragma unroll
    for (int j = 0; j < kTauPer; ++j)
      if (key[j] != 0u) atomicAdd(&hist[key[j] >> 20], 1u);
    __syncthreads();
    find_bin<kBins1>(hist, m, sc);
    const uint32_t b1 = sc.res[0], above1 = sc.res[1];
    __syncthreads();
    for (int i = threadIdx.x; i < 1024; i += kTopkThreads) hist[i] = 0u;
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kTauPer; ++j)
      if (key[j] != 0u && (key[j] >> 20) == b1) atomicAdd(&hist[(key[j] >> 10) & 1023u], 1u);
    __syncthreads();
    find_bin<1024>(hist, m - above1, sc);
    const uint32_t tk = (b1 << 20) | (sc.res[0] << 10);  // >= every real key's bin floor
    const uint32_t bits = (tk & 0x80000000u) ? (tk & 0x7FFFFFFFu) : ~tk;  // key -> float bits
    tf = __uint_as_float(bits);
  }
  if (threadIdx.x == 0) tau[t] = tf;
}

// List entries whose positions are kept as their low 16 bits: the list is in
// position order, so the high bits of entry i's position count the 65536-key
// boundaries at or below it (cross[j] = entries below position 65536 (j + 1)).
struct ListSrc16 {
  const uint32_t* keys;
  const uint16_t* poss;
  int64_t n;
  uint32_t cross[3];
  __device__ __forceinline__ uint32_t pos(int64_t i) const {
    const uint32_t hi = (i >= cross[0] ? 1u : 0u) + (i >= cross[1] ? 1u : 0u) + (i >= cross[2] ? 1u : 0u);
    return static_cast<uint32_t>(poss[i]) | (hi << 16);
  }
  __device__ __forceinline__ void load4(int64_t i0, uint32_t (&key)[4], uint32_t (&pos4)[4]) const {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int64_t i = i0 + e;
      const bool in = i < n;
      key[e] = in ? keys[i] : 0u;
      pos4[e] = in ? pos(i) : 0u;
    }
  }
};

__device__ __forceinline__ uint32_t entry_pos(const ListSrc& s, uint32_t i) { return s.poss[i]; }
__device__ __forceinline__ uint32_t entry_pos(const ListSrc16& s, uint32_t i) { return s.pos(i); }

// ordered_select over a list of at most 65535 entries with a single block
// scan: each thread takes a contiguous run of entries, so the runs' counts in
// thread order give every kept entry its slot in list order.  The run length
// is odd, so a warp's lanes read 32 different shared-memory banks.
template <class Src, class Emit>
__device__ uint32_t ordered_select_runs(const Src& src, uint32_t T, uint32_t need, const Emit& emit,
                                        SmemCtl& sc) {
  const uint32_t n = static_cast<uint32_t>(src.n);
  const uint32_t per = ((n + kTopkThreads - 1) / kTopkThreads) | 1u;
  const uint32_t i0 = min(threadIdx.x * per, n), i1 = min(i0 + per, n);
  uint32_t gt = 0, eq = 0;
  for (uint32_t i = i0; i < i1; ++i) {
    const uint32_t key = src.keys[i];
    gt += key > T;
    eq += key == T && key != 0u;
  }
  uint32_t total;
  const uint32_t excl = block_excl_scan(gt | (eq << 16), sc, total);
  uint32_t eq_rank = excl >> 16;
  uint32_t slot = (excl & 0xFFFFu) + min(eq_rank, need);
  for (uint32_t i = i0; i < i1; ++i) {
    const uint32_t key = src.keys[i];
    if (key > T) {
      emit(slot++, key, entry_pos(src, i));
    } else if (key == T && key != 0u) {
      if (eq_rank < need) emit(slot++, key, entry_pos(src, i));
      ++eq_rank;
    }
  }
  return (total & 0xFFFFu) + min(total >> 16, need);
}

// Per row: the exact top-k among the logits the select-mode scoring kept (the
// bits of the row's pass mask; their values stored in place).  They hold the
// whole top-k whenever at least min(k, visible) of them passed.  Rows short of
// that, or with more than list_cap kept, raise their repair flag (and the
// any-row flag gate[0]) and write nothing.  P16 (large k): positions are
// staged as 16-bit halves (6 bytes per list entry instead of 8), so the long
// lists of large k still fit two CTAs per SM.
template <bool P16>
__global__ void __launch_bounds__(kTopkThreads)
fused_finish_kernel(const float* __restrict__ logits, int64_t ld, const uint32_t* __restrict__ mask,
                    int64_t mask_ld, int64_t q_pos0, int64_t n_k, int k, int32_t* __restrict__ idx,
                    int* __restrict__ gate, int list_cap) {
  using Pos = typename std::conditional<P16, uint16_t, uint32_t>::type;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  SmemCtl& sc = *reinterpret_cast<SmemCtl*>(smem_raw + kBins1 * 4);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kBins1 * 4 + sizeof(SmemCtl));
  Pos* poss = reinterpret_cast<Pos*>(keys + list_cap);
  const int t = blockIdx.x;
  const int64_t visible = min(q_pos0 + t + 1, n_k);
  // every thread owns a run of 4-word units (the scoring pass wrote whole
  // 128-key tiles, so the words up to the next multiple of 4 exist and hold
  // no bit past the row's last visible key)
  const uint32_t units = static_cast<uint32_t>((visible + 127) / 128);
  const uint32_t per = (units + kTopkThreads - 1) / kTopkThreads;
  const uint32_t u0 = min(threadIdx.x * per, units), u1 = min(u0 + per, units);
  const uint4* mrow = reinterpret_cast<const uint4*>(mask + static_cast<int64_t>(t) * mask_ld);
  if (P16) {
    // res[1 + j]: entries below position 65536 (j + 1), i.e. in units below 512 (j + 1)
    if (threadIdx.x < 3) sc.res[1 + threadIdx.x] = 0u;
    __syncthreads();
  }
  // the first kHold units of the run are loaded at once and stay in registers
  // for the second pass (all of it while n_k <= 131072)
  constexpr uint32_t kHold = 4;
  uint4 mh[kHold];
#pragma unroll
  for (uint32_t j = 0; j < kHold; ++j)
    mh[j] = u0 + j < u1 ? __ldg(mrow + u0 + j) : make_uint4(0u, 0u, 0u, 0u);
  uint32_t c = 0, c_lo[3] = {0u, 0u, 0u};
  auto count_unit = [&](uint32_t u, const uint4& m) {
    const uint32_t cu = __popc(m.x) + __popc(m.y) + __popc(m.z) + __popc(m.w);
    c += cu;
#pragma unroll
    for (int j = 0; j < 3; ++j)
      if (u < 512u * (j + 1)) c_lo[j] += cu;
  };
#pragma unroll
  for (uint32_t j = 0; j < kHold; ++j) count_unit(u0 + j, mh[j]);  // (zero past u1)
  for (uint32_t u = u0 + kHold; u < u1; ++u) count_unit(u, __ldg(mrow + u));
  if (P16) {
#pragma unroll
    for (int j = 0; j < 3; ++j)
      if (c_lo[j]) atomicAdd(&sc.res[1 + j], c_lo[j]);
  }
  uint32_t total;
  uint32_t slot = block_excl_scan(c, sc, total);  // (also publishes res[1..3])
  const uint32_t cross[3] = {P16 ? sc.res[1] : 0u, P16 ? sc.res[2] : 0u, P16 ? sc.res[3] : 0u};
  __syncthreads();  // every thread has read res before the selection reuses it
  const uint32_t need_total = static_cast<uint32_t>(visible < k ? visible : k);
  if (total < need_total || total > static_cast<uint32_t>(list_cap)) {
    if (threadIdx.x == 0) {
      gate[1 + t] = 1;
      atomicOr(gate, 1);
    }
    return;
  }
  // kept positions in ascending order, then their logits (batches of
  // independent loads)
  auto emit_unit = [&](uint32_t u, const uint4& m4) {
    const uint32_t mw[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t m = mw[q];
      while (m) {
        poss[slot++] = static_cast<Pos>((u * 4u + q) * 32u + static_cast<uint32_t>(__ffs(m) - 1));
        m &= m - 1u;
      }
    }
  };
#pragma unroll
  for (uint32_t j = 0; j < kHold; ++j) emit_unit(u0 + j, mh[j]);
  for (uint32_t u = u0 + kHold; u < u1; ++u) emit_unit(u, __ldg(mrow + u));
  __syncthreads();
  const float* row = logits + static_cast<int64_t>(t) * ld;
  const ListSrc16 ls16{keys, reinterpret_cast<const uint16_t*>(poss), static_cast<int64_t>(total),
                       {cross[0], cross[1], cross[2]}};
  auto pos_of = [&](uint32_t i) { return P16 ? ls16.pos(i) : static_cast<uint32_t>(poss[i]); };
  constexpr int kBatch = 16;
  for (uint32_t b0 = 0; b0 < total; b0 += kBatch * kTopkThreads) {
    float v[kBatch];
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const uint32_t i = b0 + j * kTopkThreads + threadIdx.x;
      v[j] = i < total ? __ldg(row + pos_of(i)) : 0.0f;
    }
#pragma unroll
    for (int j = 0; j < kBatch; ++j) {
      const uint32_t i = b0 + j * kTopkThreads + threadIdx.x;
      if (i < total) keys[i] = f2key(v[j]);
    }
  }
  __syncthreads();
  const OutEmit out{idx + static_cast<int64_t>(t) * k, static_cast<uint32_t>(k)};
  uint32_t T = 0u, need = 0u, kept;
  if constexpr (P16) {
    if (total > static_cast<uint32_t>(k))
      T = kth_largest_spread<ListSrc16, true>(ls16, static_cast<uint32_t>(k), hist, sc, need);
    kept = ordered_select_runs(ls16, T, need, out, sc);
  } else {
    const ListSrc ls{keys, reinterpret_cast<const uint32_t*>(poss), static_cast<int64_t>(total)};
    if (total > static_cast<uint32_t>(k))
      T = kth_largest_spread<ListSrc, true>(ls, static_cast<uint32_t>(k), hist, sc, need);
    kept = ordered_select_runs(ls, T, need, out, sc);
  }
  for (uint32_t i = min(kept, static_cast<uint32_t>(k)) + threadIdx.x; i < static_cast<uint32_t>(k);
       i += kTopkThreads)
    out.out[i] = -1;
}

// ---------------------------------------------------------------- candidate rows
// MISA-dagger final selection (Variante Hierarquica: the top-k among the
// re-scored candidates).  Row t holds the all-head scores vals[t*ldv + i] of
// the candidate tokens cand[t*kp + i]; a candidate is absent when its token
// lies outside 0..pos(t) (the -1 padding included) or its score is -inf.  The
// k present candidates of largest score are kept, ties to the lower TOKEN, and
// their tokens written ascending, -1 padded, whatever order the candidates
// come in.  The row (scores as order-preserving keys, and tokens) is staged in
// shared memory; three radix rounds over it give the exact k-th key T.
//   ascending rows (present tokens strictly increasing, absent entries only at
//   the end, which is what the coarse selection emits): one ordered pass, since
//   position order is token order;
//   any other row: the tokens tied at T are sorted and the lowest kept, then
//   the kept tokens are sorted and written.  Two kept entries with the same
//   token break the contract (distinct candidates) and are reported.
__device__ void select_candidates_row(const float* __restrict__ vals, int64_t ldv,
                                      const int32_t* __restrict__ cand, int kp, int64_t q_pos0,
                                      int64_t n_k, int k, int32_t* __restrict__ idx, int tmp_cap,
                                      const DevCtl& ctl, int t, uint8_t* smem_raw) {
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  SmemCtl& sc = *reinterpret_cast<SmemCtl*>(smem_raw + kBins1 * 4);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kBins1 * 4 + sizeof(SmemCtl));
  uint32_t* toks = keys + kp;
  uint32_t* tmp = toks + kp;  // tmp_cap entries: the next power of two >= kp
  const int64_t pos = q_pos0 + t;
  const float* vrow = vals + static_cast<int64_t>(t) * ldv;
  const int32_t* crow = cand + static_cast<int64_t>(t) * kp;
  int32_t* out = idx + static_cast<int64_t>(t) * k;
  const uint32_t kk = static_cast<uint32_t>(k);

  auto stage = [&](int i, float v, int32_t tok) {
    const bool valid = tok >= 0 && tok <= pos && tok < n_k;
    const uint32_t key = valid ? f2key(v) : 0u;
    keys[i] = key;
    toks[i] = static_cast<uint32_t>(tok);
    return key != 0u ? 1u : 0u;
  };
  uint32_t c = 0;
  const bool vec = (kp & 3) == 0 && (reinterpret_cast<uintptr_t>(vrow) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(crow) & 15u) == 0;
  if (vec) {
    for (int i = threadIdx.x * 4; i < kp; i += kTopkThreads * 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(vrow + i));
      const int4 tk = __ldg(reinterpret_cast<const int4*>(crow + i));
      c += stage(i, v.x, tk.x) + stage(i + 1, v.y, tk.y) + stage(i + 2, v.z, tk.z) +
           stage(i + 3, v.w, tk.w);
    }
  } else {
    for (int i = threadIdx.x; i < kp; i += kTopkThreads) c += stage(i, __ldg(vrow + i), __ldg(crow + i));
  }
  uint32_t present;
  block_excl_scan(c, sc, present);  // (also orders the stores above before the reads below)
  bool unordered = false;
  for (int i = threadIdx.x; i + 1 < kp; i += kTopkThreads)
    if (keys[i + 1] != 0u && (keys[i] == 0u || toks[i] >= toks[i + 1])) unordered = true;
  unordered = __syncthreads_or(unordered) != 0;

  const ListSrc ls{keys, toks, static_cast<int64_t>(kp)};
  uint32_t T = 0u, need = 0u;  // present <= k: every present entry (key > 0)
  if (present > kk)  // (ordered rows take entries only by key > T and `need` of key == T)
    T = unordered ? kth_largest_spread(ls, kk, hist, sc, need)
                  : kth_largest_spread<ListSrc, true>(ls, kk, hist, sc, need);
  if (!unordered) {
    const uint32_t kept = ordered_select(ls, T, need, kk, OutEmit{out, kk}, sc);
    for (uint32_t i = min(kept, kk) + threadIdx.x; i < kk; i += kTopkThreads) out[i] = -1;
    return;
  }
  // tokens tied at T: keep the `need` lowest (those <= cut)
  uint32_t cut = 0xFFFFFFFFu;
  if (present > kk) {
    if (threadIdx.x == 0) sc.res[2] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < kp; i += kTopkThreads)
      if (keys[i] == T) tmp[atomicAdd(&sc.res[2], 1u)] = toks[i];
    __syncthreads();
    const uint32_t n_eq = sc.res[2];
    if (n_eq > need) {
      bitonic_sort_asc(tmp, n_eq);
      cut = tmp[need - 1];
    }
  }
  if (threadIdx.x == 0) sc.res[3] = 0u;
  __syncthreads();  // every thread has read cut before tmp is refilled
  for (int i = threadIdx.x; i < kp; i += kTopkThreads) {
    const uint32_t key = keys[i];
    if (key > T || (key == T && key != 0u && toks[i] <= cut)) tmp[atomicAdd(&sc.res[3], 1u)] = toks[i];
  }
  __syncthreads();
  const uint32_t n_win = min(sc.res[3], static_cast<uint32_t>(tmp_cap));
  bitonic_sort_asc(tmp, n_win);
  bool dup = false;
  for (uint32_t i = threadIdx.x; i + 1 < n_win; i += kTopkThreads) dup |= tmp[i] == tmp[i + 1];
  if (__syncthreads_or(dup) && threadIdx.x == 0) report(ctl, DEV_BAD_INPUT);
  for (uint32_t i = threadIdx.x; i < kk; i += kTopkThreads)
    out[i] = i < n_win ? static_cast<int32_t>(tmp[i]) : -1;
}

// The rows the ordered kernel below marked (idx row starting with kUnorderedRow)
// — candidates in any order — over a persistent grid.
constexpr int32_t kUnorderedRow = -2;

__global__ void __launch_bounds__(kTopkThreads)
select_candidates_kernel(const float* __restrict__ vals, int64_t ldv,
                         const int32_t* __restrict__ cand, int kp, int n_q, int64_t q_pos0,
                         int64_t n_k, int k, int32_t* __restrict__ idx, int tmp_cap, DevCtl ctl) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  for (int t = blockIdx.x; t < n_q; t += gridDim.x) {
    if (idx[static_cast<int64_t>(t) * k] != kUnorderedRow) continue;
    __syncthreads();  // every thread has read the marker before the row is rewritten
    select_candidates_row(vals, ldv, cand, kp, q_pos0, n_k, k, idx, tmp_cap, ctl, t, smem_raw);
    __syncthreads();  // shared memory is reused by the next marked row
  }
}

// Candidate entries: keys staged in shared memory, tokens read where they are.
struct CandSrc {
  const uint32_t* keys;
  const int32_t* toks;
  int64_t n;
  __device__ __forceinline__ void load4(int64_t i0, uint32_t (&key)[4], uint32_t (&pos)[4]) const {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const bool in = i0 + e < n;
      key[e] = in ? keys[i0 + e] : 0u;
      pos[e] = in ? static_cast<uint32_t>(__ldg(toks + i0 + e)) : 0u;
    }
  }
};

// Rows whose valid candidates ascend, with only absent entries after them (what
// the coarse selection emits): only the keys are staged (48 KB of shared
// memory, four CTAs per SM), the tokens are read from the candidate row, and
// one ordered pass writes the selection.  Any other row gets kUnorderedRow in
// its first output slot and is left to select_candidates_kernel.
__global__ void __launch_bounds__(kTopkThreads)
select_candidates_ordered_kernel(const float* __restrict__ vals, int64_t ldv,
                                 const int32_t* __restrict__ cand, int kp, int64_t q_pos0,
                                 int64_t n_k, int k, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  SmemCtl& sc = *reinterpret_cast<SmemCtl*>(smem_raw + kBins1 * 4);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + kBins1 * 4 + sizeof(SmemCtl));
  const int t = blockIdx.x;
  const int64_t pos = q_pos0 + t;
  const float* vrow = vals + static_cast<int64_t>(t) * ldv;
  const int32_t* crow = cand + static_cast<int64_t>(t) * kp;
  int32_t* out = idx + static_cast<int64_t>(t) * k;
  const uint32_t kk = static_cast<uint32_t>(k);
  auto stage = [&](int i, float v, int32_t tok) {
    const bool valid = tok >= 0 && tok <= pos && tok < n_k;
    const uint32_t key = valid ? f2key(v) : 0u;
    keys[i] = key;
    return key != 0u ? 1u : 0u;
  };
  uint32_t c = 0;
  bool unordered = false;
  const bool vec = (kp & 3) == 0 && (reinterpret_cast<uintptr_t>(vrow) & 15u) == 0 &&
                   (reinterpret_cast<uintptr_t>(crow) & 15u) == 0;
  if (vec) {
    for (int i = threadIdx.x * 4; i < kp; i += kTopkThreads * 4) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(vrow + i));
      const int4 tk = __ldg(reinterpret_cast<const int4*>(crow + i));
      c += stage(i, v.x, tk.x) + stage(i + 1, v.y, tk.y) + stage(i + 2, v.z, tk.z) +
           stage(i + 3, v.w, tk.w);
    }
  } else {
    for (int i = threadIdx.x; i < kp; i += kTopkThreads) c += stage(i, __ldg(vrow + i), __ldg(crow + i));
  }
  uint32_t present;
  block_excl_scan(c, sc, present);  // (also orders the key writes before the reads below)
  for (int i = threadIdx.x; i + 1 < kp; i += kTopkThreads)
    if (keys[i + 1] != 0u && (keys[i] == 0u || __ldg(crow + i) >= __ldg(crow + i + 1))) unordered = true;
  if (__syncthreads_or(unordered)) {
    if (threadIdx.x == 0) out[0] = kUnorderedRow;
    return;
  }
  const CandSrc src{keys, crow, static_cast<int64_t>(kp)};
  uint32_t T = 0u, need = 0u;  // present <= k: every present entry (key > 0)
  if (present > kk) T = kth_largest_spread<CandSrc, true>(src, kk, hist, sc, need);
  const uint32_t kept = ordered_select(src, T, need, kk, OutEmit{out, kk}, sc);
  for (uint32_t i = min(kept, kk) + threadIdx.x; i < kk; i += kTopkThreads) out[i] = -1;
}

}  // namespace

cudaError_t launch_topk(const float* vals, int64_t ld, int n_q, int64_t q_pos0, int64_t n_k,
                        int k, int32_t* idx, const DevCtl& ctl, cudaStream_t s, const int* gate,
                        const int32_t* row_len) {
  if (n_q <= 0 || k <= 0) return cudaSuccess;
  // list capacity: kFastCap for k <= 2048 (three CTAs per SM); larger k need
  // room for ~1.4 k sampled-threshold entries (fast path; the list is split into
  // equal per-warp regions, so with headroom for the warps' uneven shares) or
  // for the entries in or above the k-th histogram bin (fallback)
  int cap = k <= 2048 ? kFastCap
                      : (k <= 4096 ? (2 * k + 1023) / 1024 * 1024
                                   : std::min(24576, ((2 * k + 4096) + 1023) / 1024 * 1024));
  const size_t smem = kBins1 * 4 + sizeof(SmemCtl) + static_cast<size_t>(cap) * 8 +
                      (k <= kFastMaxK ? (kEqMax + kWarps) * 4 : 0);
  TopkParams p{vals, ld, n_q, q_pos0, n_k, k, idx, cap, ctl, gate, row_len};
  if (gate) {
    cudaError_t e = cudaFuncSetAttribute(topk_gated_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem));
    if (e != cudaSuccess) return e;
    const int grid = std::min(n_q, kCtasPerSm * sm_count());
    topk_gated_kernel<<<grid, kTopkThreads, smem, s>>>(p);
    return cudaGetLastError();
  }
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  topk_kernel<<<n_q, kTopkThreads, smem, s>>>(p);
  return cudaGetLastError();
}

cudaError_t launch_gather_sample(const void* K, const float* k_scale, const KeyPages& kpg,
                                 int row_bytes, int64_t span, int n_blocks, void* Ks,
                                 float* ks_scale, const DevCtl& ctl, cudaStream_t s) {
  gather_sample_kernel<<<n_blocks, 256, 0, s>>>(static_cast<const uint8_t*>(K), k_scale, kpg,
                                                row_bytes, span, n_blocks,
                                                static_cast<uint8_t*>(Ks), ks_scale, ctl);
  return cudaGetLastError();
}

cudaError_t launch_fused_tau(const float* sample, int64_t lds, int n_s, int n_q, int64_t q_pos0,
                             int64_t n_k, int k, float* tau, int* gate, cudaStream_t s) {
  if (n_q <= 0) return cudaSuccess;
  if (n_s > kTauPer * kTopkThreads) return cudaErrorInvalidValue;
  const size_t smem = kBins1 * 4 + sizeof(SmemCtl);
  cudaError_t e = cudaFuncSetAttribute(fused_tau_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  fused_tau_kernel<<<n_q, kTopkThreads, smem, s>>>(sample, lds, n_s, q_pos0, n_k, k, tau, gate);
  return cudaGetLastError();
}

cudaError_t launch_select_candidates(const float* vals, int64_t ldv, const int32_t* cand, int kp,
                                     int n_q, int64_t q_pos0, int64_t n_k, int k, int32_t* idx,
                                     const DevCtl& ctl, cudaStream_t s) {
  if (n_q <= 0 || k <= 0 || kp <= 0) return cudaSuccess;
  // every row through the ordered kernel; rows it marks through the general one
  const size_t smem1 = kBins1 * 4 + sizeof(SmemCtl) + static_cast<size_t>(kp) * 4;
  cudaError_t e = cudaFuncSetAttribute(select_candidates_ordered_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem1));
  if (e != cudaSuccess) return e;
  select_candidates_ordered_kernel<<<n_q, kTopkThreads, smem1, s>>>(vals, ldv, cand, kp, q_pos0,
                                                                    n_k, k, idx);
  int cap = 1;
  while (cap < kp) cap <<= 1;
  const size_t smem = kBins1 * 4 + sizeof(SmemCtl) + (2 * static_cast<size_t>(kp) + cap) * 4;
  e = cudaFuncSetAttribute(select_candidates_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int grid = std::min(n_q, 2 * sm_count());
  select_candidates_kernel<<<grid, kTopkThreads, smem, s>>>(vals, ldv, cand, kp, n_q, q_pos0, n_k,
                                                            k, idx, cap, ctl);
  return cudaGetLastError();
}

// k <= 4096: 8-byte entries, max(6144, 3k) of them (three CTAs per SM at k =
// 2048); larger k: 6-byte entries, 2k of them (two CTAs per SM at k = 8192, whose
// kept lists run ~1.5 k on the chunk with threshold margin 1.4).
int fused_list_cap(int k) {
  return k <= 4096 ? std::max(6144, (3 * k + 1023) / 1024 * 1024) : (2 * k + 1023) / 1024 * 1024;
}

cudaError_t launch_fused_finish(const float* logits, int64_t ld, const uint32_t* mask,
                                int64_t mask_ld, int n_q, int64_t q_pos0, int64_t n_k, int k,
                                int32_t* idx, int* gate, cudaStream_t s) {
  if (n_q <= 0 || k <= 0) return cudaSuccess;
  const int cap = fused_list_cap(k);
  const bool p16 = k > 4096;
  const size_t smem = kBins1 * 4 + sizeof(SmemCtl) + static_cast<size_t>(cap) * (p16 ? 6 : 8);
  auto kern = p16 ? fused_finish_kernel<true> : fused_finish_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  kern<<<n_q, kTopkThreads, smem, s>>>(logits, ld, mask, mask_ld, q_pos0, n_k, k, idx, gate, cap);
  return cudaGetLastError();
}


}  // namespace misa
