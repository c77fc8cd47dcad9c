// Stage 5 — exact per-row top-k selection.
//
// For each row keep the k largest values, ties to the lower position, and
// write the kept positions in ascending order, padded with -1 ("MISA"
// technical summary, Metodologia step 2: the final top-k tokens are chosen from
// the routed scores).  Two row kinds share the kernel:
//   token rows      logits[t, 0 .. min(pos(t), n_k-1)]; output = token index;
//   candidate rows  full[t, 0 .. kp-1] (-inf = absent); output = cand[t, i]
//                   (MISA-dagger: final top-k among the re-scored candidates).
//
// Values are mapped to order-preserving 32-bit keys (-0.0 folded onto +0.0,
// -inf and padding to the reserved key 0).  One CTA per row:
//   pass 1   stream the row once from HBM, 4096-bin histogram of key >> 20;
//            the bin holding the k-th largest key follows from a block scan;
//   pass 2   (fast path) stream the row again — normally from L2 — and append,
//            in position order, every entry whose key is in or above that bin
//            to a shared-memory list (block scans give each thread its slots);
//   refine   two 10-bit histogram rounds over the list pin the exact k-th key
//            T and how many entries equal to T are still needed;
//   select   one ordered pass over the list keeps key > T, and keys == T while
//            their rank among equals is below the need: output is ascending by
//            construction and ties resolve to the lower position.
// If the candidate list would not fit in shared memory (massive ties), the
// refine rounds and the ordered selection run over the row in global memory.
#include "internal.h"

namespace misa {
namespace {

constexpr int kTopkThreads = 512;
constexpr int kWarps = kTopkThreads / 32;
constexpr int kBins1 = 4096;
constexpr int kChunk = 4 * kTopkThreads;  // entries per block-wide step

struct TopkParams {
  const float* vals;
  int64_t ld;
  int n_q;
  int64_t q_pos0;
  int64_t n_k;
  int row_len;           // candidate rows only
  const int32_t* cand;   // nullptr: token rows
  int k;
  int32_t* idx;
  int cap;               // shared-memory list capacity (entries)
  DevCtl ctl;
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

struct OutEmit {
  int32_t* out;           // idx row
  const int32_t* cand;    // candidate row or nullptr
  uint32_t k;
  __device__ __forceinline__ void operator()(uint32_t slot, uint32_t, uint32_t pos) const {
    if (slot < k) out[slot] = cand ? __ldg(cand + pos) : static_cast<int32_t>(pos);
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

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const TopkParams p) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);
  SmemCtl& sc = *reinterpret_cast<SmemCtl*>(smem_raw + kBins1 * 4);
  uint32_t* lkeys = reinterpret_cast<uint32_t*>(smem_raw + kBins1 * 4 + sizeof(SmemCtl));
  uint32_t* lposs = lkeys + p.cap;

  const int t = blockIdx.x;
  const uint32_t k = static_cast<uint32_t>(p.k);
  int64_t n;
  const int32_t* cand_row = nullptr;
  if (p.cand) {
    n = p.row_len;
    cand_row = p.cand + static_cast<int64_t>(t) * p.row_len;
  } else {
    n = min(p.q_pos0 + t + 1, p.n_k);
  }
  const float* row = p.vals + static_cast<int64_t>(t) * p.ld;
  const RowSrc src{row, n, (reinterpret_cast<uintptr_t>(row) & 15u) == 0u};
  const OutEmit out{p.idx + static_cast<int64_t>(t) * p.k, cand_row, k};
  if (k == 0) return;

  // ---- pass 1: histogram of key >> 20
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
      // ---- pass 2: ordered list of the entries in or above bin b1
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

}  // namespace

cudaError_t launch_topk(const float* vals, int64_t ld, int n_q, int64_t q_pos0, int64_t n_k,
                        int row_len, const int32_t* cand, int k, int32_t* idx,
                        const DevCtl& ctl, cudaStream_t s) {
  if (n_q <= 0 || k <= 0) return cudaSuccess;
  int cap = std::max(8192, ((2 * k + 4096) + 1023) / 1024 * 1024);
  if (cand) cap = std::max(cap, ((row_len + 1023) / 1024) * 1024);
  cap = std::min(cap, 24576);
  const size_t smem = kBins1 * 4 + sizeof(SmemCtl) + static_cast<size_t>(cap) * 8;
  cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  TopkParams p{vals, ld, n_q, q_pos0, n_k, row_len, cand, k, idx, cap, ctl};
  topk_kernel<<<n_q, kTopkThreads, smem, s>>>(p);
  return cudaGetLastError();
}

}  // namespace misa
