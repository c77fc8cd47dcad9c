// MISA-dagger fine stage, scoring part — all-head scores of gathered candidates.
//
//   full[t, i] = sum_{j<H} w[t, j] * ReLU(q[t, j] . k_c),  c = cand[t, i] in 0..pos(t)
//
// ("MISA" technical summary, Variante Hierarquica: the original all-head DSA
// indexer re-scores only the k' candidates kept by the routed coarse pass.)
// The top-k among the candidates is taken afterwards by the top-k kernel in
// candidate mode.
//
// Per query, a dense contraction on the tensor cores: A = 128 candidate key
// rows gathered from K (16-byte loads into the swizzled K-major layout; FP8 keys
// are decoded to bf16 on the way, exactly), B = the query's H head rows, D =
// 128 x H fp32 in TMEM.  TMEM lane = candidate, so each epilogue thread reduces
// ReLU * w over the H columns of its own lane.  The work is bound by the gather
// from L2, not by the MMA.
//
// Warp roles (416 threads): warps 0-3 gather producers, warp 4 TMEM allocator
// and MMA issuer, warps 5-12 epilogue in two groups of four: group g takes the
// tiles of accumulator g (even / odd tiles of the CTA's sequence).  Queries are
// distributed round-robin over a persistent grid.
#include "internal.h"

namespace misa {
namespace {

constexpr int kCand = 128;  // MMA M: candidates per tile
constexpr int kRerankThreads = 416;
constexpr int kProducers = 128;
constexpr uint64_t kDrainNs = 2000000;

template <int D, int NB>
struct RerankLayout {
  static constexpr int ROWB = D >= 64 ? 128 : 64;
  static constexpr int A_CHUNK = kCand * ROWB;
  static constexpr int A_BYTES = kCand * D * 2;
  static constexpr int B_CHUNK = NB * ROWB;
  static constexpr int B_BYTES = NB * D * 2;
  static constexpr int STAGES = 4;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_W = OFF_B + ((B_BYTES + 1023) / 1024) * 1024;  // 8 warps x NB floats
  static constexpr int OFF_BAR = OFF_W + 8 * NB * 4;
  static constexpr int NBAR = 2 * STAGES + 6;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
};

struct RerankParams {
  const uint16_t* Q;
  const float* w;
  const uint8_t* K;
  const float* k_scale;
  const int32_t* cand;
  int kp;
  int n_q;
  int64_t q_pos0;
  int64_t n_k;
  int H;
  float* full;
  int64_t ldf;
  DevCtl ctl;
  KeyPages kpg;  // paged key cache (kpg.bt != nullptr) or contiguous
};

template <int D, int NB, bool FP8>
__global__ void __launch_bounds__(kRerankThreads, 1)
rerank_scores_kernel(const RerankParams p) {
  using L = RerankLayout<D, NB>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const uint32_t sA = smem_u32(smem + L::OFF_A);
  const uint32_t sB = smem_u32(smem + L::OFF_B);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = L::STAGES, BFULL = 2 * L::STAGES, BEMPTY = BFULL + 1,
            ACCFULL = BFULL + 2, ACCEMPTY = BFULL + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  constexpr uint32_t kTmemCols = 2 * NB <= 32 ? 32 : (2 * NB <= 64 ? 64 : (2 * NB <= 128 ? 128 : 256));

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::STAGES; ++i) {
      mbar_init(bar(FULL + i), kProducers);
      mbar_init(bar(EMPTY + i), 1);
    }
    mbar_init(bar(BFULL), kProducers);
    mbar_init(bar(BEMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(ACCFULL + i), 1);
      mbar_init(bar(ACCEMPTY + i), 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 4) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int tiles = (p.kp + kCand - 1) / kCand;
  constexpr int UPC = L::ROWB / 16;      // 16-byte units per swizzle-chunk row
  constexpr int UPR = D / 8;             // bf16 16-byte units per key row

  if (warp < 4) {
    // ------------------------------------------------------------ gather producers
    const int tid = threadIdx.x;  // 0..127
    int stage = 0;
    uint32_t phase = 0, qcount = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < p.n_q && ok; t += gridDim.x) {
      const int64_t pos = p.q_pos0 + t;
      // B: the query's H head rows, zero rows up to NB
      ok = mbar_wait(bar(BEMPTY), (qcount & 1) ^ 1, abort_flag, p.ctl);
      if (!ok) break;
      for (int x = tid; x < NB * UPR; x += kProducers) {
        const int n = x / UPR, u = x % UPR;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (n < p.H)
          v = __ldg(reinterpret_cast<const uint4*>(p.Q + (static_cast<int64_t>(t) * p.H + n) * D + u * 8));
        const uint32_t off = (u / UPC) * L::B_CHUNK + swz_offset(n, u % UPC, L::ROWB);
        asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(sB + off), "r"(v.x), "r"(v.y),
                     "r"(v.z), "r"(v.w)
                     : "memory");
      }
      fence_proxy_async_smem();
      mbar_arrive(bar(BFULL));
      ++qcount;
      // each producer thread holds one candidate of every tile: its index is
      // loaded kAhead tiles ahead and checked (and mapped to a physical row) one
      // tile ahead, so no index load stalls the copies; all of a tile's copies
      // are in flight at once (bf16: asynchronous 16-byte copies, whole rows per
      // warp instruction, arriving on the stage barrier when they land; FP8:
      // each thread loads its own row's codes for the next tile while decoding
      // this tile's)
      const int32_t* crow = p.cand + static_cast<int64_t>(t) * p.kp;
      auto raw_of = [&](int tile) -> int32_t {
        const int i = tile * kCand + tid;
        return (tile < tiles && i < p.kp) ? __ldg(crow + i) : -1;
      };
      // physical key row of a candidate (-1: ignored)
      auto row_of = [&](int32_t c) -> int64_t {
        return (c >= 0 && c <= pos && c < p.n_k) ? p.kpg.row(c, p.ctl) : -1;
      };
      constexpr int kAhead = 4;
      int32_t rq[kAhead];
#pragma unroll
      for (int i = 0; i < kAhead; ++i) rq[i] = raw_of(i);
      constexpr int U8 = D / 16;  // 16-byte units of an e4m3 row
      int64_t c_next = tiles > 0 ? row_of(rq[0]) : -1;
      uint4 raw_next[FP8 ? U8 : 1];
      if constexpr (FP8) {
#pragma unroll
        for (int u = 0; u < U8; ++u)
          raw_next[u] = c_next >= 0 ? __ldg(reinterpret_cast<const uint4*>(p.K + c_next * D) + u)
                                    : make_uint4(0u, 0u, 0u, 0u);
      }
      for (int tile = 0; tile < tiles; ++tile) {
        const int64_t c = c_next;
        uint4 raw[FP8 ? U8 : 1];
        if constexpr (FP8) {
#pragma unroll
          for (int u = 0; u < U8; ++u) raw[u] = raw_next[u];
        }
#pragma unroll
        for (int i = 0; i + 1 < kAhead; ++i) rq[i] = rq[i + 1];
        rq[kAhead - 1] = raw_of(tile + kAhead);
        if (tile + 1 < tiles) c_next = row_of(rq[0]);
        if constexpr (FP8) {
#pragma unroll
          for (int u = 0; u < U8; ++u)
            raw_next[u] = (tile + 1 < tiles && c_next >= 0)
                              ? __ldg(reinterpret_cast<const uint4*>(p.K + c_next * D) + u)
                              : make_uint4(0u, 0u, 0u, 0u);
        }
        ok = mbar_wait(bar(EMPTY + stage), phase ^ 1, abort_flag, p.ctl);
        if (!ok) break;
        const uint32_t dstA = sA + stage * L::A_BYTES;
        if constexpr (FP8) {
#pragma unroll
          for (int u = 0; u < U8; ++u) {
            const uint32_t wv[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {  // 8 codes -> 8 bf16 (exact)
              const uint32_t b0 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh] & 0xFFFF));
              const uint32_t b1 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh] >> 16));
              const uint32_t b2 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh + 1] & 0xFFFF));
              const uint32_t b3 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh + 1] >> 16));
              const int u2 = 2 * u + hh;
              const uint32_t off = (u2 / UPC) * L::A_CHUNK + swz_offset(tid, u2 % UPC, L::ROWB);
              asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dstA + off), "r"(b0),
                           "r"(b1), "r"(b2), "r"(b3)
                           : "memory");
            }
          }
          fence_proxy_async_smem();
          mbar_arrive(bar(FULL + stage));
        } else {
          // warp w copies rows 32w..32w+31, UPR lanes per row so that one
          // instruction reads whole rows (full 128-byte lines); lane i holds the
          // candidate of row 32w+i
          constexpr int RPI = 32 / UPR;  // rows per instruction
          const int wr0 = tid & ~31;
#pragma unroll
          for (int j = 0; j < UPR; ++j) {
            const int rr = j * RPI + lane / UPR;
            const int u = lane % UPR;
            const int64_t cr = __shfl_sync(0xffffffffu, c, rr);
            const uint32_t off = (u / UPC) * L::A_CHUNK + swz_offset(wr0 + rr, u % UPC, L::ROWB);
            cp_async16(dstA + off, p.K + ((cr >= 0 ? cr : 0) * D + u * 8) * 2, cr >= 0 ? 16u : 0u);
          }
          cp_async_mbar_arrive_noinc(bar(FULL + stage));
        }
        if (++stage == L::STAGES) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0, acc = 0;
    uint32_t phase = 0, accph = 0, qcount = 0;
    bool ok = true;
    constexpr uint32_t idesc = umma_idesc_bf16_f32(kCand, NB);
    for (int t = blockIdx.x; t < p.n_q && ok; t += gridDim.x) {
      if (lane == 0) {
        ok = mbar_wait(bar(BFULL), qcount & 1, abort_flag, p.ctl);
        for (int tile = 0; tile < tiles && ok; ++tile) {
          ok = mbar_wait(bar(FULL + stage), phase, abort_flag, p.ctl) &&
               mbar_wait(bar(ACCEMPTY + acc), accph ^ 1, abort_flag, p.ctl);
          if (!ok) break;
          fence_proxy_async_smem();  // copies observed through the barrier -> MMA operand reads
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * NB);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int c = (kk * 32) / L::ROWB, within = (kk * 32) % L::ROWB;
            const uint64_t ad =
                umma_desc_kmajor(sA + stage * L::A_BYTES + c * L::A_CHUNK + within, L::ROWB);
            const uint64_t bd = umma_desc_kmajor(sB + c * L::B_CHUNK + within, L::ROWB);
            tc_mma_bf16(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(EMPTY + stage));
          tc_commit(bar(ACCFULL + acc));
          if (tile == tiles - 1) tc_commit(bar(BEMPTY));
          if (++stage == L::STAGES) {
            stage = 0;
            phase ^= 1;
          }
          if (++acc == 2) {
            acc = 0;
            accph ^= 1;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      stage = __shfl_sync(0xffffffffu, stage, 0);
      phase = __shfl_sync(0xffffffffu, phase, 0);
      acc = __shfl_sync(0xffffffffu, acc, 0);
      accph = __shfl_sync(0xffffffffu, accph, 0);
      ++qcount;
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;
    const int grp = (warp - 5) >> 2;  // accumulator (and tile parity) of this group
    float* w_s = reinterpret_cast<float*>(smem + L::OFF_W) + (warp - 5) * NB;
    uint32_t accph = 0;
    int64_t gtile = 0;  // tiles of the CTA's sequence before this query
    bool ok = true;
    for (int t = blockIdx.x; t < p.n_q && ok; t += gridDim.x) {
      const int64_t pos = p.q_pos0 + t;
      for (int i = lane; i < NB; i += 32)
        w_s[i] = i < p.H ? __ldg(p.w + static_cast<int64_t>(t) * p.H + i) : 0.0f;
      __syncwarp();
      // this lane's candidate of each of the group's tiles: its index loaded
      // two of the group's tiles ahead and checked one ahead (and, for FP8
      // keys, its scale loaded one ahead)
      const int first = static_cast<int>((grp - gtile % 2 + 2) % 2);
      const int32_t* crow = p.cand + static_cast<int64_t>(t) * p.kp;
      auto raw_of = [&](int tile) -> int32_t {
        const int i = tile * kCand + quad * 32 + lane;
        return (tile < tiles && i < p.kp) ? __ldg(crow + i) : -1;
      };
      // a candidate's physical key row (for the FP8 scale), -1 when ignored
      auto row_of = [&](int32_t c) -> int64_t {
        if (c < 0 || c > pos || c >= p.n_k) return -1;
        return FP8 ? p.kpg.row(c, p.ctl) : c;
      };
      int32_t r_nxt = raw_of(first + 2), r_far = raw_of(first + 4);
      int64_t c_cur = row_of(raw_of(first));
      float ks_cur = (FP8 && c_cur >= 0) ? __ldg(p.k_scale + c_cur) : 1.0f;
      for (int tile = first; tile < tiles; tile += 2) {
        if (lane == 0) ok = mbar_wait(bar(ACCFULL + grp), accph, abort_flag, p.ctl);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tbase = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                               static_cast<uint32_t>(grp * NB);
        float2 a0 = make_float2(0.0f, 0.0f), a1 = make_float2(0.0f, 0.0f);
        if (NB >= 32) {
#pragma unroll 1
          for (int c = 0; c < NB / 32; ++c) {
            uint32_t v[32];
            tmem_ld32(tbase + static_cast<uint32_t>(c * 32), v);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 32; e += 4) {
              const float4 w4 = *reinterpret_cast<const float4*>(w_s + c * 32 + e);
              a0 = fma2(make_float2(w4.x, w4.y),
                        make_float2(relu(__uint_as_float(v[e])), relu(__uint_as_float(v[e + 1]))), a0);
              a1 = fma2(make_float2(w4.z, w4.w),
                        make_float2(relu(__uint_as_float(v[e + 2])), relu(__uint_as_float(v[e + 3]))), a1);
            }
          }
        } else {
          uint32_t v[16];
          tmem_ld16(tbase, v);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; e += 4) {
            const float4 w4 = *reinterpret_cast<const float4*>(w_s + e);
            a0 = fma2(make_float2(w4.x, w4.y),
                      make_float2(relu(__uint_as_float(v[e])), relu(__uint_as_float(v[e + 1]))), a0);
            a1 = fma2(make_float2(w4.z, w4.w),
                      make_float2(relu(__uint_as_float(v[e + 2])), relu(__uint_as_float(v[e + 3]))), a1);
          }
        }
        const float sum = (a0.x + a0.y) + (a1.x + a1.y);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ACCEMPTY + grp));
        accph ^= 1;
        const int i = tile * kCand + quad * 32 + lane;
        if (i < p.kp)
          p.full[static_cast<int64_t>(t) * p.ldf + i] =
              c_cur >= 0 ? (FP8 ? sum * ks_cur : sum) : -INFINITY;
        c_cur = row_of(r_nxt);
        r_nxt = r_far;
        r_far = raw_of(tile + 6);
        ks_cur = (FP8 && c_cur >= 0) ? __ldg(p.k_scale + c_cur) : 1.0f;
      }
      gtile += tiles;
      __syncwarp();  // w_s is rewritten for the next query
    }
  }

  __syncthreads();
  if (*abort_flag) drain_pause(kDrainNs);
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

template <int D, int NB, bool FP8>
cudaError_t launch3(const RerankParams& p, cudaStream_t s) {
  using L = RerankLayout<D, NB>;
  auto kern = rerank_scores_kernel<D, NB, FP8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  const int grid = std::min(sm_count(), p.n_q);
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, kRerankThreads, L::ALLOC, s>>>(p);
  return cudaGetLastError();
}

template <int D, bool FP8>
cudaError_t launch2(const RerankParams& p, cudaStream_t s) {
  if (p.H <= 16) return launch3<D, 16, FP8>(p, s);
  if (p.H <= 32) return launch3<D, 32, FP8>(p, s);
  if (p.H <= 64) return launch3<D, 64, FP8>(p, s);
  if (p.H <= 128) return launch3<D, 128, FP8>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_rerank_scores(const uint16_t* Q, const float* w, const void* K,
                                 const float* k_scale, const KeyPages& kpg, bool fp8,
                                 const int32_t* cand, int kp, int n_q, int64_t q_pos0, int64_t n_k,
                                 int H, int d, float* full, int64_t ldf, const DevCtl& ctl,
                                 cudaStream_t s) {
  if (n_q <= 0 || kp <= 0) return cudaSuccess;
  RerankParams p{Q, w, static_cast<const uint8_t*>(K), k_scale, cand, kp, n_q, q_pos0, n_k, H, full,
                 ldf, ctl, kpg};
  if (fp8) {
    switch (d) {
      case 32: return launch2<32, true>(p, s);
      case 64: return launch2<64, true>(p, s);
      case 128: return launch2<128, true>(p, s);
    }
  } else {
    switch (d) {
      case 32: return launch2<32, false>(p, s);
      case 64: return launch2<64, false>(p, s);
      case 128: return launch2<128, false>(p, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace misa
