// Stages 2-3 — block-pooled router and top-h head selection.
//
//   r[t, j] = w[t, j] * sum_{m in C(t)} ReLU(q[t, j] . kbar_m)
//   heads[t] = the h heads of largest r (ties: lower head index), ascending
//
// ("MISA" technical summary, Metodologia step 1: per-head affinities against
// the mean-pooled block keys are aggregated into one importance per head and
// the top-h heads are kept; C(t) = the complete blocks whose last key is at or
// before pos(t).)
//
// A dense contraction on the tensor cores: A = 128 consecutive (query, head)
// rows of Q (128/H queries), B = a 128-block tile of the pooled keys, twice —
// once for hi = bf16(kbar) and once for lo = bf16(kbar - hi) — accumulated into
// the same fp32 TMEM tile, so the pooled keys carry ~16 significant bits.  TMEM
// lane = (query, head), column = block: each epilogue thread sums ReLU over its
// own row's causal columns, then the 4 epilogue warps exchange r through shared
// memory and one warp per query runs the top-h as h rounds of a warp argmax.
//
// Work unit: NA consecutive 128-row tiles contracted against the same stream
// of pooled-key tiles (prefill: NA = 2, so each hi/lo tile pair read from L2
// feeds 256 rows; decode: NA = 1, each query has pooled keys of its own).
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocator and MMA issuer, then
// 4 * NA epilogue warps (one per TMEM lane quadrant and row tile: one
// tcgen05.ld of the 128 block columns per tile, the accumulator handed back
// right after it lands), then 2 top-h warps.  The epilogue hands each unit's
// partial sums to the top-h warps through a double-buffered shared array, so
// the (latency-bound) selection of one unit overlaps the contraction of the
// next.  Pooled-key tiles stream through a 2- or 3-stage ring.  Units are
// distributed round-robin over a persistent grid.
#include "internal.h"

namespace misa {
namespace {

constexpr int kRows = 128;    // MMA M: (query, head) rows per tile
constexpr int kBlkN = 128;    // MMA N: pooled blocks per tile
constexpr int kRouteTopWarps = 2;
constexpr uint64_t kDrainNs = 2000000;
constexpr int kMaxDynSmem = 232448;  // per block (227 KB)

// NA = row tiles a CTA contracts against each pooled-key tile (prefill: 2, so
// each pooled-key tile read from L2 serves 256 (query, head) rows; decode: 1,
// every query has pooled keys of its own).  Four epilogue warps per row tile.
template <int NA>
struct RouteRoles {
  static constexpr int EPI = 4 * NA;
  static constexpr int THREADS = 64 + 32 * (EPI + kRouteTopWarps);
};

template <int D, int NA>
struct RouteLayout {
  static constexpr int ROWB = D >= 64 ? 128 : 64;
  static constexpr int KCH = D * 2 / ROWB;
  static constexpr int A_CHUNK = kRows * ROWB;
  static constexpr int A_BYTES = kRows * D * 2;
  static constexpr int B_CHUNK = kBlkN * ROWB;
  static constexpr int B_HALF = kBlkN * D * 2;           // hi or lo tile
  static constexpr int R_BYTES = 2 * NA * kRows * 4;     // [2 buf][NA * kRows] block sums
  static constexpr int STAGES_FIT = (kMaxDynSmem - 1024 - 512 - R_BYTES - NA * A_BYTES) / (2 * B_HALF);
  static constexpr int STAGES = STAGES_FIT < 3 ? STAGES_FIT : 3;
  static_assert(STAGES >= 2, "pooled-key ring needs two stages");
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NA * A_BYTES;
  static constexpr int OFF_R = OFF_B + STAGES * 2 * B_HALF;
  static constexpr int OFF_BAR = OFF_R + R_BYTES;
  static constexpr int NBAR = 2 * STAGES + 10;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static_assert(ALLOC <= kMaxDynSmem, "shared memory");
};

struct RouteParams {
  const float* w;
  int32_t* heads;
  float* r_out;
  int n_q;
  int64_t q_pos0;
  int64_t n_k;
  int H;
  int B;
  int h;
  int row_tiles;
  DevCtl ctl;
  // decode (lens != nullptr): query t is the last key of its own sequence of
  // lens[t] keys, with its own pooled keys (slices 2t, 2t+1 of the pooled-key
  // map, M = blocks per slice); each row tile holds one query's H rows
  const int32_t* lens;
};

__device__ __forceinline__ int64_t causal_blocks(const RouteParams& p, int64_t pos) {
  return min((pos + 1) / p.B, p.n_k / p.B);
}

// Complete causal blocks of query t (decode: every complete block of its own
// sequence, at most the slice's M).
__device__ __forceinline__ int64_t query_blocks(const RouteParams& p, int t, int64_t M) {
  if (p.lens) {
    const int64_t len = __ldg(p.lens + t);
    return len <= 0 ? 0 : min(len / p.B, M);
  }
  return causal_blocks(p, p.q_pos0 + t);
}

// Queries per row tile.
__device__ __forceinline__ int queries_per_tile(const RouteParams& p) {
  return p.lens ? 1 : kRows / p.H;
}

// Number of 128-block N tiles a row tile needs (its last query has the most).
__device__ __forceinline__ int ntiles_of(const RouteParams& p, int rt, int64_t M) {
  const int QT = queries_per_tile(p);
  const int t_last = min((rt + 1) * QT, p.n_q) - 1;
  const int64_t nc = query_blocks(p, t_last, M);
  return static_cast<int>((nc + kBlkN - 1) / kBlkN);
}

// warp-uniform argmax by (r desc, head asc)
__device__ __forceinline__ void better(float& br, int& bj, float r, int j) {
  if (r > br || (r == br && j < bj)) {
    br = r;
    bj = j;
  }
}

template <int D, int NA>
__global__ void __launch_bounds__(RouteRoles<NA>::THREADS, 1)
route_heads_kernel(const __grid_constant__ CUtensorMap qmap,
                   const __grid_constant__ CUtensorMap kbmap, const RouteParams p, int64_t M) {
  using L = RouteLayout<D, NA>;
  constexpr int EPI = RouteRoles<NA>::EPI;
  constexpr int kRouteStages = L::STAGES;
  constexpr int TM_COLS = 2 * NA * kBlkN;  // two accumulators per row tile
  // work unit: NA consecutive row tiles (the last unit may hold fewer)
  const int units = (p.row_tiles + NA - 1) / NA;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const uint32_t sA = smem_u32(smem + L::OFF_A);
  const uint32_t sB = smem_u32(smem + L::OFF_B);
  float* r_s = reinterpret_cast<float*>(smem + L::OFF_R);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = kRouteStages, AFULL = 2 * kRouteStages, AEMPTY = AFULL + 1,
            ACCFULL = AFULL + 2, ACCEMPTY = AFULL + 4, RFULL = AFULL + 6, REMPTY = AFULL + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRouteStages; ++i) {
      mbar_init(bar(FULL + i), 1);
      mbar_init(bar(EMPTY + i), 1);
    }
    mbar_init(bar(AFULL), 1);
    mbar_init(bar(AEMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(ACCFULL + i), 1);
      mbar_init(bar(ACCEMPTY + i), EPI);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(RFULL + i), EPI);
      mbar_init(bar(REMPTY + i), kRouteTopWarps);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&qmap);
    tma_prefetch_desc(&kbmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), TM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0, tcount = 0;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int rt = u * NA, na = min(NA, p.row_tiles - rt);
      const int nN = ntiles_of(p, rt + na - 1, M);  // the unit's last row tile sees the most
      if (nN == 0) continue;
      // decode: the tile's rows start at query rt's first head row, and its
      // pooled keys are slices 2rt (hi) and 2rt+1 (lo)
      const int row0 = p.lens ? rt * p.H : rt * kRows;
      const int z0 = p.lens ? 2 * rt : 0;
      if (lane == 0) {
        ok = mbar_wait(bar(AEMPTY), (tcount & 1) ^ 1, abort_flag, p.ctl);
        if (ok) {
          mbar_arrive_expect_tx(bar(AFULL), na * L::A_BYTES);
          for (int a = 0; a < na; ++a)
            for (int c = 0; c < L::KCH; ++c)
              tma_load_2d(sA + a * L::A_BYTES + c * L::A_CHUNK, &qmap, bar(AFULL), c * (L::ROWB / 2),
                          row0 + a * kRows);
        }
        for (int nb = 0; nb < nN && ok; ++nb) {
          ok = mbar_wait(bar(EMPTY + stage), phase ^ 1, abort_flag, p.ctl);
          if (!ok) break;
          mbar_arrive_expect_tx(bar(FULL + stage), 2 * L::B_HALF);
          const uint32_t dst = sB + stage * 2 * L::B_HALF;
          for (int half = 0; half < 2; ++half)
            for (int c = 0; c < L::KCH; ++c)
              tma_load_3d(dst + half * L::B_HALF + c * L::B_CHUNK, &kbmap, bar(FULL + stage),
                          c * (L::ROWB / 2), nb * kBlkN, z0 + half);
          if (++stage == kRouteStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      stage = __shfl_sync(0xffffffffu, stage, 0);
      phase = __shfl_sync(0xffffffffu, phase, 0);
      ++tcount;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0, acc = 0;
    uint32_t phase = 0, accph = 0, tcount = 0;
    bool ok = true;
    constexpr uint32_t idesc = umma_idesc_bf16_f32(kRows, kBlkN);
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int rt = u * NA, na = min(NA, p.row_tiles - rt);
      const int nN = ntiles_of(p, rt + na - 1, M);
      if (nN == 0) continue;
      if (lane == 0) {
        ok = mbar_wait(bar(AFULL), tcount & 1, abort_flag, p.ctl);
        for (int nb = 0; nb < nN && ok; ++nb) {
          ok = mbar_wait(bar(FULL + stage), phase, abort_flag, p.ctl) &&
               mbar_wait(bar(ACCEMPTY + acc), accph ^ 1, abort_flag, p.ctl);
          if (!ok) break;
          tc_fence_after();
          const uint32_t bstage = sB + stage * 2 * L::B_HALF;
          for (int a = 0; a < na; ++a) {
            const uint32_t d_tmem = tmem_base + static_cast<uint32_t>((acc * NA + a) * kBlkN);
            for (int half = 0; half < 2; ++half) {
#pragma unroll
              for (int kk = 0; kk < D / 16; ++kk) {
                const int c = (kk * 32) / L::ROWB, within = (kk * 32) % L::ROWB;
                const uint64_t ad =
                    umma_desc_kmajor(sA + a * L::A_BYTES + c * L::A_CHUNK + within, L::ROWB);
                const uint64_t bd =
                    umma_desc_kmajor(bstage + half * L::B_HALF + c * L::B_CHUNK + within, L::ROWB);
                tc_mma_bf16(d_tmem, ad, bd, idesc, (half > 0 || kk > 0) ? 1u : 0u);
              }
            }
          }
          tc_commit(bar(EMPTY + stage));
          tc_commit(bar(ACCFULL + acc));
          if (++stage == kRouteStages) {
            stage = 0;
            phase ^= 1;
          }
          if (++acc == 2) {
            acc = 0;
            accph ^= 1;
          }
        }
        if (ok) tc_commit(bar(AEMPTY));
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      stage = __shfl_sync(0xffffffffu, stage, 0);
      phase = __shfl_sync(0xffffffffu, phase, 0);
      acc = __shfl_sync(0xffffffffu, acc, 0);
      accph = __shfl_sync(0xffffffffu, accph, 0);
      ++tcount;
    }
  } else {
    // ------------------------------------------------------------ epilogue / top-h
    const bool top_role = warp >= 2 + EPI;
    const int QT = queries_per_tile(p);
    uint32_t rcount = 0;  // units handed over so far (buffer = rcount & 1)
    bool ok = true;
    if (!top_role) {
      const int quad = warp & 3;
      const int a = (warp - 2) / 4;       // row tile of the unit
      const int row = quad * 32 + lane;   // TMEM lane of this thread
      int acc = 0;
      uint32_t accph = 0;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++rcount) {
        const int rt0 = u * NA, na = min(NA, p.row_tiles - rt0);
        const int nN = ntiles_of(p, rt0 + na - 1, M);
        const int rt = rt0 + a;
        const int t = rt * QT + row / p.H;
        const bool valid = a < na && t < p.n_q && row / p.H < QT;
        const int64_t nc = valid ? query_blocks(p, t, M) : 0;
        float sum = 0.0f;
        for (int nb = 0; nb < nN; ++nb) {
          if (lane == 0) ok = mbar_wait(bar(ACCFULL + acc), accph, abort_flag, p.ctl);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          tc_fence_after();
          uint32_t v[kBlkN];
          tmem_ld128(tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                         static_cast<uint32_t>((acc * NA + a) * kBlkN),
                     v);
          tmem_wait_ld();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(ACCEMPTY + acc));
          if (++acc == 2) {
            acc = 0;
            accph ^= 1;
          }
          const int64_t m0 = static_cast<int64_t>(nb) * kBlkN;
          if (m0 + kBlkN <= nc) {
            float s0 = 0.0f, s1 = 0.0f, s2 = 0.0f, s3 = 0.0f;
#pragma unroll
            for (int i = 0; i < kBlkN; i += 4) {
              s0 += relu(__uint_as_float(v[i]));
              s1 += relu(__uint_as_float(v[i + 1]));
              s2 += relu(__uint_as_float(v[i + 2]));
              s3 += relu(__uint_as_float(v[i + 3]));
            }
            sum += (s0 + s1) + (s2 + s3);
          } else {
#pragma unroll
            for (int i = 0; i < kBlkN; ++i)
              if (m0 + i < nc) sum += relu(__uint_as_float(v[i]));
          }
        }
        if (!ok) break;
        // hand the partial sums of this row tile to the top-h warps
        const uint32_t buf = rcount & 1;
        if (lane == 0) ok = mbar_wait(bar(REMPTY + buf), ((rcount >> 1) & 1) ^ 1, abort_flag, p.ctl);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        r_s[buf * NA * kRows + a * kRows + row] = sum;
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(RFULL + buf));
      }
    } else {
      // top-h: one warp per query, h rounds of a warp argmax by (r desc, head asc)
      const int tw = warp - 2 - EPI;
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x, ++rcount) {
        const uint32_t buf = rcount & 1;
        if (lane == 0) ok = mbar_wait(bar(RFULL + buf), (rcount >> 1) & 1, abort_flag, p.ctl);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const float* rb = r_s + buf * NA * kRows;
        const int rt0 = u * NA, na = min(NA, p.row_tiles - rt0);
        for (int qq = tw; qq < na * QT; qq += kRouteTopWarps) {
          const int tq = rt0 * QT + qq;
          if (tq >= p.n_q) break;
          constexpr int SL = 4;  // slots per lane: H <= 128
          float rv[SL];
          bool taken[SL];
#pragma unroll
          for (int i = 0; i < SL; ++i) {
            const int jj = lane + 32 * i;
            taken[i] = jj >= p.H;
            rv[i] = 0.0f;
            if (!taken[i]) {
              const int rr = qq * p.H + jj;
              rv[i] = __ldg(p.w + static_cast<int64_t>(tq) * p.H + jj) * rb[rr];
              if (p.r_out) p.r_out[static_cast<int64_t>(tq) * p.H + jj] = rv[i];
            }
          }
          for (int round = 0; round < p.h; ++round) {
            float br = -INFINITY;
            int bj = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < SL; ++i)
              if (!taken[i]) better(br, bj, rv[i], lane + 32 * i);
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
              const float orr = __shfl_xor_sync(0xffffffffu, br, off);
              const int oj = __shfl_xor_sync(0xffffffffu, bj, off);
              better(br, bj, orr, oj);
            }
            if (bj < p.H && (bj & 31) == lane) taken[bj >> 5] = true;
          }
          // selected heads, written in ascending order
          int before = 0;
#pragma unroll
          for (int i = 0; i < SL; ++i) {
            const int jj = lane + 32 * i;
            const bool sel = jj < p.H && taken[i];
            const uint32_t m = __ballot_sync(0xffffffffu, sel);
            if (sel)
              p.heads[static_cast<int64_t>(tq) * p.h + before + __popc(m & ((1u << lane) - 1u))] = jj;
            before += __popc(m);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(REMPTY + buf));
      }
    }
  }

  __syncthreads();
  if (*abort_flag) drain_pause(kDrainNs);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TM_COLS);
  }
}

template <int D, int NA>
cudaError_t launch_dn(const RouteParams& p, const CUtensorMap& qm, const CUtensorMap& km,
                      int64_t M, cudaStream_t s) {
  using L = RouteLayout<D, NA>;
  auto kern = route_heads_kernel<D, NA>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  const int grid = std::min(sm_count(), (p.row_tiles + NA - 1) / NA);
  if (grid <= 0) return cudaSuccess;
  kern<<<grid, RouteRoles<NA>::THREADS, L::ALLOC, s>>>(qm, km, p, M);
  return cudaGetLastError();
}

// Prefill: two row tiles per pooled-key tile once there are enough of them to
// keep every SM busy; decode: one (each query has its own pooled keys).
template <int D>
cudaError_t launch_d(const RouteParams& p, const CUtensorMap& qm, const CUtensorMap& km, int64_t M,
                     cudaStream_t s) {
  if (!p.lens && p.row_tiles >= 2 * sm_count()) return launch_dn<D, 2>(p, qm, km, M, s);
  return launch_dn<D, 1>(p, qm, km, M, s);
}

// Tensor maps and launch: Q as [n_q * H, d] rows; the pooled keys as [slices,
// M, d] (slices = 2: hi, lo; decode: 2 per sequence).
cudaError_t launch_route(const uint16_t* Q, const uint16_t* kbar_hl, const RouteParams& p, int d,
                         int64_t M, int64_t slices, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(p.n_q) * p.H;
  const int rowb = d >= 64 ? 128 : 64;
  const CUtensorMapSwizzle swz = rowb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  CUtensorMap qm, km;
  {
    const uint64_t dims[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(rows)};
    const uint64_t strides[1] = {static_cast<uint64_t>(d) * 2};
    const uint32_t box[2] = {static_cast<uint32_t>(rowb / 2), static_cast<uint32_t>(kRows)};
    if (encode_tensor_map(&qm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Q, dims, strides, box, swz) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    const uint64_t dims[3] = {static_cast<uint64_t>(d), static_cast<uint64_t>(M),
                              static_cast<uint64_t>(slices)};
    const uint64_t strides[2] = {static_cast<uint64_t>(d) * 2, static_cast<uint64_t>(M * d * 2)};
    const uint32_t box[3] = {static_cast<uint32_t>(rowb / 2), static_cast<uint32_t>(kBlkN), 1};
    if (encode_tensor_map(&km, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, kbar_hl, dims, strides, box,
                          swz) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  switch (d) {
    case 32: return launch_d<32>(p, qm, km, M, s);
    case 64: return launch_d<64>(p, qm, km, M, s);
    case 128: return launch_d<128>(p, qm, km, M, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_route_heads(const uint16_t* Q, const float* w, const uint16_t* kbar_hl,
                               int n_q, int64_t q_pos0, int64_t n_k, int H, int d, int B, int h,
                               int32_t* heads, float* r_out, const DevCtl& ctl, cudaStream_t s) {
  if (n_q <= 0) return cudaSuccess;
  const int64_t M = (n_k + B - 1) / B;
  const int64_t rows = static_cast<int64_t>(n_q) * H;
  const int row_tiles = static_cast<int>((rows + kRows - 1) / kRows);
  const RouteParams p{w, heads, r_out, n_q, q_pos0, n_k, H, B, h, row_tiles, ctl, nullptr};
  return launch_route(Q, kbar_hl, p, d, M, 2, s);
}

cudaError_t launch_route_heads_decode(const uint16_t* Q, const float* w, const uint16_t* kbar_hl,
                                      int64_t M_max, const int32_t* lens, int n_seq, int H, int d,
                                      int B, int h, int32_t* heads, float* r_out, const DevCtl& ctl,
                                      cudaStream_t s) {
  if (n_seq <= 0) return cudaSuccess;
  // n_k only bounds the complete blocks in prefill mode; decode reads lens
  const RouteParams p{w, heads, r_out, n_seq, 0, M_max * B, H, B, h, n_seq, ctl, lens};
  return launch_route(Q, kbar_hl, p, d, M_max, 2 * static_cast<int64_t>(n_seq), s);
}

}  // namespace misa
