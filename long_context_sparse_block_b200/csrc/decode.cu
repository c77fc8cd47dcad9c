// Decode-shaped routed scoring: many sequences, one new query each, the keys of
// every sequence in a paged cache.
//
//   logit[b, s] = sum_{i<h} w[b, j_i] * ReLU(q[b, j_i] . k_{b,s}),  s < len(b)
//
// ("MISA" technical summary, Metodologia step 2, for the query at the end of
// each sequence: it sees all len(b) keys of its own cache.)  With one query per
// sequence the keys of a tile serve only that query's h routed heads, so the
// work is a stream over the key caches (about 8 flop per byte for h = 8), not a
// dense contraction.  The prefill kernel would spend a 256-column MMA group on
// h live columns; here the tensor core runs M = 128 keys x N = NB (16, 32 or
// 64 >= h) columns, the query's routed head rows padded with zero rows, so the
// MMA costs ~5 % of the time the HBM stream takes and the kernel reads each key
// once.
//
// Work items are (sequence, chunk of kChunkTiles 128-key tiles), spread
// round-robin over a persistent grid (one CTA per SM).  Warp roles (192
// threads): warp 0 producer (gathers the query's head rows by cp.async into one
// of two buffers, so the next item's rows land while this item's tiles stream,
// and streams key tiles with TMA through the sequence's block table, one box
// per page),
// warp 1 TMEM allocator and MMA issuer, warps 2-5 epilogue (one per TMEM lane
// quadrant: one tcgen05.ld of the NB columns per tile, ReLU * w head-sum in the
// prefill kernel's order, logits stored for s < len(b)).  The top-k per
// sequence then runs on those rows (topk.cu, per-row lengths).
#include <cstring>

#include "internal.h"

namespace misa {
namespace {

constexpr int kTile = 128;        // keys per tile (MMA M)
constexpr int kChunkTiles = 16;   // tiles per work item
constexpr int kStages = 4;        // key ring
constexpr uint64_t kDrainNs = 2000000;

template <int D, int NB, bool F8>
struct DecLayout {
  // FP8 pages: e4m3 -> bf16 converter warps (fewer for the widest epilogue,
  // whose registers leave room for fewer threads)
  static constexpr int CONV = F8 ? (NB <= 32 ? 8 : 4) : 0;
  static constexpr int THREADS = 192 + 32 * CONV;
  static constexpr int ROWB = D >= 64 ? 128 : 64;  // bytes per row of one swizzle chunk
  static constexpr int KCH = D * 2 / ROWB;
  static constexpr int A_CHUNK = kTile * ROWB;
  static constexpr int A_BYTES = kTile * D * 2;
  static constexpr int B_CHUNK = NB * ROWB;
  static constexpr int B_BYTES = NB * D * 2;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + kStages * A_BYTES;
  static constexpr int B_STRIDE = (B_BYTES + 1023) / 1024 * 1024;
  static constexpr int RAW_BYTES = F8 ? kTile * D : 0;    // e4m3 codes of a tile
  static constexpr int OFF_RAW = OFF_B + 2 * B_STRIDE;     // two B buffers before
  static constexpr int OFF_BAR = OFF_RAW + kStages * RAW_BYTES;
  static constexpr int NBAR = 2 * kStages + 8 + (F8 ? 2 * kStages : 0);
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;
  static constexpr uint32_t TMEM_COLS = 2 * NB < 32 ? 32 : 2 * NB;
};

struct DecParams {
  const uint16_t* Q;      // [n_seq, H, d]
  const float* w;         // [n_seq, H]
  const int32_t* heads;   // [n_seq, h], nullptr: heads 0..h-1 (h == H)
  const int32_t* bts;     // [n_seq, max_blocks] block tables
  const int32_t* lens;    // [n_seq] keys per sequence
  const float* k_scale;   // FP8 pages: [n_pages, page_size] per-row scales
  int max_blocks;
  int page_shift;
  int64_t n_pages;
  int64_t key_rows;       // rows of the page pool (tensor map)
  int n_seq;
  int H;
  int h;
  int cps;                // work items per sequence
  float* logits;          // [n_seq, ld]
  int64_t ld;
  DevCtl ctl;
};

// Keys of sequence b (clamped to what its block table holds; a longer length
// is reported).
__device__ __forceinline__ int64_t seq_len(const DecParams& p, int b) {
  int64_t len = __ldg(p.lens + b);
  const int64_t cap = static_cast<int64_t>(p.max_blocks) << p.page_shift;
  if (len > cap) {
    report(p.ctl, DEV_BAD_INPUT);
    len = cap;
  }
  return len < 0 ? 0 : len;
}

// Tiles [t0, t1) of work item c of sequence b (empty when t0 >= t1).
__device__ __forceinline__ void item_tiles(const DecParams& p, int64_t c, int& b, int64_t& len,
                                           int64_t& t0, int64_t& t1) {
  b = static_cast<int>(c / p.cps);
  len = seq_len(p, b);
  t0 = (c % p.cps) * kChunkTiles;
  const int64_t nt = (len + kTile - 1) / kTile;
  t1 = min(t0 + kChunkTiles, nt);
}

// F8: the pages hold e4m3 codes; their tiles land in a raw ring by TMA and the
// converter warps decode them exactly to bf16 into the MMA's key ring; the
// row's scale multiplies the head-sum.
template <int D, int NB, bool F8>
__global__ void __launch_bounds__(DecLayout<D, NB, F8>::THREADS, 1)
decode_score_kernel(const __grid_constant__ CUtensorMap kmap, const DecParams p) {
  using L = DecLayout<D, NB, F8>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const uint32_t sA = smem_u32(smem + L::OFF_A);
  const uint32_t sB = smem_u32(smem + L::OFF_B);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = kStages, BFULL = 2 * kStages, BEMPTY = BFULL + 2, ACCFULL = BFULL + 4,
            ACCEMPTY = BFULL + 6, RFULL = BFULL + 8, REMPTY = RFULL + kStages;
  const uint32_t sRaw = smem_u32(smem + L::OFF_RAW);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);
  const int64_t total = static_cast<int64_t>(p.n_seq) * p.cps;

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bar(FULL + i), F8 ? L::CONV : 1);
      mbar_init(bar(EMPTY + i), 1);
      if (F8) {
        mbar_init(bar(RFULL + i), 1);
        mbar_init(bar(REMPTY + i), L::CONV);
      }
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(BFULL + i), 32);
      mbar_init(bar(BEMPTY + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(ACCFULL + i), 1);
      mbar_init(bar(ACCEMPTY + i), 4);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&kmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int stage = 0;
    uint32_t phase = 0, icount = 0;
    bool ok = true;
    constexpr int UPR = D * 2 / 16;    // 16-byte units per head row
    constexpr int UPC = L::ROWB / 16;  // units per swizzle-chunk row
    for (int64_t c = blockIdx.x; c < total && ok; c += gridDim.x) {
      int b;
      int64_t len, t0, t1;
      item_tiles(p, c, b, len, t0, t1);
      if (t0 >= t1) continue;
      // B: the query's routed head rows, zero rows up to NB, into one of two
      // buffers; the copies land asynchronously (each lane arrives on the
      // buffer's barrier when its own copies are done) while the key tiles of
      // this item are already being requested
      const int bb = icount & 1;
      const uint32_t sBb = sB + bb * L::B_STRIDE;
      if (lane == 0) ok = mbar_wait(bar(BEMPTY + bb), ((icount >> 1) & 1) ^ 1, abort_flag, p.ctl);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      for (int x = lane; x < NB * UPR; x += 32) {
        const int n = x / UPR, u = x % UPR;
        int j = -1;
        if (n < p.h) {
          j = p.heads ? __ldg(p.heads + static_cast<int64_t>(b) * p.h + n) : n;
          if (j < 0 || j >= p.H) {
            report(p.ctl, DEV_BAD_INPUT);
            j = 0;
          }
        }
        const uint16_t* src = p.Q + (static_cast<int64_t>(b) * p.H + (j >= 0 ? j : 0)) * D + u * 8;
        cp_async16(sBb + (u / UPC) * L::B_CHUNK + swz_offset(n, u % UPC, L::ROWB), src,
                   j >= 0 ? 16u : 0u);
      }
      cp_async_mbar_arrive_noinc(bar(BFULL + bb));
      ++icount;
      const int32_t* bt = p.bts + static_cast<int64_t>(b) * p.max_blocks;
      const int ps = 1 << p.page_shift;
      for (int64_t kt = t0; kt < t1; ++kt) {
        if (lane == 0) {
          // bf16 pages: straight into the key ring; e4m3 pages: into the raw
          // ring (same stage index), freed by the converters
          ok = mbar_wait(bar((F8 ? REMPTY : EMPTY) + stage), phase ^ 1, abort_flag, p.ctl);
          if (ok) {
            mbar_arrive_expect_tx(bar((F8 ? RFULL : FULL) + stage), F8 ? L::RAW_BYTES : L::A_BYTES);
            for (int jp = 0; jp < kTile / ps; ++jp) {
              const int64_t s0 = kt * kTile + jp * ps;
              int64_t y = p.key_rows;  // past the sequence: a box of fill rows
              if (s0 < len) {
                int64_t pg = __ldg(bt + (s0 >> p.page_shift));
                if (pg < 0 || pg >= p.n_pages) {
                  report(p.ctl, DEV_BAD_INPUT);
                  pg = 0;
                }
                y = pg << p.page_shift;
              }
              if constexpr (F8) {
                tma_load_2d(sRaw + stage * L::RAW_BYTES + jp * ps * D, &kmap, bar(RFULL + stage), 0,
                            static_cast<int>(y));
              } else {
#pragma unroll
                for (int cc = 0; cc < L::KCH; ++cc)
                  tma_load_2d(sA + stage * L::A_BYTES + cc * L::A_CHUNK + jp * ps * L::ROWB, &kmap,
                              bar(FULL + stage), cc * (L::ROWB / 2), static_cast<int>(y));
              }
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        if (++stage == kStages) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    int stage = 0, acc = 0;
    uint32_t phase = 0, accph = 0, icount = 0;
    bool ok = true;
    constexpr uint32_t idesc = umma_idesc_bf16_f32(kTile, NB);
    for (int64_t c = blockIdx.x; c < total && ok; c += gridDim.x) {
      int b;
      int64_t len, t0, t1;
      item_tiles(p, c, b, len, t0, t1);
      if (t0 >= t1) continue;
      const int bb = icount & 1;
      const uint32_t sBb = sB + bb * L::B_STRIDE;
      if (lane == 0) {
        ok = mbar_wait(bar(BFULL + bb), (icount >> 1) & 1, abort_flag, p.ctl);
        fence_proxy_async_smem();  // the copies, observed through the barrier -> MMA operand reads
        for (int64_t kt = t0; kt < t1 && ok; ++kt) {
          ok = mbar_wait(bar(FULL + stage), phase, abort_flag, p.ctl) &&
               mbar_wait(bar(ACCEMPTY + acc), accph ^ 1, abort_flag, p.ctl);
          if (!ok) break;
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * NB);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const int cc = (kk * 32) / L::ROWB, within = (kk * 32) % L::ROWB;
            const uint64_t ad =
                umma_desc_kmajor(sA + stage * L::A_BYTES + cc * L::A_CHUNK + within, L::ROWB);
            const uint64_t bd = umma_desc_kmajor(sBb + cc * L::B_CHUNK + within, L::ROWB);
            tc_mma_bf16(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(EMPTY + stage));
          tc_commit(bar(ACCFULL + acc));
          if (kt == t1 - 1) tc_commit(bar(BEMPTY + bb));
          if (++stage == kStages) {
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
      ++icount;
    }
  } else if (warp >= 6) {
    // ------------------------------------------------------------ e4m3 -> bf16 converters
    if constexpr (F8) {
      static_assert(L::KCH >= 1, "decoded rows span whole swizzle chunks");
      const int cw = warp - 6;          // rows cw*RPW .. cw*RPW+RPW-1 of every tile
      constexpr int RPW = kTile / L::CONV;  // rows per converter warp
      constexpr int U8 = D / 16;        // 16-byte units of an e4m3 row
      constexpr int RPI = 32 / U8;      // rows per warp instruction
      constexpr int UPC = L::ROWB / 16; // bf16 units per swizzle-chunk row
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int64_t c = blockIdx.x; c < total && ok; c += gridDim.x) {
        int b;
        int64_t len, t0, t1;
        item_tiles(p, c, b, len, t0, t1);
        for (int64_t kt = t0; kt < t1; ++kt) {
          if (lane == 0)
            ok = mbar_wait(bar(RFULL + stage), phase, abort_flag, p.ctl) &&
                 mbar_wait(bar(EMPTY + stage), phase ^ 1, abort_flag, p.ctl);
          if (!__shfl_sync(0xffffffffu, ok, 0)) break;
          const uint32_t src = sRaw + stage * L::RAW_BYTES;
          const uint32_t dst = sA + stage * L::A_BYTES;
#pragma unroll
          for (int it = 0; it < RPW / RPI; ++it) {
            const int r = cw * RPW + it * RPI + lane / U8, u = lane % U8;
            uint32_t wv[4];
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(wv[0]), "=r"(wv[1]), "=r"(wv[2]), "=r"(wv[3])
                         : "r"(src + static_cast<uint32_t>(r * D + u * 16)));
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {  // 8 codes -> 8 bf16 (exact)
              const uint32_t b0 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh] & 0xFFFF));
              const uint32_t b1 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh] >> 16));
              const uint32_t b2 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh + 1] & 0xFFFF));
              const uint32_t b3 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh + 1] >> 16));
              const int bu = 2 * u + hh;  // bf16 unit of the row
              const uint32_t off = (bu / UPC) * L::A_CHUNK + swz_offset(r, bu % UPC, L::ROWB);
              asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + off), "r"(b0),
                           "r"(b1), "r"(b2), "r"(b3)
                           : "memory");
            }
          }
          fence_proxy_async_smem();  // the decoded tile -> MMA operand reads
          __syncwarp();              // every lane has read its raw codes and written its rows
          if (lane == 0) {
            mbar_arrive(bar(FULL + stage));
            mbar_arrive(bar(REMPTY + stage));
          }
          if (++stage == kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int quad = warp & 3;  // TMEM lanes quad*32 .. quad*32+31
    int acc = 0;
    uint32_t accph = 0;
    bool ok = true;
    for (int64_t c = blockIdx.x; c < total && ok; c += gridDim.x) {
      int b;
      int64_t len, t0, t1;
      item_tiles(p, c, b, len, t0, t1);
      if (t0 >= t1) continue;
      float wv[NB];
#pragma unroll
      for (int i = 0; i < NB; ++i) {
        float x = 0.0f;
        if (i < p.h) {
          int j = p.heads ? __ldg(p.heads + static_cast<int64_t>(b) * p.h + i) : i;
          if (j < 0 || j >= p.H) j = 0;
          x = __ldg(p.w + static_cast<int64_t>(b) * p.H + j);
        }
        wv[i] = x;
      }
      float* row = p.logits + static_cast<int64_t>(b) * p.ld;
      const int32_t* bt = p.bts + static_cast<int64_t>(b) * p.max_blocks;
      (void)bt;
      for (int64_t kt = t0; kt < t1; ++kt) {
        if (lane == 0) ok = mbar_wait(bar(ACCFULL + acc), accph, abort_flag, p.ctl);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        tc_fence_after();
        uint32_t v[NB];
        const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                               static_cast<uint32_t>(acc * NB);
        if constexpr (NB == 16) {
          tmem_ld16(taddr, v);
        } else if constexpr (NB == 32) {
          tmem_ld32(taddr, v);
        } else {
          tmem_ld64(taddr, v);
        }
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ACCEMPTY + acc));
        if (++acc == 2) {
          acc = 0;
          accph ^= 1;
        }
        // the head-sum in the order the prefill kernel uses: for h >= 4 two
        // interleaved FMA chains (heads 0, 2, 4, .. and 1, 3, 5, ..), then their sum
        float sum;
        if (p.h == 1) {
          sum = wv[0] * relu(__uint_as_float(v[0]));
        } else if (p.h == 2) {
          sum = fmaf(wv[1], relu(__uint_as_float(v[1])), wv[0] * relu(__uint_as_float(v[0])));
        } else {
          float2 a2 = make_float2(0.0f, 0.0f);
#pragma unroll
          for (int j = 0; j < NB; j += 4) {
            if (j < p.h) {
              a2 = fma2(make_float2(wv[j], wv[j + 1]),
                        make_float2(relu(__uint_as_float(v[j])), relu(__uint_as_float(v[j + 1]))), a2);
              a2 = fma2(make_float2(wv[j + 2], wv[j + 3]),
                        make_float2(relu(__uint_as_float(v[j + 2])), relu(__uint_as_float(v[j + 3]))),
                        a2);
            }
          }
          sum = a2.x + a2.y;
        }
        const int64_t s = kt * kTile + quad * 32 + lane;
        if constexpr (F8) {
          // the row's scale > 0 commutes with the ReLU: w * ReLU(scale * dot)
          float ks = 0.0f;
          if (s < len) {
            int64_t pg = __ldg(bt + (s >> p.page_shift));
            if (pg < 0 || pg >= p.n_pages) pg = 0;  // (reported by the producer)
            ks = __ldg(p.k_scale + ((pg << p.page_shift) | (s & ((int64_t(1) << p.page_shift) - 1))));
          }
          sum *= ks;
        }
        if (s < len) row[s] = sum;
      }
    }
  }

  __syncthreads();
  if (*abort_flag) drain_pause(kDrainNs);  // let issued copies / MMAs land
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, L::TMEM_COLS);
  }
}

template <int D, int NB, bool F8>
cudaError_t launch_dn(const DecParams& p, const CUtensorMap& map, cudaStream_t s) {
  using L = DecLayout<D, NB, F8>;
  auto kern = decode_score_kernel<D, NB, F8>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  const int64_t items = static_cast<int64_t>(p.n_seq) * p.cps;
  const int64_t grid = std::min<int64_t>(sm_count(), items);
  if (grid <= 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(grid), L::THREADS, L::ALLOC, s>>>(map, p);
  return cudaGetLastError();
}

template <int D, bool F8>
cudaError_t launch_d(const DecParams& p, const CUtensorMap& map, cudaStream_t s) {
  if (p.h <= 16) return launch_dn<D, 16, F8>(p, map, s);
  if (p.h <= 32) return launch_dn<D, 32, F8>(p, map, s);
  if (p.h <= 64) return launch_dn<D, 64, F8>(p, map, s);
  return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_decode_score(const uint16_t* Q, const float* w, const int32_t* heads,
                                const void* pages, const float* k_scale, bool fp8,
                                const int32_t* block_tables, int max_blocks, int page_shift,
                                int64_t n_pages, const int32_t* lens, int n_seq, int H, int d, int h,
                                float* logits, int64_t ld, const DevCtl& ctl, cudaStream_t s) {
  if (n_seq <= 0) return cudaSuccess;
  const int64_t max_len = static_cast<int64_t>(max_blocks) << page_shift;
  const int cps = static_cast<int>((max_len + kTile * kChunkTiles - 1) / (kTile * kChunkTiles));
  const int64_t key_rows = n_pages << page_shift;
  DecParams p{Q, w, heads, block_tables, lens, k_scale, max_blocks, page_shift, n_pages, key_rows,
              n_seq, H, h, cps, logits, ld, ctl};
  CUtensorMap map;
  std::memset(&map, 0, sizeof map);
  if (fp8) {  // e4m3 rows into the raw ring: one row-major box per page
    const uint64_t dims[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(key_rows)};
    const uint64_t strides[1] = {static_cast<uint64_t>(d)};
    const uint32_t box[2] = {static_cast<uint32_t>(d), 1u << page_shift};
    if (encode_tensor_map(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, pages, dims, strides, box,
                          CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    switch (d) {
      case 32: return launch_d<32, true>(p, map, s);
      case 64: return launch_d<64, true>(p, map, s);
      case 128: return launch_d<128, true>(p, map, s);
    }
    return cudaErrorInvalidValue;
  }
  const int rowb = d >= 64 ? 128 : 64;
  const uint64_t dims[2] = {static_cast<uint64_t>(d), static_cast<uint64_t>(key_rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(d) * 2};
  const uint32_t box[2] = {static_cast<uint32_t>(rowb / 2), 1u << page_shift};
  if (encode_tensor_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, pages, dims, strides, box,
                        rowb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) !=
      CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  switch (d) {
    case 32: return launch_d<32, false>(p, map, s);
    case 64: return launch_d<64, false>(p, map, s);
    case 128: return launch_d<128, false>(p, map, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace misa
