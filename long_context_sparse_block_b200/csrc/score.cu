// Stage 4 — routed token scoring on the 5th-generation tensor cores.
//
//   logit[t, s] = sum_{i<h} w[t, j_i] * ReLU(q[t, j_i] . k_s),  s <= pos(t)
//
// ("MISA" technical summary, Metodologia step 2: only the h routed heads score
// every prefix token; with all heads routed this is the dense DSA lightning
// indexer of Declaracao do Problema.)
//
// Because every head shares the same key vector k_s, the h routed head rows of
// a group of queries can be stacked into one dense operand: for h = 8, 32
// queries x 8 heads = 256 rows.  The kernel makes the KEYS the MMA M dimension
// ("swap-AB"): A = a 128-key tile of K streamed by TMA, B = the 256 gathered
// (query, head) rows of Q held in shared memory for the whole group, D = 128 x
// 256 fp32 in TMEM.  TMEM lane = key, column = (query, head), so the epilogue
// thread that owns a key finds all h heads of a query in its own consecutive
// columns: ReLU, the head weights and the head-sum are applied in registers and
// only the fused logit is written to HBM (per-head logits never leave the SM).
//
// Warp roles (608 threads for h <= 64, else 352, plus a warp for FP8 keys
// decoded in the kernel; one CTA per SM, persistent):
//   warp 0     producer: gathers B for each query group (16-byte cp.async into
//              the 128-byte-swizzled K-major layout) and streams key tiles with
//              TMA into a STAGES-deep ring;
//   warp 1     allocates TMEM (512 columns = two 256-column accumulators) and
//              issues tcgen05.mma from one thread;
//   warp 2     store mode: issues one TMA store per tile of the logits the
//              epilogue staged in shared memory (double-buffered);
//   (warp 3    FP8 keys decoded here: e4m3 rows -> bf16 into the key tile;)
//   then       epilogue, four warps per TMEM lane quadrant each owning 64 of
//              the 256 columns (two warps owning 128 when h = 128): one
//              tcgen05.ld of its columns, the accumulator released right after
//              the load lands, then the fused ReLU * w head-sum (packed fp32
//              FMA) and, per mode:
//                store   the causal-masked logits staged for the TMA store;
//                select  each logit compared with its row's threshold: a ballot
//                        per query gives the row's 32-key pass-mask word, the
//                        kept logits are stored in place (fused top-k);
//                repair  store mode over only the query groups that hold a row
//                        flagged by the fused top-k (nothing when none is).
// Work is the flattened list of (query group, key tile) pairs, split evenly
// over the CTAs, so causal triangles stay balanced.
//
// With e4m3 queries and keys (a scale per (query, head) row and per key) the
// same roles run on one-byte operands: key tiles of 128 x d bytes, gathered
// rows of d bytes, tcgen05.mma.kind::f8f6f4; the row scale is folded into the
// head weight and the key scale multiplies the head-sum.
#include <cstring>

#include "internal.h"

namespace misa {
namespace {

constexpr int kTileKeys = 128;   // MMA M
constexpr int kCols = 256;       // MMA N: (query, head) columns per group
// epilogue warps: 4 per TMEM lane quadrant (64 columns each) when a query's h
// columns fit in 64, else 2 per quadrant (128 columns each).  Warp 2 issues the
// TMA stores of the staged logits; FP8 keys add a converter warp (e4m3 -> bf16
// into the swizzled key tile) before the epilogue warps.
template <int HT, bool FP8, bool SEL = false>
struct Epi {
  static constexpr int WARPS = HT <= 64 ? 16 : 8;
  static constexpr int COLS = kCols / (WARPS / 4);
  static constexpr int CONV = FP8 ? 1 : 0;
  static constexpr int BASE = 3 + CONV;  // first epilogue warp
  static constexpr int THREADS = 32 * (BASE + WARPS);
  // a block's warps are spread over the 4 SM sub-partitions (16K registers
  // each): the largest per-thread count that still lets THREADS threads launch
  static constexpr int MAXREG_RAW = 16384 / (((THREADS / 32) + 3) / 4 * 32) / 8 * 8;
  static constexpr int MAXREG = MAXREG_RAW > 255 ? 255 : MAXREG_RAW;
};
constexpr uint64_t kDrainNs = 2000000;  // 2 ms

// EB = bytes per operand element: 2 for bf16 operands, 1 when both Q and K are
// e4m3 (kind::f8f6f4).
template <int D, int HT, bool FP8, bool SEL = false, int EB = 2>
struct ScoreLayout {
  static_assert(D * EB >= 64, "operand rows of at least 64 bytes");
  static constexpr int ROWB = D * EB >= 128 ? 128 : 64;  // bytes per row of one swizzle chunk
  static constexpr int KCH = D * EB / ROWB;              // swizzle chunks along d
  static constexpr int A_CHUNK = kTileKeys * ROWB;
  static constexpr int A_BYTES = kTileKeys * D * EB;
  static constexpr int B_CHUNK = kCols * ROWB;
  static constexpr int B_BYTES = kCols * D * EB;
  // fused logits of a tile are staged in shared memory ([QG queries][128 keys]
  // fp32, double-buffered) and written by one TMA store (h >= 4)
  static constexpr bool TMA_STORE = HT >= 4 && !SEL;
  static constexpr int QG = kCols / HT;
  static constexpr int STG_BYTES = TMA_STORE ? QG * kTileKeys * 4 : 0;
  static constexpr int SMEM_BUDGET = 227 * 1024 - 1024 - 8 * 1024;  // minus alignment, small data
  // FP8 keys decoded in the kernel: raw e4m3 tiles staged by cp.async, two
  // (the next one prefetched) when that still leaves two key stages, else one
  static constexpr int RAW_TILE = FP8 ? kTileKeys * D : 0;
  static constexpr int NRAW =
      !FP8 ? 0 : ((SMEM_BUDGET - B_BYTES - 2 * STG_BYTES - 2 * RAW_TILE) / A_BYTES >= 2 ? 2 : 1);
  static constexpr int STAGES_FIT =
      (SMEM_BUDGET - B_BYTES - 2 * STG_BYTES - NRAW * RAW_TILE) / A_BYTES;
  static constexpr int STAGES_MAX = D * EB == 256 ? 4 : 8;
  static constexpr int STAGES = STAGES_FIT < STAGES_MAX ? STAGES_FIT : STAGES_MAX;
  static_assert(STAGES >= 2, "key ring needs two stages");
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
  static constexpr int OFF_STG = OFF_B + B_BYTES;       // 2 staging buffers (1024-aligned)
  static constexpr int OFF_RAW = OFF_STG + 2 * STG_BYTES;  // FP8: 2 raw key tiles
  static constexpr int OFF_W = OFF_RAW + NRAW * RAW_TILE;  // per epilogue warp: its columns' w
  static constexpr int OFF_TAU = OFF_W + Epi<HT, FP8>::WARPS * Epi<HT, FP8>::COLS * 4;  // select: tau
  static constexpr int OFF_HEADS = OFF_TAU + (SEL ? Epi<HT, FP8>::WARPS * 16 * 4 : 0);  // producer
  static constexpr int OFF_BAR = OFF_HEADS + kCols * 4;
  static constexpr int NBAR = 2 * STAGES + 10;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int BYTES = OFF_MISC + 16;
  static constexpr int ALLOC = BYTES + 1024;            // room to align the base to 1024
};

struct ScoreParams {
  const uint16_t* Q;
  const float* w;
  const int32_t* heads;  // nullptr: all heads
  const float* k_scale;  // FP8 keys only
  const uint8_t* K8;     // FP8 keys only
  float* logits;
  int64_t ld;
  int n_q;
  int64_t q_pos0;
  int64_t n_k;
  int H;
  int64_t total_tiles;
  DevCtl ctl;
  // select mode (fused top-k): only logits >= tau[t] are stored, and flagged
  const float* tau;
  uint32_t* mask;        // [n_q][mask_ld] pass bits, bit s%32 of word s/32
  int64_t mask_ld;
  // repair launch: nothing unless gate[0] != 0, then only the query groups
  // holding a row t with gate[1 + t] != 0
  const int* gate;
  const float* q_scale;  // e4m3 queries only: [n_q, H] per (query, head) row
  KeyPages kpg;          // paged key cache (kpg.bt != nullptr) or contiguous
  int64_t key_rows;      // rows of the key tensor map (n_k, or the page pool's rows)
};

// Flattened schedule over (group g, key tile kt): each role of a CTA walks the
// same contiguous range, so they agree on every group switch.
template <int QG>
struct Sched {
  int g;
  int64_t kt, nt, left;

  __device__ static int64_t tiles_of(const ScoreParams& p, int g) {
    const int t_last = min((g + 1) * QG, p.n_q) - 1;
    const int64_t last = min(p.q_pos0 + t_last, p.n_k - 1);  // queries may see every key
    return last / kTileKeys + 1;
  }
  __device__ void init(const ScoreParams& p) {
    const int64_t start = p.total_tiles * blockIdx.x / gridDim.x;
    const int64_t end = p.total_tiles * (blockIdx.x + 1) / gridDim.x;
    left = end - start;
    g = 0;
    kt = 0;
    nt = 0;
    if (left <= 0) return;
    int64_t acc = 0;
    while (true) {
      const int64_t n = tiles_of(p, g);
      if (acc + n > start) {
        kt = start - acc;
        nt = n;
        break;
      }
      acc += n;
      ++g;
    }
    skip_dead(p);
  }
  // repair launches (gate set) score only the groups holding a flagged row
  __device__ static bool live(const ScoreParams& p, int g) {
    if (!p.gate) return true;
    const int t1 = min((g + 1) * QG, p.n_q);
    for (int t = g * QG; t < t1; ++t)
      if (p.gate[1 + t]) return true;
    return false;
  }
  __device__ void skip_dead(const ScoreParams& p) {
    while (left > 0 && !live(p, g)) {
      left -= nt - kt;
      if (left <= 0) {
        left = 0;
        break;
      }
      ++g;
      kt = 0;
      nt = tiles_of(p, g);
    }
  }
  __device__ bool last_of_group() const { return kt == nt - 1 || left == 1; }
  __device__ void next(const ScoreParams& p) {
    --left;
    if (++kt == nt && left > 0) {
      ++g;
      kt = 0;
      nt = tiles_of(p, g);
      skip_dead(p);
    }
  }
};

// Key modes: KM 0 = bf16 keys; KM 1 = FP8 E4M3 keys decoded by converter
// warps in the kernel; KM 2 = FP8 keys already decoded to bf16 (exact) by the
// caller; KM 3 = E4M3 queries and keys multiplied as they are (kind::f8f6f4),
// each (query, head) row's scale folded into its head weight.  KM 1, 2 and 3
// multiply each logit by the key's scale.
template <int D, int HT, int KM, bool SEL>
__global__ void __maxnreg__((Epi<HT, KM == 1>::MAXREG))
score_tokens_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap lmap,
                    const ScoreParams p) {
  constexpr bool FP8 = KM == 1;  // converter warps
  constexpr bool KSC = KM != 0;  // per-key scale
  constexpr bool QK8 = KM == 3;  // e4m3 operands
  constexpr int EB = QK8 ? 1 : 2;
  using L = ScoreLayout<D, HT, FP8, SEL, EB>;
  static_assert(!SEL || HT >= 4, "select mode needs h >= 4");
  if (p.gate && *p.gate == 0) return;  // repair launch with nothing to repair
  constexpr int EW = Epi<HT, FP8>::WARPS;
  constexpr int EC = Epi<HT, FP8>::COLS;
  constexpr int QG = kCols / HT;  // queries per group
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const uint32_t sA = smem_u32(smem + L::OFF_A);
  const uint32_t sB = smem_u32(smem + L::OFF_B);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  auto bar = [&](int i) { return smem_u32(bars + i); };
  const int FULL = 0, EMPTY = L::STAGES, BFULL = 2 * L::STAGES, BEMPTY = BFULL + 1,
            ACCFULL = BFULL + 2, ACCEMPTY = BFULL + 4, SFULL = BFULL + 6, SFREE = BFULL + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_MISC + 4);

  const int warp = warp_id(), lane = lane_id();
  if (threadIdx.x == 0) {
    for (int i = 0; i < L::STAGES; ++i) {
      mbar_init(bar(FULL + i), 1);
      mbar_init(bar(EMPTY + i), 1);
    }
    mbar_init(bar(BFULL), 32);
    mbar_init(bar(BEMPTY), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(ACCFULL + i), 1);
      mbar_init(bar(ACCEMPTY + i), EW);
      mbar_init(bar(SFULL + i), EW);
      mbar_init(bar(SFREE + i), 1);
    }
    *abort_flag = 0;
    fence_mbar_init();
    if (!FP8) tma_prefetch_desc(&kmap);
    if (L::TMA_STORE) tma_prefetch_desc(&lmap);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    Sched<QG> it;
    it.init(p);
    int stage = 0;
    uint32_t phase = 0, gcount = 0;
    int prev_g = -1;
    for (; it.left > 0; it.next(p)) {
      if (it.g != prev_g) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(bar(BEMPTY), (gcount & 1) ^ 1, abort_flag, p.ctl);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        // gather the routed (query, head) rows of group g into B: the group's
        // head ids first (independent loads), then one cp.async per 16 bytes
        int32_t* hs = reinterpret_cast<int32_t*>(smem + L::OFF_HEADS);
        for (int n = lane; n < kCols; n += 32) {
          const int t = it.g * QG + n / HT;
          int j = -1;
          if (t < p.n_q) {
            j = p.heads ? __ldg(p.heads + static_cast<int64_t>(t) * HT + n % HT) : n % HT;
            if (j < 0 || j >= p.H) {
              report(p.ctl, DEV_BAD_INPUT);
              j = 0;
            }
          }
          hs[n] = j;
        }
        __syncwarp();
        constexpr int UPR = D * EB / 16;       // 16-byte units per row
        constexpr int UPC = L::ROWB / 16;      // units per swizzle chunk row
        const uint8_t* qb = reinterpret_cast<const uint8_t*>(p.Q);
        for (int x = lane; x < kCols * UPR; x += 32) {
          const int n = x / UPR, u = x % UPR;
          const int j = hs[n];
          const int t = it.g * QG + n / HT;
          const uint8_t* src = j >= 0 ? qb + (static_cast<int64_t>(t) * p.H + j) * (D * EB) + u * 16 : qb;
          const uint32_t off = (u / UPC) * L::B_CHUNK + swz_offset(n, u % UPC, L::ROWB);
          cp_async16(sB + off, src, j >= 0 ? 16u : 0u);
        }
        cp_async_wait_all();
        fence_proxy_async_smem();
        mbar_arrive(bar(BFULL));
        prev_g = it.g;
        ++gcount;
      }
      if (FP8) continue;  // key tiles come from the converter warps
      bool ok = true;
      if (lane == 0) {
        ok = mbar_wait(bar(EMPTY + stage), phase ^ 1, abort_flag, p.ctl);
        if (ok) {
          mbar_arrive_expect_tx(bar(FULL + stage), L::A_BYTES);
          if (!p.kpg.paged()) {
#pragma unroll
            for (int c = 0; c < L::KCH; ++c)
              tma_load_2d(sA + stage * L::A_BYTES + c * L::A_CHUNK, &kmap, bar(FULL + stage),
                          c * (L::ROWB / EB), static_cast<int>(it.kt * kTileKeys));
          } else {
            // one box per page of the tile; pages past the last key are read as
            // fill (a box at the end of the pool), never through the table
            const int ps = 1 << p.kpg.page_shift;
            for (int j = 0; j < kTileKeys / ps; ++j) {
              const int64_t s0 = it.kt * kTileKeys + j * ps;
              const int y = static_cast<int>(s0 < p.n_k ? p.kpg.row(s0, p.ctl) : p.key_rows);
#pragma unroll
              for (int c = 0; c < L::KCH; ++c)
                tma_load_2d(sA + stage * L::A_BYTES + c * L::A_CHUNK + j * ps * L::ROWB, &kmap,
                            bar(FULL + stage), c * (L::ROWB / EB), y);
            }
          }
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (++stage == L::STAGES) {
        stage = 0;
        phase ^= 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    Sched<QG> it;
    it.init(p);
    int stage = 0, acc = 0;
    uint32_t phase = 0, accph = 0, gcount = 0;
    int prev_g = -1;
    constexpr uint32_t idesc =
        QK8 ? umma_idesc_e4m3_f32(kTileKeys, kCols) : umma_idesc_bf16_f32(kTileKeys, kCols);
    for (; it.left > 0; it.next(p)) {
      const bool new_group = it.g != prev_g;
      bool ok = true;
      if (lane == 0) {
        if (new_group) ok = mbar_wait(bar(BFULL), gcount & 1, abort_flag, p.ctl);
        ok = ok && mbar_wait(bar(FULL + stage), phase, abort_flag, p.ctl);
        ok = ok && mbar_wait(bar(ACCEMPTY + acc), accph ^ 1, abort_flag, p.ctl);
        if (ok) {
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * kCols);
          // one instruction per 32 bytes of the rows (16 bf16 or 32 e4m3 elements)
#pragma unroll
          for (int kk = 0; kk < D * EB / 32; ++kk) {
            const int c = (kk * 32) / L::ROWB, within = (kk * 32) % L::ROWB;
            const uint64_t ad =
                umma_desc_kmajor(sA + stage * L::A_BYTES + c * L::A_CHUNK + within, L::ROWB);
            const uint64_t bd = umma_desc_kmajor(sB + c * L::B_CHUNK + within, L::ROWB);
            if constexpr (QK8)
              tc_mma_e4m3(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
            else
              tc_mma_bf16(d_tmem, ad, bd, idesc, kk > 0 ? 1u : 0u);
          }
          tc_commit(bar(EMPTY + stage));
          tc_commit(bar(ACCFULL + acc));
          if (it.last_of_group()) tc_commit(bar(BEMPTY));
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      if (new_group) {
        prev_g = it.g;
        ++gcount;
      }
      if (++stage == L::STAGES) {
        stage = 0;
        phase ^= 1;
      }
      if (++acc == 2) {
        acc = 0;
        accph ^= 1;
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ logit store issuer
    if constexpr (L::TMA_STORE) {
      if (lane == 0) {
        Sched<QG> it;
        it.init(p);
        uint32_t tcount = 0;
        for (; it.left > 0; it.next(p), ++tcount) {
          const uint32_t buf = tcount & 1;
          if (!mbar_wait(bar(SFULL + buf), (tcount >> 1) & 1, abort_flag, p.ctl)) break;
          tma_store_2d(&lmap, smem_u32(smem + L::OFF_STG) + buf * L::STG_BYTES,
                       static_cast<int>(it.kt * kTileKeys),
                       static_cast<int>(static_cast<int64_t>(it.g) * QG));
          bulk_commit();
          bulk_wait_read<1>();  // the previous tile's store has read its buffer
          if (tcount > 0) mbar_arrive(bar(SFREE + (buf ^ 1)));
        }
        bulk_wait_all();
      }
      __syncwarp();
    }
  } else if (warp < Epi<HT, FP8>::BASE) {
    // ------------------------------------------------------------ FP8 key converters
    // e4m3 key rows -> bf16 (exact) straight into the swizzled key tile
    if constexpr (FP8) {
      // the e4m3 rows of the next tile are copied into a raw staging tile by
      // cp.async while this tile's are decoded (shared memory to shared memory)
      constexpr int U8 = D / 16;        // 16-byte e4m3 units per key row
      constexpr int UPC = L::ROWB / 16; // bf16 16-byte units per swizzle-chunk row
      const uint32_t raw0 = smem_u32(smem + L::OFF_RAW);
      auto issue = [&](int64_t kt, int rb) {
        for (int x = lane; x < kTileKeys * U8; x += 32) {
          const int r = x / U8, u = x % U8;
          const int64_t key = kt * kTileKeys + r;
          const bool in = key < p.n_k;
          cp_async16(raw0 + rb * L::RAW_TILE + x * 16,
                     p.K8 + (in ? p.kpg.row(key, p.ctl) : 0) * D + u * 16, in ? 16u : 0u);
        }
        cp_async_commit();
      };
      Sched<QG> it, nx;
      it.init(p);
      nx = it;
      int stage = 0, rb = 0;
      uint32_t phase = 0;
      if (L::NRAW == 2 && it.left > 0) {
        issue(it.kt, 0);
        nx.next(p);
      }
      for (; it.left > 0; it.next(p)) {
        if constexpr (L::NRAW == 2) {
          if (nx.left > 0) {
            issue(nx.kt, rb ^ 1);
            nx.next(p);
          } else {
            cp_async_commit();  // (empty group: keeps the wait below uniform)
          }
          cp_async_wait_group<1>();  // this tile's rows have landed
        } else {
          issue(it.kt, 0);
          cp_async_wait_group<0>();
        }
        __syncwarp();
        bool ok = true;
        if (lane == 0) ok = mbar_wait(bar(EMPTY + stage), phase ^ 1, abort_flag, p.ctl);
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        const uint32_t dst = sA + stage * L::A_BYTES;
        const uint32_t src = raw0 + rb * L::RAW_TILE;
#pragma unroll 4
        for (int x = lane; x < kTileKeys * U8; x += 32) {
          const int r = x / U8, u = x % U8;
          uint32_t wv[4];
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(wv[0]), "=r"(wv[1]), "=r"(wv[2]), "=r"(wv[3])
                       : "r"(src + x * 16));
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const uint32_t b0 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh] & 0xFFFF));
            const uint32_t b1 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh] >> 16));
            const uint32_t b2 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh + 1] & 0xFFFF));
            const uint32_t b3 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[2 * hh + 1] >> 16));
            const int u2 = 2 * u + hh;  // bf16 unit of the row
            const uint32_t off = (u2 / UPC) * L::A_CHUNK + swz_offset(r, u2 % UPC, L::ROWB);
            asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(dst + off), "r"(b0),
                         "r"(b1), "r"(b2), "r"(b3)
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        __syncwarp();  // every lane has read the raw tile before it is refilled
        if (lane == 0) mbar_arrive(bar(FULL + stage));
        if (++stage == L::STAGES) {
          stage = 0;
          phase ^= 1;
        }
        if constexpr (L::NRAW == 2) rb ^= 1;
      }
      cp_async_wait_all();
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int e = warp - Epi<HT, FP8>::BASE;
    const int quad = warp & 3;   // TMEM lanes quad*32 .. quad*32+31
    const int part = e >> 2;     // columns part*EC .. part*EC+EC-1
    constexpr int QPW = EC / HT;  // queries per warp
    float* w_s = reinterpret_cast<float*>(smem + L::OFF_W) + e * EC;  // private to this warp
    Sched<QG> it;
    it.init(p);
    int acc = 0;
    uint32_t accph = 0, tcount = 0;
    int prev_g = -1;
    float* tau_s = reinterpret_cast<float*>(smem + L::OFF_TAU) + e * 16;  // select: thresholds
    (void)tau_s;
    for (; it.left > 0; it.next(p), ++tcount) {
      if (it.g != prev_g) {
        for (int i = lane; i < EC; i += 32) {
          const int col = part * EC + i;
          const int t = it.g * QG + col / HT;
          float wv = 0.0f;
          if (t < p.n_q) {
            int j = p.heads ? __ldg(p.heads + static_cast<int64_t>(t) * HT + col % HT) : col % HT;
            if (j < 0 || j >= p.H) j = 0;
            wv = __ldg(p.w + static_cast<int64_t>(t) * p.H + j);
            // e4m3 queries: the row's scale > 0 commutes with the ReLU
            if constexpr (QK8) wv *= __ldg(p.q_scale + static_cast<int64_t>(t) * p.H + j);
          }
          w_s[i] = wv;
        }
        if constexpr (SEL) {
          for (int qq = lane; qq < QPW; qq += 32) {
            const int64_t t = static_cast<int64_t>(it.g) * QG + part * QPW + qq;
            tau_s[qq] = t < p.n_q ? __ldg(p.tau + t) : INFINITY;
          }
        }
        __syncwarp();
        prev_g = it.g;
      }
      bool ok = true;
      if (lane == 0) ok = mbar_wait(bar(ACCFULL + acc), accph, abort_flag, p.ctl);
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) +
                             static_cast<uint32_t>(acc * kCols + part * EC);
      float sums[HT >= 4 ? QPW : 1];
      // w * ReLU head-sum of query qq (of this warp) from its h columns x[0..HT)
      auto qsum_of = [&](int qq, const uint32_t* x) {
        float2 a2 = make_float2(0.0f, 0.0f);
#pragma unroll
        for (int j = 0; j < HT; j += 4) {
          const float4 w4 = *reinterpret_cast<const float4*>(w_s + qq * HT + j);
          a2 = fma2(make_float2(w4.x, w4.y),
                    make_float2(relu(__uint_as_float(x[j])), relu(__uint_as_float(x[j + 1]))), a2);
          a2 = fma2(make_float2(w4.z, w4.w),
                    make_float2(relu(__uint_as_float(x[j + 2])), relu(__uint_as_float(x[j + 3]))),
                    a2);
        }
        return a2.x + a2.y;
      };
      auto release_acc = [&]() {  // the accumulator is in registers: back to the MMA warp
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(ACCEMPTY + acc));
        if (++acc == 2) {
          acc = 0;
          accph ^= 1;
        }
      };
      // h <= 32: the warp's 64 columns are read 32 at a time (whole queries),
      // the next load in flight while the current queries are summed; only two
      // CW-column buffers are live, which leaves registers for the selection
      constexpr bool CHUNKED = EC == 64 && HT >= 4 && HT <= 32;
      if constexpr (CHUNKED) {
        constexpr int CW = HT <= 64 ? 32 : 16;  // columns per TMEM load (16: 2% slower)
        constexpr int NCH = EC / CW;            // loads per tile
        constexpr int QPC = CW / HT;            // queries per load
        uint32_t vb[2][CW];
        auto ld_cols = [&](uint32_t addr, uint32_t (&r)[CW]) {
          if constexpr (CW == 16)
            tmem_ld16(addr, r);
          else
            tmem_ld32(addr, r);
        };
        ld_cols(taddr, vb[0]);
        tmem_wait_ld_regs(vb[0]);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          if (c + 1 < NCH)
            ld_cols(taddr + static_cast<uint32_t>((c + 1) * CW), vb[(c + 1) & 1]);
          else
            release_acc();
#pragma unroll
          for (int q = 0; q < QPC; ++q) sums[c * QPC + q] = qsum_of(c * QPC + q, vb[c & 1] + q * HT);
          if (c + 1 < NCH) tmem_wait_ld_regs(vb[(c + 1) & 1]);
        }
      }
      uint32_t v[CHUNKED ? 1 : EC];
      if constexpr (!CHUNKED) {
        if constexpr (EC == 64)
          tmem_ld64(taddr, v);
        else
          tmem_ld128(taddr, v);
        tmem_wait_ld();
        release_acc();
      }
      const int64_t s = it.kt * kTileKeys + quad * 32 + lane;
      const bool s_ok = s < p.n_k;
      const int64_t tq0 = static_cast<int64_t>(it.g) * QG + part * QPW;
      float* dst = p.logits + tq0 * p.ld + s;
      (void)dst;
      if constexpr (HT >= 4) {
        if constexpr (!CHUNKED) {
#pragma unroll
          for (int qq = 0; qq < QPW; ++qq) sums[qq] = qsum_of(qq, v + qq * HT);
        }
        if constexpr (KSC) {
          // per-token scale > 0: w * ReLU(scale * dot) = scale * w * ReLU(dot)
          const float ks = s_ok ? __ldg(p.k_scale + p.kpg.row(s, p.ctl)) : 0.0f;
#pragma unroll
          for (int qq = 0; qq < QPW; ++qq) sums[qq] *= ks;
        }
        if constexpr (SEL) {
          // fused top-k: a logit at or above its row's threshold is stored in
          // place and flagged in the row's pass mask (one word per 32 keys);
          // the others are neither stored nor flagged
          const int64_t rows_left = p.n_q - tq0;
          const int q_end = static_cast<int>(rows_left < QPW ? rows_left : QPW);
          // the warp's 32 keys are causal for all its queries and inside n_k: no
          // per-query validity test (every tile but the diagonal and edge ones)
          const int64_t s_last = it.kt * kTileKeys + quad * 32 + 31;
          const bool full = s_last <= p.q_pos0 + tq0 && s_last < p.n_k && q_end == QPW;
          uint32_t m[QPW];
          if (full) {
#pragma unroll
            for (int qq = 0; qq < QPW; ++qq) {
              const bool pass = sums[qq] >= tau_s[qq];
              m[qq] = __ballot_sync(0xffffffffu, pass);
              if (pass) *dst = sums[qq];
              dst += p.ld;
            }
          } else {
            const int64_t cut64 = s - p.q_pos0 - tq0;  // query qq is causal for key s iff qq >= cut
            const int cut = static_cast<int>(cut64 < 0 ? 0 : (cut64 > QPW ? QPW : cut64));
            const uint32_t valid = s_ok ? (((1u << q_end) - 1u) & ~((1u << cut) - 1u)) : 0u;
#pragma unroll
            for (int qq = 0; qq < QPW; ++qq) {
              const bool pass = ((valid >> qq) & 1u) && sums[qq] >= tau_s[qq];
              m[qq] = __ballot_sync(0xffffffffu, pass);
              if (pass) *dst = sums[qq];
              dst += p.ld;
            }
          }
          // lane qq stores the mask word of query qq (a select tree on the lane bits)
          uint32_t mine = m[0];
#pragma unroll
          for (int bit = 1; bit < QPW; bit <<= 1) {
#pragma unroll
            for (int qq = 0; qq < QPW; qq += 2 * bit) m[qq] = (lane & bit) ? m[qq + bit] : m[qq];
          }
          mine = m[0];
          if (lane < q_end)
            p.mask[(tq0 + lane) * p.mask_ld + it.kt * (kTileKeys / 32) + quad] = mine;
        } else {
        // stage [query][key] in shared memory, then one TMA store per tile
          // (rows past n_q and keys past n_k fall outside the map and are not written)
          const uint32_t buf = tcount & 1;
          const uint32_t sbuf = smem_u32(smem + L::OFF_STG) + buf * L::STG_BYTES;
          bool sok = true;
          if (lane == 0) sok = mbar_wait(bar(SFREE + buf), ((tcount >> 1) & 1) ^ 1, abort_flag, p.ctl);
          if (!__shfl_sync(0xffffffffu, sok, 0)) break;
          const int64_t cut64 = s - p.q_pos0 - tq0;  // query qq is causal for key s iff qq >= cut
          const int cut = static_cast<int>(cut64 < 0 ? 0 : (cut64 > QPW ? QPW : cut64));
#pragma unroll
          for (int qq = 0; qq < QPW; ++qq) {
            const float val = qq >= cut ? sums[qq] : -INFINITY;
            const uint32_t a = sbuf + static_cast<uint32_t>(((part * QPW + qq) * kTileKeys + quad * 32 + lane) * 4);
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(a), "f"(val) : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(bar(SFULL + buf));
        }
        (void)s_ok;
      } else {
#pragma unroll
        for (int qq = 0; qq < QPW; ++qq) {
          float sum;
          if constexpr (HT == 1) {
            sum = w_s[qq] * relu(__uint_as_float(v[qq]));
          } else {
            const float2 w2 = *reinterpret_cast<const float2*>(w_s + qq * 2);
            sum = fmaf(w2.y, relu(__uint_as_float(v[qq * 2 + 1])), w2.x * relu(__uint_as_float(v[qq * 2])));
          }
          if constexpr (KSC) sum *= s_ok ? __ldg(p.k_scale + p.kpg.row(s, p.ctl)) : 0.0f;
          const int64_t t = tq0 + qq;
          if (t < p.n_q && s_ok) *dst = (s <= p.q_pos0 + t) ? sum : -INFINITY;
          dst += p.ld;
        }
      }
    }
  }

  __syncthreads();
  if (*abort_flag) drain_pause(kDrainNs);  // let issued copies / MMAs land
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int D, int HT, int KM, bool SEL>
cudaError_t launch_dhs(const ScoreParams& p, const CUtensorMap& map, cudaStream_t s) {
  constexpr bool FP8 = KM == 1;
  using L = ScoreLayout<D, HT, FP8, SEL, KM == 3 ? 1 : 2>;
  // fused-logit store map: [n_q rows][n_k keys] fp32 with row pitch ld, box 128 keys x QG queries
  CUtensorMap lmap;
  std::memset(&lmap, 0, sizeof lmap);
  if (L::TMA_STORE) {
    // the store covers whole 16-byte units: keys up to n_k rounded up to 4 (< ld)
    const uint64_t dims[2] = {static_cast<uint64_t>((p.n_k + 3) / 4 * 4), static_cast<uint64_t>(p.n_q)};
    const uint64_t strides[1] = {static_cast<uint64_t>(p.ld) * 4};
    const uint32_t box[2] = {static_cast<uint32_t>(kTileKeys), static_cast<uint32_t>(L::QG)};
    if (encode_tensor_map(&lmap, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, p.logits, dims, strides, box,
                          CU_TENSOR_MAP_SWIZZLE_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  auto kern = score_tokens_kernel<D, HT, KM, SEL>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, L::ALLOC);
  if (e != cudaSuccess) return e;
  const int64_t grid = std::min<int64_t>(sm_count(), p.total_tiles);
  if (grid <= 0) return cudaSuccess;
  kern<<<static_cast<unsigned>(grid), Epi<HT, FP8>::THREADS, L::ALLOC, s>>>(map, lmap, p);
  return cudaGetLastError();
}

template <int D, int KM>
cudaError_t launch_d(const ScoreParams& p, int h, bool sel, const CUtensorMap& map, cudaStream_t s) {
  if (sel) {
    switch (h) {
      case 4: return launch_dhs<D, 4, KM, true>(p, map, s);
      case 8: return launch_dhs<D, 8, KM, true>(p, map, s);
      case 16: return launch_dhs<D, 16, KM, true>(p, map, s);
      case 32: return launch_dhs<D, 32, KM, true>(p, map, s);
      case 64: return launch_dhs<D, 64, KM, true>(p, map, s);
    }
    return cudaErrorNotSupported;
  }
  switch (h) {
    case 1: return launch_dhs<D, 1, KM, false>(p, map, s);
    case 2: return launch_dhs<D, 2, KM, false>(p, map, s);
    case 4: return launch_dhs<D, 4, KM, false>(p, map, s);
    case 8: return launch_dhs<D, 8, KM, false>(p, map, s);
    case 16: return launch_dhs<D, 16, KM, false>(p, map, s);
    case 32: return launch_dhs<D, 32, KM, false>(p, map, s);
    case 64: return launch_dhs<D, 64, KM, false>(p, map, s);
    case 128: return launch_dhs<D, 128, KM, false>(p, map, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool score_select_supported(int h) { return h == 4 || h == 8 || h == 16 || h == 32 || h == 64; }

cudaError_t launch_score(const ScoreLaunch& a, const DevCtl& ctl, cudaStream_t s) {
  if (a.n_q <= 0) return cudaSuccess;
  const bool sel = a.tau != nullptr;
  if (sel && !score_select_supported(a.h)) return cudaErrorNotSupported;
  const int QG = kCols / a.h;
  const int n_groups = (a.n_q + QG - 1) / QG;
  int64_t total = 0;
  for (int g = 0; g < n_groups; ++g) {
    const int t_last = std::min((g + 1) * QG, a.n_q) - 1;
    total += std::min<int64_t>(a.q_pos0 + t_last, a.n_k - 1) / kTileKeys + 1;
  }
  // key tensor map: [key_rows, d] with one box per 128-key tile, or per page
  const bool paged = a.kpg.paged();
  const int64_t key_rows = paged ? (a.kpg.n_pages << a.kpg.page_shift) : a.n_k;
  const uint32_t box_rows = paged ? (1u << a.kpg.page_shift) : static_cast<uint32_t>(kTileKeys);
  if (paged && (box_rows > static_cast<uint32_t>(kTileKeys) || box_rows < 8)) return cudaErrorInvalidValue;
  ScoreParams p{a.Q, a.w, a.heads, a.k_scale, static_cast<const uint8_t*>(a.K), a.logits, a.ld,
                a.n_q, a.q_pos0, a.n_k, a.H, total, ctl, a.tau, a.mask, a.mask_ld,
                a.gate, a.q_scale, a.kpg, key_rows};
  CUtensorMap map;
  std::memset(&map, 0, sizeof map);
  if (a.q8) {  // e4m3 queries and keys: one-byte key tiles by TMA, kind::f8f6f4
    if (!a.fp8 || a.k_bf16 || (a.d != 64 && a.d != 128)) return cudaErrorNotSupported;
    const uint64_t dims[2] = {static_cast<uint64_t>(a.d), static_cast<uint64_t>(key_rows)};
    const uint64_t strides[1] = {static_cast<uint64_t>(a.d)};
    const uint32_t box[2] = {static_cast<uint32_t>(a.d), box_rows};
    if (encode_tensor_map(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, a.K, dims, strides, box,
                          a.d == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    return a.d == 128 ? launch_d<128, 3>(p, a.h, sel, map, s) : launch_d<64, 3>(p, a.h, sel, map, s);
  }
  if (a.fp8 && !a.k_bf16) {  // converter warps read the e4m3 keys; no key tensor map
    switch (a.d) {
      case 32: return launch_d<32, 1>(p, a.h, sel, map, s);
      case 64: return launch_d<64, 1>(p, a.h, sel, map, s);
      case 128: return launch_d<128, 1>(p, a.h, sel, map, s);
    }
    return cudaErrorInvalidValue;
  }
  const uint64_t dims[2] = {static_cast<uint64_t>(a.d), static_cast<uint64_t>(key_rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(a.d) * 2};
  const int rowb = a.d >= 64 ? 128 : 64;
  const uint32_t box[2] = {static_cast<uint32_t>(rowb / 2), box_rows};
  if (encode_tensor_map(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, a.K, dims, strides, box,
                        rowb == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) !=
      CUDA_SUCCESS)
    return cudaErrorInvalidValue;
  if (a.fp8) {  // decoded FP8 keys: bf16 operand, per-key scale in the epilogue
    switch (a.d) {
      case 32: return launch_d<32, 2>(p, a.h, sel, map, s);
      case 64: return launch_d<64, 2>(p, a.h, sel, map, s);
      case 128: return launch_d<128, 2>(p, a.h, sel, map, s);
    }
    return cudaErrorInvalidValue;
  }
  switch (a.d) {
    case 32: return launch_d<32, 0>(p, a.h, sel, map, s);
    case 64: return launch_d<64, 0>(p, a.h, sel, map, s);
    case 128: return launch_d<128, 0>(p, a.h, sel, map, s);
  }
  return cudaErrorInvalidValue;
}

}  // namespace misa
