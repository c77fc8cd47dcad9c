#include <algorithm>
// Stage 1 — block mean-pooling of the shared index keys.
//
// kbar[m, :] = (1/n_m) * sum of K rows mB .. mB+n_m-1, n_m = min(B, n_k - mB)
// ("MISA" technical summary, Metodologia step 1: the prefix is split into
// M = ceil(L/B) blocks summarised by mean-pooled index keys).
//
// HBM-bound stream: one CTA per block, 16-byte loads along d, fp32 partial sums
// per (row phase, column group), combined in shared memory.  Also writes the
// hi/lo bf16 split of kbar that the router's tensor-core contraction reads.
#include "internal.h"

namespace misa {
namespace {

constexpr int kPoolThreads = 256;

// Many sequences at once (decode): sequence blockIdx.y has lens[y] keys through
// block table bts[y]; its pooled keys are kbar[y] ([M_max, d]) and kbar_hl[y]
// ([2, M_max, d]); the CTA pools block M_y - n_last + blockIdx.x of it, where
// M_y = ceil(lens[y] / B) (nothing when that block does not exist).
struct PoolBatch {
  const int32_t* bts;    // nullptr: one sequence (the kernel's own arguments)
  int max_blocks;
  const int32_t* lens;
  int64_t M_max;
  int64_t n_last;
};

template <int D, bool FP8>
__global__ void __launch_bounds__(kPoolThreads)
pool_keys_kernel(const uint8_t* __restrict__ K, const float* __restrict__ k_scale, KeyPages kpg,
                 int64_t n_k, int B, int64_t M, int64_t m0, float* __restrict__ kbar,
                 uint16_t* __restrict__ kbar_hl, DevCtl ctl, PoolBatch batch) {
  // elements per 16-byte unit and units per row
  constexpr int EPU = FP8 ? 16 : 8;
  constexpr int UPR = D / EPU;                 // column groups
  constexpr int PHASES = kPoolThreads / UPR;   // rows handled in parallel
  static_assert(kPoolThreads % UPR == 0, "column groups must tile the block");
  __shared__ float part[PHASES][D];

  int64_t m = m0 + blockIdx.x;  // this CTA's block
  if (batch.bts) {
    const int y = blockIdx.y;
    kpg.bt = batch.bts + static_cast<int64_t>(y) * batch.max_blocks;
    n_k = __ldg(batch.lens + y);
    const int64_t cap = static_cast<int64_t>(batch.max_blocks) << kpg.page_shift;
    if (n_k > cap) {
      report(ctl, DEV_BAD_INPUT);
      n_k = cap;
    }
    const int64_t My = (n_k + B - 1) / B;
    m = My - batch.n_last + blockIdx.x;
    if (n_k <= 0 || m < 0 || m >= My || My > batch.M_max) return;
    M = batch.M_max;
    if (kbar) kbar += static_cast<int64_t>(y) * batch.M_max * D;
    if (kbar_hl) kbar_hl += static_cast<int64_t>(y) * 2 * batch.M_max * D;
  }
  const int64_t first = m * B;
  const int n_m = static_cast<int>(n_k - first < B ? n_k - first : static_cast<int64_t>(B));
  const int u = threadIdx.x % UPR;
  const int ph = threadIdx.x / UPR;
  constexpr int ROW_BYTES = D * (FP8 ? 1 : 2);

  float acc[EPU];
#pragma unroll
  for (int e = 0; e < EPU; ++e) acc[e] = 0.0f;

  // physical row of the block's r-th key (contiguous or paged cache)
  auto prow = [&](int r) { return kpg.row(first + r, ctl); };
  const uint8_t* base = K + u * 16;
  int r = ph;
  // two rows in flight per iteration
  for (; r + PHASES < n_m; r += 2 * PHASES) {
    const int64_t ra = prow(r), rb = prow(r + PHASES);
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(base + ra * ROW_BYTES));
    const uint4 b = __ldg(reinterpret_cast<const uint4*>(base + rb * ROW_BYTES));
    const uint4 ab[2] = {a, b};
    float sc[2] = {1.0f, 1.0f};
    if (FP8) {
      sc[0] = __ldg(k_scale + ra);
      sc[1] = __ldg(k_scale + rb);
    }
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint32_t* wv = reinterpret_cast<const uint32_t*>(&ab[q]);
      if (FP8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t bf2 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[i >> 1] >> ((i & 1) * 16)));
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bf2));
          acc[2 * i] += f.x * sc[q];
          acc[2 * i + 1] += f.y * sc[q];
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[i]));
          acc[2 * i] += f.x;
          acc[2 * i + 1] += f.y;
        }
      }
    }
  }
  for (; r < n_m; r += PHASES) {
    const int64_t ra = prow(r);
    const uint4 a = __ldg(reinterpret_cast<const uint4*>(base + ra * ROW_BYTES));
    const uint32_t* wv = reinterpret_cast<const uint32_t*>(&a);
    if (FP8) {
      const float sc = __ldg(k_scale + ra);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint32_t bf2 = e4m3x2_to_bf16x2(static_cast<uint16_t>(wv[i >> 1] >> ((i & 1) * 16)));
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&bf2));
        acc[2 * i] += f.x * sc;
        acc[2 * i + 1] += f.y * sc;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[i]));
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
  }
#pragma unroll
  for (int e = 0; e < EPU; ++e) part[ph][u * EPU + e] = acc[e];
  __syncthreads();
  for (int c = threadIdx.x; c < D; c += kPoolThreads) {
    float s = 0.0f;
#pragma unroll 8
    for (int p = 0; p < PHASES; ++p) s += part[p][c];
    const float mean = s / static_cast<float>(n_m);
    if (kbar) kbar[m * D + c] = mean;
    if (kbar_hl) {
      const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
      const __nv_bfloat16 lo = __float2bfloat16_rn(mean - __bfloat162float(hi));
      kbar_hl[m * D + c] = __bfloat16_as_ushort(hi);
      kbar_hl[(M + m) * D + c] = __bfloat16_as_ushort(lo);
    }
  }
}

template <int D, bool FP8>
cudaError_t launch_batch(const void* K, const float* k_scale, const KeyPages& kpg, int B,
                         const PoolBatch& batch, int n_seq, float* kbar, uint16_t* kbar_hl,
                         const DevCtl& ctl, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>(batch.n_last), static_cast<unsigned>(n_seq));
  pool_keys_kernel<D, FP8><<<grid, kPoolThreads, 0, s>>>(static_cast<const uint8_t*>(K), k_scale,
                                                        kpg, 0, B, batch.M_max, 0, kbar, kbar_hl,
                                                        ctl, batch);
  return cudaGetLastError();
}

// Large ranges of bf16 keys: one persistent CTA per SM takes a contiguous share
// of the blocks and streams them through a ring of shared-memory stages that
// bulk copies (the TMA engine: a block's rows, or its runs inside pages) fill
// `stages` blocks ahead, so every SM keeps ~200 KB in flight.  Each block is
// summed with the per-block kernel's thread-to-row mapping and order (rows
// ph, ph + PHASES, ... per thread, then the phases in order), so both kernels
// give the same bits.
template <int D>
__global__ void __launch_bounds__(kPoolThreads, 1)
pool_stream_kernel(const uint8_t* __restrict__ K, KeyPages kpg, int64_t n_k, int B, int64_t M,
                   int64_t m0, int64_t m1, float* __restrict__ kbar, uint16_t* __restrict__ kbar_hl,
                   int stages, DevCtl ctl) {
  constexpr int EPU = 8;
  constexpr int UPR = D / EPU;
  constexpr int PHASES = kPoolThreads / UPR;
  constexpr int ROW_BYTES = D * 2;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  float(*part)[D] = reinterpret_cast<float(*)[D]>(smem_raw);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + PHASES * D * 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(full + stages);
  uint8_t* ring = smem_raw + ((PHASES * D * 4 + 8 * stages + 16 + 127) / 128) * 128;
  const int64_t stage_bytes = static_cast<int64_t>(B) * ROW_BYTES;
  const int64_t nblk = m1 - m0;
  const int64_t b0 = m0 + nblk * blockIdx.x / gridDim.x;
  const int nb = static_cast<int>(m0 + nblk * (blockIdx.x + 1) / gridDim.x - b0);
  const int tid = threadIdx.x, u = tid % UPR, ph = tid / UPR;
  if (tid == 0) {
    for (int i = 0; i < stages; ++i) mbar_init(smem_u32(full + i), 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // (thread 0) block b0 + j into stage j % stages
  auto issue = [&](int j) {
    const int64_t first = (b0 + j) * B;
    const int n_m = static_cast<int>(n_k - first < B ? n_k - first : static_cast<int64_t>(B));
    const uint32_t bar = smem_u32(full + j % stages);
    const uint32_t dst = smem_u32(ring + (j % stages) * stage_bytes);
    mbar_arrive_expect_tx(bar, static_cast<uint32_t>(n_m) * ROW_BYTES);
    if (!kpg.paged()) {
      bulk_load(dst, K + first * ROW_BYTES, static_cast<uint32_t>(n_m) * ROW_BYTES, bar);
      return;
    }
    const int ps = 1 << kpg.page_shift;
    for (int r = 0; r < n_m;) {
      const int64_t s = first + r;
      const int in_page = ps - static_cast<int>(s & (ps - 1));
      const int run = in_page < n_m - r ? in_page : n_m - r;
      bulk_load(dst + r * ROW_BYTES, K + kpg.row(s, ctl) * ROW_BYTES,
                static_cast<uint32_t>(run) * ROW_BYTES, bar);
      r += run;
    }
  };
  if (tid == 0)
    for (int j = 0; j < nb && j < stages; ++j) issue(j);
  for (int j = 0; j < nb; ++j) {
    const int64_t m = b0 + j;
    const int64_t first = m * B;
    const int n_m = static_cast<int>(n_k - first < B ? n_k - first : static_cast<int64_t>(B));
    const bool ok = mbar_wait(smem_u32(full + j % stages), (j / stages) & 1, abort_flag, ctl);
    float acc[EPU];
#pragma unroll
    for (int e = 0; e < EPU; ++e) acc[e] = 0.0f;
    const uint8_t* blk = ring + (j % stages) * stage_bytes + u * 16;
    for (int r = ph; ok && r < n_m; r += PHASES) {
      const uint4 a = *reinterpret_cast<const uint4*>(blk + r * ROW_BYTES);
      const uint32_t* wv = reinterpret_cast<const uint32_t*>(&a);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wv[i]));
        acc[2 * i] += f.x;
        acc[2 * i + 1] += f.y;
      }
    }
#pragma unroll
    for (int e = 0; e < EPU; ++e) part[ph][u * EPU + e] = acc[e];
    if (!__syncthreads_and(ok)) break;
    // the stage is read: refill it
    if (tid == 0 && j + stages < nb) issue(j + stages);
    for (int c = tid; c < D; c += kPoolThreads) {
      float sum = 0.0f;
#pragma unroll 8
      for (int p = 0; p < PHASES; ++p) sum += part[p][c];
      const float mean = sum / static_cast<float>(n_m);
      if (kbar) kbar[m * D + c] = mean;
      if (kbar_hl) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(mean);
        const __nv_bfloat16 lo = __float2bfloat16_rn(mean - __bfloat162float(hi));
        kbar_hl[m * D + c] = __bfloat16_as_ushort(hi);
        kbar_hl[(M + m) * D + c] = __bfloat16_as_ushort(lo);
      }
    }
    __syncthreads();  // part is rewritten by the next block
  }
  if (*abort_flag) drain_pause(2000000);  // let issued copies land
}

template <int D, bool FP8>
cudaError_t launch(const void* K, const float* k_scale, const KeyPages& kpg, int64_t n_k, int B,
                   int64_t m0, int64_t m1, float* kbar, uint16_t* kbar_hl, const DevCtl& ctl,
                   cudaStream_t s) {
  const int64_t M = (n_k + B - 1) / B;
  if (m1 > M) m1 = M;
  if (m1 <= m0) return cudaSuccess;
  const int sms = sm_count();
  if constexpr (!FP8) {
    // the streaming kernel when every SM gets two or more blocks and three
    // block stages fit
    constexpr int PHASES = kPoolThreads / (D / 8);
    const int64_t stage_bytes = static_cast<int64_t>(B) * D * 2;
    const int64_t fixed = ((PHASES * D * 4 + 8 * 8 + 16 + 127) / 128) * 128 + 128;
    const int64_t budget = 227 * 1024 - fixed;
    const int stages = static_cast<int>(std::min<int64_t>(8, budget / stage_bytes));
    if (m1 - m0 >= 2 * static_cast<int64_t>(sms) && stages >= 3) {
      const size_t smem = static_cast<size_t>(fixed + stages * stage_bytes);
      cudaError_t e = cudaFuncSetAttribute(pool_stream_kernel<D>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           static_cast<int>(smem));
      if (e != cudaSuccess) return e;
      pool_stream_kernel<D><<<static_cast<unsigned>(sms), kPoolThreads, smem, s>>>(
          static_cast<const uint8_t*>(K), kpg, n_k, B, M, m0, m1, kbar, kbar_hl, stages, ctl);
      return cudaGetLastError();
    }
  }
  pool_keys_kernel<D, FP8><<<static_cast<unsigned>(m1 - m0), kPoolThreads, 0, s>>>(
      static_cast<const uint8_t*>(K), k_scale, kpg, n_k, B, M, m0, kbar, kbar_hl, ctl,
      PoolBatch{nullptr, 0, nullptr, 0, 0});
  return cudaGetLastError();
}

// 16 E4M3 codes per thread -> 16 bf16 codes (exact: every E4M3 value is a bf16
// value).
__global__ void __launch_bounds__(256)
e4m3_to_bf16_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst, int64_t n16) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const uint4 raw = __ldg(src + i);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      o[2 * j] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w[j] & 0xFFFF));
      o[2 * j + 1] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w[j] >> 16));
    }
    dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// Logical key rows 0..n_k-1 of an e4m3 cache (paged or contiguous) decoded to
// bf16 codes (exact) in logical order, 16 codes per thread; with dst_scale the
// rows' scales are gathered into logical order too.
__global__ void __launch_bounds__(256)
e4m3_rows_to_bf16_kernel(const uint8_t* __restrict__ src, const float* __restrict__ scale,
                         KeyPages kpg, int64_t n_k, int d, uint4* __restrict__ dst,
                         float* __restrict__ dst_scale, DevCtl ctl) {
  const int upr = d / 16;  // 16-byte units of an e4m3 row
  const int64_t n16 = n_k * upr;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n16;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t srow = i / upr;
    const int u = static_cast<int>(i - srow * upr);
    const int64_t prow = kpg.row(srow, ctl);
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src + prow * d) + u);
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t o[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      o[2 * j] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w[j] & 0xFFFF));
      o[2 * j + 1] = e4m3x2_to_bf16x2(static_cast<uint16_t>(w[j] >> 16));
    }
    dst[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    if (dst_scale && u == 0) dst_scale[srow] = __ldg(scale + prow);
  }
}

}  // namespace

cudaError_t launch_e4m3_rows_to_bf16(const uint8_t* src, const float* scale, const KeyPages& kpg,
                                     int64_t n_k, int d, uint16_t* dst, float* dst_scale,
                                     const DevCtl& ctl, cudaStream_t s) {
  const int64_t n16 = n_k * (d / 16);
  if (n16 <= 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n16 + 255) / 256, static_cast<int64_t>(sm_count()) * 8);
  e4m3_rows_to_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      src, scale, kpg, n_k, d, reinterpret_cast<uint4*>(dst), dst_scale, ctl);
  return cudaGetLastError();
}

cudaError_t launch_e4m3_to_bf16(const uint8_t* src, uint16_t* dst, int64_t n, cudaStream_t s) {
  const int64_t n16 = n / 16;
  if (n16 <= 0) return cudaSuccess;
  const int64_t blocks = std::min<int64_t>((n16 + 255) / 256, static_cast<int64_t>(sm_count()) * 8);
  e4m3_to_bf16_kernel<<<static_cast<unsigned>(blocks), 256, 0, s>>>(
      reinterpret_cast<const uint4*>(src), reinterpret_cast<uint4*>(dst), n16);
  return cudaGetLastError();
}

cudaError_t launch_pool_keys_batch(const void* pages, const float* k_scale, bool fp8,
                                   const int32_t* block_tables, int max_blocks, int page_shift,
                                   int64_t n_pages, const int32_t* lens, int n_seq, int d, int B,
                                   int64_t M_max, int64_t n_last, float* kbar, uint16_t* kbar_hl,
                                   const DevCtl& ctl, cudaStream_t s) {
  if (n_seq <= 0 || n_last <= 0) return cudaSuccess;
  const KeyPages kpg{nullptr, page_shift, n_pages};  // the table is set per sequence
  const PoolBatch batch{block_tables, max_blocks, lens, M_max, n_last};
  if (fp8) {
    switch (d) {
      case 32: return launch_batch<32, true>(pages, k_scale, kpg, B, batch, n_seq, kbar, kbar_hl, ctl, s);
      case 64: return launch_batch<64, true>(pages, k_scale, kpg, B, batch, n_seq, kbar, kbar_hl, ctl, s);
      case 128: return launch_batch<128, true>(pages, k_scale, kpg, B, batch, n_seq, kbar, kbar_hl, ctl, s);
    }
  } else {
    switch (d) {
      case 32: return launch_batch<32, false>(pages, k_scale, kpg, B, batch, n_seq, kbar, kbar_hl, ctl, s);
      case 64: return launch_batch<64, false>(pages, k_scale, kpg, B, batch, n_seq, kbar, kbar_hl, ctl, s);
      case 128: return launch_batch<128, false>(pages, k_scale, kpg, B, batch, n_seq, kbar, kbar_hl, ctl, s);
    }
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_pool_keys(const void* K, const float* k_scale, const KeyPages& kpg, bool fp8,
                             int64_t n_k, int d, int B, int64_t m0, int64_t m1, float* kbar,
                             uint16_t* kbar_hl, const DevCtl& ctl, cudaStream_t s) {
  if (fp8) {
    switch (d) {
      case 32: return launch<32, true>(K, k_scale, kpg, n_k, B, m0, m1, kbar, kbar_hl, ctl, s);
      case 64: return launch<64, true>(K, k_scale, kpg, n_k, B, m0, m1, kbar, kbar_hl, ctl, s);
      case 128: return launch<128, true>(K, k_scale, kpg, n_k, B, m0, m1, kbar, kbar_hl, ctl, s);
    }
  } else {
    switch (d) {
      case 32: return launch<32, false>(K, k_scale, kpg, n_k, B, m0, m1, kbar, kbar_hl, ctl, s);
      case 64: return launch<64, false>(K, k_scale, kpg, n_k, B, m0, m1, kbar, kbar_hl, ctl, s);
      case 128: return launch<128, false>(K, k_scale, kpg, n_k, B, m0, m1, kbar, kbar_hl, ctl, s);
    }
  }
  return cudaErrorInvalidValue;
}

}  // namespace misa
