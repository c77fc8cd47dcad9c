// C ABI of libmisa (declared in include/misa.h): argument validation, the
// per-device status word, the bounded-wait budget, TMA descriptor encoding and
// the stage launches.  Nothing here allocates device memory.
#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"
#include "misa.h"

namespace misa {

namespace {

__device__ int g_device_status;  // one per device that loads the library

constexpr int kMaxDevices = 64;
std::mutex g_mu;
int* g_status_ptr[kMaxDevices] = {};
int g_sm_count[kMaxDevices] = {};
std::atomic<unsigned long long> g_wait_ns{2000000000ull};

int current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

int* status_ptr() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_status) != cudaSuccess) return nullptr;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  return g_status_ptr[dev];
}

bool make_ctl(DevCtl& ctl) {
  ctl.status = status_ptr();
  ctl.wait_ns = g_wait_ns.load();
  return ctl.status != nullptr;
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                              const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                              CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                              CUtensorMapFloatOOBfill);
EncodeFn g_encode = nullptr;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool good_d(int d) { return d == 32 || d == 64 || d == 128; }
bool pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }
cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }
int cuda_status(cudaError_t e) { return e == cudaSuccess ? MISA_OK : MISA_ERR_CUDA; }

// Fused score + top-k: the routed logits of a 32 x 128-key sample of the
// visible prefix set per-row thresholds; the scoring pass then stores only the
// logits at or above them (flagged in per-row pass masks) and an exact
// selection over the flagged logits finishes.
constexpr int kSampleBlocks = 32;
constexpr int kSampleKeys = kSampleBlocks * 128;
constexpr int64_t kFusedMaxKeys = int64_t(1) << 18;  // a 4096-key sample stays representative
constexpr int kFusedMaxK = 8192;                    // the finish kernel's list fits in shared memory

size_t round256(size_t x) { return (x + 255) / 256 * 256; }

// The key cache of an entry point: contiguous ([n_k, d] rows) or paged (pages
// of page_size rows in a pool of n_pages pages, logical block b of the
// sequence in page block_table[b]); FP8 scales follow the physical rows.
struct KeyArg {
  const void* K;
  const float* k_scale;
  int kdtype;
  KeyPages kpg;
  bool fp8() const { return kdtype == MISA_K_FP8E4M3; }
};

KeyArg contiguous_keys(const void* K, const float* k_scale, int kdtype) {
  return KeyArg{K, k_scale, kdtype, KeyPages{nullptr, 0, 0}};
}

// page_size must be 16, 32, 64 or 128 (a 128-key tile holds whole pages); an
// unsupported size leaves page_shift at -1 for check_keys to refuse.
KeyArg paged_keys(const void* pages, const float* k_scale, int kdtype, const int32_t* block_table,
                  int page_size, int64_t n_pages) {
  int shift = -1;
  for (int sh = 4; sh <= 7; ++sh)
    if (page_size == (1 << sh)) shift = sh;
  return KeyArg{pages, k_scale, kdtype, KeyPages{block_table, shift, n_pages}};
}

// scaled_bf16_ok: the call takes MISA_K_BF16_SCALED (contiguous keys only).
int check_keys(const KeyArg& k, int64_t n_k, bool scaled_bf16_ok = false) {
  if (!k.K || !aligned16(k.K)) return MISA_ERR_INVALID_ARG;
  const bool scaled = k.kdtype == MISA_K_BF16_SCALED && scaled_bf16_ok && !k.kpg.bt;
  if (k.kdtype != MISA_K_BF16 && k.kdtype != MISA_K_FP8E4M3 && !scaled) return MISA_ERR_INVALID_ARG;
  if ((k.fp8() || scaled) && (!k.k_scale || !aligned4(k.k_scale))) return MISA_ERR_INVALID_ARG;
  if (n_k > 0x7fffffffLL) return MISA_ERR_INVALID_ARG;
  if (k.kpg.bt) {
    if (!aligned4(k.kpg.bt)) return MISA_ERR_INVALID_ARG;
    if (k.kpg.page_shift < 0) return MISA_ERR_UNSUPPORTED;
    if (k.kpg.n_pages < 1 || (k.kpg.n_pages << k.kpg.page_shift) > 0x7fffffffLL)
      return MISA_ERR_INVALID_ARG;
  }
  return MISA_OK;
}

// Optional per-stage timing of misa_score_topk: while enabled, every launch of
// the fused sequence is bracketed by a pair of CUDA events on its stream.
constexpr int kStages = 7;
const char* const kStageNames[kStages] = {"prepare",       "sample_score", "threshold",
                                          "select_score",  "finish",       "repair_score",
                                          "repair_topk"};
struct Profiler {
  std::mutex mu;
  std::atomic<bool> on{false};
  std::vector<cudaEvent_t> start[kStages], stop[kStages];
};
Profiler g_prof;

struct StageMark {
  int stage;
  cudaStream_t s;
  cudaEvent_t a = nullptr;
  StageMark(int st, cudaStream_t str) : stage(st), s(str) {
    if (g_prof.on.load() && cudaEventCreate(&a) == cudaSuccess) cudaEventRecord(a, s);
  }
  ~StageMark() {
    if (!a) return;
    cudaEvent_t b = nullptr;
    if (cudaEventCreate(&b) != cudaSuccess) {
      cudaEventDestroy(a);
      return;
    }
    cudaEventRecord(b, s);
    std::lock_guard<std::mutex> lk(g_prof.mu);
    g_prof.start[stage].push_back(a);
    g_prof.stop[stage].push_back(b);
  }
};

int64_t mask_words(int64_t n_k) { return ((n_k + 31) / 32 + 3) / 4 * 4; }

struct FusedLayout {
  size_t gate, tau, ks, ks_scale, sample, mask, kbf, kbf_scale, total;
  FusedLayout(int n_q, int64_t n_k) {
    const size_t nq = static_cast<size_t>(n_q);
    size_t o = 0;
    gate = o;
    o += round256((nq + 1) * 4);
    tau = o;
    o += round256(nq * 4);
    ks = o;
    o += round256(static_cast<size_t>(kSampleKeys) * 256);  // d <= 128 bf16
    ks_scale = o;
    o += round256(static_cast<size_t>(kSampleKeys) * 4);
    sample = o;
    o += round256(nq * kSampleKeys * 4);
    mask = o;
    o += round256(nq * static_cast<size_t>(mask_words(n_k)) * 4);
    kbf = o;  // FP8 keys decoded to bf16 (d <= 128), in logical order
    o += round256(static_cast<size_t>(n_k) * 256);
    kbf_scale = o;  // their scales, in logical order (paged caches)
    o += round256(static_cast<size_t>(n_k) * 4);
    total = o;
  }
};

}  // namespace

int* device_status_word() { return status_ptr(); }

unsigned long long wait_limit_ns() { return g_wait_ns.load(); }

int sm_count() {
  const int dev = current_device();
  if (dev < 0 || dev >= kMaxDevices) return 148;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_sm_count[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    g_sm_count[dev] = n;
  }
  return g_sm_count[dev];
}

CUresult encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank, const void* base,
                           const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box,
                           CUtensorMapSwizzle swz) {
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return CUDA_ERROR_NOT_FOUND;
      g_encode = reinterpret_cast<EncodeFn>(fn);
    }
  }
  cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(map, dtype, static_cast<cuuint32_t>(rank), const_cast<void*>(base),
                  reinterpret_cast<const cuuint64_t*>(dims),
                  reinterpret_cast<const cuuint64_t*>(strides_bytes),
                  reinterpret_cast<const cuuint32_t*>(box), estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
}

}  // namespace misa

using namespace misa;

namespace {

int pool_impl(const KeyArg& key, int64_t n_k, int d, int B, int64_t m0, int64_t m1, float* kbar,
              uint16_t* kbar_hl, void* stream) {
  if (n_k < 1 || !good_d(d) || B < 1 || B > 4096) return MISA_ERR_INVALID_ARG;
  if (const int st = check_keys(key, n_k)) return st;
  if (!kbar && !kbar_hl) return MISA_ERR_INVALID_ARG;
  if ((kbar && !aligned4(kbar)) || (kbar_hl && (reinterpret_cast<uintptr_t>(kbar_hl) & 1u)))
    return MISA_ERR_INVALID_ARG;
  const int64_t M = (n_k + B - 1) / B;
  if (M > 0x7fffffff || m0 < 0 || m1 < m0 || m1 > M) return MISA_ERR_INVALID_ARG;
  if (m0 == m1) return MISA_OK;
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  return cuda_status(launch_pool_keys(key.K, key.k_scale, key.kpg, key.fp8(), n_k, d, B, m0, m1,
                                      kbar, kbar_hl, ctl, as_stream(stream)));
}

}  // namespace

namespace {

int score_impl(const uint16_t* Q, const float* w, const int32_t* heads, const KeyArg& key, int n_q,
               int64_t q_pos0, int64_t n_k, int H, int d, int h, float* logits, int64_t ld,
               void* stream) {
  if (!Q || !aligned16(Q) || !w || !aligned4(w) || !logits || !aligned16(logits))
    return MISA_ERR_INVALID_ARG;
  if (heads && !aligned4(heads)) return MISA_ERR_INVALID_ARG;
  if (n_q < 0 || q_pos0 < 0 || n_k < 1 || q_pos0 + n_q > n_k || H < 1 || h < 1 || h > H ||
      ld < n_k || ld % 4 != 0)
    return MISA_ERR_INVALID_ARG;
  if (!heads && h != H) return MISA_ERR_INVALID_ARG;
  if (const int st = check_keys(key, n_k)) return st;
  if (!good_d(d) || !pow2(h) || h > 128) return MISA_ERR_UNSUPPORTED;
  if (n_q == 0) return MISA_OK;
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  ScoreLaunch a{};
  a.Q = Q;
  a.w = w;
  a.heads = heads;
  a.K = key.K;
  a.k_scale = key.k_scale;
  a.fp8 = key.fp8();
  a.kpg = key.kpg;
  a.n_q = n_q;
  a.q_pos0 = q_pos0;
  a.n_k = n_k;
  a.H = H;
  a.d = d;
  a.h = h;
  a.logits = logits;
  a.ld = ld;
  return cuda_status(launch_score(a, ctl, as_stream(stream)));
}

}  // namespace

namespace {

int rerank_impl(const uint16_t* Q, const float* w, const KeyArg& key, const int32_t* cand, int kp,
                int n_q, int64_t q_pos0, int64_t n_k, int H, int d, int k, int32_t* idx,
                float* full_logits, void* ws, size_t ws_bytes, void* stream) {
  if (!Q || !aligned16(Q) || !w || !aligned4(w) || !cand || !aligned4(cand) ||
      (k > 0 && (!idx || !aligned4(idx))))
    return MISA_ERR_INVALID_ARG;
  if (full_logits && !aligned4(full_logits)) return MISA_ERR_INVALID_ARG;
  if (n_q < 0 || q_pos0 < 0 || n_k < 1 || q_pos0 + n_q > n_k || kp < 1 || kp > 16384 || k < 0 ||
      k > kp || H < 1)
    return MISA_ERR_INVALID_ARG;
  if (const int st = check_keys(key, n_k)) return st;
  if (!good_d(d) || H > 128) return MISA_ERR_UNSUPPORTED;
  if (n_q == 0) return MISA_OK;
  float* full = full_logits;
  if (!full) {
    const size_t need = misa_workspace_size("rerank", n_q, n_k, k, kp);
    if (!ws || ws_bytes < need || !aligned16(ws)) return MISA_ERR_WORKSPACE;
    full = static_cast<float*>(ws);
  }
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  const cudaStream_t s = as_stream(stream);
  cudaError_t e = launch_rerank_scores(Q, w, key.K, key.k_scale, key.kpg, key.fp8(), cand, kp, n_q,
                                       q_pos0, n_k, H, d, full, kp, ctl, s);
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  if (k == 0) return MISA_OK;
  return cuda_status(launch_select_candidates(full, kp, cand, kp, n_q, q_pos0, n_k, k, idx, ctl, s));
}

}  // namespace

namespace {

int score_topk_impl(const uint16_t* Q, const float* w, const int32_t* heads, const KeyArg& key,
                    int n_q, int64_t q_pos0, int64_t n_k, int H, int d, int h, int k, int32_t* idx,
                    float* logits, int64_t ld, void* ws, size_t ws_bytes, void* stream) {
  if (!Q || !aligned16(Q) || !w || !aligned4(w) || !logits || !aligned16(logits) ||
      (k > 0 && (!idx || !aligned4(idx))))
    return MISA_ERR_INVALID_ARG;
  if (heads && !aligned4(heads)) return MISA_ERR_INVALID_ARG;
  if (n_q < 0 || q_pos0 < 0 || n_k < 1 || q_pos0 + n_q > n_k || H < 1 || h < 1 || h > H ||
      ld < n_k || ld % 4 != 0 || k < 0 || k > 16384)
    return MISA_ERR_INVALID_ARG;
  if (!heads && h != H) return MISA_ERR_INVALID_ARG;
  if (const int st = check_keys(key, n_k, true)) return st;
  if (!good_d(d) || !pow2(h) || h > 128) return MISA_ERR_UNSUPPORTED;
  if (n_q == 0 || k == 0) return MISA_OK;
  const size_t need = misa_workspace_size("score_topk", n_q, n_k, k, 0);
  if (need > 0 && (!ws || ws_bytes < need || !aligned16(ws))) return MISA_ERR_WORKSPACE;
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  const cudaStream_t s = as_stream(stream);
  const bool fp8 = key.fp8();                               // e4m3 codes
  const bool decoded = key.kdtype == MISA_K_BF16_SCALED;     // bf16 codes + scales
  ScoreLaunch a{};
  a.Q = Q;
  a.w = w;
  a.heads = heads;
  a.K = key.K;
  a.k_scale = key.k_scale;
  a.fp8 = fp8 || decoded;  // a per-key scale in the epilogue
  a.k_bf16 = decoded;
  a.kpg = key.kpg;
  a.n_q = n_q;
  a.q_pos0 = q_pos0;
  a.n_k = n_k;
  a.H = H;
  a.d = d;
  a.h = h;
  a.logits = logits;
  a.ld = ld;
  const bool fused = need > 0 && q_pos0 + 1 >= kSampleKeys && score_select_supported(h);
  if (!fused) {  // unfused: every logit, then the selection
    cudaError_t e = launch_score(a, ctl, s);
    if (e != cudaSuccess) return MISA_ERR_CUDA;
    return cuda_status(launch_topk(logits, ld, n_q, q_pos0, n_k, k, idx, ctl, s));
  }
  const FusedLayout L(n_q, n_k);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* gate = reinterpret_cast<int*>(base + L.gate);
  float* tau = reinterpret_cast<float*>(base + L.tau);
  void* Ks = base + L.ks;
  float* ks_scale = reinterpret_cast<float*>(base + L.ks_scale);
  float* sample = reinterpret_cast<float*>(base + L.sample);
  uint32_t* mask = reinterpret_cast<uint32_t*>(base + L.mask);
  const int64_t mld = mask_words(n_k);
  cudaError_t e;
  {
    StageMark m(0, s);
    if (fp8) {
      // decode the keys once, in logical order (with their scales when paged);
      // every scoring pass then reads contiguous bf16 codes
      uint16_t* kbf = reinterpret_cast<uint16_t*>(base + L.kbf);
      float* kbf_scale = key.kpg.paged() ? reinterpret_cast<float*>(base + L.kbf_scale) : nullptr;
      e = launch_e4m3_rows_to_bf16(static_cast<const uint8_t*>(key.K), key.k_scale, key.kpg, n_k, d,
                                   kbf, kbf_scale, ctl, s);
      if (e != cudaSuccess) return MISA_ERR_CUDA;
      a.K = kbf;
      a.k_bf16 = true;
      if (kbf_scale) a.k_scale = kbf_scale;
      a.kpg = KeyPages{nullptr, 0, 0};
    }
    e = launch_gather_sample(a.K, a.fp8 ? a.k_scale : nullptr, a.kpg, 2 * d, q_pos0 + 1,
                             kSampleBlocks, Ks, a.fp8 ? ks_scale : nullptr, ctl, s);
  }
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  ScoreLaunch sa = a;  // the sample: every sampled key is visible to every query
  sa.K = Ks;
  sa.k_scale = a.fp8 ? ks_scale : nullptr;
  sa.kpg = KeyPages{nullptr, 0, 0};
  sa.q_pos0 = kSampleKeys - 1;
  sa.n_k = kSampleKeys;
  sa.logits = sample;
  sa.ld = kSampleKeys;
  {
    StageMark m(1, s);
    e = launch_score(sa, ctl, s);
  }
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  {
    StageMark m(2, s);
    e = launch_fused_tau(sample, kSampleKeys, kSampleKeys, n_q, q_pos0, n_k, k, tau, gate, s);
  }
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  ScoreLaunch se = a;  // select mode
  se.tau = tau;
  se.mask = mask;
  se.mask_ld = mld;
  {
    StageMark m(3, s);
    e = launch_score(se, ctl, s);
  }
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  {
    StageMark m(4, s);
    e = launch_fused_finish(logits, ld, mask, mld, n_q, q_pos0, n_k, k, idx, gate, s);
  }
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  // exact fallback for the rows the thresholds missed (a no-op launch when none)
  ScoreLaunch ra = a;
  ra.gate = gate;
  {
    StageMark m(5, s);
    e = launch_score(ra, ctl, s);
  }
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  StageMark m(6, s);
  return cuda_status(launch_topk(logits, ld, n_q, q_pos0, n_k, k, idx, ctl, s, gate));
}

}  // namespace

extern "C" {

int misa_pool_keys_range(const void* K, const float* k_scale, int kdtype, int64_t n_k, int d,
                         int B, int64_t m0, int64_t m1, float* kbar, uint16_t* kbar_hl,
                         void* stream) {
  return pool_impl(contiguous_keys(K, k_scale, kdtype), n_k, d, B, m0, m1, kbar, kbar_hl, stream);
}

int misa_pool_keys(const void* K, const float* k_scale, int kdtype, int64_t n_k, int d, int B,
                   float* kbar, uint16_t* kbar_hl, void* stream) {
  if (B < 1) return MISA_ERR_INVALID_ARG;
  return misa_pool_keys_range(K, k_scale, kdtype, n_k, d, B, 0, (n_k + B - 1) / B, kbar, kbar_hl,
                              stream);
}

int misa_pool_keys_paged(const void* pages, const float* k_scale, int kdtype,
                         const int32_t* block_table, int page_size, int64_t n_pages, int64_t n_k,
                         int d, int B, int64_t m0, int64_t m1, float* kbar, uint16_t* kbar_hl,
                         void* stream) {
  if (!block_table) return MISA_ERR_INVALID_ARG;
  return pool_impl(paged_keys(pages, k_scale, kdtype, block_table, page_size, n_pages), n_k, d, B,
                   m0, m1, kbar, kbar_hl, stream);
}

int misa_route_heads(const uint16_t* Q, const float* w, const uint16_t* kbar_hl, int n_q,
                     int64_t q_pos0, int64_t n_k, int H, int d, int B, int h, int32_t* heads,
                     float* r_out, void* stream) {
  if (!Q || !aligned16(Q) || !w || !aligned4(w) || !kbar_hl || !aligned16(kbar_hl) || !heads ||
      !aligned4(heads))
    return MISA_ERR_INVALID_ARG;
  if (r_out && !aligned4(r_out)) return MISA_ERR_INVALID_ARG;
  if (n_q < 0 || q_pos0 < 0 || n_k < 1 || q_pos0 + n_q > n_k || B < 1 || h < 1 || h > H)
    return MISA_ERR_INVALID_ARG;
  if (!good_d(d) || !pow2(H) || H > 128) return MISA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(n_q) * H > 0x7fffffffLL) return MISA_ERR_INVALID_ARG;
  if (n_q == 0) return MISA_OK;
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  return cuda_status(launch_route_heads(Q, w, kbar_hl, n_q, q_pos0, n_k, H, d, B, h, heads, r_out,
                                        ctl, as_stream(stream)));
}

int misa_score_tokens(const uint16_t* Q, const float* w, const int32_t* heads, const void* K,
                      const float* k_scale, int kdtype, int n_q, int64_t q_pos0, int64_t n_k, int H,
                      int d, int h, float* logits, int64_t ld, void* stream) {
  return score_impl(Q, w, heads, contiguous_keys(K, k_scale, kdtype), n_q, q_pos0, n_k, H, d, h,
                    logits, ld, stream);
}

int misa_score_tokens_paged(const uint16_t* Q, const float* w, const int32_t* heads,
                            const void* pages, const float* k_scale, int kdtype,
                            const int32_t* block_table, int page_size, int64_t n_pages, int n_q,
                            int64_t q_pos0, int64_t n_k, int H, int d, int h, float* logits,
                            int64_t ld, void* stream) {
  if (!block_table) return MISA_ERR_INVALID_ARG;
  return score_impl(Q, w, heads, paged_keys(pages, k_scale, kdtype, block_table, page_size, n_pages),
                    n_q, q_pos0, n_k, H, d, h, logits, ld, stream);
}

int misa_score_tokens_fp8(const uint8_t* Q8, const float* q_scale, const float* w,
                          const int32_t* heads, const uint8_t* K8, const float* k_scale, int n_q,
                          int64_t q_pos0, int64_t n_k, int H, int d, int h, float* logits,
                          int64_t ld, void* stream) {
  if (!Q8 || !aligned16(Q8) || !q_scale || !aligned4(q_scale) || !w || !aligned4(w) || !K8 ||
      !aligned16(K8) || !k_scale || !aligned4(k_scale) || !logits || !aligned16(logits))
    return MISA_ERR_INVALID_ARG;
  if (heads && !aligned4(heads)) return MISA_ERR_INVALID_ARG;
  if (n_q < 0 || q_pos0 < 0 || n_k < 1 || q_pos0 + n_q > n_k || H < 1 || h < 1 || h > H ||
      ld < n_k || ld % 4 != 0)
    return MISA_ERR_INVALID_ARG;
  if (!heads && h != H) return MISA_ERR_INVALID_ARG;
  if ((d != 64 && d != 128) || !pow2(h) || h > 128) return MISA_ERR_UNSUPPORTED;
  if (n_k > 0x7fffffffLL) return MISA_ERR_INVALID_ARG;
  if (n_q == 0) return MISA_OK;
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  ScoreLaunch a{};
  a.Q = reinterpret_cast<const uint16_t*>(Q8);
  a.q8 = true;
  a.q_scale = q_scale;
  a.w = w;
  a.heads = heads;
  a.K = K8;
  a.k_scale = k_scale;
  a.fp8 = true;
  a.n_q = n_q;
  a.q_pos0 = q_pos0;
  a.n_k = n_k;
  a.H = H;
  a.d = d;
  a.h = h;
  a.logits = logits;
  a.ld = ld;
  return cuda_status(launch_score(a, ctl, as_stream(stream)));
}

int misa_topk(const float* logits, int64_t ld, int n_q, int64_t q_pos0, int64_t n_k, int k,
              int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  (void)ws;
  (void)ws_bytes;
  if (!logits || !aligned4(logits) || (k > 0 && (!idx || !aligned4(idx)))) return MISA_ERR_INVALID_ARG;
  if (n_q < 0 || q_pos0 < 0 || n_k < 1 || q_pos0 + n_q > n_k || k < 0 || k > 16384)
    return MISA_ERR_INVALID_ARG;
  if (ld < std::min<int64_t>(n_k, q_pos0 + n_q)) return MISA_ERR_INVALID_ARG;
  if (n_k > 0x7fffffffLL) return MISA_ERR_INVALID_ARG;
  if (n_q == 0 || k == 0) return MISA_OK;
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  return cuda_status(
      launch_topk(logits, ld, n_q, q_pos0, n_k, k, idx, ctl, as_stream(stream)));
}

int misa_rerank(const uint16_t* Q, const float* w, const void* K, const float* k_scale, int kdtype,
                const int32_t* cand, int kp, int n_q, int64_t q_pos0, int64_t n_k, int H, int d,
                int k, int32_t* idx, float* full_logits, void* ws, size_t ws_bytes, void* stream) {
  return rerank_impl(Q, w, contiguous_keys(K, k_scale, kdtype), cand, kp, n_q, q_pos0, n_k, H, d, k,
                     idx, full_logits, ws, ws_bytes, stream);
}

int misa_rerank_paged(const uint16_t* Q, const float* w, const void* pages, const float* k_scale,
                      int kdtype, const int32_t* block_table, int page_size, int64_t n_pages,
                      const int32_t* cand, int kp, int n_q, int64_t q_pos0, int64_t n_k, int H,
                      int d, int k, int32_t* idx, float* full_logits, void* ws, size_t ws_bytes,
                      void* stream) {
  if (!block_table) return MISA_ERR_INVALID_ARG;
  return rerank_impl(Q, w, paged_keys(pages, k_scale, kdtype, block_table, page_size, n_pages), cand,
                     kp, n_q, q_pos0, n_k, H, d, k, idx, full_logits, ws, ws_bytes, stream);
}

int misa_score_topk(const uint16_t* Q, const float* w, const int32_t* heads, const void* K,
                    const float* k_scale, int kdtype, int n_q, int64_t q_pos0, int64_t n_k, int H,
                    int d, int h, int k, int32_t* idx, float* logits, int64_t ld, void* ws,
                    size_t ws_bytes, void* stream) {
  return score_topk_impl(Q, w, heads, contiguous_keys(K, k_scale, kdtype), n_q, q_pos0, n_k, H, d,
                         h, k, idx, logits, ld, ws, ws_bytes, stream);
}

int misa_keys_e4m3_to_bf16(const uint8_t* K8, int64_t n_k, int d, uint16_t* Kbf, void* stream) {
  if (!K8 || !aligned16(K8) || !Kbf || !aligned16(Kbf) || n_k < 0 || n_k > 0x7fffffffLL)
    return MISA_ERR_INVALID_ARG;
  if (!good_d(d)) return MISA_ERR_UNSUPPORTED;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(K8), a1 = a0 + static_cast<uintptr_t>(n_k) * d;
  const uintptr_t b0 = reinterpret_cast<uintptr_t>(Kbf), b1 = b0 + static_cast<uintptr_t>(n_k) * d * 2;
  if (n_k > 0 && a0 < b1 && b0 < a1) return MISA_ERR_INVALID_ARG;  // overlapping buffers
  // n_k * d is a multiple of 16 (d is): whole 16-code units
  return cuda_status(launch_e4m3_to_bf16(K8, Kbf, n_k * d, as_stream(stream)));
}

int misa_score_topk_paged(const uint16_t* Q, const float* w, const int32_t* heads,
                          const void* pages, const float* k_scale, int kdtype,
                          const int32_t* block_table, int page_size, int64_t n_pages, int n_q,
                          int64_t q_pos0, int64_t n_k, int H, int d, int h, int k, int32_t* idx,
                          float* logits, int64_t ld, void* ws, size_t ws_bytes, void* stream) {
  if (!block_table) return MISA_ERR_INVALID_ARG;
  return score_topk_impl(Q, w, heads,
                         paged_keys(pages, k_scale, kdtype, block_table, page_size, n_pages), n_q,
                         q_pos0, n_k, H, d, h, k, idx, logits, ld, ws, ws_bytes, stream);
}

int misa_decode_pool_keys(const void* pages, const float* k_scale, int kdtype,
                          const int32_t* block_tables, int max_blocks, int page_size,
                          int64_t n_pages, const int32_t* seq_lens, int n_seq, int d, int B,
                          int64_t M_max, int64_t n_last, float* kbar, uint16_t* kbar_hl,
                          void* stream) {
  const KeyArg key = paged_keys(pages, k_scale, kdtype, block_tables, page_size, n_pages);
  if (!block_tables || !seq_lens || !aligned4(seq_lens) || n_seq < 0 || n_seq > 65535 ||
      max_blocks < 1 || !good_d(d) || B < 1 || B > 4096 || n_last < 0 || n_last > 0x7fffffffLL)
    return MISA_ERR_INVALID_ARG;
  const int64_t max_len = static_cast<int64_t>(max_blocks) * page_size;
  if (const int st = check_keys(key, max_len)) return st;
  if (M_max < (max_len + B - 1) / B || M_max > 0x7fffffffLL) return MISA_ERR_INVALID_ARG;
  if (!kbar && !kbar_hl) return MISA_ERR_INVALID_ARG;
  if ((kbar && !aligned4(kbar)) || (kbar_hl && (reinterpret_cast<uintptr_t>(kbar_hl) & 1u)))
    return MISA_ERR_INVALID_ARG;
  if (n_seq == 0 || n_last == 0) return MISA_OK;
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  return cuda_status(launch_pool_keys_batch(pages, k_scale, key.fp8(), block_tables, max_blocks,
                                            key.kpg.page_shift, n_pages, seq_lens, n_seq, d, B,
                                            M_max, std::min<int64_t>(n_last, M_max), kbar, kbar_hl,
                                            ctl, as_stream(stream)));
}

int misa_decode_route_heads(const uint16_t* Q, const float* w, const uint16_t* kbar_hl,
                            int64_t M_max, const int32_t* seq_lens, int n_seq, int H, int d, int B,
                            int h, int32_t* heads, float* r_out, void* stream) {
  if (!Q || !aligned16(Q) || !w || !aligned4(w) || !kbar_hl || !aligned16(kbar_hl) || !heads ||
      !aligned4(heads) || !seq_lens || !aligned4(seq_lens))
    return MISA_ERR_INVALID_ARG;
  if (r_out && !aligned4(r_out)) return MISA_ERR_INVALID_ARG;
  if (n_seq < 0 || M_max < 1 || M_max > 0x7fffffffLL || B < 1 || h < 1 || h > H)
    return MISA_ERR_INVALID_ARG;
  if (!good_d(d) || !pow2(H) || H > 128) return MISA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(n_seq) * H > 0x7fffffffLL) return MISA_ERR_INVALID_ARG;
  if (n_seq == 0) return MISA_OK;
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  return cuda_status(launch_route_heads_decode(Q, w, kbar_hl, M_max, seq_lens, n_seq, H, d, B, h,
                                               heads, r_out, ctl, as_stream(stream)));
}

int misa_decode_score_topk(const uint16_t* Q, const float* w, const int32_t* heads,
                           const void* pages, const float* k_scale, int kdtype,
                           const int32_t* block_tables, int max_blocks, int page_size,
                           int64_t n_pages, const int32_t* seq_lens, int n_seq, int H, int d,
                           int h, int k, int32_t* idx, float* logits, int64_t ld, void* stream) {
  const KeyArg key = paged_keys(pages, k_scale, kdtype, block_tables, page_size, n_pages);
  if (!Q || !aligned16(Q) || !w || !aligned4(w) || !block_tables || !seq_lens ||
      !aligned4(seq_lens) || !logits || !aligned4(logits) || (k > 0 && (!idx || !aligned4(idx))))
    return MISA_ERR_INVALID_ARG;
  if (heads && !aligned4(heads)) return MISA_ERR_INVALID_ARG;
  if (n_seq < 0 || max_blocks < 1 || H < 1 || h < 1 || h > H || k < 0 || k > 16384)
    return MISA_ERR_INVALID_ARG;
  if (!heads && h != H) return MISA_ERR_INVALID_ARG;
  const int64_t max_len = static_cast<int64_t>(max_blocks) * page_size;
  if (const int st = check_keys(key, max_len)) return st;
  if (ld < max_len) return MISA_ERR_INVALID_ARG;
  if (!good_d(d) || !pow2(h) || h > 64) return MISA_ERR_UNSUPPORTED;
  if (n_seq == 0) return MISA_OK;
  DevCtl ctl;
  if (!make_ctl(ctl)) return MISA_ERR_CUDA;
  const cudaStream_t s = as_stream(stream);
  cudaError_t e = launch_decode_score(Q, w, heads, pages, k_scale, key.fp8(), block_tables,
                                      max_blocks, key.kpg.page_shift, n_pages, seq_lens, n_seq, H, d,
                                      h, logits, ld, ctl, s);
  if (e != cudaSuccess) return MISA_ERR_CUDA;
  if (k == 0) return MISA_OK;
  return cuda_status(launch_topk(logits, ld, n_seq, 0, max_len, k, idx, ctl, s, nullptr, seq_lens));
}

int misa_profile_start(void) {
  std::lock_guard<std::mutex> lk(g_prof.mu);
  for (int i = 0; i < kStages; ++i) {
    for (cudaEvent_t e : g_prof.start[i]) cudaEventDestroy(e);
    for (cudaEvent_t e : g_prof.stop[i]) cudaEventDestroy(e);
    g_prof.start[i].clear();
    g_prof.stop[i].clear();
  }
  g_prof.on.store(true);
  return MISA_OK;
}

int misa_profile_stop(double* ms, int* counts, int n) {
  g_prof.on.store(false);
  std::lock_guard<std::mutex> lk(g_prof.mu);
  int status = MISA_OK;
  for (int i = 0; i < kStages; ++i) {
    double sum = 0.0;
    for (size_t j = 0; j < g_prof.start[i].size(); ++j) {
      float t = 0.0f;
      if (cudaEventSynchronize(g_prof.stop[i][j]) != cudaSuccess ||
          cudaEventElapsedTime(&t, g_prof.start[i][j], g_prof.stop[i][j]) != cudaSuccess)
        status = MISA_ERR_CUDA;
      sum += t;
      cudaEventDestroy(g_prof.start[i][j]);
      cudaEventDestroy(g_prof.stop[i][j]);
    }
    if (i < n) {
      if (ms) ms[i] = sum;
      if (counts) counts[i] = static_cast<int>(g_prof.start[i].size());
    }
    g_prof.start[i].clear();
    g_prof.stop[i].clear();
  }
  return status;
}

const char* misa_profile_stage_name(int i) {
  return (i >= 0 && i < kStages) ? kStageNames[i] : nullptr;
}

size_t misa_workspace_size(const char* op, int n_q, int64_t n_k, int k, int kp) {
  if (!op || n_q <= 0) return 0;
  if (std::strcmp(op, "rerank") == 0 && kp > 0)
    return static_cast<size_t>(n_q) * static_cast<size_t>(kp) * sizeof(float);
  if (std::strcmp(op, "score_topk") == 0) {
    // fused only where the sample lies inside every row's prefix and the
    // position bitmap fits; 0 selects the unfused sequence
    if (k <= 0 || k > kFusedMaxK || n_k > kFusedMaxKeys || n_k < kSampleKeys) return 0;
    return FusedLayout(n_q, n_k).total;
  }
  return 0;
}

const char* misa_status_string(int status) {
  switch (status) {
    case MISA_OK: return "ok";
    case MISA_ERR_INVALID_ARG: return "invalid argument";
    case MISA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MISA_ERR_CUDA: return "CUDA error";
    case MISA_ERR_TIMEOUT: return "device wait timed out";
    case MISA_ERR_WORKSPACE: return "workspace missing or too small";
    case MISA_ERR_DEVICE: return "device detected an input outside its contract";
  }
  return "unknown status";
}

int misa_last_device_status(void* stream) {
  if (cudaStreamSynchronize(as_stream(stream)) != cudaSuccess) return MISA_ERR_CUDA;
  int* p = status_ptr();
  if (!p) return MISA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MISA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(p, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return MISA_ERR_CUDA;
  switch (v) {
    case DEV_OK: return MISA_OK;
    case DEV_TIMEOUT: return MISA_ERR_TIMEOUT;
    default: return MISA_ERR_DEVICE;
  }
}

int misa_set_wait_limit_ns(uint64_t ns) {
  g_wait_ns.store(ns ? ns : 2000000000ull);
  return MISA_OK;
}

}  // extern "C"
