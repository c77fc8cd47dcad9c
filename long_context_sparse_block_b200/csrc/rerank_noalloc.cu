// misa_rerank_noalloc: the MISA-dagger fine stage for callers that cannot
// allocate device memory.
//
// misa_rerank needs n_q * kp floats of scratch for the all-head candidate
// scores (unless the caller asks for them in full_logits), and takes that
// scratch as caller workspace.  Some callers cannot provide it: code running
// under a memory pool or allocator it does not own (an inference server whose
// pool is fixed at start-up, a framework's graph-capture region where
// cudaMalloc is forbidden), or a plain C host that has no device allocator at
// hand.  For them this entry point keeps its scratch in a file-scope device
// array of fixed size, so it allocates nothing at all.
//
// Limits and sharing:
//   * at most kNoAllocMaxScores (4,194,304 = 16 MiB of fp32) candidate scores
//     per call, i.e. n_q * kp <= 4,194,304; larger calls are rejected with
//     MISA_ERR_WORKSPACE before any launch (split the queries into chunks);
//   * every GPU that loads the library holds the 16 MiB array until exit;
//   * all calls on a device share the array: calls whose work overlaps on the
//     GPU (different streams, no ordering between them) race on it;
//   * each call writes every score it reads, so nothing needs clearing between
//     calls; the array keeps the last call's scores.
//   * the first call on each device looks up the array's device address with
//     cudaGetSymbolAddress (a runtime call), so make that first call outside
//     any stream capture.
#include <mutex>

#include "internal.h"
#include "misa.h"

namespace misa {
namespace {

constexpr int64_t kNoAllocMaxScores = 4194304;  // fp32 scores (16 MiB)

static __device__ __align__(256) float g_rerank_scratch[kNoAllocMaxScores];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of this device's scratch array (looked up once per device,
// with that device current).
float* scratch_for_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_scratch_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_rerank_scratch) != cudaSuccess || !p) return nullptr;
    g_scratch_ptr[dev] = static_cast<float*>(p);
  }
  return g_scratch_ptr[dev];
}

}  // namespace
}  // namespace misa

extern "C" int misa_rerank_noalloc(const uint16_t* Q, const float* w, const void* K,
                                   const float* k_scale, int kdtype, const int32_t* cand, int kp,
                                   int n_q, int64_t q_pos0, int64_t n_k, int H, int d, int k,
                                   int32_t* idx, void* stream) {
  using namespace misa;
  const auto a16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
  const auto a4 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; };
  if (!Q || !a16(Q) || !w || !a4(w) || !K || !a16(K) || !cand || !a4(cand) ||
      (k > 0 && (!idx || !a4(idx))))
    return MISA_ERR_INVALID_ARG;
  if (n_q < 0 || q_pos0 < 0 || n_k < 1 || q_pos0 + n_q > n_k || kp < 1 || kp > 16384 || k < 0 ||
      k > kp || H < 1)
    return MISA_ERR_INVALID_ARG;
  if (kdtype != MISA_K_BF16 && kdtype != MISA_K_FP8E4M3) return MISA_ERR_INVALID_ARG;
  if (kdtype == MISA_K_FP8E4M3 && (!k_scale || !a4(k_scale))) return MISA_ERR_INVALID_ARG;
  if (!(d == 32 || d == 64 || d == 128) || H > 128) return MISA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(n_q) * kp > kNoAllocMaxScores) return MISA_ERR_WORKSPACE;
  if (n_q == 0) return MISA_OK;
  float* scratch = scratch_for_current_device();
  if (!scratch) return MISA_ERR_CUDA;
  // the library's per-device status word (the one misa_last_device_status reads)
  int* status = device_status_word();
  if (!status) return MISA_ERR_CUDA;
  DevCtl ctl{status, wait_limit_ns()};
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_rerank_scores(Q, w, K, k_scale, KeyPages{nullptr, 0, 0}, kdtype == MISA_K_FP8E4M3,
                           cand, kp, n_q, q_pos0, n_k, H, d, scratch, kp, ctl, s) != cudaSuccess)
    return MISA_ERR_CUDA;
  if (k == 0) return MISA_OK;
  return launch_select_candidates(scratch, kp, cand, kp, n_q, q_pos0, n_k, k, idx, ctl, s) ==
                     cudaSuccess
             ? MISA_OK
             : MISA_ERR_CUDA;
}
