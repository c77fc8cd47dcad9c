// Launchers the C ABI layer (api.cu) calls; each lives beside its kernel.
// Arguments are validated by the caller; launchers only pick configurations.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace misa {

int sm_count();  // of the current device

// The current device's status word and the bounded-wait budget (api.cu).
int* device_status_word();
unsigned long long wait_limit_ns();

// Pools blocks m0 <= m < min(m1, ceil(n_k / B)) of a contiguous or paged key
// cache (pool.cu).
cudaError_t launch_pool_keys(const void* K, const float* k_scale, const KeyPages& kpg, bool fp8,
                             int64_t n_k, int d, int B, int64_t m0, int64_t m1, float* kbar,
                             uint16_t* kbar_hl, const DevCtl& ctl, cudaStream_t s);

cudaError_t launch_route_heads(const uint16_t* Q, const float* w, const uint16_t* kbar_hl,
                               int n_q, int64_t q_pos0, int64_t n_k, int H, int d, int B, int h,
                               int32_t* heads, float* r_out, const DevCtl& ctl, cudaStream_t s);

// Decode (route.cu, pool.cu, decode.cu): n_seq sequences, one query each at the
// last of its lens[b] keys, keys in paged caches (block_tables [n_seq,
// max_blocks]), pooled keys per sequence in kbar_hl [n_seq, 2, M_max, d].
cudaError_t launch_route_heads_decode(const uint16_t* Q, const float* w, const uint16_t* kbar_hl,
                                      int64_t M_max, const int32_t* lens, int n_seq, int H, int d,
                                      int B, int h, int32_t* heads, float* r_out, const DevCtl& ctl,
                                      cudaStream_t s);
// Pools blocks M_b - n_last .. M_b - 1 of every sequence (M_b = ceil(lens[b] / B)).
cudaError_t launch_pool_keys_batch(const void* pages, const float* k_scale, bool fp8,
                                   const int32_t* block_tables, int max_blocks, int page_shift,
                                   int64_t n_pages, const int32_t* lens, int n_seq, int d, int B,
                                   int64_t M_max, int64_t n_last, float* kbar, uint16_t* kbar_hl,
                                   const DevCtl& ctl, cudaStream_t s);
// logits[b, s] for s < lens[b] (bf16 pages, or e4m3 pages with per-row scales).
cudaError_t launch_decode_score(const uint16_t* Q, const float* w, const int32_t* heads,
                                const void* pages, const float* k_scale, bool fp8,
                                const int32_t* block_tables, int max_blocks, int page_shift,
                                int64_t n_pages, const int32_t* lens, int n_seq, int H, int d, int h,
                                float* logits, int64_t ld, const DevCtl& ctl, cudaStream_t s);

// Score kernel launch description: store mode writes fused logits (logits,
// ld); select mode (tau != nullptr) keeps logits >= tau[t] in per-row
// candidate lists instead.  gate (nullable): do nothing unless *gate != 0.
struct ScoreLaunch {
  const uint16_t* Q;
  const float* w;
  const int32_t* heads;
  const void* K;
  const float* k_scale;
  bool fp8;
  bool k_bf16;            // FP8 keys given already decoded to bf16 codes at K
  int n_q;
  int64_t q_pos0;
  int64_t n_k;
  int H;
  int d;
  int h;
  float* logits;
  int64_t ld;
  const float* tau;       // select mode: per-row thresholds (else nullptr)
  uint32_t* mask;         // select mode: [n_q][mask_ld] pass bits
  int64_t mask_ld;
  const int* gate;        // nullable: launch does nothing unless *gate != 0
  bool q8;                // Q holds e4m3 codes ([n_q, H, d] bytes) with q_scale [n_q, H]
  const float* q_scale;
  KeyPages kpg;           // key rows through a block table (kpg.bt != nullptr)
};
cudaError_t launch_score(const ScoreLaunch& a, const DevCtl& ctl, cudaStream_t s);
bool score_select_supported(int h);

// Top-k over token rows: row t is vals[t*ld ..] with min(pos(t)+1, n_k)
// visible entries (min(row_len[t], n_k) when row_len is given); writes token
// indices.
cudaError_t launch_topk(const float* vals, int64_t ld, int n_q, int64_t q_pos0, int64_t n_k,
                        int k, int32_t* idx, const DevCtl& ctl, cudaStream_t s,
                        const int* gate = nullptr, const int32_t* row_len = nullptr);

// Top-k over candidate rows: row t holds the scores vals[t*ldv + i] of tokens
// cand[t*kp + i] (absent: token outside 0..pos(t), or -inf); ties to the lower
// token; tokens written ascending whatever the candidate order (kp <= 16384).
cudaError_t launch_select_candidates(const float* vals, int64_t ldv, const int32_t* cand, int kp,
                                     int n_q, int64_t q_pos0, int64_t n_k, int k, int32_t* idx,
                                     const DevCtl& ctl, cudaStream_t s);

// Exact decode of FP8 E4M3 key codes to bf16 codes (pool.cu); n multiple of 16.
cudaError_t launch_e4m3_to_bf16(const uint8_t* src, uint16_t* dst, int64_t n, cudaStream_t s);
// The same for the logical rows 0..n_k-1 of a paged or contiguous e4m3 cache,
// written in logical order, their scales gathered into dst_scale (nullable).
cudaError_t launch_e4m3_rows_to_bf16(const uint8_t* src, const float* scale, const KeyPages& kpg,
                                     int64_t n_k, int d, uint16_t* dst, float* dst_scale,
                                     const DevCtl& ctl, cudaStream_t s);

// Fused top-k helpers (topk.cu): sample gather, per-row thresholds from the
// scored sample, and the exact selection over the select-mode candidates.
cudaError_t launch_gather_sample(const void* K, const float* k_scale, const KeyPages& kpg,
                                 int row_bytes, int64_t span, int n_blocks, void* Ks,
                                 float* ks_scale, const DevCtl& ctl, cudaStream_t s);
cudaError_t launch_fused_tau(const float* sample, int64_t lds, int n_s, int n_q, int64_t q_pos0,
                             int64_t n_k, int k, float* tau, int* gate, cudaStream_t s);
cudaError_t launch_fused_finish(const float* logits, int64_t ld, const uint32_t* mask,
                                int64_t mask_ld, int n_q, int64_t q_pos0, int64_t n_k, int k,
                                int32_t* idx, int* gate, cudaStream_t s);

// All-head scores of candidate keys: full[t*ldf + i] (-inf where ignored).
cudaError_t launch_rerank_scores(const uint16_t* Q, const float* w, const void* K,
                                 const float* k_scale, const KeyPages& kpg, bool fp8,
                                 const int32_t* cand, int kp, int n_q, int64_t q_pos0, int64_t n_k,
                                 int H, int d, float* full, int64_t ldf, const DevCtl& ctl,
                                 cudaStream_t s);

// Driver entry point for cuTensorMapEncodeTiled (resolved once).
CUresult encode_tensor_map(CUtensorMap* map, CUtensorMapDataType dtype, int rank,
                           const void* base, const uint64_t* dims, const uint64_t* strides_bytes,
                           const uint32_t* box, CUtensorMapSwizzle swz);

}  // namespace misa
