/*
 * misa.h — C ABI of the MISA token indexer library (libmisa.so, sm_100a).
 *
 * MISA ("MISA: Mixture of Indexer Sparse Attention for Long-Context LLM
 * Inference") replaces the DeepSeek-Sparse-Attention lightning indexer.  Per
 * query it (1) mean-pools the shared index keys into M = ceil(L/B) block keys,
 * (2-3) routes: scores every indexer head against the pooled keys and keeps the
 * top-h heads, (4) lets only those heads score the causal prefix token by token,
 * and (5) keeps the top-k tokens.  The hierarchical variant (MISA-dagger) keeps a
 * larger routed candidate set and re-scores it with all heads.  (Technical
 * summary, Metodologia steps 1-2 and Variante Hierarquica; abstract.)
 *
 * Shapes and layouts (all row-major, all pointers are DEVICE pointers owned by
 * the caller unless stated otherwise):
 *   Q       [n_q, H, d]  bf16 (uint16 codes)  index queries, H = H_I heads
 *   Q8      [n_q, H, d]  FP8 E4M3 codes with q_scale [n_q, H] fp32 (the FP8
 *                        scoring call only; value = e4m3(code) * q_scale[t, j])
 *   K       [n_k, d]     bf16 codes, or FP8 E4M3 codes with k_scale [n_k] fp32
 *                        (value = e4m3(code) * k_scale[s])
 *   w       [n_q, H]     fp32 per-query head weights
 *   kbar    [M, d]       fp32 pooled block keys
 *   kbar_hl [2, M, d]    bf16: hi = bf16(kbar), lo = bf16(kbar - hi)
 *   heads   [n_q, h]     int32 routed heads, ascending head index
 *   logits  [n_q, ld]    fp32
 *   idx     [n_q, k]     int32 token indices, ascending, padded with -1
 * Query t sits at position pos(t) = q_pos0 + t and sees keys 0..pos(t); every
 * call requires q_pos0 >= 0 and q_pos0 + n_q <= n_k.  d must be 32, 64 or 128.
 *
 * Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 * stream), validates its arguments before launching anything and returns a
 * misa_status.  Argument errors launch nothing.  Device-side faults detected by
 * the kernels' own checks (a bounded wait that ran out, a value outside its
 * contract) are recorded in a per-device status word read by
 * misa_last_device_status().  No entry point allocates device memory.
 */
#ifndef MISA_H_
#define MISA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum misa_status {
    MISA_OK = 0,
    MISA_ERR_INVALID_ARG = -1,  /* null/misaligned pointer, size out of range */
    MISA_ERR_UNSUPPORTED = -2,  /* a shape the kernels do not implement (d, H, h) */
    MISA_ERR_CUDA = -3,         /* a CUDA runtime/driver call failed */
    MISA_ERR_TIMEOUT = -4,      /* a kernel's bounded wait ran out (device status) */
    MISA_ERR_WORKSPACE = -5,    /* workspace pointer/size too small */
    MISA_ERR_DEVICE = -6        /* a kernel detected an input outside its contract */
} misa_status;

typedef enum misa_kdtype {
    MISA_K_BF16 = 0,
    MISA_K_FP8E4M3 = 1,
    /* bf16 codes with a per-token fp32 scale k_scale[n_k] > 0 that multiplies
     * the dot product like the e4m3 scale: e4m3 keys decoded once by
     * misa_keys_e4m3_to_bf16 and kept with their scales.  Accepted only by
     * misa_score_topk with contiguous keys; the other calls refuse it. */
    MISA_K_BF16_SCALED = 2
} misa_kdtype;

/*
 * Stage 1 — block mean-pooling of the index keys (Metodologia step 1: keys split
 * into M = ceil(n_k/B) blocks, each summarised by its mean key).
 *   kbar[m, :] = (1/n_m) * sum_{s = mB}^{mB+n_m-1} K[s, :],  n_m = min(B, n_k - mB)
 * Sums in fp32.  Writes kbar (nullable) and kbar_hl (nullable; hi/lo bf16 split
 * used by misa_route_heads).  K: 16-byte aligned; k_scale required iff
 * kdtype == MISA_K_FP8E4M3.  1 <= B <= 4096.
 */
int misa_pool_keys(const void* K, const float* k_scale, int kdtype, int64_t n_k, int d, int B,
                   float* kbar, uint16_t* kbar_hl, void* stream);

/*
 * Stage 1 for a growing key cache (decode): misa_pool_keys restricted to blocks
 * m0 <= m < m1 of the n_k keys, M = ceil(n_k/B); every other entry of kbar and
 * kbar_hl is left as it is.  kbar_hl keeps the [2, M, d] layout of the current
 * n_k, so after appending keys: while M is unchanged only the last block needs
 * pooling again (m0 = M-1, m1 = M); when M grows, pool every block (the lo
 * plane moves).  Pooling each block is the same arithmetic whatever the range,
 * so the result equals misa_pool_keys bit for bit.  0 <= m0 <= m1 <= M (m0 == m1
 * is a no-op); other arguments as misa_pool_keys.  (Not a step of the pages'
 * method, which they evaluate on prefill only: an incremental form of stage 1.)
 */
int misa_pool_keys_range(const void* K, const float* k_scale, int kdtype, int64_t n_k, int d,
                         int B, int64_t m0, int64_t m1, float* kbar, uint16_t* kbar_hl,
                         void* stream);

/*
 * Stages 2-3 — router and top-h (Metodologia step 1: per-head affinities
 * against the pooled keys, aggregated into one importance per head; keep the
 * top-h heads).  The aggregate is
 *   r[t, j] = w[t, j] * sum_{m in C(t)} ReLU(q[t, j] . kbar_m),
 *   C(t) = { m : (m+1)B - 1 <= pos(t), m < floor(n_k/B) }  (complete causal blocks)
 * with kbar_m = hi_m + lo_m read from kbar_hl ([2, M, d], M = ceil(n_k/B)).
 * heads[t, :] = the h heads of largest r, ties to the lower index, written in
 * ascending head order.  r_out (nullable) receives r.  H must divide 128
 * (H in {1,2,4,...,128}); 1 <= h <= H.  Q and kbar_hl 16-byte aligned.
 */
int misa_route_heads(const uint16_t* Q, const float* w, const uint16_t* kbar_hl, int n_q,
                     int64_t q_pos0, int64_t n_k, int H, int d, int B, int h, int32_t* heads,
                     float* r_out, void* stream);

/*
 * Stage 4 — routed token scoring (Metodologia step 2: only the h routed heads
 * score the prefix token by token).
 *   logits[t, s] = sum_{i < h} w[t, j_i] * ReLU(q[t, j_i] . k_s),  j_i = heads[t, i],
 * for s <= pos(t).  heads == NULL scores with all H heads (h must equal H): the
 * dense DSA lightning indexer (Declaracao do Problema).  For FP8 keys the
 * product uses the decoded code and the per-token scale multiplies the dot
 * product before the ReLU.  Entries s > pos(t) are not part of the result:
 * those in a 128-key tile that also holds causal keys are written -inf (up to
 * column n_k rounded up to a multiple of 4), the rest are left untouched.  h must be a power of two <= 128; ld >= n_k and a
 * multiple of 4 (16-byte rows: tiles are written by TMA stores).  Q, K, logits
 * 16-byte aligned.
 */
int misa_score_tokens(const uint16_t* Q, const float* w, const int32_t* heads, const void* K,
                      const float* k_scale, int kdtype, int n_q, int64_t q_pos0, int64_t n_k,
                      int H, int d, int h, float* logits, int64_t ld, void* stream);

/*
 * Stage 4 with FP8 queries as well as FP8 keys, multiplied on the tensor cores
 * as E4M3 (kind::f8f6f4, twice the bf16 rate).  The integration issue runs the
 * indexer with FP8 operands in vLLM but fixes no scale rule; here every
 * (query, head) row and every key row carries its own fp32 scale:
 *   q[t, j] = e4m3(Q8[t, j, :]) * q_scale[t, j],  k_s = e4m3(K8[s, :]) * k_scale[s]
 *   logits[t, s] = sum_{i < h} w[t, j_i] * ReLU(q[t, j_i] . k_s),  s <= pos(t)
 * computed as k_scale[s] * sum_i (w[t, j_i] * q_scale[t, j_i]) * ReLU(e4m3 dot),
 * the same in real arithmetic because every scale must be positive and finite
 * (not checked).  Q8 [n_q, H, d] and K8 [n_k, d] hold e4m3 codes (NaN codes
 * not allowed), 16-byte aligned; q_scale [n_q, H], k_scale [n_k] fp32.
 * d in {64, 128}; the other arguments, the layout of logits and the -inf
 * entries are those of misa_score_tokens.  Returns MISA_ERR_UNSUPPORTED for
 * other d, MISA_ERR_INVALID_ARG for bad pointers or sizes.
 */
int misa_score_tokens_fp8(const uint8_t* Q8, const float* q_scale, const float* w,
                          const int32_t* heads, const uint8_t* K8, const float* k_scale, int n_q,
                          int64_t q_pos0, int64_t n_k, int H, int d, int h, float* logits,
                          int64_t ld, void* stream);

/*
 * Stage 5 — top-k token selection (technical summary, Metodologia step 2: the
 * final top-k tokens come from the reduced scores).  For each row t, among
 * logits[t, 0..min(pos(t), n_k-1)] keep the k largest, ties to the lower token
 * index (-0.0 equals +0.0), and write their indices ascending into idx[t, :],
 * padded with -1 when fewer than k tokens are visible.  Rows must hold no NaN.
 * logits 16-byte aligned with ld a multiple of 4.  0 <= k <= 16384.
 * ws/ws_bytes: workspace, size from misa_workspace_size("topk", ...) (may be 0).
 */
int misa_topk(const float* logits, int64_t ld, int n_q, int64_t q_pos0, int64_t n_k, int k,
              int32_t* idx, void* ws, size_t ws_bytes, void* stream);

/*
 * MISA-dagger fine stage (Variante Hierarquica: the original all-head indexer
 * re-scores the k' routed candidates and the final top-k comes from them).
 *   full[t, i] = sum_{j < H} w[t, j] * ReLU(q[t, j] . k_{c}),  c = cand[t, i]
 * Entries c outside 0..pos(t) (including the -1 padding) are ignored.  The k
 * candidates of largest full score, ties to the lower token index, are written
 * ascending to idx[t, :], -1 padded, whatever order a row's candidates come in
 * (rows whose valid candidates ascend, as the coarse selection emits them,
 * take a faster path).  full_logits (nullable, [n_q, kp]) receives full, -inf
 * where ignored.  The valid candidates of a row must be distinct: a token kept
 * twice records MISA_ERR_DEVICE in the device status.  H <= 128; 1 <= kp <=
 * 16384; 0 <= k <= kp.
 * ws/ws_bytes: workspace, size from misa_workspace_size("rerank", ...).
 */
int misa_rerank(const uint16_t* Q, const float* w, const void* K, const float* k_scale, int kdtype,
                const int32_t* cand, int kp, int n_q, int64_t q_pos0, int64_t n_k, int H, int d,
                int k, int32_t* idx, float* full_logits, void* ws, size_t ws_bytes, void* stream);

/*
 * misa_rerank for callers that cannot allocate device memory.  The MISA pages
 * have no counterpart: this is a packaging variant of misa_rerank, not a step of
 * the method.  Callers inside a fixed memory pool they do not own, inside a
 * region where cudaMalloc is forbidden, or without a device allocator cannot
 * hand misa_rerank its n_q * kp floats of workspace; this entry point keeps
 * that scratch in a 16 MiB device array inside the library instead (held on
 * every GPU that loads the library until exit) and allocates nothing.
 * Arguments and results are those of misa_rerank without full_logits and
 * workspace.  Limit: n_q * kp <= 4194304, else MISA_ERR_WORKSPACE before any
 * launch (call it on smaller query chunks).  All calls on a device share the
 * scratch: calls that overlap on the GPU (unordered streams) race on it.  The
 * first call on each device looks the array's address up (a CUDA runtime
 * call), so make it outside any stream capture.
 */
int misa_rerank_noalloc(const uint16_t* Q, const float* w, const void* K, const float* k_scale,
                        int kdtype, const int32_t* cand, int kp, int n_q, int64_t q_pos0,
                        int64_t n_k, int H, int d, int k, int32_t* idx, void* stream);

/*
 * Stages 4-5 fused — routed token scoring and top-k in one call (Metodologia
 * step 2).  Same result as misa_score_tokens followed by misa_topk on its
 * logits: idx[t, :] = the k tokens s <= pos(t) of largest routed logit, ties to
 * the lower index, ascending, -1 padded.  Instead of writing all n_q x n_k
 * logits it scores a 4096-key sample of the prefix 0..q_pos0 first, sets a
 * per-row threshold from it, stores only the logits at or above the threshold
 * (a few k per row, flagged in a per-row bit mask) while scoring, and selects
 * exactly among them.  Rows whose threshold kept fewer than min(k, visible)
 * logits, or more than the finish's list holds (max(6144, 3k) entries up to
 * k = 4096, 2k above, rounded up to a multiple of 1024), are recomputed by the
 * unfused sequence, so the result is exact for every input.
 *   logits [n_q, ld]: scratch for the kept logits and the fallback (contents
 *     unspecified afterwards; ld >= n_k, a multiple of 4, 16-byte aligned).
 *   ws/ws_bytes: misa_workspace_size("score_topk", n_q, n_k, k, 0) bytes,
 *     16-byte aligned (it includes room for FP8 keys decoded to bf16, which
 *     every scoring pass of the fused sequence then reads).  That size is 0 (and the call runs the unfused
 *     sequence) unless 4096 <= n_k <= 262144 and 1 <= k <= 8192.  The fused
 *     sequence also needs q_pos0 >= 4095 and h in {4, 8, 16, 32, 64}, else the
 *     call is unfused.  After a fused call, ws holds n_q + 1 int32 repair flags
 *     at offset 0: [0] != 0 iff any row took the fallback, [1 + t] for row t.
 * kdtype may also be MISA_K_BF16_SCALED (contiguous keys): the fused sequence
 * then reads the given bf16 codes and their scales directly, where e4m3 keys
 * are decoded into the workspace on every call, so a caller that scores the
 * same FP8 keys in several query pieces decodes them once.  The logits equal
 * those of the e4m3 keys the codes were decoded from.
 * Shapes and other limits as misa_score_tokens; 0 <= k <= 16384.
 */
int misa_score_topk(const uint16_t* Q, const float* w, const int32_t* heads, const void* K,
                    const float* k_scale, int kdtype, int n_q, int64_t q_pos0, int64_t n_k, int H,
                    int d, int h, int k, int32_t* idx, float* logits, int64_t ld, void* ws,
                    size_t ws_bytes, void* stream);

/*
 * FP8 index keys (the FP8 indexer of the integration issue "Clarification on
 * the Figure 3 baseline...": e4m3 codes with a per-token scale) decoded to bf16
 * codes: Kbf[s, i] = bf16(e4m3(K8[s, i])), exact (every e4m3 value is a bf16
 * value; NaN codes give a bf16 NaN); the scales are not applied (pass them with
 * the codes as MISA_K_BF16_SCALED).
 *   K8 [n_k, d] e4m3 codes, Kbf [n_k, d] bf16 codes: caller-owned device
 *   memory, 16-byte aligned, not overlapping; d in {32, 64, 128}.
 * Asynchronous on `stream`.  Returns MISA_ERR_INVALID_ARG for bad pointers or
 * sizes, MISA_ERR_UNSUPPORTED for other d.
 */
int misa_keys_e4m3_to_bf16(const uint8_t* K8, int64_t n_k, int d, uint16_t* Kbf, void* stream);

/*
 * Paged key caches.  The integration issue ("Clarification on the Figure 3
 * baseline...", measurement table and the use_misa call path) measures the
 * indexer at the vLLM boundary, where the index keys live in a paged cache and
 * the indexer's time includes the cache handling.  These entry points take the
 * keys in that form instead of as one contiguous [n_k, d] array:
 *   pages        [n_pages, page_size, d] key rows (bf16 codes, or e4m3 codes
 *                with k_scale [n_pages, page_size] fp32: a scale per row),
 *                16-byte aligned; n_pages * page_size < 2^31
 *   block_table  [ceil(n_k / page_size)] int32: logical key s of the sequence
 *                is row s % page_size of page block_table[s / page_size]
 *   page_size    16, 32, 64 or 128 (else MISA_ERR_UNSUPPORTED)
 * Every other argument, and the result, is that of the contiguous entry point
 * of the same name: the result equals the contiguous call on the keys gathered
 * in logical order, bit for bit (the same arithmetic on the same values).  A
 * block-table entry outside 0..n_pages-1 is reported as MISA_ERR_DEVICE and
 * read as page 0.  Table entries are read only for keys below n_k.
 */
int misa_pool_keys_paged(const void* pages, const float* k_scale, int kdtype,
                         const int32_t* block_table, int page_size, int64_t n_pages, int64_t n_k,
                         int d, int B, int64_t m0, int64_t m1, float* kbar, uint16_t* kbar_hl,
                         void* stream);  /* misa_pool_keys_range over a paged cache */
int misa_score_tokens_paged(const uint16_t* Q, const float* w, const int32_t* heads,
                            const void* pages, const float* k_scale, int kdtype,
                            const int32_t* block_table, int page_size, int64_t n_pages, int n_q,
                            int64_t q_pos0, int64_t n_k, int H, int d, int h, float* logits,
                            int64_t ld, void* stream);
int misa_score_topk_paged(const uint16_t* Q, const float* w, const int32_t* heads,
                          const void* pages, const float* k_scale, int kdtype,
                          const int32_t* block_table, int page_size, int64_t n_pages, int n_q,
                          int64_t q_pos0, int64_t n_k, int H, int d, int h, int k, int32_t* idx,
                          float* logits, int64_t ld, void* ws, size_t ws_bytes, void* stream);
int misa_rerank_paged(const uint16_t* Q, const float* w, const void* pages, const float* k_scale,
                      int kdtype, const int32_t* block_table, int page_size, int64_t n_pages,
                      const int32_t* cand, int kp, int n_q, int64_t q_pos0, int64_t n_k, int H,
                      int d, int k, int32_t* idx, float* full_logits, void* ws, size_t ws_bytes,
                      void* stream);

/*
 * Decode over paged caches: n_seq sequences, each with one new query at the
 * last of its own seq_lens[b] keys (the pages evaluate prefill only; this is
 * stages 1-5 for the token-by-token generation that follows it, batched over
 * sequences the way a serving engine calls the indexer).  Layouts:
 *   Q            [n_seq, H, d] bf16: the new query of each sequence
 *   w            [n_seq, H] fp32
 *   pages, k_scale, page_size, n_pages: one shared page pool, as above
 *   block_tables [n_seq, max_blocks] int32: row b is sequence b's block table
 *   seq_lens     [n_seq] int32 (device): keys of sequence b, 0..max_blocks *
 *                page_size (a longer length is reported as MISA_ERR_DEVICE and
 *                clamped); query b sits at position seq_lens[b] - 1
 *   kbar, kbar_hl per-sequence pooled keys: [n_seq, M_max, d] fp32 and
 *                [n_seq, 2, M_max, d] bf16 hi/lo (sequence b's slice in the
 *                layout misa_pool_keys writes for M = M_max)
 * n_seq <= 65535 for the pooling call.
 */
/* Stage 1: re-pools the last n_last blocks of every sequence (blocks
 * M_b - n_last .. M_b - 1, M_b = ceil(seq_lens[b] / B)): n_last = 1 after one
 * key was appended, n_last = M_max for a whole cache.  M_max >=
 * ceil(max_blocks * page_size / B).  Each block's arithmetic is that of
 * misa_pool_keys. */
int misa_decode_pool_keys(const void* pages, const float* k_scale, int kdtype,
                          const int32_t* block_tables, int max_blocks, int page_size,
                          int64_t n_pages, const int32_t* seq_lens, int n_seq, int d, int B,
                          int64_t M_max, int64_t n_last, float* kbar, uint16_t* kbar_hl,
                          void* stream);
/* Stages 2-3 for each sequence's query against its own pooled keys: the router
 * of misa_route_heads with C(b) = the complete blocks of sequence b
 * (floor(seq_lens[b] / B), at most M_max).  heads [n_seq, h], r_out [n_seq, H]
 * (nullable).  H a power of two <= 128. */
int misa_decode_route_heads(const uint16_t* Q, const float* w, const uint16_t* kbar_hl,
                            int64_t M_max, const int32_t* seq_lens, int n_seq, int H, int d, int B,
                            int h, int32_t* heads, float* r_out, void* stream);
/* Stages 4-5 for each sequence's query over all its keys:
 *   logits[b, s] = sum_{i<h} w[b, j_i] * ReLU(q[b, j_i] . k_{b,s}),  s < seq_lens[b]
 * (heads [n_seq, h], NULL = all H heads with h == H), then idx[b, :] = the k
 * keys of largest logit, ties to the lower index, ascending, -1 padded.  A
 * scoring pass shaped for one query per sequence: 128-key tiles against the
 * query's h head rows padded to 16, 32 or 64 MMA columns, so the keys are read
 * once and the MMA stays small.  bf16 or e4m3 pages (e4m3: decoded exactly to
 * bf16 in the kernel, the row's scale multiplying the head-sum, as in
 * misa_score_tokens); h a power of two <= 64.  logits [n_seq, ld] fp32
 * scratch (ld >= max_blocks * page_size; entries s < seq_lens[b] hold the
 * logits afterwards). */
int misa_decode_score_topk(const uint16_t* Q, const float* w, const int32_t* heads,
                           const void* pages, const float* k_scale, int kdtype,
                           const int32_t* block_tables, int max_blocks, int page_size,
                           int64_t n_pages, const int32_t* seq_lens, int n_seq, int H, int d,
                           int h, int k, int32_t* idx, float* logits, int64_t ld, void* stream);

/*
 * Stage timing of misa_score_topk (diagnostic; not a step of the method).
 * Between misa_profile_start() and misa_profile_stop(), each launch of the fused
 * sequence is bracketed by CUDA events on the call's stream.  misa_profile_stop
 * synchronises on those events and writes, for stage i < n, the summed device
 * milliseconds ms[i] and the number of launches counts[i] (either array may be
 * NULL); misa_profile_stage_name(i) names stage i (NULL past the last).  The
 * fused call's stages: prepare (FP8 key decode and sample gather),
 * sample_score, threshold, select_score, finish, repair_score, repair_topk.  Not for use inside stream capture.
 */
int misa_profile_start(void);
int misa_profile_stop(double* ms, int* counts, int n);
const char* misa_profile_stage_name(int i);

/* Workspace bytes needed by op "topk", "rerank" or "score_topk" for the given
 * sizes (0 if none). */
size_t misa_workspace_size(const char* op, int n_q, int64_t n_k, int k, int kp);

/* Static text for a misa_status value. */
const char* misa_status_string(int status);

/* Synchronises `stream`, returns and clears the device status word of the
 * current device (MISA_OK, MISA_ERR_TIMEOUT or MISA_ERR_DEVICE). */
int misa_last_device_status(void* stream);

/* Sets the time budget of every bounded device-side wait, in nanoseconds
 * (default 2e9; 0 restores the default).  Diagnostic knob: a tiny value makes
 * kernels give up and report MISA_ERR_TIMEOUT instead of waiting. */
int misa_set_wait_limit_ns(uint64_t ns);

#ifdef __cplusplus
}
#endif
#endif /* MISA_H_ */
