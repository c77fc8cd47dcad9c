/*
 * CPU oracle for the MISA token indexer.  TEST INFRASTRUCTURE ONLY: the tests,
 * the smoke check and the benchmark's CPU-baseline leg call it; the product path
 * never does.  It shares no code with the CUDA library.
 *
 * Plain, slow, single-threaded, fp64.  Every function restates one step of the
 * method in the order the MISA pages give it ("MISA: Mixture of Indexer Sparse
 * Attention for Long-Context LLM Inference"; technical summary, Metodologia steps
 * 1-2 and "Variante Hierarquica"; abstract):
 *
 *   pool     kbar_m = mean of the key rows of block m, M = ceil(L/B) blocks
 *            (Metodologia step 1: "chaves de indexacao com media agrupada").
 *   route    r[t,j] = sum over the complete causal blocks m of
 *                     w[t,j] * ReLU(q[t,j] . kbar_m)
 *            (step 1 only says the router "aggregates" per-head block
 *            affinities; this sum is the reading used throughout).
 *   top-h    the h heads of largest r, ties to the lower head index, returned
 *            in ascending head order (step 1: "seleciona as top-h cabecas").
 *   score    logit[t,s] = sum over routed heads j (ascending) of
 *                     w[t,j] * ReLU(q[t,j] . k_s),  s <= pos(t)
 *            (step 2: only the h routed heads score tokens).  With every head
 *            routed this is the dense DSA lightning indexer (Declaracao do
 *            Problema: all H_I heads score every prefix token).
 *   top-k    the k tokens of largest logit, ties to the lower token index,
 *            returned in ascending token order, padded with -1.
 *   rerank   MISA-dagger fine stage: all H_I heads re-score the k' candidates
 *            kept by the routed coarse pass, then top-k among them (Variante
 *            Hierarquica, "Etapa Grossa" / "Etapa Fina").
 *
 * Conventions.  Query t sits at position pos(t) = q_pos0 + t and sees keys
 * 0..pos(t) (inclusive).  Block m covers keys mB .. mB+n_m-1 with
 * n_m = min(B, L - mB); the router uses only complete blocks whose last key is
 * <= pos(t), so no key after pos(t) reaches query t.  Inputs are the stored
 * values (bf16 codes, or e4m3 codes times a per-token fp32 scale) decoded
 * exactly to fp64.
 *
 * Optional counters (`macs`) add the multiply-adds each function performs, for
 * the per-query cost model O(h L + H_I M) of the pages (Metodologia).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---- storage formats -------------------------------------------------- */

/* bf16: the upper 16 bits of an IEEE-754 binary32. */
double oracle_bf16_to_double(uint16_t code) {
    uint32_t u = (uint32_t)code << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP FP8 E4M3: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent
 * field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; there are no infinities. */
double oracle_e4m3_to_double(uint8_t code) {
    int sign = (code >> 7) & 1;
    int ex = (code >> 3) & 0xF;
    int man = code & 0x7;
    double mag;
    if (ex == 0xF && man == 0x7) return NAN;
    if (ex == 0)
        mag = ldexp((double)man / 8.0, -6);
    else
        mag = ldexp(1.0 + (double)man / 8.0, ex - 7);
    return sign ? -mag : mag;
}

void oracle_decode_bf16(const uint16_t* in, int64_t n, double* out) {
    for (int64_t i = 0; i < n; ++i) out[i] = oracle_bf16_to_double(in[i]);
}

/* K[s,c] = e4m3(code[s,c]) * scale[s] */
void oracle_decode_e4m3_keys(const uint8_t* codes, const float* scale, int64_t n_k, int d,
                             double* out) {
    for (int64_t s = 0; s < n_k; ++s)
        for (int c = 0; c < d; ++c)
            out[s * d + c] = oracle_e4m3_to_double(codes[s * d + c]) * (double)scale[s];
}

/* ---- helpers ---------------------------------------------------------- */

static double dot(const double* a, const double* b, int d) {
    double acc = 0.0;
    for (int c = 0; c < d; ++c) acc += a[c] * b[c];
    return acc;
}

static double relu(double x) { return x > 0.0 ? x : 0.0; }

/* ---- stage 1: block mean-pooling --------------------------------------- */

void oracle_pool_keys(const double* K, int64_t n_k, int d, int B, double* kbar) {
    int64_t M = (n_k + B - 1) / B;
    for (int64_t m = 0; m < M; ++m) {
        int64_t first = m * B;
        int64_t n_m = n_k - first < B ? n_k - first : B;
        for (int c = 0; c < d; ++c) {
            double sum = 0.0;
            for (int64_t r = 0; r < n_m; ++r) sum += K[(first + r) * d + c];
            kbar[m * d + c] = sum / (double)n_m;
        }
    }
}

/* Number of complete blocks whose last key is <= pos. */
int64_t oracle_causal_blocks(int64_t pos, int64_t n_k, int B) {
    int64_t complete_in_prefix = (pos + 1) / B;
    int64_t complete_in_keys = n_k / B;
    return complete_in_prefix < complete_in_keys ? complete_in_prefix : complete_in_keys;
}

/* ---- stages 2-3: router and top-h --------------------------------------- */

/* Strict "ranks before" for heads: larger score first, then lower head index. */
static int head_before(double ra, int ja, double rb, int jb) {
    if (ra > rb) return 1;
    if (ra < rb) return 0;
    return ja < jb;
}

void oracle_route(const double* Q, const double* w, const double* kbar, int n_q,
                  int64_t q_pos0, int64_t n_k, int H, int d, int B, int h, double* r_out,
                  int32_t* heads, int64_t* macs) {
    double* r = (double*)malloc(sizeof(double) * (size_t)H);
    int* taken = (int*)malloc(sizeof(int) * (size_t)H);
    for (int t = 0; t < n_q; ++t) {
        int64_t pos = q_pos0 + t;
        int64_t nC = oracle_causal_blocks(pos, n_k, B);
        for (int j = 0; j < H; ++j) {
            const double* q = Q + ((int64_t)t * H + j) * d;
            double wt = w[(int64_t)t * H + j];
            double acc = 0.0;
            for (int64_t m = 0; m < nC; ++m) acc += wt * relu(dot(q, kbar + m * d, d));
            r[j] = acc;
            if (macs) *macs += nC * d;
            if (r_out) r_out[(int64_t)t * H + j] = acc;
        }
        /* top-h by repeated selection of the best head not yet taken */
        for (int j = 0; j < H; ++j) taken[j] = 0;
        for (int i = 0; i < h; ++i) {
            int best = -1;
            for (int j = 0; j < H; ++j) {
                if (taken[j]) continue;
                if (best < 0 || head_before(r[j], j, r[best], best)) best = j;
            }
            taken[best] = 1;
        }
        int o = 0;
        for (int j = 0; j < H; ++j)
            if (taken[j]) heads[(int64_t)t * h + o++] = j;
    }
    free(taken);
    free(r);
}

/* ---- stage 4: routed token scoring and the dense indexer ---------------- */

/* logits is [n_q, ld]; entries s > pos(t) (and s < n_k) are -inf. */
void oracle_score(const double* Q, const double* w, const int32_t* heads, const double* K,
                  int n_q, int64_t q_pos0, int64_t n_k, int H, int d, int h, double* logits,
                  int64_t ld, int64_t* macs) {
    for (int t = 0; t < n_q; ++t) {
        int64_t pos = q_pos0 + t;
        for (int64_t s = 0; s < n_k; ++s) {
            double v;
            if (s > pos) {
                v = -INFINITY;
            } else {
                v = 0.0;
                for (int i = 0; i < h; ++i) {
                    int j = heads[(int64_t)t * h + i];
                    const double* q = Q + ((int64_t)t * H + j) * d;
                    v += w[(int64_t)t * H + j] * relu(dot(q, K + s * d, d));
                }
                if (macs) *macs += (int64_t)h * d;
            }
            logits[(int64_t)t * ld + s] = v;
        }
    }
}

/* The DSA lightning indexer: every one of the H heads scores every prefix token. */
void oracle_dense_logits(const double* Q, const double* w, const double* K, int n_q,
                         int64_t q_pos0, int64_t n_k, int H, int d, double* logits, int64_t ld) {
    for (int t = 0; t < n_q; ++t) {
        int64_t pos = q_pos0 + t;
        for (int64_t s = 0; s < n_k; ++s) {
            double v = -INFINITY;
            if (s <= pos) {
                v = 0.0;
                for (int j = 0; j < H; ++j)
                    v += w[(int64_t)t * H + j] *
                         relu(dot(Q + ((int64_t)t * H + j) * d, K + s * d, d));
            }
            logits[(int64_t)t * ld + s] = v;
        }
    }
}

/* ---- stage 5: top-k ------------------------------------------------------ */

typedef struct { double v; int64_t s; } scored;

/* larger value first, then lower token index */
static int cmp_scored(const void* pa, const void* pb) {
    const scored* a = (const scored*)pa;
    const scored* b = (const scored*)pb;
    if (a->v > b->v) return -1;
    if (a->v < b->v) return 1;
    return (a->s < b->s) ? -1 : (a->s > b->s);
}

static int cmp_i64(const void* pa, const void* pb) {
    int64_t a = *(const int64_t*)pa, b = *(const int64_t*)pb;
    return (a > b) - (a < b);
}

/* Pick the k best of n (value, token) pairs; write their tokens ascending, then -1. */
static void select_k(scored* items, int64_t n, int k, int32_t* out) {
    qsort(items, (size_t)n, sizeof(scored), cmp_scored);
    int64_t take = n < k ? n : k;
    int64_t* tok = (int64_t*)malloc(sizeof(int64_t) * (size_t)(take > 0 ? take : 1));
    for (int64_t i = 0; i < take; ++i) tok[i] = items[i].s;
    qsort(tok, (size_t)take, sizeof(int64_t), cmp_i64);
    for (int64_t i = 0; i < k; ++i) out[i] = i < take ? (int32_t)tok[i] : -1;
    free(tok);
}

/* Top-k over logits rows given in fp64 ([n_q, ld]); only s <= pos(t) are read. */
void oracle_topk(const double* logits, int64_t ld, int n_q, int64_t q_pos0, int64_t n_k, int k,
                 int32_t* idx) {
    scored* items = (scored*)malloc(sizeof(scored) * (size_t)(n_k > 0 ? n_k : 1));
    for (int t = 0; t < n_q; ++t) {
        int64_t pos = q_pos0 + t;
        int64_t n = pos + 1 < n_k ? pos + 1 : n_k;
        for (int64_t s = 0; s < n; ++s) {
            items[s].v = logits[(int64_t)t * ld + s];
            items[s].s = s;
        }
        select_k(items, n, k, idx + (int64_t)t * k);
    }
    free(items);
}

/* Same selection over fp32 rows (for logits produced elsewhere); each value is
 * widened exactly to fp64, so -0.0 and +0.0 compare equal. */
void oracle_topk_f32(const float* logits, int64_t ld, int n_q, int64_t q_pos0, int64_t n_k, int k,
                     int32_t* idx) {
    scored* items = (scored*)malloc(sizeof(scored) * (size_t)(n_k > 0 ? n_k : 1));
    for (int t = 0; t < n_q; ++t) {
        int64_t pos = q_pos0 + t;
        int64_t n = pos + 1 < n_k ? pos + 1 : n_k;
        for (int64_t s = 0; s < n; ++s) {
            items[s].v = (double)logits[(int64_t)t * ld + s];
            items[s].s = s;
        }
        select_k(items, n, k, idx + (int64_t)t * k);
    }
    free(items);
}

/* ---- MISA-dagger fine stage -------------------------------------------- */

/* cand is [n_q, kp], -1 padded; entries outside 0..pos(t) are ignored.
 * full_logits (nullable) is [n_q, kp]: the all-head logit of each candidate,
 * -inf where the entry is ignored. */
void oracle_rerank(const double* Q, const double* w, const double* K, const int32_t* cand, int kp,
                   int n_q, int64_t q_pos0, int64_t n_k, int H, int d, int k, int32_t* idx,
                   double* full_logits, int64_t* macs) {
    scored* items = (scored*)malloc(sizeof(scored) * (size_t)(kp > 0 ? kp : 1));
    for (int t = 0; t < n_q; ++t) {
        int64_t pos = q_pos0 + t;
        int64_t n = 0;
        for (int i = 0; i < kp; ++i) {
            int64_t c = cand[(int64_t)t * kp + i];
            double v = -INFINITY;
            if (c >= 0 && c <= pos && c < n_k) {
                v = 0.0;
                for (int j = 0; j < H; ++j)
                    v += w[(int64_t)t * H + j] *
                         relu(dot(Q + ((int64_t)t * H + j) * d, K + c * d, d));
                if (macs) *macs += (int64_t)H * d;
                items[n].v = v;
                items[n].s = c;
                ++n;
            }
            if (full_logits) full_logits[(int64_t)t * kp + i] = v;
        }
        select_k(items, n, k, idx + (int64_t)t * k);
    }
    free(items);
}

/* Top-k among candidate scores given in fp32 (scores produced elsewhere):
 * row t holds vals[t*kp + i] for token cand[t*kp + i].  Entries whose token is
 * outside 0..pos(t) or whose value is -inf are ignored; selection by (value
 * desc, token asc); tokens written ascending, -1 padded. */
void oracle_select_candidates_f32(const float* vals, const int32_t* cand, int kp, int n_q,
                                  int64_t q_pos0, int64_t n_k, int k, int32_t* idx) {
    scored* items = (scored*)malloc(sizeof(scored) * (size_t)(kp > 0 ? kp : 1));
    for (int t = 0; t < n_q; ++t) {
        int64_t pos = q_pos0 + t;
        int64_t n = 0;
        for (int i = 0; i < kp; ++i) {
            int64_t c = cand[(int64_t)t * kp + i];
            double v = (double)vals[(int64_t)t * kp + i];
            if (c < 0 || c > pos || c >= n_k || v == -INFINITY) continue;
            items[n].v = v;
            items[n].s = c;
            ++n;
        }
        select_k(items, n, k, idx + (int64_t)t * k);
    }
    free(items);
}
