/*
 * Paged-attention ORACLE: a plain, slow, fp64 CPU statement of what the paged
 * decode path computes.  TEST INFRASTRUCTURE ONLY: tests, the smoke check and
 * the benchmark's CPU-baseline leg call it; the library never does.  It shares
 * no source, header or table with the CUDA library.
 *
 * Sources, by page title and section:
 *  [FSAH]  "PagedAttention Paper Breakdown: Virtual Memory Allocation for LLM KV
 *          Cache Serving" (fullstackaihub.com), section 2 "Virtual Memory Paging &
 *          Block Table Architecture", Address Translation Formula and the block
 *          diagram under it.
 *  [INIT]  "PagedAttention and vLLM Architecture: Virtual Memory for LLM Serving"
 *          (initnode.dev), section 1 "Logical vs Physical Blocks", section 2
 *          "PagedAttention Attention CUDA Kernel Mechanics", section 3
 *          "Copy-on-Write (CoW) for Parallel Sampling & Beam Search".
 *
 * Layout of the KV pools (one for K, one for V): [num_blocks][kv_heads][B][D],
 * element (slot, h, d) of physical block p = slot / B at offset o = slot % B.
 *
 * Pins (tests/test_oracle_pins.py): the printed translation examples, contiguous
 * attention from torch's scaled_dot_product_attention when the block table is
 * the identity, invariance under any permutation of physical blocks, closed
 * forms (one token, equal keys, one dominant logit), weights summing to one,
 * pure-Python brute force on tiny inputs.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* [FSAH] Address Translation Formula: b = floor(i/B), o = i mod B,
 * PhysicalAddr(K_i) = T[b]*B + o.  The address is a token-slot index. */
int64_t oracle_physical_slot(const int32_t* table, int block_size, int64_t i)
{
    int64_t b = i / block_size;
    int64_t o = i % block_size;
    return (int64_t)table[b] * block_size + o;
}

/* Offset, in elements, of (slot, kv_head, d=0) in a [num_blocks][kv_heads][B][D] pool. */
static size_t pool_row(int64_t slot, int kv_head, int kv_heads, int block_size, int head_dim)
{
    int64_t p = slot / block_size;
    int64_t o = slot % block_size;
    return ((size_t)(p * kv_heads + kv_head) * block_size + (size_t)o) * head_dim;
}

struct decode_job {
    double* out;                 /* [S][Hq][D] */
    double* weights;             /* optional [S][Hq][wstride] */
    int64_t wstride;
    const float* q;              /* [S][Hq][D] */
    const float* k_cache;        /* [NB][Hkv][B][D] */
    const float* v_cache;
    const int32_t* block_tables; /* [S][MB] */
    const int32_t* context_lens; /* [S] */
    int S, Hq, Hkv, D, B, MB;
    double scale;
    int nthreads;
    int tid;
};

/*
 * Decode attention for one (sequence s, query head h), as a plain two-pass
 * softmax over the sequence's logical tokens 0..L-1 ([INIT] section 2: the
 * kernel walks the block table, dots q with each key, softmaxes over all
 * blocks and weights the values).  Query head h reads kv head h / (Hq/Hkv).
 * L = 0 gives a zero output row.
 */
static void decode_one(const struct decode_job* j, int s, int h)
{
    const int D = j->D;
    const int group = j->Hq / j->Hkv;
    const int kvh = h / group;
    const int L = j->context_lens[s];
    const float* q = j->q + ((size_t)s * j->Hq + h) * D;
    const int32_t* T = j->block_tables + (size_t)s * j->MB;
    double* out = j->out + ((size_t)s * j->Hq + h) * D;

    for (int d = 0; d < D; ++d) out[d] = 0.0;
    if (L <= 0) return;

    double* z = (double*)malloc(sizeof(double) * (size_t)L);
    double zmax = -INFINITY;
    for (int i = 0; i < L; ++i) {
        int64_t slot = oracle_physical_slot(T, j->B, i);
        const float* k = j->k_cache + pool_row(slot, kvh, j->Hkv, j->B, D);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += (double)q[d] * (double)k[d];
        z[i] = j->scale * dot;
        if (z[i] > zmax) zmax = z[i];
    }
    double denom = 0.0;
    for (int i = 0; i < L; ++i) denom += exp(z[i] - zmax);
    for (int i = 0; i < L; ++i) {
        double w = exp(z[i] - zmax) / denom;
        if (j->weights) j->weights[((size_t)s * j->Hq + h) * (size_t)j->wstride + i] = w;
        int64_t slot = oracle_physical_slot(T, j->B, i);
        const float* v = j->v_cache + pool_row(slot, kvh, j->Hkv, j->B, D);
        for (int d = 0; d < D; ++d) out[d] += w * (double)v[d];
    }
    free(z);
}

static void* decode_worker(void* arg)
{
    const struct decode_job* j = (const struct decode_job*)arg;
    int64_t n = (int64_t)j->S * j->Hq;
    for (int64_t u = j->tid; u < n; u += j->nthreads) decode_one(j, (int)(u / j->Hq), (int)(u % j->Hq));
    return NULL;
}

/*
 * out[s][h][:] = softmax_i(scale * q[s][h].K_i) . V_i over i < context_lens[s].
 * Inputs are fp32 (bf16 values widen to fp32 exactly); arithmetic is fp64.
 * weights (nullable) receives the softmax weights, row stride wstride >= max L.
 * nthreads > 1 splits the (s, h) pairs over POSIX threads; the arithmetic of
 * each pair is the same.  Returns 0, or -1 on a bad argument.
 */
int oracle_decode(double* out, double* weights, int64_t wstride, const float* q, const float* k_cache,
                  const float* v_cache, const int32_t* block_tables, const int32_t* context_lens, int S,
                  int Hq, int Hkv, int D, int B, int MB, double scale, int nthreads)
{
    if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || B <= 0 || MB < 0) return -1;
    for (int s = 0; s < S; ++s) {
        if (context_lens[s] < 0 || context_lens[s] > (int64_t)MB * B) return -1;
        if (weights && context_lens[s] > wstride) return -1;
    }
    if (nthreads < 1) nthreads = 1;
    struct decode_job* jobs = (struct decode_job*)calloc((size_t)nthreads, sizeof(struct decode_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        struct decode_job* j = &jobs[t];
        j->out = out; j->weights = weights; j->wstride = wstride;
        j->q = q; j->k_cache = k_cache; j->v_cache = v_cache;
        j->block_tables = block_tables; j->context_lens = context_lens;
        j->S = S; j->Hq = Hq; j->Hkv = Hkv; j->D = D; j->B = B; j->MB = MB;
        j->scale = scale; j->nthreads = nthreads; j->tid = t;
    }
    if (nthreads == 1) {
        decode_worker(&jobs[0]);
    } else {
        for (int t = 0; t < nthreads; ++t) pthread_create(&th[t], NULL, decode_worker, &jobs[t]);
        for (int t = 0; t < nthreads; ++t) pthread_join(th[t], NULL);
    }
    free(th);
    free(jobs);
    return 0;
}

/*
 * Partial softmax state of one (s, h) over the logical token range [t0, t1):
 * m = max z_i, l = sum exp(z_i - m), acc[d] = sum exp(z_i - m) V_i[d].
 * An empty range gives m = -inf, l = 0, acc = 0.  This is the per-partition
 * state of a context split; oracle_merge_partials combines such states.
 */
int oracle_partial(double* m_out, double* l_out, double* acc_out, const float* q, const float* k_cache,
                   const float* v_cache, const int32_t* table, int Hq, int Hkv, int D, int B, int h,
                   int t0, int t1, double scale)
{
    if (Hq % Hkv != 0 || t0 < 0 || t1 < t0) return -1;
    const int kvh = h / (Hq / Hkv);
    double m = -INFINITY;
    for (int i = t0; i < t1; ++i) {
        const float* k = k_cache + pool_row(oracle_physical_slot(table, B, i), kvh, Hkv, B, D);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += (double)q[d] * (double)k[d];
        if (scale * dot > m) m = scale * dot;
    }
    double l = 0.0;
    for (int d = 0; d < D; ++d) acc_out[d] = 0.0;
    for (int i = t0; i < t1; ++i) {
        int64_t slot = oracle_physical_slot(table, B, i);
        const float* k = k_cache + pool_row(slot, kvh, Hkv, B, D);
        const float* v = v_cache + pool_row(slot, kvh, Hkv, B, D);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += (double)q[d] * (double)k[d];
        double e = exp(scale * dot - m);
        l += e;
        for (int d = 0; d < D; ++d) acc_out[d] += e * (double)v[d];
    }
    *m_out = m;
    *l_out = l;
    return 0;
}

/*
 * Log-sum-exp merge of n partial states: M = max m_p,
 * out = sum_p exp(m_p - M) acc_p / sum_p exp(m_p - M) l_p.
 * States with l = 0 (empty ranges) are skipped; if all are empty, out = 0.
 */
void oracle_merge_partials(double* out, const double* m, const double* l, const double* acc, int n, int D)
{
    double M = -INFINITY;
    for (int p = 0; p < n; ++p)
        if (l[p] > 0.0 && m[p] > M) M = m[p];
    double denom = 0.0;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    for (int p = 0; p < n; ++p) {
        if (!(l[p] > 0.0)) continue;
        double w = exp(m[p] - M);
        denom += w * l[p];
        for (int d = 0; d < D; ++d) out[d] += w * acc[(size_t)p * D + d];
    }
    if (denom > 0.0)
        for (int d = 0; d < D; ++d) out[d] /= denom;
}

/*
 * Slot-mapped append: for token t with slot_mapping[t] >= 0, the D elements of
 * key[t][h] (and value[t][h]) are written to the pool row of that slot for
 * kv head h.  Negative slots are padding and are skipped.  Works on raw
 * elements of elt_bytes bytes, so the copy is exact for any dtype.
 * Returns 0, or -1 if a slot is >= num_blocks * B.
 */
int oracle_reshape_and_cache(const void* key, const void* value, void* k_cache, void* v_cache,
                             const int64_t* slot_mapping, int N, int Hkv, int D, int B, int num_blocks,
                             int elt_bytes)
{
    for (int t = 0; t < N; ++t)
        if (slot_mapping[t] >= (int64_t)num_blocks * B) return -1;
    const size_t row = (size_t)D * elt_bytes;
    for (int t = 0; t < N; ++t) {
        int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        for (int h = 0; h < Hkv; ++h) {
            size_t dst = pool_row(slot, h, Hkv, B, D) * elt_bytes;
            size_t src = ((size_t)t * Hkv + h) * row;
            memcpy((char*)k_cache + dst, (const char*)key + src, row);
            memcpy((char*)v_cache + dst, (const char*)value + src, row);
        }
    }
    return 0;
}

/*
 * Copy-on-write block copy ([INIT] section 3): for each pair (src, dst), in
 * pair order, the whole physical block dst (all kv heads, all B slots) of the
 * K pool and of the V pool becomes a copy of block src.
 * Returns 0, or -1 if an index is out of range.
 */
int oracle_copy_blocks(void* k_cache, void* v_cache, const int64_t* block_mapping, int num_pairs, int Hkv,
                       int D, int B, int num_blocks, int elt_bytes)
{
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
        if (src < 0 || dst < 0 || src >= num_blocks || dst >= num_blocks) return -1;
    }
    const size_t block_bytes = (size_t)Hkv * B * D * elt_bytes;
    for (int i = 0; i < num_pairs; ++i) {
        int64_t src = block_mapping[2 * i], dst = block_mapping[2 * i + 1];
        memmove((char*)k_cache + (size_t)dst * block_bytes, (const char*)k_cache + (size_t)src * block_bytes,
                block_bytes);
        memmove((char*)v_cache + (size_t)dst * block_bytes, (const char*)v_cache + (size_t)src * block_bytes,
                block_bytes);
    }
    return 0;
}

/*
 * Chunked prefill over the paged cache (the multi-token case of the same
 * attention: [INIT] section 3 "When a prompt is processed" assigns the prompt's
 * blocks; the new tokens' K/V are in the pools before the call, as for decode).
 * Sequence s holds L_s = context_lens[s] tokens, of which the last
 * n_s = q_start[s+1] - q_start[s] are queries: query i of s sits at position
 * p = L_s - n_s + i and attends causally to tokens 0..p, i.e. it is the decode
 * attention of that row with context length p + 1.  q and out are packed by
 * q_start: row q_start[s] + i, head h.  Plain loops, fp64; nothing is shared
 * with the decode function above except the address translation.
 */
struct prefill_job {
    double* out;                 /* [Nq][Hq][D] */
    const float* q;              /* [Nq][Hq][D] */
    const float* k_cache;
    const float* v_cache;
    const int32_t* block_tables; /* [S][MB] */
    const int32_t* context_lens; /* [S] */
    const int32_t* q_start;      /* [S+1] */
    int S, Hq, Hkv, D, B, MB;
    double scale;
    int nthreads, tid;
};

static void prefill_row(const struct prefill_job* j, int s, int i, int h)
{
    const int D = j->D;
    const int kvh = h / (j->Hq / j->Hkv);
    const int n = j->q_start[s + 1] - j->q_start[s];
    const int64_t row = (int64_t)j->q_start[s] + i;
    const int p = j->context_lens[s] - n + i;          /* position of this query token */
    const float* q = j->q + ((size_t)row * j->Hq + h) * D;
    const int32_t* T = j->block_tables + (size_t)s * j->MB;
    double* out = j->out + ((size_t)row * j->Hq + h) * D;
    for (int d = 0; d < D; ++d) out[d] = 0.0;
    const int L = p + 1;                                /* tokens 0..p */
    if (L <= 0) return;
    double* z = (double*)malloc(sizeof(double) * (size_t)L);
    double zmax = -INFINITY;
    for (int t = 0; t < L; ++t) {
        const float* k = j->k_cache + pool_row(oracle_physical_slot(T, j->B, t), kvh, j->Hkv, j->B, D);
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += (double)q[d] * (double)k[d];
        z[t] = j->scale * dot;
        if (z[t] > zmax) zmax = z[t];
    }
    double denom = 0.0;
    for (int t = 0; t < L; ++t) denom += exp(z[t] - zmax);
    for (int t = 0; t < L; ++t) {
        const double w = exp(z[t] - zmax) / denom;
        const float* v = j->v_cache + pool_row(oracle_physical_slot(T, j->B, t), kvh, j->Hkv, j->B, D);
        for (int d = 0; d < D; ++d) out[d] += w * (double)v[d];
    }
    free(z);
}

static void* prefill_worker(void* arg)
{
    const struct prefill_job* j = (const struct prefill_job*)arg;
    const int64_t rows = j->q_start[j->S];
    int64_t u = 0;
    for (int s = 0; s < j->S; ++s)
        for (int i = 0; i < j->q_start[s + 1] - j->q_start[s]; ++i)
            for (int h = 0; h < j->Hq; ++h, ++u)
                if (u % j->nthreads == j->tid) prefill_row(j, s, i, h);
    (void)rows;
    return NULL;
}

/* Returns 0, or -1 on a bad argument (a sequence with more queries than tokens,
 * a context beyond its table, q_start not non-decreasing). */
int oracle_prefill(double* out, const float* q, const float* k_cache, const float* v_cache,
                   const int32_t* block_tables, const int32_t* context_lens, const int32_t* q_start, int S, int Hq,
                   int Hkv, int D, int B, int MB, double scale, int nthreads)
{
    if (S < 0 || Hq <= 0 || Hkv <= 0 || Hq % Hkv != 0 || D <= 0 || B <= 0 || MB < 0 || q_start[0] != 0) return -1;
    for (int s = 0; s < S; ++s) {
        const int n = q_start[s + 1] - q_start[s];
        if (n < 0 || n > context_lens[s] || context_lens[s] > (int64_t)MB * B) return -1;
    }
    if (nthreads < 1) nthreads = 1;
    struct prefill_job* jobs = (struct prefill_job*)calloc((size_t)nthreads, sizeof(struct prefill_job));
    pthread_t* th = (pthread_t*)calloc((size_t)nthreads, sizeof(pthread_t));
    for (int t = 0; t < nthreads; ++t) {
        struct prefill_job* j = &jobs[t];
        j->out = out; j->q = q; j->k_cache = k_cache; j->v_cache = v_cache;
        j->block_tables = block_tables; j->context_lens = context_lens; j->q_start = q_start;
        j->S = S; j->Hq = Hq; j->Hkv = Hkv; j->D = D; j->B = B; j->MB = MB;
        j->scale = scale; j->nthreads = nthreads; j->tid = t;
    }
    for (int t = 1; t < nthreads; ++t) pthread_create(&th[t], NULL, prefill_worker, &jobs[t]);
    prefill_worker(&jobs[0]);
    for (int t = 1; t < nthreads; ++t) pthread_join(th[t], NULL);
    free(jobs);
    free(th);
    return 0;
}
