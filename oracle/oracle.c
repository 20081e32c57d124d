/*
 * CPU oracle for attention over a block-paged bf16 KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or
 * call this file: it exists so that tests, the smoke check and the benchmark's
 * CPU-baseline leg can compare the CUDA kernels against a plain, slow, obviously
 * correct restatement of what the path computes.  It shares no code, header,
 * table or helper with the CUDA library.
 *
 * Everything is evaluated in fp64 from the same bf16 inputs the kernels get.
 * The steps follow the order in which the pages state the problem:
 *
 *   store    "3.1 Project overview and the four-layer architecture", section 3
 *            (Layer 4: the attention layer first writes the new K/V into the
 *            cache, then runs attention) and section 4, step 4; "Nano-vLLM
 *            Architecture and Performance", Key Features 4 (store_kvcache writes
 *            KV entries into the paged cache blocks chosen by the slot mapping).
 *   gather   "nano-vllm" README, PagedAttention (a sequence's KV lives in
 *            fixed-size blocks allocated on demand, not contiguously);
 *            "Nano-vLLM Architecture and Performance", Key Features 2 and
 *            How It Works End-to-End (block tables and slot mappings).
 *   head map "nano-vllm" README, X-Ray Mode, step 1 (32 query heads share 8 KV
 *            heads, 4:1): query head h uses KV head h / (Hq / Hkv).
 *   scores   same page, X-Ray Mode, step 2: scores = Q K^T / sqrt(head_dim).
 *   mask     same page, Tutorial Mode chapter 3 (the causal mask: a token sees
 *            only itself and earlier tokens) and Features: Chunked Prefill (a
 *            chunk of new rows sits at the tail of its sequence, so row i of an
 *            n-row chunk is at absolute position L - n + i).
 *   softmax  exact softmax over the visible keys, then the weighted sum of V.
 *            The FlashAttention family (README, Features) only re-arranges this
 *            result, so the oracle is the plain definition.
 *
 *   rope     "Nano-vLLM Architecture and Performance", project structure
 *            (layers/rotary_embedding.py: RoPE, the rotary position embedding
 *            applied to q and k before the attention layer stores k).  The
 *            pages name the step only; oracle_rope states the rotary embedding
 *            of Su et al., "RoFormer" (2021), section 3.4, in the rotate-half
 *            pairing of dimension i with i + D/2 that Qwen3 uses.
 *
 * Readings where the pages are silent (each also listed in the design notes):
 *   - slot s addresses block s / block_size, offset s % block_size;
 *   - a negative slot is a padding row and writes nothing;
 *   - context_lens[b] counts the tokens stored by this step's store;
 *   - block-table entries past ceil(L_b / block_size) are never read.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

enum {
    ORACLE_OK = 0,
    ORACLE_ERR_ARG = 1,   /* a shape or pointer argument is invalid */
    ORACLE_ERR_DATA = 2,  /* a slot, block id or length is out of range */
    ORACLE_ERR_NOMEM = 3,
};

/* bf16 bit pattern -> double: the 16 bits are the top half of an fp32. */
static double bf16_to_double(uint16_t bits)
{
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

double oracle_bf16_to_double(uint16_t bits) { return bf16_to_double(bits); }

/*
 * Store: for every new token t with slot s = slot_mapping[t] >= 0, copy its
 * [Hkv, D] key row into k_pool[s / BS][s % BS] and its value row into v_pool.
 * key/value rows are kv_token_stride elements apart.  Bit-for-bit copy.
 */
int oracle_store_kvcache(const uint16_t *key, const uint16_t *value, int64_t kv_token_stride,
                         uint16_t *k_pool, uint16_t *v_pool, const int32_t *slot_mapping,
                         int32_t num_tokens, int32_t num_blocks, int32_t block_size,
                         int32_t num_kv_heads, int32_t head_dim)
{
    if (num_tokens < 0 || num_blocks <= 0 || block_size <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return ORACLE_ERR_ARG;
    if (num_tokens == 0)
        return ORACLE_OK;
    if (!key || !value || !k_pool || !v_pool || !slot_mapping)
        return ORACLE_ERR_ARG;
    const int64_t row = (int64_t)num_kv_heads * head_dim;
    if (kv_token_stride < row)
        return ORACLE_ERR_ARG;
    const int64_t num_slots = (int64_t)num_blocks * block_size;
    int status = ORACLE_OK;
    for (int32_t t = 0; t < num_tokens; ++t) {
        const int64_t s = slot_mapping[t];
        if (s < 0)
            continue;
        if (s >= num_slots) {
            status = ORACLE_ERR_DATA;
            continue;
        }
        const int64_t block = s / block_size;
        const int64_t offset = s % block_size;
        const int64_t dst = (block * block_size + offset) * row;
        memcpy(k_pool + dst, key + (int64_t)t * kv_token_stride, (size_t)row * sizeof(uint16_t));
        memcpy(v_pool + dst, value + (int64_t)t * kv_token_stride, (size_t)row * sizeof(uint16_t));
    }
    return status;
}

typedef struct {
    double *out;
    const uint16_t *q;
    const int32_t *cu_seqlens_q;
    const uint16_t *k_pool;
    const uint16_t *v_pool;
    const int32_t *block_tables;
    int32_t max_blocks_per_seq;
    const int32_t *context_lens;
    int32_t num_seqs, num_q_heads, num_kv_heads, head_dim, num_blocks, block_size;
    double scale;
    int64_t num_units;       /* total_q * num_q_heads */
    int64_t next_unit;       /* shared work counter */
    int32_t max_context_len;
    int error;
} attn_job;

/* Index of the sequence that owns packed query row r (cu_seqlens_q is nondecreasing). */
static int32_t seq_of_row(const attn_job *job, int64_t r)
{
    int32_t lo = 0, hi = job->num_seqs - 1;
    while (lo < hi) {
        int32_t mid = (lo + hi + 1) / 2;
        if (job->cu_seqlens_q[mid] <= r)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo;
}

/* One output row for query row r, query head hq. */
static int attend_row(const attn_job *job, int64_t r, int32_t hq, double *scores)
{
    const int32_t b = seq_of_row(job, r);
    const int32_t n_b = job->cu_seqlens_q[b + 1] - job->cu_seqlens_q[b];
    const int32_t L_b = job->context_lens[b];
    const int32_t i = (int32_t)(r - job->cu_seqlens_q[b]);
    const int32_t D = job->head_dim;
    const int32_t BS = job->block_size;

    /* head map: consecutive query heads share one KV head */
    const int32_t group = job->num_q_heads / job->num_kv_heads;
    const int32_t hk = hq / group;

    /* causal: row i of the n_b new rows sits at absolute position L_b - n_b + i */
    const int32_t pos = L_b - n_b + i;
    const int32_t visible = pos + 1;

    const uint16_t *qrow = job->q + (r * job->num_q_heads + hq) * (int64_t)D;
    double *orow = job->out + (r * job->num_q_heads + hq) * (int64_t)D;

    /* scores s_j = scale * <q, K_j> over the gathered keys j = 0 .. pos */
    for (int32_t j = 0; j < visible; ++j) {
        const int32_t blk = job->block_tables[(int64_t)b * job->max_blocks_per_seq + j / BS];
        if (blk < 0 || blk >= job->num_blocks)
            return ORACLE_ERR_DATA;
        const uint16_t *krow = job->k_pool + (((int64_t)blk * BS + j % BS) * job->num_kv_heads + hk) * D;
        double dot = 0.0;
        for (int32_t d = 0; d < D; ++d)
            dot += bf16_to_double(qrow[d]) * bf16_to_double(krow[d]);
        scores[j] = job->scale * dot;
    }

    /* softmax: subtract the maximum, exponentiate, normalise */
    double m = -INFINITY;
    for (int32_t j = 0; j < visible; ++j)
        if (scores[j] > m)
            m = scores[j];
    double denom = 0.0;
    for (int32_t j = 0; j < visible; ++j) {
        scores[j] = exp(scores[j] - m);
        denom += scores[j];
    }

    /* output o = sum_j p_j V_j / sum_j p_j */
    for (int32_t d = 0; d < D; ++d)
        orow[d] = 0.0;
    for (int32_t j = 0; j < visible; ++j) {
        const int32_t blk = job->block_tables[(int64_t)b * job->max_blocks_per_seq + j / BS];
        const uint16_t *vrow = job->v_pool + (((int64_t)blk * BS + j % BS) * job->num_kv_heads + hk) * D;
        for (int32_t d = 0; d < D; ++d)
            orow[d] += scores[j] * bf16_to_double(vrow[d]);
    }
    for (int32_t d = 0; d < D; ++d)
        orow[d] /= denom;
    return ORACLE_OK;
}

static void *attn_worker(void *arg)
{
    attn_job *job = (attn_job *)arg;
    double *scores = (double *)malloc(sizeof(double) * (size_t)(job->max_context_len > 0 ? job->max_context_len : 1));
    if (!scores) {
        __atomic_store_n(&job->error, ORACLE_ERR_NOMEM, __ATOMIC_RELAXED);
        return NULL;
    }
    for (;;) {
        int64_t u = __atomic_fetch_add(&job->next_unit, 1, __ATOMIC_RELAXED);
        if (u >= job->num_units)
            break;
        int rc = attend_row(job, u / job->num_q_heads, (int32_t)(u % job->num_q_heads), scores);
        if (rc != ORACLE_OK)
            __atomic_store_n(&job->error, rc, __ATOMIC_RELAXED);
    }
    free(scores);
    return NULL;
}

/*
 * Attention for packed query rows against the paged cache.
 *   out          [total_q, Hq, D] fp64 (written)
 *   q            [total_q, Hq, D] bf16 bits, rows of sequence b at
 *                cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1
 *   k/v_pool     [num_blocks, block_size, Hkv, D] bf16 bits
 *   block_tables [num_seqs, max_blocks_per_seq]
 *   context_lens [num_seqs], L_b (including this step's new rows)
 *   scale        <= 0 selects 1 / sqrt(head_dim)
 *   num_threads  worker threads over (row, query head) units
 * Decode is the case cu_seqlens_q = 0, 1, ..., num_seqs.
 */
int oracle_paged_attention(double *out, const uint16_t *q, const int32_t *cu_seqlens_q,
                           const uint16_t *k_pool, const uint16_t *v_pool,
                           const int32_t *block_tables, int32_t max_blocks_per_seq,
                           const int32_t *context_lens, int32_t num_seqs, int32_t num_q_heads,
                           int32_t num_kv_heads, int32_t head_dim, int32_t num_blocks,
                           int32_t block_size, double scale, int32_t num_threads)
{
    if (num_seqs < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 || num_blocks <= 0 ||
        block_size <= 0 || max_blocks_per_seq < 0)
        return ORACLE_ERR_ARG;
    if (num_q_heads % num_kv_heads != 0)
        return ORACLE_ERR_ARG;
    if (num_seqs == 0)
        return ORACLE_OK;
    if (!cu_seqlens_q || !context_lens)
        return ORACLE_ERR_ARG;

    int32_t max_ctx = 0;
    for (int32_t b = 0; b < num_seqs; ++b) {
        const int32_t n_b = cu_seqlens_q[b + 1] - cu_seqlens_q[b];
        const int32_t L_b = context_lens[b];
        if (n_b < 0 || L_b < n_b || (int64_t)L_b > (int64_t)max_blocks_per_seq * block_size)
            return ORACLE_ERR_DATA;
        if (L_b > max_ctx)
            max_ctx = L_b;
    }
    const int64_t total_q = cu_seqlens_q[num_seqs] - cu_seqlens_q[0];
    if (cu_seqlens_q[0] != 0)
        return ORACLE_ERR_ARG;
    if (total_q == 0)
        return ORACLE_OK;
    if (!out || !q || !k_pool || !v_pool || !block_tables)
        return ORACLE_ERR_ARG;

    attn_job job;
    memset(&job, 0, sizeof job);
    job.out = out;
    job.q = q;
    job.cu_seqlens_q = cu_seqlens_q;
    job.k_pool = k_pool;
    job.v_pool = v_pool;
    job.block_tables = block_tables;
    job.max_blocks_per_seq = max_blocks_per_seq;
    job.context_lens = context_lens;
    job.num_seqs = num_seqs;
    job.num_q_heads = num_q_heads;
    job.num_kv_heads = num_kv_heads;
    job.head_dim = head_dim;
    job.num_blocks = num_blocks;
    job.block_size = block_size;
    job.scale = scale > 0.0 ? scale : 1.0 / sqrt((double)head_dim);
    job.num_units = total_q * num_q_heads;
    job.next_unit = 0;
    job.max_context_len = max_ctx;
    job.error = ORACLE_OK;

    if (num_threads < 1)
        num_threads = 1;
    if (num_threads > 256)
        num_threads = 256;
    if ((int64_t)num_threads > job.num_units)
        num_threads = (int32_t)job.num_units;

    if (num_threads == 1) {
        attn_worker(&job);
    } else {
        pthread_t tid[256];
        int started = 0;
        for (int t = 0; t < num_threads; ++t) {
            if (pthread_create(&tid[t], NULL, attn_worker, &job) != 0)
                break;
            ++started;
        }
        if (started == 0)
            attn_worker(&job);
        for (int t = 0; t < started; ++t)
            pthread_join(tid[t], NULL);
    }
    return job.error;
}

/*
 * Rotary position embedding of num_tokens x num_heads rows of head_dim bf16
 * values (token rows token_stride elements apart), written to out as fp64
 * [num_tokens][num_heads][head_dim].  Token t sits at position p = positions[t];
 * for i < D/2 the pair (x[i], x[i + D/2]) is turned by the angle p * theta_i,
 * theta_i = base^(-2i/D):
 *     out[i]       = x[i] cos(p theta_i) - x[i + D/2] sin(p theta_i)
 *     out[i + D/2] = x[i + D/2] cos(p theta_i) + x[i] sin(p theta_i)
 * i.e. the complex number x[i] + j x[i + D/2] times exp(j p theta_i).
 */
int oracle_rope(double *out, const uint16_t *x, int64_t num_tokens, int32_t num_heads, int32_t head_dim,
                int64_t token_stride, const int32_t *positions, double base)
{
    if (num_tokens < 0 || num_heads <= 0 || head_dim <= 0 || head_dim % 2 != 0 || !(base > 0.0))
        return ORACLE_ERR_ARG;
    if (token_stride < (int64_t)num_heads * head_dim)
        return ORACLE_ERR_ARG;
    if (num_tokens == 0)
        return ORACLE_OK;
    if (!out || !x || !positions)
        return ORACLE_ERR_ARG;
    const int32_t half = head_dim / 2;
    for (int64_t t = 0; t < num_tokens; ++t) {
        const double p = (double)positions[t];
        for (int32_t i = 0; i < half; ++i) {
            const double theta = pow(base, -2.0 * (double)i / (double)head_dim);
            const double angle = p * theta;
            const double c = cos(angle), s = sin(angle);
            for (int32_t h = 0; h < num_heads; ++h) {
                const uint16_t *row = x + t * token_stride + (int64_t)h * head_dim;
                double *o = out + (t * num_heads + h) * (int64_t)head_dim;
                const double x1 = bf16_to_double(row[i]);
                const double x2 = bf16_to_double(row[i + half]);
                o[i] = x1 * c - x2 * s;
                o[i + half] = x2 * c + x1 * s;
            }
        }
    }
    return ORACLE_OK;
}

/*
 * The bf16 value nearest to v, ties to even (IEEE 754 round-to-nearest for an
 * 8-bit significand with fp32's exponent range); NaN gives the quiet NaN 0x7FC0
 * and magnitudes that round past the largest finite value give infinity.
 */
uint16_t oracle_double_to_bf16(double v)
{
    if (isnan(v))
        return 0x7FC0;
    const uint16_t sign = signbit(v) ? 0x8000 : 0;
    const double a = fabs(v);
    if (a == 0.0)
        return sign;
    int e;
    frexp(a, &e);          /* a = m 2^e with 0.5 <= m < 1 */
    int q = e - 8;         /* spacing of the 8-bit significands in [2^(e-1), 2^e) */
    if (q < -133)
        q = -133;          /* subnormal spacing, 2^-126 / 2^7 */
    const double y = ldexp(nearbyint(ldexp(a, -q)), q);
    if (y > ldexp(255.0, 120))  /* largest finite bf16: (2 - 2^-7) 2^127 */
        return sign | 0x7F80;
    const float f = (float)y;   /* exact: at most 8 significant bits */
    uint32_t u;
    memcpy(&u, &f, sizeof u);
    return (uint16_t)(sign | (u >> 16));
}
