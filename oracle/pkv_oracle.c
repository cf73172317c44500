/*
 * pkv_oracle.c -- plain, slow, obviously-correct CPU oracle for the paged
 * KV-cache decode hot path (TEST INFRASTRUCTURE ONLY).
 *
 * Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may
 * load this library.  The product path (paged_kv_cache_373_b200) never
 * imports, links or calls it, and it shares no code, header, table or
 * constant with the CUDA kernels.
 *
 * Everything is computed in fp64 from the stored bytes.  Each function names
 * the passage it follows:
 *   - per-token KV size      : zwxr.cn "PagedAttention 与 Continuous Batching"
 *                              section 一 (the 2 x layers x kv_heads x dim x bytes
 *                              formula and its Llama-2-7B / Llama-3-8B values)
 *   - slot / block addressing: same page, sections 3.1 (a token takes a slot
 *                              when produced) and 3.2 (logical -> physical
 *                              block table, e.g. 0->3, 1->11, 2->7)
 *   - decode attention       : thinkmoon.cn "PagedAttention不够用了之后",
 *                              section "PagedAttention 的计算优化" (gather the
 *                              sequence's blocks, q.K^T / sqrt(d), softmax, .V),
 *                              restricted to the sequence's logical length
 *                              (ttlab.hopto.org section 2: only the last block
 *                              holds unused slots)
 *   - block-wise softmax     : zwxr.cn section 3.3 (per-block max m and
 *                              normaliser l, rescale-merge, exactly equal to the
 *                              global softmax)
 *   - copy-on-write copy     : zwxr.cn section 3.4, ttlab.hopto.org section 2
 *                              "共享区块"
 *   - FP8 E4M3 cache         : zwxr.cn section 五 (--kv-cache-dtype fp8, E4M3);
 *                              the encoder is written from the bit format
 *                              (1 sign, 4 exponent bits with bias 7, 3 mantissa
 *                              bits, no infinities, S.1111.111 = NaN, max 448)
 *
 * Parity status of every function is pinned by tests/test_oracle_*.py (none is
 * "parity unpinned").
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { OR_F32 = 0, OR_F16 = 1, OR_BF16 = 2, OR_FP8_E4M3 = 3 };
enum { OR_OK = 0, OR_EINVAL = 1, OR_ERANGE = 2 };

/* ------------------------------------------------------------------------- */
/* number formats, written from their IEEE-754 / OCP bit layouts             */
/* ------------------------------------------------------------------------- */

/* Decode an IEEE-style binary format with `ebits` exponent bits and `mbits`
 * mantissa bits (sign in the top bit) into an exact double. */
static double ieee_decode(uint32_t bits, int ebits, int mbits)
{
    uint32_t sign = (bits >> (ebits + mbits)) & 1u;
    uint32_t e = (bits >> mbits) & ((1u << ebits) - 1u);
    uint32_t m = bits & ((1u << mbits) - 1u);
    int bias = (1 << (ebits - 1)) - 1;
    double v;
    if (e == (1u << ebits) - 1u)
        v = m ? NAN : INFINITY;
    else if (e == 0)
        v = ldexp((double)m, 1 - bias - mbits);           /* subnormal */
    else
        v = ldexp((double)((1u << mbits) | m), (int)e - bias - mbits);
    return sign ? -v : v;
}

/* Round-half-to-even of a non-negative double to an integer-valued double. */
static double rint_half_even(double a)
{
    double f = floor(a);
    double r = a - f;
    if (r > 0.5) return f + 1.0;
    if (r < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/* Encode a double into an IEEE-style binary format with round-to-nearest-even
 * and overflow to infinity (f16 / bf16 behaviour). */
static uint32_t ieee_encode_rne(double x, int ebits, int mbits)
{
    int bias = (1 << (ebits - 1)) - 1;
    uint32_t emax_field = (1u << ebits) - 1u;
    uint32_t sign = signbit(x) ? 1u : 0u;
    uint32_t sbit = sign << (ebits + mbits);
    if (isnan(x)) return sbit | (emax_field << mbits) | (1u << (mbits - 1));
    double a = fabs(x);
    if (isinf(a)) return sbit | (emax_field << mbits);
    int min_exp = 1 - bias;                              /* exponent of min normal */
    if (a < ldexp(1.0, min_exp)) {
        /* subnormal range: quantum 2^(min_exp - mbits) */
        double q = rint_half_even(ldexp(a, mbits - min_exp));
        return sbit | (uint32_t)q;                       /* q == 2^mbits is min normal */
    }
    int e;
    frexp(a, &e);                                        /* a = f * 2^e, f in [0.5,1) */
    e -= 1;                                              /* a in [2^e, 2^(e+1)) */
    double q = rint_half_even(ldexp(a, mbits - e));      /* in [2^mbits, 2^(mbits+1)] */
    if (q == ldexp(1.0, mbits + 1)) { q = ldexp(1.0, mbits); e += 1; }
    int ef = e + bias;
    if (ef >= (int)emax_field) return sbit | (emax_field << mbits); /* overflow -> inf */
    return sbit | ((uint32_t)ef << mbits) | ((uint32_t)q - (1u << mbits));
}

double oracle_f16_decode(uint16_t b) { return ieee_decode(b, 5, 10); }
double oracle_bf16_decode(uint16_t b) { return ieee_decode(b, 8, 7); }
uint16_t oracle_f16_encode(double x) { return (uint16_t)ieee_encode_rne(x, 5, 10); }
uint16_t oracle_bf16_encode(double x) { return (uint16_t)ieee_encode_rne(x, 8, 7); }

/* FP8 E4M3 ("fn" variant: no infinities, only S.1111.111 is NaN). */
double oracle_fp8_e4m3_decode(uint8_t b)
{
    uint32_t sign = (b >> 7) & 1u, e = (b >> 3) & 0xFu, m = b & 7u;
    double v;
    if (e == 0xF && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);                /* m/8 * 2^(1-7) */
    else v = ldexp((double)(8u | m), (int)e - 7 - 3);    /* (1+m/8) * 2^(e-7) */
    return sign ? -v : v;
}

/* Round-to-nearest-even with saturation to the largest finite value (+-448);
 * NaN maps to the canonical NaN 0x7F. */
uint8_t oracle_fp8_e4m3_encode(float xf)
{
    double x = (double)xf;
    if (isnan(x)) return 0x7F;
    uint8_t sbit = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (a >= 448.0) return sbit | 0x7E;                  /* satfinite */
    if (a < ldexp(1.0, -6)) {                            /* below min normal 2^-6 */
        double q = rint_half_even(ldexp(a, 9));          /* quantum 2^-9 */
        return sbit | (uint8_t)q;                        /* q == 8 is min normal */
    }
    int e;
    frexp(a, &e);
    e -= 1;                                              /* a in [2^e, 2^(e+1)) */
    double q = rint_half_even(ldexp(a, 3 - e));          /* in [8, 16] */
    if (q == 16.0) { q = 8.0; e += 1; }
    int ef = e + 7;
    uint8_t code = (uint8_t)((ef << 3) | ((int)q - 8));
    if (code > 0x7E) code = 0x7E;                        /* rounds above 448 */
    return sbit | code;
}

/* Exact widening of one stored element. */
static double load_elem(const void* base, int64_t idx, int dtype)
{
    switch (dtype) {
    case OR_F32: return (double)((const float*)base)[idx];
    case OR_F16: return oracle_f16_decode(((const uint16_t*)base)[idx]);
    case OR_BF16: return oracle_bf16_decode(((const uint16_t*)base)[idx]);
    case OR_FP8_E4M3: return oracle_fp8_e4m3_decode(((const uint8_t*)base)[idx]);
    default: return NAN;
    }
}

static int dtype_bytes(int dtype)
{
    switch (dtype) {
    case OR_F32: return 4;
    case OR_F16: case OR_BF16: return 2;
    case OR_FP8_E4M3: return 1;
    default: return 0;
    }
}

/* ------------------------------------------------------------------------- */
/* per-token KV size (zwxr.cn section 一)                                     */
/* ------------------------------------------------------------------------- */
int64_t oracle_kv_bytes_per_token(int layers, int kv_heads, int head_dim, int bytes)
{
    return (int64_t)2 * layers * kv_heads * head_dim * bytes;   /* K and V */
}

/* ------------------------------------------------------------------------- */
/* reshape_and_cache: write each new token's K/V into its slot               */
/* (zwxr.cn 3.1 / 3.2: slot = physical block * block_size + offset)           */
/* ------------------------------------------------------------------------- */
static void store_cache_elem(void* cache, int64_t idx, int cache_dtype, double x,
                             int src_dtype, float scale)
{
    switch (cache_dtype) {
    case OR_F32: ((float*)cache)[idx] = (float)x; break;            /* exact copy */
    case OR_F16: ((uint16_t*)cache)[idx] = oracle_f16_encode(x); break;
    case OR_BF16: ((uint16_t*)cache)[idx] = oracle_bf16_encode(x); break;
    case OR_FP8_E4M3: {
        /* x / scale in IEEE fp32 (the widened source value is exactly a float) */
        float xf = (float)x;
        volatile float q = xf / scale;
        (void)src_dtype;
        ((uint8_t*)cache)[idx] = oracle_fp8_e4m3_encode(q);
        break;
    }
    }
}

int oracle_reshape_and_cache(const void* key, const void* value, int src_dtype,
                             void* key_cache, void* value_cache, int cache_dtype,
                             const int64_t* slot_mapping, int64_t num_tokens,
                             int64_t num_blocks, int block_size, int num_kv_heads,
                             int head_dim, float k_scale, float v_scale)
{
    if (cache_dtype != OR_FP8_E4M3 && cache_dtype != src_dtype) return OR_EINVAL;
    int64_t row = (int64_t)num_kv_heads * head_dim;
    for (int64_t i = 0; i < num_tokens; ++i) {
        int64_t slot = slot_mapping[i];
        if (slot < 0) continue;                            /* padding token */
        if (slot >= num_blocks * block_size) return OR_ERANGE;
        int64_t blk = slot / block_size, off = slot % block_size;
        int64_t dst = (blk * block_size + off) * row;     /* [NB, bs, Hkv, D] */
        if (cache_dtype == src_dtype) {                   /* same dtype: a byte copy */
            size_t nb = (size_t)row * dtype_bytes(src_dtype);
            memcpy((char*)key_cache + dst * dtype_bytes(src_dtype),
                   (const char*)key + i * row * dtype_bytes(src_dtype), nb);
            memcpy((char*)value_cache + dst * dtype_bytes(src_dtype),
                   (const char*)value + i * row * dtype_bytes(src_dtype), nb);
            continue;
        }
        for (int64_t j = 0; j < row; ++j) {
            store_cache_elem(key_cache, dst + j, cache_dtype,
                             load_elem(key, i * row + j, src_dtype), src_dtype, k_scale);
            store_cache_elem(value_cache, dst + j, cache_dtype,
                             load_elem(value, i * row + j, src_dtype), src_dtype, v_scale);
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* copy_blocks: copy-on-write duplication of whole blocks (zwxr.cn 3.4)       */
/* ------------------------------------------------------------------------- */
int oracle_copy_blocks(void* const* key_caches, void* const* value_caches, int num_layers,
                       const int64_t* block_mapping, int64_t num_pairs,
                       int64_t block_bytes, int64_t num_blocks)
{
    for (int64_t p = 0; p < num_pairs; ++p) {
        int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
        if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) return OR_ERANGE;
        for (int l = 0; l < num_layers; ++l) {
            memcpy((char*)key_caches[l] + dst * block_bytes,
                   (const char*)key_caches[l] + src * block_bytes, (size_t)block_bytes);
            memcpy((char*)value_caches[l] + dst * block_bytes,
                   (const char*)value_caches[l] + src * block_bytes, (size_t)block_bytes);
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* swap_blocks: whole blocks from one pool to another (zwxr.cn 4.3, swapping   */
/* a preempted sequence's KV blocks out to host memory and back in)           */
/* ------------------------------------------------------------------------- */
int oracle_swap_blocks(void* const* dst_key_caches, void* const* dst_value_caches,
                       int64_t dst_num_blocks, void* const* src_key_caches,
                       void* const* src_value_caches, int64_t src_num_blocks, int num_layers,
                       const int64_t* block_mapping, int64_t num_pairs, int64_t block_bytes)
{
    for (int64_t p = 0; p < num_pairs; ++p) {
        int64_t src = block_mapping[2 * p], dst = block_mapping[2 * p + 1];
        if (src < 0 || src >= src_num_blocks || dst < 0 || dst >= dst_num_blocks) return OR_ERANGE;
        for (int l = 0; l < num_layers; ++l) {
            memcpy((char*)dst_key_caches[l] + dst * block_bytes,
                   (const char*)src_key_caches[l] + src * block_bytes, (size_t)block_bytes);
            memcpy((char*)dst_value_caches[l] + dst * block_bytes,
                   (const char*)src_value_caches[l] + src * block_bytes, (size_t)block_bytes);
        }
    }
    return OR_OK;
}

/* ------------------------------------------------------------------------- */
/* decode attention (thinkmoon.cn pseudocode, masked to the logical length)   */
/* ------------------------------------------------------------------------- */

/* Gather sequence s's first L token rows for one kv head into contiguous
 * fp64 arrays K[L][D], V[L][D] through the block table. */
static int gather_sequence(double* K, double* V, const void* key_cache, const void* value_cache,
                           int cache_dtype, const int32_t* table_row, int L, int block_size,
                           int64_t num_blocks, int num_kv_heads, int kvh, int head_dim,
                           double ks, double vs)
{
    for (int t = 0; t < L; ++t) {
        int32_t phys = table_row[t / block_size];        /* logical block -> physical */
        int off = t % block_size;
        if (phys < 0 || phys >= num_blocks) return OR_ERANGE;
        int64_t base = (((int64_t)phys * block_size + off) * num_kv_heads + kvh) * head_dim;
        for (int d = 0; d < head_dim; ++d) {
            K[(int64_t)t * head_dim + d] = load_elem(key_cache, base + d, cache_dtype) * ks;
            V[(int64_t)t * head_dim + d] = load_elem(value_cache, base + d, cache_dtype) * vs;
        }
    }
    return OR_OK;
}

/* softmax(scale * q.K^T) . V over L rows, fp64; writes out[D].  L == 0 -> 0. */
static void attend(double* out, const double* q, const double* K, const double* V, int L,
                   int head_dim, double scale, double* score)
{
    if (L == 0) { for (int d = 0; d < head_dim; ++d) out[d] = 0.0; return; }
    double m = -INFINITY;
    for (int t = 0; t < L; ++t) {
        double acc = 0.0;
        for (int d = 0; d < head_dim; ++d) acc += q[d] * K[(int64_t)t * head_dim + d];
        score[t] = scale * acc;
        if (score[t] > m) m = score[t];
    }
    double denom = 0.0;
    for (int t = 0; t < L; ++t) { score[t] = exp(score[t] - m); denom += score[t]; }
    for (int d = 0; d < head_dim; ++d) {
        double acc = 0.0;
        for (int t = 0; t < L; ++t) acc += score[t] * V[(int64_t)t * head_dim + d];
        out[d] = acc / denom;
    }
}

/*
 * out      : fp64 [num_seqs, num_heads, head_dim]; only the rows of the
 *            sequences listed in seq_subset are written (all when n_subset < 0)
 * q        : [num_seqs, num_heads, head_dim] in q_dtype
 * caches   : [num_blocks, block_size, num_kv_heads, head_dim] in cache_dtype
 * FP8      : element value = decode(code) * k_scale (resp. v_scale)
 * GQA      : q head h reads kv head h / (num_heads / num_kv_heads)
 */
int oracle_paged_attention_decode(double* out, const void* q, int q_dtype,
                                  const void* key_cache, const void* value_cache, int cache_dtype,
                                  const int32_t* block_tables, int max_blocks_per_seq,
                                  const int32_t* seq_lens, int num_seqs, int num_heads,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int64_t num_blocks, double scale, float k_scale, float v_scale,
                                  const int32_t* seq_subset, int n_subset, int num_threads)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0) return OR_EINVAL;
    if (dtype_bytes(q_dtype) == 0 || dtype_bytes(cache_dtype) == 0) return OR_EINVAL;
    int g = num_heads / num_kv_heads;
    int n = n_subset < 0 ? num_seqs : n_subset;
    double ks = cache_dtype == OR_FP8_E4M3 ? (double)k_scale : 1.0;
    double vs = cache_dtype == OR_FP8_E4M3 ? (double)v_scale : 1.0;
    int status = OR_OK;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int i = 0; i < n; ++i) {
        int s = n_subset < 0 ? i : seq_subset[i];
        int L = seq_lens[s];
        if (L < 0 || (int64_t)(L + block_size - 1) / block_size > max_blocks_per_seq) {
            status = OR_ERANGE;
            continue;
        }
        double* K = (double*)malloc(sizeof(double) * ((size_t)L * head_dim + 1));
        double* V = (double*)malloc(sizeof(double) * ((size_t)L * head_dim + 1));
        double* score = (double*)malloc(sizeof(double) * ((size_t)L + 1));
        double* qh = (double*)malloc(sizeof(double) * (size_t)head_dim);
        for (int kvh = 0; kvh < num_kv_heads; ++kvh) {
            if (gather_sequence(K, V, key_cache, value_cache, cache_dtype,
                                block_tables + (int64_t)s * max_blocks_per_seq, L, block_size,
                                num_blocks, num_kv_heads, kvh, head_dim, ks, vs) != OR_OK) {
                status = OR_ERANGE;
                break;
            }
            for (int h = kvh * g; h < (kvh + 1) * g; ++h) {
                int64_t qo = ((int64_t)s * num_heads + h) * head_dim;
                for (int d = 0; d < head_dim; ++d) qh[d] = load_elem(q, qo + d, q_dtype);
                attend(out + qo, qh, K, V, L, head_dim, scale, score);
            }
        }
        free(K); free(V); free(score); free(qh);
    }
    return status;
}

/*
 * Chunked prefill (ttlab.hopto.org "LLM KV cache 02", section 3, "新问题：
 * 长 Prefill 会暂停解码": a long prompt is cut into chunks processed over
 * several steps).  Sequence s contributes the C_s = query_start[s+1] -
 * query_start[s] query rows of its current chunk; its cache already holds
 * all seq_lens[s] tokens (the context and this chunk), so the chunk's i-th
 * token sits at position p = seq_lens[s] - C_s + i and attends to the
 * cached tokens t <= p (causal attention through the block table).
 * out  : fp64 [T, num_heads, head_dim], T = query_start[num_seqs]
 * q    : [T, num_heads, head_dim] in q_dtype; other arguments as decode.
 */
int oracle_paged_prefill(double* out, const void* q, int q_dtype,
                         const void* key_cache, const void* value_cache, int cache_dtype,
                         const int32_t* block_tables, int max_blocks_per_seq,
                         const int32_t* seq_lens, const int32_t* query_start, int num_seqs,
                         int num_heads, int num_kv_heads, int head_dim, int block_size,
                         int64_t num_blocks, double scale, float k_scale, float v_scale,
                         int num_threads)
{
    if (num_kv_heads <= 0 || num_heads % num_kv_heads != 0) return OR_EINVAL;
    if (dtype_bytes(q_dtype) == 0 || dtype_bytes(cache_dtype) == 0) return OR_EINVAL;
    int g = num_heads / num_kv_heads;
    double ks = cache_dtype == OR_FP8_E4M3 ? (double)k_scale : 1.0;
    double vs = cache_dtype == OR_FP8_E4M3 ? (double)v_scale : 1.0;
    int status = OR_OK;
#ifdef _OPENMP
    if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (int s = 0; s < num_seqs; ++s) {
        int L = seq_lens[s];
        int C = query_start[s + 1] - query_start[s];
        if (L < 0 || C < 0 || C > L ||
            (int64_t)(L + block_size - 1) / block_size > max_blocks_per_seq) {
            status = OR_ERANGE;
            continue;
        }
        double* K = (double*)malloc(sizeof(double) * ((size_t)L * head_dim + 1));
        double* V = (double*)malloc(sizeof(double) * ((size_t)L * head_dim + 1));
        double* score = (double*)malloc(sizeof(double) * ((size_t)L + 1));
        double* qh = (double*)malloc(sizeof(double) * (size_t)head_dim);
        for (int kvh = 0; kvh < num_kv_heads; ++kvh) {
            if (gather_sequence(K, V, key_cache, value_cache, cache_dtype,
                                block_tables + (int64_t)s * max_blocks_per_seq, L, block_size,
                                num_blocks, num_kv_heads, kvh, head_dim, ks, vs) != OR_OK) {
                status = OR_ERANGE;
                break;
            }
            for (int i = 0; i < C; ++i) {
                int64_t row = (int64_t)query_start[s] + i;
                int pos = L - C + i;                      /* the token's position */
                for (int h = kvh * g; h < (kvh + 1) * g; ++h) {
                    int64_t qo = (row * num_heads + h) * head_dim;
                    for (int d = 0; d < head_dim; ++d) qh[d] = load_elem(q, qo + d, q_dtype);
                    attend(out + qo, qh, K, V, pos + 1, head_dim, scale, score);  /* t <= pos */
                }
            }
        }
        free(K); free(V); free(score); free(qh);
    }
    return status;
}

/*
 * Block-wise softmax (zwxr.cn 3.3): the L rows are cut into partitions of
 * `part` tokens; each partition keeps its own max m_p, normaliser
 * l_p = sum exp(s - m_p) and unnormalised o_p = sum exp(s - m_p) v; the
 * partitions are then merged with M = max m_p:
 *   out = sum_p exp(m_p - M) o_p / sum_p exp(m_p - M) l_p.
 * Used by the tests to pin that this merge equals the global softmax.
 * One (sequence, head) at a time: q[D], K[L][D], V[L][D] already contiguous.
 */
int oracle_blockwise_attend(double* out, const double* q, const double* K, const double* V,
                            int L, int head_dim, double scale, int part)
{
    if (part <= 0) return OR_EINVAL;
    if (L == 0) { for (int d = 0; d < head_dim; ++d) out[d] = 0.0; return OR_OK; }
    int np = (L + part - 1) / part;
    double* m = (double*)malloc(sizeof(double) * np);
    double* l = (double*)malloc(sizeof(double) * np);
    double* o = (double*)calloc((size_t)np * head_dim, sizeof(double));
    double* sc = (double*)malloc(sizeof(double) * part);
    for (int p = 0; p < np; ++p) {
        int t0 = p * part, t1 = t0 + part < L ? t0 + part : L;
        m[p] = -INFINITY;
        for (int t = t0; t < t1; ++t) {
            double acc = 0.0;
            for (int d = 0; d < head_dim; ++d) acc += q[d] * K[(int64_t)t * head_dim + d];
            sc[t - t0] = scale * acc;
            if (sc[t - t0] > m[p]) m[p] = sc[t - t0];
        }
        l[p] = 0.0;
        for (int t = t0; t < t1; ++t) {
            double e = exp(sc[t - t0] - m[p]);
            l[p] += e;
            for (int d = 0; d < head_dim; ++d) o[(int64_t)p * head_dim + d] += e * V[(int64_t)t * head_dim + d];
        }
    }
    double M = -INFINITY;
    for (int p = 0; p < np; ++p) if (m[p] > M) M = m[p];
    double denom = 0.0;
    for (int p = 0; p < np; ++p) denom += exp(m[p] - M) * l[p];
    for (int d = 0; d < head_dim; ++d) {
        double acc = 0.0;
        for (int p = 0; p < np; ++p) acc += exp(m[p] - M) * o[(int64_t)p * head_dim + d];
        out[d] = acc / denom;
    }
    free(m); free(l); free(o); free(sc);
    return OR_OK;
}

/* Plain contiguous attention for one (sequence, head): the global softmax
 * reference the block-wise merge is compared with. */
int oracle_contiguous_attend(double* out, const double* q, const double* K, const double* V,
                             int L, int head_dim, double scale)
{
    double* score = (double*)malloc(sizeof(double) * ((size_t)L + 1));
    attend(out, q, K, V, L, head_dim, scale, score);
    free(score);
    return OR_OK;
}

int oracle_num_threads_available(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* Exported gather (zwxr.cn 3.2 translation) so the tests can pin the
 * logical -> physical indexing on its own: K/V rows t = 0..L-1 of kv head
 * `kvh` of the sequence whose table row is `table_row`, widened to fp64. */
int oracle_gather_kv(double* K, double* V, const void* key_cache, const void* value_cache,
                     int cache_dtype, const int32_t* table_row, int L, int block_size,
                     int64_t num_blocks, int num_kv_heads, int kvh, int head_dim,
                     float k_scale, float v_scale)
{
    double ks = cache_dtype == OR_FP8_E4M3 ? (double)k_scale : 1.0;
    double vs = cache_dtype == OR_FP8_E4M3 ? (double)v_scale : 1.0;
    return gather_sequence(K, V, key_cache, value_cache, cache_dtype, table_row, L, block_size,
                           num_blocks, num_kv_heads, kvh, head_dim, ks, vs);
}
