/*
 * Oracle for the paged KV-cache decode path: plain, slow, fp64, CPU only.
 *
 * TEST INFRASTRUCTURE. Only the test suite, the smoke check and the CPU
 * baseline leg of the benchmark may load this library. It shares no code,
 * header, table or helper with the CUDA library; the two meet only through
 * the seeded inputs the tests hand to both.
 *
 * What it follows (cited as page title + section):
 *  - "别再让GPU内存拖后腿了：vLLM的PagedAttention如何像操作系统一样管理KV Cache",
 *    section 3.1 (分块注意力计算), the paged_attention code: for every page in the
 *    sequence's page table, score the query against that page; concatenate the
 *    page scores; softmax(scores / sqrt(dim)); then the output is the sum over
 *    pages of (that page's slice of the weights) @ (that page).
 *  - same page, section 2.1 (分页式存储架构): fixed-size pages in one physical
 *    pool reached through a per-sequence page table.
 *  - "vLLM架构深度解析：PagedAttention如何实现高吞吐LLM推理", section PagedAttention:
 *    blocks hold the keys and values of a fixed number of tokens (usually 16)
 *    and need not be contiguous; section KV Cache内存共享: copy-on-write copies a
 *    shared block before a sequence appends to it.
 *  - "VLLM ... PageAttention 分页 KV Cache ..." (m.nxbn.cn), section 一: decode
 *    computes only the new token's K/V, appends it to the cache, then attends.
 *
 * Readings where the pages are silent or garbled (each one is listed in the
 * design notes of the repository):
 *  - K and V live in two pools [num_blocks][num_kv_heads][block_size][head_dim];
 *    the printed code uses one tensor for both and leaves seq_id undefined.
 *  - Only the first context_len tokens count; the printed code scores whole
 *    pages, which would include unwritten tail slots.
 *  - The scale is an argument (the configurations pass 1/sqrt(head_dim)).
 *  - Grouped-query attention: query head h reads KV head h / (H / H_kv).
 *  - context_len == 0 gives a zero output row.
 *  - 8-bit caches (section 3.2 of the first page, 内存压缩技术): one scale per
 *    tensor, per KV head, or per (physical block, KV head); a block's scale
 *    applies to every token written into that block.
 *
 * Element formats: fp16 is IEEE 754 binary16; bf16 is the upper half of an
 * IEEE 754 binary32. Both are decoded here from their bit fields.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

enum { ORACLE_F16 = 0, ORACLE_BF16 = 1 };

/* Decode one 16-bit element to double, from the bit-field definitions. */
double oracle_to_double(uint16_t bits, int dtype)
{
    int sign = (bits >> 15) & 1;
    double mag;
    if (dtype == ORACLE_F16) {
        int e = (bits >> 10) & 0x1f;      /* 5-bit exponent, bias 15 */
        int m = bits & 0x3ff;             /* 10-bit fraction */
        if (e == 0)
            mag = ldexp((double)m, -24);  /* subnormal: m * 2^(1-15-10) */
        else if (e == 31)
            mag = m ? NAN : INFINITY;
        else
            mag = ldexp((double)(m + 1024), e - 25);
    } else {
        int e = (bits >> 7) & 0xff;       /* 8-bit exponent, bias 127 */
        int m = bits & 0x7f;              /* 7-bit fraction */
        if (e == 0)
            mag = ldexp((double)m, -133); /* subnormal: m * 2^(1-127-7) */
        else if (e == 255)
            mag = m ? NAN : INFINITY;
        else
            mag = ldexp((double)(m + 128), e - 134);
    }
    return sign ? -mag : mag;
}

/*
 * 8-bit E4M3 ("fp8 e4m3fn"): 1 sign bit, 4 exponent bits (bias 7), 3 fraction
 * bits, no infinities, one NaN pattern per sign (exponent and fraction all
 * ones), largest finite magnitude 448. Quantised KV cache of
 * "别再让GPU内存拖后腿了：vLLM的PagedAttention如何像操作系统一样管理KV Cache",
 * section 3.2 (内存压缩技术: store K/V in fewer bits). Decoded here from the
 * bit fields.
 */
double oracle_e4m3_to_double(uint8_t code)
{
    const int sign = (code >> 7) & 1;
    const int e = (code >> 3) & 0xf;
    const int m = code & 7;
    double mag;
    if (e == 15 && m == 7)
        mag = NAN;
    else if (e == 0)
        mag = ldexp((double)m, -9);          /* subnormal: m * 2^(1-7-3) */
    else
        mag = ldexp((double)(m + 8), e - 10);
    return sign ? -mag : mag;
}

/*
 * Nearest E4M3 code to y, ties to even, magnitudes past 448 saturated to 448
 * (NaN stays NaN). Works on the value exactly (y is a float, so y * 2^k is
 * exact in double).
 */
uint8_t oracle_e4m3_encode(float y)
{
    if (isnan(y))
        return 0x7f;
    const uint8_t sign = signbit(y) ? 0x80 : 0;
    double a = fabs((double)y);
    if (a >= 464.0)                         /* rounds past 448: saturate */
        return sign | 0x7e;
    int e;
    if (a < ldexp(1.0, -6)) {               /* subnormal range, step 2^-9 */
        double q = a * 512.0;
        double r = floor(q);
        double f = q - r;
        if (f > 0.5 || (f == 0.5 && fmod(r, 2.0) == 1.0))
            r += 1.0;
        return sign | (uint8_t)r;           /* r == 8 is the smallest normal */
    }
    frexp(a, &e);                           /* a = f * 2^e, f in [0.5, 1) */
    e -= 1;                                 /* a in [2^e, 2^(e+1)) */
    double q = ldexp(a, 3 - e);             /* in [8, 16): 8 + fraction * 8 */
    double r = floor(q);
    double f = q - r;
    if (f > 0.5 || (f == 0.5 && fmod(r, 2.0) == 1.0))
        r += 1.0;
    if (r == 16.0) {
        r = 8.0;
        e += 1;
    }
    if (e > 8 || (e == 8 && r > 14.0))      /* above 448 after rounding */
        return sign | 0x7e;
    return sign | (uint8_t)(((e + 7) << 3) | ((int)r - 8));
}

int oracle_max_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/*
 * Paged decode attention.
 *   out          [num_seqs][num_heads][head_dim]          fp64 result
 *   q            [num_seqs][num_heads][head_dim]          16-bit elements
 *   k_pool,v_pool[num_blocks][num_kv_heads][block_size][head_dim]
 *   block_tables [num_seqs][max_blocks_per_seq]           physical page ids
 *   context_lens [num_seqs]
 * num_threads > 0 sets the OpenMP thread count; the (sequence, head) pairs are
 * independent, so threads only split that outer loop.
 */
void oracle_paged_attention(double *out, const uint16_t *q,
                            const uint16_t *k_pool, const uint16_t *v_pool,
                            const int32_t *block_tables, const int32_t *context_lens,
                            int num_seqs, int num_heads, int num_kv_heads,
                            int head_dim, int block_size, int max_blocks_per_seq,
                            double scale, int dtype, int num_threads)
{
    const int group = num_heads / num_kv_heads;
    const long pairs = (long)num_seqs * num_heads;
#ifdef _OPENMP
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long sh = 0; sh < pairs; sh++) {
        const int s = (int)(sh / num_heads);
        const int h = (int)(sh % num_heads);
        const int kvh = h / group;
        const int n = context_lens[s];
        double *o = out + (size_t)sh * head_dim;
        for (int d = 0; d < head_dim; d++)
            o[d] = 0.0;
        if (n <= 0)
            continue;

        double *qd = (double *)malloc(sizeof(double) * head_dim);
        double *scores = (double *)malloc(sizeof(double) * n);
        for (int d = 0; d < head_dim; d++)
            qd[d] = oracle_to_double(q[(size_t)sh * head_dim + d], dtype);

        const int pages = (n + block_size - 1) / block_size;
        const int32_t *table = block_tables + (size_t)s * max_blocks_per_seq;

        /* Page by page: scores of the query against the page's valid keys,
           appended in logical order (the concatenation). */
        for (int i = 0; i < pages; i++) {
            const size_t page = (size_t)table[i];
            for (int r = 0; r < block_size; r++) {
                const int t = i * block_size + r;
                if (t >= n)
                    break;
                const uint16_t *key =
                    k_pool + ((page * num_kv_heads + kvh) * block_size + r) * head_dim;
                double dot = 0.0;
                for (int d = 0; d < head_dim; d++)
                    dot += qd[d] * oracle_to_double(key[d], dtype);
                scores[t] = dot;
            }
        }

        /* softmax(scale * scores) over the concatenated scores. */
        double mx = -INFINITY;
        for (int t = 0; t < n; t++)
            if (scale * scores[t] > mx)
                mx = scale * scores[t];
        double total = 0.0;
        for (int t = 0; t < n; t++) {
            scores[t] = exp(scale * scores[t] - mx);
            total += scores[t];
        }
        for (int t = 0; t < n; t++)
            scores[t] /= total;

        /* Page by page: that page's slice of the weights times its values. */
        for (int i = 0; i < pages; i++) {
            const size_t page = (size_t)table[i];
            for (int r = 0; r < block_size; r++) {
                const int t = i * block_size + r;
                if (t >= n)
                    break;
                const uint16_t *val =
                    v_pool + ((page * num_kv_heads + kvh) * block_size + r) * head_dim;
                for (int d = 0; d < head_dim; d++)
                    o[d] += scores[t] * oracle_to_double(val[d], dtype);
            }
        }
        free(scores);
        free(qd);
    }
}

/*
 * Paged decode attention over an E4M3 KV cache: the same computation as
 * oracle_paged_attention with every key element k_scale * decode(code) and
 * every value element v_scale * decode(code), in fp64.
 */
void oracle_paged_attention_fp8(double *out, const uint16_t *q,
                                const uint8_t *k_pool, const uint8_t *v_pool,
                                const int32_t *block_tables, const int32_t *context_lens,
                                int num_seqs, int num_heads, int num_kv_heads,
                                int head_dim, int block_size, int max_blocks_per_seq,
                                double scale, int q_dtype, double k_scale, double v_scale,
                                int num_threads)
{
    const int group = num_heads / num_kv_heads;
    const long pairs = (long)num_seqs * num_heads;
#ifdef _OPENMP
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long sh = 0; sh < pairs; sh++) {
        const int s = (int)(sh / num_heads);
        const int h = (int)(sh % num_heads);
        const int kvh = h / group;
        const int n = context_lens[s];
        double *o = out + (size_t)sh * head_dim;
        for (int d = 0; d < head_dim; d++)
            o[d] = 0.0;
        if (n <= 0)
            continue;
        double *qd = (double *)malloc(sizeof(double) * head_dim);
        double *scores = (double *)malloc(sizeof(double) * n);
        for (int d = 0; d < head_dim; d++)
            qd[d] = oracle_to_double(q[(size_t)sh * head_dim + d], q_dtype);
        const int pages = (n + block_size - 1) / block_size;
        const int32_t *table = block_tables + (size_t)s * max_blocks_per_seq;
        for (int i = 0; i < pages; i++) {
            const size_t page = (size_t)table[i];
            for (int r = 0; r < block_size; r++) {
                const int t = i * block_size + r;
                if (t >= n)
                    break;
                const uint8_t *key = k_pool + ((page * num_kv_heads + kvh) * block_size + r) * head_dim;
                double dot = 0.0;
                for (int d = 0; d < head_dim; d++)
                    dot += qd[d] * (k_scale * oracle_e4m3_to_double(key[d]));
                scores[t] = dot;
            }
        }
        double mx = -INFINITY;
        for (int t = 0; t < n; t++)
            if (scale * scores[t] > mx)
                mx = scale * scores[t];
        double total = 0.0;
        for (int t = 0; t < n; t++) {
            scores[t] = exp(scale * scores[t] - mx);
            total += scores[t];
        }
        for (int t = 0; t < n; t++)
            scores[t] /= total;
        for (int i = 0; i < pages; i++) {
            const size_t page = (size_t)table[i];
            for (int r = 0; r < block_size; r++) {
                const int t = i * block_size + r;
                if (t >= n)
                    break;
                const uint8_t *val = v_pool + ((page * num_kv_heads + kvh) * block_size + r) * head_dim;
                for (int d = 0; d < head_dim; d++)
                    o[d] += scores[t] * (v_scale * oracle_e4m3_to_double(val[d]));
            }
        }
        free(scores);
        free(qd);
    }
}

/*
 * Quantising cache write: like oracle_reshape_and_cache, but each element x
 * (fp16/bf16) is stored as oracle_e4m3_encode(x / scale) with the division in
 * fp32 (float operands, IEEE single, round to nearest).
 */
void oracle_reshape_and_cache_fp8(const uint16_t *k, const uint16_t *v,
                                  uint8_t *k_pool, uint8_t *v_pool,
                                  const int64_t *slot_mapping, int num_tokens,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int dtype, float k_scale, float v_scale)
{
    for (int t = 0; t < num_tokens; t++) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        const int64_t block = slot / block_size;
        const int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; h++) {
            const size_t src = ((size_t)t * num_kv_heads + h) * head_dim;
            const size_t dst = (((size_t)block * num_kv_heads + h) * block_size + offset) * head_dim;
            for (int d = 0; d < head_dim; d++) {
                const float kx = (float)oracle_to_double(k[src + d], dtype);
                const float vx = (float)oracle_to_double(v[src + d], dtype);
                k_pool[dst + d] = oracle_e4m3_encode(kx / k_scale);
                v_pool[dst + d] = oracle_e4m3_encode(vx / v_scale);
            }
        }
    }
}

/*
 * 8-bit signed integer KV cache, the INT8 row of the compression table of
 * "别再让GPU内存拖后腿了：vLLM的PagedAttention如何像操作系统一样管理KV Cache",
 * section 3.2 (内存压缩技术; section 4.3 applies it to older pages). Stored
 * excess-128: byte u holds the integer u - 128. An element x with scale s is
 * stored as clamp(round(x / s), -127, 127) + 128, the rounding to nearest with
 * ties to even, the division in fp32 (float operands, IEEE single). NaN stores
 * 128 (zero); infinities clamp.
 */
double oracle_int8_to_double(uint8_t code)
{
    return (double)code - 128.0;
}

uint8_t oracle_int8_encode(float y)
{
    if (isnan(y))
        return 128;
    if (y >= 127.0f)
        return 255;
    if (y <= -127.0f)
        return 1;
    const double a = (double)y;
    double r = floor(a);
    const double f = a - r;                 /* exact: |a| < 127 */
    if (f > 0.5 || (f == 0.5 && fmod(r, 2.0) != 0.0))
        r += 1.0;
    return (uint8_t)(int)(r + 128.0);
}

enum { ORACLE_KV_E4M3 = 0, ORACLE_KV_INT8 = 1 };

static double kv8_to_double(uint8_t code, int format)
{
    return format == ORACLE_KV_INT8 ? oracle_int8_to_double(code) : oracle_e4m3_to_double(code);
}

/*
 * The scale of KV head kvh of physical block `page`: one per (block, KV head)
 * ([num_blocks][num_kv_heads] arrays) when per_block, else one per KV head.
 */
static double kv8_scale(const double *scales, int per_block, size_t page, int kvh, int num_kv_heads)
{
    return per_block ? scales[page * (size_t)num_kv_heads + kvh] : scales[kvh];
}

static void paged_attention_kv8(double *out, const uint16_t *q,
                                const uint8_t *k_pool, const uint8_t *v_pool,
                                const int32_t *block_tables, const int32_t *context_lens,
                                int num_seqs, int num_heads, int num_kv_heads,
                                int head_dim, int block_size, int max_blocks_per_seq,
                                double scale, int q_dtype, int format,
                                const double *k_scales, const double *v_scales, int per_block,
                                int num_threads);

/*
 * Paged decode attention over an 8-bit KV cache (E4M3 or INT8 codes) with one
 * scale per KV head: key element of KV head j = k_scales[j] * decode(code),
 * value element = v_scales[j] * decode(code). Otherwise the computation of
 * oracle_paged_attention, in fp64.
 */
void oracle_paged_attention_kv8(double *out, const uint16_t *q,
                                const uint8_t *k_pool, const uint8_t *v_pool,
                                const int32_t *block_tables, const int32_t *context_lens,
                                int num_seqs, int num_heads, int num_kv_heads,
                                int head_dim, int block_size, int max_blocks_per_seq,
                                double scale, int q_dtype, int format,
                                const double *k_scales, const double *v_scales, int num_threads)
{
    paged_attention_kv8(out, q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads, num_kv_heads,
                        head_dim, block_size, max_blocks_per_seq, scale, q_dtype, format, k_scales, v_scales, 0,
                        num_threads);
}

/*
 * The same with one scale per (physical block, KV head): the key element of KV
 * head j in block b = k_scales[b * num_kv_heads + j] * decode(code), the value
 * element likewise with v_scales.
 */
void oracle_paged_attention_kv8_blocks(double *out, const uint16_t *q,
                                       const uint8_t *k_pool, const uint8_t *v_pool,
                                       const int32_t *block_tables, const int32_t *context_lens,
                                       int num_seqs, int num_heads, int num_kv_heads,
                                       int head_dim, int block_size, int max_blocks_per_seq,
                                       double scale, int q_dtype, int format,
                                       const double *k_scales, const double *v_scales, int num_threads)
{
    paged_attention_kv8(out, q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads, num_kv_heads,
                        head_dim, block_size, max_blocks_per_seq, scale, q_dtype, format, k_scales, v_scales, 1,
                        num_threads);
}

static void paged_attention_kv8(double *out, const uint16_t *q,
                                const uint8_t *k_pool, const uint8_t *v_pool,
                                const int32_t *block_tables, const int32_t *context_lens,
                                int num_seqs, int num_heads, int num_kv_heads,
                                int head_dim, int block_size, int max_blocks_per_seq,
                                double scale, int q_dtype, int format,
                                const double *k_scales, const double *v_scales, int per_block,
                                int num_threads)
{
    const int group = num_heads / num_kv_heads;
    const long pairs = (long)num_seqs * num_heads;
#ifdef _OPENMP
    if (num_threads > 0)
        omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
    for (long sh = 0; sh < pairs; sh++) {
        const int s = (int)(sh / num_heads);
        const int h = (int)(sh % num_heads);
        const int kvh = h / group;
        const int n = context_lens[s];
        double *o = out + (size_t)sh * head_dim;
        for (int d = 0; d < head_dim; d++)
            o[d] = 0.0;
        if (n <= 0)
            continue;
        double *qd = (double *)malloc(sizeof(double) * head_dim);
        double *scores = (double *)malloc(sizeof(double) * n);
        for (int d = 0; d < head_dim; d++)
            qd[d] = oracle_to_double(q[(size_t)sh * head_dim + d], q_dtype);
        const int pages = (n + block_size - 1) / block_size;
        const int32_t *table = block_tables + (size_t)s * max_blocks_per_seq;
        for (int i = 0; i < pages; i++) {
            const size_t page = (size_t)table[i];
            const double ks = kv8_scale(k_scales, per_block, page, kvh, num_kv_heads);
            for (int r = 0; r < block_size; r++) {
                const int t = i * block_size + r;
                if (t >= n)
                    break;
                const uint8_t *key = k_pool + ((page * num_kv_heads + kvh) * block_size + r) * head_dim;
                double dot = 0.0;
                for (int d = 0; d < head_dim; d++)
                    dot += qd[d] * (ks * kv8_to_double(key[d], format));
                scores[t] = dot;
            }
        }
        double mx = -INFINITY;
        for (int t = 0; t < n; t++)
            if (scale * scores[t] > mx)
                mx = scale * scores[t];
        double total = 0.0;
        for (int t = 0; t < n; t++) {
            scores[t] = exp(scale * scores[t] - mx);
            total += scores[t];
        }
        for (int t = 0; t < n; t++)
            scores[t] /= total;
        for (int i = 0; i < pages; i++) {
            const size_t page = (size_t)table[i];
            const double vs = kv8_scale(v_scales, per_block, page, kvh, num_kv_heads);
            for (int r = 0; r < block_size; r++) {
                const int t = i * block_size + r;
                if (t >= n)
                    break;
                const uint8_t *val = v_pool + ((page * num_kv_heads + kvh) * block_size + r) * head_dim;
                for (int d = 0; d < head_dim; d++)
                    o[d] += scores[t] * (vs * kv8_to_double(val[d], format));
            }
        }
        free(scores);
        free(qd);
    }
}

static void reshape_and_cache_kv8(const uint16_t *k, const uint16_t *v, uint8_t *k_pool, uint8_t *v_pool,
                                  const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                  int block_size, int dtype, int format, const float *k_scales,
                                  const float *v_scales, int per_block);

/*
 * Quantising cache write with one scale per KV head: element x of head h is
 * stored as encode(x / k_scales[h]) (keys) or encode(x / v_scales[h])
 * (values), the division in fp32, encode being the E4M3 or the INT8 encoder.
 */
void oracle_reshape_and_cache_kv8(const uint16_t *k, const uint16_t *v,
                                  uint8_t *k_pool, uint8_t *v_pool,
                                  const int64_t *slot_mapping, int num_tokens,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int dtype, int format, const float *k_scales, const float *v_scales)
{
    reshape_and_cache_kv8(k, v, k_pool, v_pool, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size, dtype,
                          format, k_scales, v_scales, 0);
}

/*
 * The same with one scale per (physical block, KV head): a token written into
 * block b divides by k_scales[b * num_kv_heads + h] (v_scales for values).
 */
void oracle_reshape_and_cache_kv8_blocks(const uint16_t *k, const uint16_t *v,
                                         uint8_t *k_pool, uint8_t *v_pool,
                                         const int64_t *slot_mapping, int num_tokens,
                                         int num_kv_heads, int head_dim, int block_size,
                                         int dtype, int format, const float *k_scales, const float *v_scales)
{
    reshape_and_cache_kv8(k, v, k_pool, v_pool, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size, dtype,
                          format, k_scales, v_scales, 1);
}

static void reshape_and_cache_kv8(const uint16_t *k, const uint16_t *v, uint8_t *k_pool, uint8_t *v_pool,
                                  const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                  int block_size, int dtype, int format, const float *k_scales,
                                  const float *v_scales, int per_block)
{
    for (int t = 0; t < num_tokens; t++) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        const int64_t block = slot / block_size;
        const int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; h++) {
            const size_t src = ((size_t)t * num_kv_heads + h) * head_dim;
            const size_t dst = (((size_t)block * num_kv_heads + h) * block_size + offset) * head_dim;
            const size_t si = per_block ? (size_t)block * num_kv_heads + h : (size_t)h;
            for (int d = 0; d < head_dim; d++) {
                const float kx = (float)oracle_to_double(k[src + d], dtype) / k_scales[si];
                const float vx = (float)oracle_to_double(v[src + d], dtype) / v_scales[si];
                k_pool[dst + d] = format == ORACLE_KV_INT8 ? oracle_int8_encode(kx) : oracle_e4m3_encode(kx);
                v_pool[dst + d] = format == ORACLE_KV_INT8 ? oracle_int8_encode(vx) : oracle_e4m3_encode(vx);
            }
        }
    }
}

/*
 * Write each new token's K and V rows into its pool slot. slot = block *
 * block_size + offset; a negative slot means "no write" for that token.
 * Pure bit copy of the 16-bit elements.
 */
void oracle_reshape_and_cache(const uint16_t *k, const uint16_t *v,
                              uint16_t *k_pool, uint16_t *v_pool,
                              const int64_t *slot_mapping, int num_tokens,
                              int num_kv_heads, int head_dim, int block_size)
{
    for (int t = 0; t < num_tokens; t++) {
        const int64_t slot = slot_mapping[t];
        if (slot < 0)
            continue;
        const int64_t block = slot / block_size;
        const int64_t offset = slot % block_size;
        for (int h = 0; h < num_kv_heads; h++) {
            const size_t src = ((size_t)t * num_kv_heads + h) * head_dim;
            const size_t dst = (((size_t)block * num_kv_heads + h) * block_size + offset) * head_dim;
            for (int d = 0; d < head_dim; d++) {
                k_pool[dst + d] = k[src + d];
                v_pool[dst + d] = v[src + d];
            }
        }
    }
}

/*
 * Copy-on-write block copies: for each (src, dst) pair in order and each pool,
 * the whole block dst becomes a byte copy of block src.
 */
void oracle_copy_blocks(uint8_t *const *pools, int num_pools,
                        const int64_t *src_dst_pairs, int num_pairs,
                        size_t block_bytes)
{
    for (int p = 0; p < num_pairs; p++) {
        const int64_t src = src_dst_pairs[2 * p];
        const int64_t dst = src_dst_pairs[2 * p + 1];
        for (int i = 0; i < num_pools; i++)
            memcpy(pools[i] + (size_t)dst * block_bytes,
                   pools[i] + (size_t)src * block_bytes, block_bytes);
    }
}

/*
 * Swap copies between two sets of pools (e.g. GPU blocks out to a host pool
 * and back), as in "vLLM架构深度解析：PagedAttention如何实现高吞吐LLM推理",
 * section 抢占与恢复 (swapping a preempted request's blocks to CPU memory over
 * PCIe and back): for each (src, dst) pair in order and each pool index i,
 * block dst of dst_pools[i] becomes a byte copy of block src of src_pools[i].
 */
void oracle_swap_blocks(uint8_t *const *dst_pools, const uint8_t *const *src_pools, int num_pools,
                        const int64_t *src_dst_pairs, int num_pairs, size_t block_bytes)
{
    for (int p = 0; p < num_pairs; p++) {
        const int64_t src = src_dst_pairs[2 * p];
        const int64_t dst = src_dst_pairs[2 * p + 1];
        for (int i = 0; i < num_pools; i++)
            memcpy(dst_pools[i] + (size_t)dst * block_bytes,
                   src_pools[i] + (size_t)src * block_bytes, block_bytes);
    }
}

/*
 * Slot of token position pos of a sequence: the page table maps logical page
 * pos / block_size to a physical page; the slot is that page's first slot plus
 * the offset inside the page.
 */
void oracle_slot_mapping(int64_t *slots, const int32_t *block_tables,
                         int max_blocks_per_seq, const int32_t *seq_ids,
                         const int32_t *positions, int n, int block_size)
{
    for (int i = 0; i < n; i++) {
        const int32_t *table = block_tables + (size_t)seq_ids[i] * max_blocks_per_seq;
        const int pos = positions[i];
        slots[i] = (int64_t)table[pos / block_size] * block_size + pos % block_size;
    }
}
