/*
 * pa.h — C ABI of the B200 (sm_100a) paged KV-cache decode library.
 *
 * Three operations, each enqueued asynchronously on the caller's CUDA stream:
 *
 *   pa_decode             paged decode attention: every sequence's one query
 *                         token attends over its KV cache, which is stored in
 *                         fixed-size blocks of a global pool and reached through
 *                         a per-sequence block table.
 *   pa_reshape_and_cache  writes new tokens' K/V rows into their pool slots.
 *   pa_copy_blocks        copy-on-write copies of whole blocks.
 *
 * Memory layouts (row-major, contiguous, device memory unless stated):
 *   q, out        [num_seqs][num_heads][head_dim]            fp16 or bf16
 *   k_pool,v_pool [num_blocks][num_kv_heads][block_size][head_dim]
 *                 One (block, KV head) chunk is contiguous: block_size*head_dim
 *                 elements (4 KB at block_size 16, head_dim 128, 16-bit).
 *   block_tables  [num_seqs][max_blocks_per_seq] int32 physical block ids;
 *                 entries at or past ceil(context_len/block_size) are never read.
 *   context_lens  [num_seqs] int32, number of cached tokens, new token included.
 *   k, v          [num_tokens][num_kv_heads][head_dim]
 *   slot_mapping  [num_tokens] int64, slot = block * block_size + offset;
 *                 a negative slot skips that token.
 *   src_dst_pairs [num_pairs][2] int64 block ids.
 * Grouped-query attention: query head h reads KV head h / (num_heads / num_kv_heads).
 *
 * Supported shapes: head_dim in {64, 128}; block_size in {16, 32, 64};
 * num_heads % num_kv_heads == 0 with group size in {1, 2, 4, 8}. All device
 * pointers must be 16-byte aligned. Anything else returns PA_ERR_UNSUPPORTED
 * (shape) or PA_ERR_INVALID (argument).
 *
 * Ownership: the caller owns every buffer, workspace included. The library
 * allocates no memory, never synchronises except in pa_device_errors(), and
 * launches only on the given stream (a cudaStream_t; NULL = legacy default).
 *
 * Errors: host-side validation returns a status before anything is launched.
 * A failed launch returns PA_ERR_CUDA (pa_last_error() gives the text).
 * Kernels never fault on bad indices: a block id, slot or copy pair out of
 * range is skipped and sets a bit in a per-device error word, and a context
 * length above the limit is clamped and flagged; read (and clear) the word
 * with pa_device_errors(). Results are then undefined but memory stays safe.
 *
 * Calls on one stream are ordered. Concurrent pa_decode calls on different
 * streams must use different workspaces.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    PA_OK = 0,
    PA_ERR_INVALID = 1,      /* bad argument: null pointer, misalignment, size */
    PA_ERR_UNSUPPORTED = 2,  /* valid but unsupported shape */
    PA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
    PA_ERR_DEVICE_CHECK = 4  /* pa_device_errors(): a kernel flagged bad input */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1 } pa_dtype;

/* Formats of an 8-bit KV cache (pa_reshape_and_cache_quant, pa_decode_quant). */
typedef enum {
    PA_KV_E4M3 = 0,  /* fp8 e4m3fn codes: value = scale * E4M3(code) */
    PA_KV_INT8 = 1   /* signed 8-bit integers stored excess-128: value = scale * (code - 128) */
} pa_kv_format;

/* Bits of the per-device error word (pa_device_errors). */
#define PA_DEVERR_BLOCK_ID 1u   /* block table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT  2u   /* context_len < 0 or above the limit (clamped) */
#define PA_DEVERR_SLOT     4u   /* slot_mapping entry >= num_blocks*block_size */
#define PA_DEVERR_PAIR     8u   /* copy pair id outside [0, num_blocks) */
#define PA_DEVERR_TIMEOUT 16u   /* a bounded device-side wait ran out */
#define PA_DEVERR_QRANGE  32u   /* pa_decode_fp8: a bf16 query element above 65504 in magnitude */

/* Opaque CUDA stream handle (cudaStream_t). */
typedef void *pa_stream_t;

/* Name of a status code. */
PA_API const char *pa_status_string(int status);

/* Text of the last failure on this host thread ("" if none). */
PA_API const char *pa_last_error(void);

/* Number of kernels this library has launched from the calling thread since
 * it was loaded, over every entry point (a decode call is 2 or 3: plan,
 * attention and, when it runs, the merge launch; a cache write 1). Host only;
 * take the difference around a region to count its launches. */
PA_API unsigned long long pa_launch_count(void);

/*
 * Paged decode attention.
 *
 * Defined by: "别再让GPU内存拖后腿了：vLLM的PagedAttention如何像操作系统一样管理KV Cache",
 * section 3.1 (分块注意力计算) — walk the sequence's page table, score the query
 * against each page, softmax(scores * scale) over the concatenation, and sum
 * each page's weight slice times its values; with blocks and block tables as
 * in "vLLM架构深度解析：PagedAttention如何实现高吞吐LLM推理", section PagedAttention.
 * Only the first context_lens[s] tokens of sequence s count.
 *
 *   out[s][h][:] = sum_t softmax_t(scale * q[s][h] . K_t) V_t,
 *   K_t = k_pool[block_tables[s][t / block_size]][h / group][t % block_size].
 *
 * Long contexts are split into partitions of partition_size tokens whose
 * partial results (max, sum, unnormalised output) are merged by the
 * log-sum-exp identity. partition_size = 0 picks one automatically: 32
 * blocks for grouped heads (group >= 2), 256 tokens for one query head per
 * KV head, or the whole context when max_context_len fits in it. Otherwise it
 * must be a multiple of 16 and of block_size, with
 * partition_size / block_size <= 32.
 *
 * max_context_len bounds every context_lens entry (larger ones are clamped and
 * flagged) and sizes the workspace. scale multiplies q.k (1/sqrt(head_dim) for
 * standard attention). context_len 0 gives a zero output row.
 *
 * workspace: device memory of at least pa_decode_workspace_size(...) bytes,
 * 256-byte aligned, owned by the caller, contents need no initialisation.
 * out is fp16/bf16 (dtype), rounded to nearest even from fp32 accumulation.
 */
PA_API pa_status pa_decode(void *out, const void *q, const void *k_pool, const void *v_pool,
                    const int32_t *block_tables, const int32_t *context_lens,
                    int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                    int block_size, int max_blocks_per_seq, int num_blocks,
                    int max_context_len, float scale, int dtype, int partition_size,
                    void *workspace, size_t workspace_bytes, pa_stream_t stream);

/*
 * Fused append + decode: for every sequence s with context_lens[s] >= 1,
 * first writes k_new[s][h][:] and v_new[s][h][:] (all KV heads h) into the
 * slot of position context_lens[s] - 1, i.e.
 *   slot = block_tables[s][pos / block_size] * block_size + pos % block_size,
 * then attends exactly as pa_decode. Same result, pool contents included, as
 * pa_reshape_and_cache with those slots followed by pa_decode, in one pass:
 * the attention unit that holds the last position writes the row and uses it
 * directly, so the new row is neither written by a separate launch nor read
 * back.
 *
 * Defined by: the m.nxbn.cn VLLM explainer, section 一 — each decode step
 * computes only the new token's K/V, appends it to the cache and attends over
 * the cache.
 *
 * k_new, v_new: [num_seqs][num_kv_heads][head_dim], fp16/bf16 like the pools,
 * 16-byte aligned. context_lens are post-append lengths. The appended slot's
 * block must be private to the sequence (a shared tail is copied first with
 * pa_copy_blocks). Other arguments as pa_decode.
 */
PA_API pa_status pa_decode_append(void *out, const void *q, const void *k_new, const void *v_new,
                                  void *k_pool, void *v_pool, const int32_t *block_tables,
                                  const int32_t *context_lens, int num_seqs, int num_heads,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int max_blocks_per_seq, int num_blocks, int max_context_len,
                                  float scale, int dtype, int partition_size, void *workspace,
                                  size_t workspace_bytes, pa_stream_t stream);

/*
 * Paged decode attention that computes over shared blocks once per group of
 * sequences. Same result as pa_decode (k_new = v_new = NULL) or
 * pa_decode_append (both set) up to the order of fp32 rounding: the
 * arithmetic is the definition of pa_decode, with the sum over tokens
 * regrouped by partition.
 *
 * Sequences forked from one another (beam search, parallel sampling) hold
 * the same physical blocks at the start of their block tables ("vLLM架构深度
 * 解析：PagedAttention如何实现高吞吐LLM推理", section KV Cache内存共享; "别再让
 * GPU内存拖后腿了", section 2.2). The library finds them on the device: it
 * sorts the sequences by their first block and, within a run of sequences
 * with the same first block, forms groups of up to 16 / (num_heads /
 * num_kv_heads) consecutive ones. A group's shared part is the leading full
 * blocks that all members have in common with its first member (with k_new,
 * only blocks below the one holding each member's last position). That part
 * is streamed once per KV head for the whole group, with the group's queries
 * side by side in the columns of the tensor-core tiles. Each member's
 * remaining tokens run as ordinary partitions, and the partitions merge by
 * the log-sum-exp identity, in a launch of its own after the attention
 * kernel (one CTA per (member, KV head)). Without shared blocks, the
 * partitions are those of pa_decode and the result equals pa_decode's up to
 * the order of the merge's fp32 sums.
 *
 * partition_size 0 picks 16 blocks for grouped heads (group >= 2; smaller
 * units balance better once the shared tiles are streamed once per group),
 * otherwise as pa_decode.
 *
 * The grouping runs in one CTA of 1024 threads: a batch of more than 1024
 * sequences runs as consecutive chunks of 1024 (in stream order, on the same
 * workspace), and sequences share work only with others of their chunk.
 *
 * Requirements beyond pa_decode's: fp16/bf16 cache (the tensor-core kernel).
 * workspace: at least pa_decode_shared_workspace_size(...) bytes (one more
 * partition per sequence than pa_decode, plus the grouping). Errors:
 * PA_ERR_UNSUPPORTED for a build without the tensor-core kernel for this
 * head group; otherwise as pa_decode / pa_decode_append.
 */
PA_API pa_status pa_decode_shared(void *out, const void *q, const void *k_new, const void *v_new,
                                  void *k_pool, void *v_pool, const int32_t *block_tables,
                                  const int32_t *context_lens, int num_seqs, int num_heads,
                                  int num_kv_heads, int head_dim, int block_size,
                                  int max_blocks_per_seq, int num_blocks, int max_context_len,
                                  float scale, int dtype, int partition_size, void *workspace,
                                  size_t workspace_bytes, pa_stream_t stream);

/*
 * pa_decode_shared over an 8-bit cache: the codes, formats and per-KV-head
 * scales of pa_decode_quant, the grouping and shared units of
 * pa_decode_shared (without the fused append). Workspace and partition:
 * pa_decode_shared_workspace_size / pa_decode_shared_partition_size. Same
 * result as pa_decode_quant up to the order of the fp32 sums.
 *
 * Defined by: the sharing of "vLLM架构深度解析：PagedAttention如何实现高吞吐LLM推理",
 * section KV Cache内存共享, over the compressed cache of "别再让GPU内存拖后腿了",
 * section 3.2.
 */
PA_API pa_status pa_decode_shared_quant(void *out, const void *q, const void *k_pool, const void *v_pool,
                                        const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                                        int num_heads, int num_kv_heads, int head_dim, int block_size,
                                        int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                                        int dtype, int kv_format, const float *k_scales, const float *v_scales,
                                        int partition_size, void *workspace, size_t workspace_bytes,
                                        pa_stream_t stream);

/* Partition and workspace bytes pa_decode_fp8 (and pa_decode_quant) uses for
 * these arguments (0 if invalid). */
PA_API int pa_decode_fp8_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                        int block_size, int max_context_len, int partition_size);
PA_API size_t pa_decode_fp8_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                           int block_size, int max_context_len, int partition_size);

/* Partition pa_decode_shared uses for these arguments (0 if invalid). */
PA_API int pa_decode_shared_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                           int block_size, int max_context_len, int partition_size);

/* Workspace bytes pa_decode_shared needs (0 for unsupported shapes). */
PA_API size_t pa_decode_shared_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                              int head_dim, int block_size, int max_context_len,
                                              int partition_size);

/*
 * Paged decode attention over an 8-bit E4M3 ("fp8 e4m3fn") KV cache with
 * per-tensor scales: key element = k_scale * E4M3 code, value element =
 * v_scale * E4M3 code; otherwise exactly pa_decode (q and out stay fp16/bf16
 * by `dtype`). k_pool, v_pool: uint8 codes [num_blocks][num_kv_heads]
 * [block_size][head_dim], written by pa_reshape_and_cache_fp8. head_dim 64 or
 * 128.
 * The products run on tensor cores with the codes widened to fp16 (exact) and
 * the queries converted to fp16 (exact for |q| in fp16's normal range; a bf16
 * query element above 65504 in magnitude has no fp16 value: the kernel sets
 * PA_DEVERR_QRANGE and that head's output is undefined). The
 * workspace is sized by pa_decode_fp8_workspace_size: partition_size 0 picks
 * 512 tokens (pa_decode_fp8_partition_size).
 *
 * Defined by: "别再让GPU内存拖后腿了：vLLM的PagedAttention如何像操作系统一样管理KV Cache",
 * section 3.2 (内存压缩技术) — keep the KV cache in fewer bits to cut its
 * memory; the attention itself is that of section 3.1.
 */
PA_API pa_status pa_decode_fp8(void *out, const void *q, const void *k_pool, const void *v_pool,
                               const int32_t *block_tables, const int32_t *context_lens,
                               int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                               int block_size, int max_blocks_per_seq, int num_blocks,
                               int max_context_len, float scale, int dtype, float k_scale,
                               float v_scale, int partition_size, void *workspace,
                               size_t workspace_bytes, pa_stream_t stream);

/*
 * Quantising cache write for an E4M3 cache: like pa_reshape_and_cache, but
 * each element x of k (v) is stored as the E4M3 code of x / k_scale
 * (x / v_scale): fp32 division rounded to nearest, then round-to-nearest-even
 * to E4M3 with magnitudes past 448 saturated to 448. k, v fp16/bf16 (dtype);
 * pools uint8, 8-byte aligned. Same slot rules and error reporting as
 * pa_reshape_and_cache. Defined by the same section 3.2.
 */
PA_API pa_status pa_reshape_and_cache_fp8(const void *k, const void *v, void *k_pool, void *v_pool,
                                          const int64_t *slot_mapping, int num_tokens,
                                          int num_kv_heads, int head_dim, int block_size,
                                          int num_blocks, int dtype, float k_scale, float v_scale,
                                          pa_stream_t stream);

/*
 * Quantising cache write with one scale per KV head, in either 8-bit format:
 * element x of KV head h (keys; values alike with v_scales) is stored as the
 * code of y = x / k_scales[h], the division in fp32 rounded to nearest.
 *   PA_KV_E4M3: the E4M3 code of y, rounded to nearest even, magnitudes past
 *               448 saturated to 448 (as pa_reshape_and_cache_fp8).
 *   PA_KV_INT8: clamp(round(y), -127, 127) + 128, rounding to nearest even;
 *               NaN stores 128 (zero).
 * k_scales, v_scales: DEVICE arrays [num_kv_heads] of positive finite floats,
 * 4-byte aligned. Pools uint8 [num_blocks][num_kv_heads][block_size][head_dim],
 * 8-byte aligned; other arguments, slot rules and error reporting as
 * pa_reshape_and_cache.
 *
 * Defined by: "别再让GPU内存拖后腿了：vLLM的PagedAttention如何像操作系统一样管理KV Cache",
 * section 3.2 (内存压缩技术) — the compression table's INT8 row (a quarter of
 * the fp32 bytes) and, in section 4.3, INT8 for older pages; the per-head
 * scale and the excess-128 storage are this library's choices.
 */
PA_API pa_status pa_reshape_and_cache_quant(const void *k, const void *v, void *k_pool, void *v_pool,
                                            const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                                            int head_dim, int block_size, int num_blocks, int dtype, int kv_format,
                                            const float *k_scales, const float *v_scales, pa_stream_t stream);

/*
 * Paged decode attention over an 8-bit cache with one scale per KV head: key
 * element of KV head j = k_scales[j] * decode(code), value element =
 * v_scales[j] * decode(code), decode being E4M3 (PA_KV_E4M3) or code - 128
 * (PA_KV_INT8); otherwise exactly pa_decode (q and out fp16/bf16 by dtype).
 * head_dim 64 or 128. The partition and the workspace are those of pa_decode_fp8
 * (pa_decode_fp8_partition_size, pa_decode_fp8_workspace_size). INT8 key
 * codes enter the tensor-core product as the exact fp16 numbers
 * 1152 + (code - 128), the constant taken off each score (per query row) in
 * fp32; value codes enter it as the exact fp16 numbers code - 128 (one fp16
 * subtraction per pair). Queries are converted to fp16 as in pa_decode_fp8
 * (PA_DEVERR_QRANGE for bf16 elements above 65504).
 *
 * Defined by: the same section 3.2; the attention is that of section 3.1.
 */
PA_API pa_status pa_decode_quant(void *out, const void *q, const void *k_pool, const void *v_pool,
                                 const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                                 int num_heads, int num_kv_heads, int head_dim, int block_size,
                                 int max_blocks_per_seq, int num_blocks, int max_context_len, float scale, int dtype,
                                 int kv_format, const float *k_scales, const float *v_scales, int partition_size,
                                 void *workspace, size_t workspace_bytes, pa_stream_t stream);

/*
 * The 8-bit cache with one scale per (physical block, KV head): k_scales and
 * v_scales are fp32 device arrays [num_blocks][num_kv_heads] of positive
 * finite floats (not checked on the device), 4-byte aligned;
 * a token written into block b of KV head h is stored as
 * encode(x / k_scales[b * num_kv_heads + h]) (v_scales for values), and
 * decoding multiplies by the same scale. Otherwise exactly
 * pa_reshape_and_cache_quant / pa_decode_quant (same codes, layouts,
 * partition, workspace and errors). A block's scale applies to every token
 * written into it, so it has to be chosen before its first token is written
 * (a serving loop sets it when it allocates the block, e.g. from prefill
 * statistics). The decode reads each unit's block scales beside its
 * block-table entries; the value product weighs each token by its block's
 * value scale relative to the unit's largest, and the denominator sums the
 * unweighted fp32 probabilities.
 *
 * Defined by: "别再让GPU内存拖后腿了：vLLM的PagedAttention如何像操作系统一样管理KV Cache",
 * section 3.2 (内存压缩技术), keep the cache in fewer bits, with the scales at the
 * granularity of the cache's own unit, the physical block of section 2.1.
 */
PA_API pa_status pa_reshape_and_cache_quant_blocks(const void *k, const void *v, void *k_pool, void *v_pool,
                                                   const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                                                   int head_dim, int block_size, int num_blocks, int dtype,
                                                   int kv_format, const float *k_scales, const float *v_scales,
                                                   pa_stream_t stream);
/* pa_decode_shared_quant with one scale per (physical block, KV head), as
 * above: the shared units stream a block once for the whole group with that
 * block's scales (the blocks are the same physical blocks for every member). */
PA_API pa_status pa_decode_shared_quant_blocks(void *out, const void *q, const void *k_pool, const void *v_pool,
                                               const int32_t *block_tables, const int32_t *context_lens,
                                               int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                               int block_size, int max_blocks_per_seq, int num_blocks,
                                               int max_context_len, float scale, int dtype, int kv_format,
                                               const float *k_scales, const float *v_scales, int partition_size,
                                               void *workspace, size_t workspace_bytes, pa_stream_t stream);
PA_API pa_status pa_decode_quant_blocks(void *out, const void *q, const void *k_pool, const void *v_pool,
                                        const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                                        int num_heads, int num_kv_heads, int head_dim, int block_size,
                                        int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                                        int dtype, int kv_format, const float *k_scales, const float *v_scales,
                                        int partition_size, void *workspace, size_t workspace_bytes,
                                        pa_stream_t stream);

/* Workspace bytes pa_decode needs for these sizes (0 if the shape is invalid). */
PA_API size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads,
                                int head_dim, int block_size, int max_context_len,
                                int partition_size);

/* The partition size pa_decode uses for these arguments (resolves 0 = auto);
 * returns 0 if the arguments are invalid. */
PA_API int pa_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                             int block_size, int max_context_len, int partition_size);

/*
 * Cache write: for each token t with slot_mapping[t] >= 0,
 *   k_pool[slot / block_size][h][slot % block_size][:] = k[t][h][:]  (all h),
 * and the same for v. Bit copy.
 *
 * Defined by: the m.nxbn.cn VLLM explainer, section 一 — decode computes only
 * the new token's K/V and appends it to the cache; prefill writes all prompt
 * tokens (section 3.2).
 *
 * Precondition: non-negative slots are distinct (two tokens into one slot race).
 * A slot >= num_blocks*block_size is skipped and flagged (PA_DEVERR_SLOT).
 */
PA_API pa_status pa_reshape_and_cache(const void *k, const void *v, void *k_pool, void *v_pool,
                               const int64_t *slot_mapping, int num_tokens,
                               int num_kv_heads, int head_dim, int block_size,
                               int num_blocks, int dtype, pa_stream_t stream);

/*
 * Copy-on-write block copies: for each pair p and each pool i,
 *   bytes [dst*block_bytes, (dst+1)*block_bytes) of pools[i] become a copy of
 *   bytes [src*block_bytes, (src+1)*block_bytes).
 *
 * Defined by: "vLLM架构深度解析：PagedAttention如何实现高吞吐LLM推理", section
 * KV Cache内存共享 — before a sequence appends into a block shared with others,
 * a new block is taken, the data copied and the block table updated.
 *
 * pools is a HOST array of num_pools device pointers (e.g. K and V of every
 * layer); src_dst_pairs is DEVICE memory. block_bytes is one block of one
 * pool (num_kv_heads*block_size*head_dim*element size) and must be a multiple
 * of 16. Precondition: destination blocks are distinct and no destination is
 * also a source in the same call (the copies run in parallel). An id outside
 * [0, num_blocks) skips that pair and sets PA_DEVERR_PAIR.
 */
PA_API pa_status pa_copy_blocks(void *const *pools, int num_pools, const int64_t *src_dst_pairs,
                         int num_pairs, size_t block_bytes, int num_blocks,
                         pa_stream_t stream);

/*
 * Swap copies of whole blocks between two sets of pools: for each pair p and
 * each pool index i, block dst of dst_pools[i] becomes a byte copy of block
 * src of src_pools[i] (block = block_bytes bytes). Used to move a preempted
 * sequence's blocks from the GPU pools to host pools and back.
 *
 * Defined by: "vLLM架构深度解析：PagedAttention如何实现高吞吐LLM推理", section
 * 抢占与恢复 — preemption by swapping moves a request's KV blocks over PCIe to
 * CPU memory and back when it resumes.
 *
 * dst_pools, src_pools: HOST arrays of num_pools pointers, each to device
 * memory or to page-locked host memory (cudaHostAlloc / cudaMallocHost /
 * cudaHostRegister), 16-byte aligned; pageable host memory is rejected with
 * PA_ERR_INVALID. src_dst_pairs: [num_pairs][2] int64 in device or page-locked
 * host memory. Source ids must be < num_src_blocks and destination ids <
 * num_dst_blocks (others are skipped and flagged PA_DEVERR_PAIR). block_bytes
 * is a multiple of 16. Destinations must be distinct; the two sides must not
 * overlap. Asynchronous on `stream`; host memory must stay valid until the
 * copy has finished.
 */
PA_API pa_status pa_swap_blocks(void *const *dst_pools, const void *const *src_pools, int num_pools,
                                const int64_t *src_dst_pairs, int num_pairs, size_t block_bytes,
                                int num_src_blocks, int num_dst_blocks, pa_stream_t stream);

/*
 * Synchronises `stream`, then returns the current device's error word in
 * *flags (PA_DEVERR_* bits) and clears it when `clear` is non-zero. Returns
 * PA_ERR_DEVICE_CHECK when any bit was set, PA_OK otherwise.
 */
PA_API pa_status pa_device_errors(unsigned int *flags, int clear, pa_stream_t stream);

/* Number of SMs the library sizes its persistent grids for (current device). */
PA_API int pa_num_sms(void);

/*
 * Self-test of the kernels' bounded device-side waits: launches one warp that
 * waits on an mbarrier nothing will ever complete, for at most limit_ns
 * nanoseconds (1 ms .. 10 s), then sets PA_DEVERR_TIMEOUT and returns — the
 * same path every pipeline wait in pa_decode takes if a copy never lands.
 * Asynchronous; read the result with pa_device_errors().
 */
PA_API pa_status pa_selftest_bounded_wait(unsigned long long limit_ns, pa_stream_t stream);

/* Size of the fixed scratch array behind pa_decode_noalloc (16 MiB). */
#define PA_NOALLOC_SCRATCH_BYTES (16u << 20)

/*
 * pa_decode without a caller-provided workspace, for callers that cannot
 * allocate device memory at decode time (a plugin whose host pre-partitions
 * all device memory, a real-time loop that must not take cudaMalloc's implicit
 * synchronisation, a process with a memory budget fixed at start-up). The
 * pages this library follows describe no such entry point; it is an addition.
 *
 * Arguments, layouts and results are those of pa_decode. The scratch lives in
 * one file-scope device array of PA_NOALLOC_SCRATCH_BYTES that every GPU which
 * loads the library holds until the process exits; nothing is allocated.
 * Sizes whose pa_decode_workspace_size() exceeds the array are rejected with
 * PA_ERR_UNSUPPORTED before anything is launched (pa_last_error() says why).
 *
 * Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress; nothing is cached, so the address stays valid after
 * a device reset or a new primary context). The first call on a device may
 * load the library's device code there: make it before any stream capture.
 * All calls share the one array: calls that overlap on the GPU
 * (different streams, or different host threads without ordering) race and
 * give undefined results. Calls ordered on one stream are safe; each call
 * re-initialises the parts of the array that must start at zero.
 */
PA_API pa_status pa_decode_noalloc(void *out, const void *q, const void *k_pool, const void *v_pool,
                                   const int32_t *block_tables, const int32_t *context_lens,
                                   int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                                   int block_size, int max_blocks_per_seq, int num_blocks,
                                   int max_context_len, float scale, int dtype, int partition_size,
                                   pa_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
