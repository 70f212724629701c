// Paged decode attention for sm_100a: two launches per call (three when a
// sequence has more partitions than the attention kernel merges itself).
//
//  1. pa_plan_kernel (one warp) cuts every sequence into partitions of P
//     tokens and writes the work list: every sequence's full partitions in
//     sequence order, then the partial last ones, longest first, so that the
//     persistent attention kernel finishes with the short ones. It also
//     zeroes the per-(sequence, KV head) merge counters. The attention warps
//     take their first units without waiting for it (they derive them from
//     the contexts). pa_plan_shared_kernel (one CTA) does the same for
//     pa_decode_shared, after grouping sequences whose tables begin with the
//     same blocks.
//  2. The attention kernel (one persistent CTA per SM, launched with
//     programmatic dependent launch so that it overlaps the plan) — every
//     warp is an independent worker. It takes (sequence, KV head, partition)
//     units from the work list with an atomic counter and streams the unit's
//     K and V tiles (16 tokens, or 32 where a 16-token tile is at most 4 KB)
//     through a private ring of shared-memory stages filled by TMA copies
//     that complete on mbarriers. The block-table entries of a unit are
//     loaded once into lane registers and handed to the copy-issuing lane by
//     a shuffle. Per tile: scores of the G query heads of the KV head, online
//     softmax, weighted sum of the values. A unit that is a whole sequence
//     writes the normalised output; otherwise it writes (max, sum,
//     unnormalised output) partials, and the last warp to finish a (sequence,
//     KV head) merges its partitions by the log-sum-exp identity, in one
//     level or two (chunks of MERGE_FANIN).
//  3. The merge launch (pa_reduce_kernel, or pa_reduce_members_kernel for
//     shared-prefix decode) merges the sequences of many partitions (every
//     sequence in shared-prefix decode) after the attention kernel.
//     The default attention kernel is the tensor-core one in
//     pa_decode_mma.cuh. This file holds the CUDA-core kernel
//     (pa_decode_kernel: 1-D bulk copies of each tile, FFMA2 dot products),
//     selected with -DPA_DECODE_TENSOR_MIN_GROUP, plus what both share: the
//     plans, the unit source and the merges.

// The arithmetic is the definition in "别再让GPU内存拖后腿了：vLLM的PagedAttention
// 如何像操作系统一样管理KV Cache", section 3.1: scores of the query against every
// page, softmax over the concatenation with the 1/sqrt(dim) scale, weighted sum
// of the pages' values. Scores are kept in the log2 domain (q is pre-scaled by
// scale*log2(e)) and accumulated in fp32.
#pragma once

#include <math.h>

#include "pa_common.cuh"

namespace pa {

struct DecodeParams {
    void *out;
    const void *q;
    const void *k_pool;
    const void *v_pool;
    const void *k_new;  // [num_seqs][num_kv_heads][head_dim] rows appended at each
    const void *v_new;  // sequence's last position first; null for plain decode
    const int32_t *block_tables;
    const int32_t *context_lens;
    int num_seqs, num_heads, num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks;
    int ctx_limit;   // context lengths are clamped to [0, ctx_limit]
    int partition;   // P, tokens per partition
    int max_parts;   // partial slots per (sequence, head): partitions, then chunk merges
    int l1_base;     // first chunk-merge slot (= the most partitions a sequence has)
    int max_chunks;  // chunk counters per (sequence, KV head); 0 without chunked merging
    float qscale;    // scale * log2(e) (times k_scale for an fp8 cache with one scale)
    float v_scale;   // fp8 cache with one scale: dequantisation scale of V (1 otherwise)
    const float *k_scales;  // 8-bit cache with one scale per KV head: [num_kv_heads]
    const float *v_scales;  // (null: the single scales above)
    int *counter;    // work-list cursor (reset by the plan kernel)
    int *num_entries;
    int4 *entries;   // {seq, partition, tokens, partitions of seq}
    float2 *ml;      // [seq][head][part] (max in log2 units, sum of weights)
    float *part_acc; // [seq][head][part][D] unnormalised outputs
    int *merge_count;// [seq][kv head] finished partitions (or finished chunks)
    int *chunk_count;// [seq][kv head][chunk] finished partitions of each chunk
    // Shared-prefix units (pa_decode_shared): a unit may serve several
    // sequences whose block tables begin with the same blocks.
    int4 *entries_b; // {first token, member offset, member count (0: one sequence), 0}
    int *members;    // sequences in grouping order
    int *member_nparts;  // partitions of members[i] to merge (0: none, or written directly)
    int append_guard;    // 1: a sequence's last position never lies in a shared block
    int early;           // 1: the attention kernel starts without waiting for the one-warp plan
    int reduce_launch;   // 1: a merge launch follows (long sequences; every sequence with shared units)
};

// Split merges: a (sequence, KV head) with more than MERGE_FANIN partitions
// merges in two levels. The last partition to finish of each chunk of
// MERGE_FANIN consecutive partitions merges that chunk into a chunk partial
// (same form: max, sum, unnormalised output); the last chunk merge merges the
// chunk partials into the output. Every merge reads a fixed set in a fixed
// order, so the result does not depend on which warp finishes when, and the
// serial merge at the end of a long sequence is MERGE_FANIN reads deep
// instead of one per partition.
constexpr int MERGE_FANIN = 8;

__host__ __device__ inline int merge_chunks(int max_parts) {
    return max_parts > MERGE_FANIN ? (max_parts + MERGE_FANIN - 1) / MERGE_FANIN : 0;
}

// Workspace layout: header (counter, entry count), work list, merge and chunk
// counters, partials (partitions, then chunk partials).
struct WsLayout {
    size_t entries, ml, acc, count, chunk_count, entries_b, members, member_nparts, total;
    int slots, chunks;
};

inline __host__ __device__ size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// max_parts: the most partitions a sequence can have. Shared-prefix decode
// merges members in one level (no chunk partials).
inline __host__ __device__ WsLayout ws_layout(int B, int H, int Hkv, int D, int max_parts, bool shared = false) {
    WsLayout L;
    L.chunks = shared ? 0 : merge_chunks(max_parts);
    L.slots = max_parts + L.chunks;
    size_t off = 256;
    L.entries = off;
    off = align256(off + sizeof(int4) * (size_t)B * max_parts);
    L.count = off;  // merge counters, then chunk counters: one region, zeroed together
    L.chunk_count = off + sizeof(int) * (size_t)B * Hkv;
    off = align256(off + sizeof(int) * (size_t)B * Hkv * (1 + L.chunks));
    L.entries_b = L.members = L.member_nparts = 0;
    if (shared) {
        L.entries_b = off;
        off = align256(off + sizeof(int4) * (size_t)B * max_parts);
        L.members = off;
        off = align256(off + sizeof(int) * (size_t)B);
        L.member_nparts = off;
        off = align256(off + sizeof(int) * (size_t)B);
    }
    const size_t parts = max_parts > 1 ? (size_t)L.slots : 0;  // no partials without a split
    L.ml = off;
    off = align256(off + sizeof(float2) * (size_t)B * H * parts);
    L.acc = off;
    off = align256(off + sizeof(float) * (size_t)B * H * parts * D);
    L.total = off;
    return L;
}

__device__ __forceinline__ int clamped_context(const DecodeParams &p, int s, bool flag) {
    int c = p.context_lens[s];
    if (c < 0 || c > p.ctx_limit) {
        if (flag) raise_error(PA_DEVERR_CONTEXT);
        c = c < 0 ? 0 : p.ctx_limit;
    }
    return c;
}

// ---- 1. work list -----------------------------------------------------------
constexpr int PLAN_THREADS = 1024;  // the grouping plan (pa_plan_shared_kernel)
static_assert(PLAN_THREADS % 32 == 0 && PLAN_THREADS <= 1024, "plan block: whole warps, at most 32");
constexpr int PLAN_MAX_BINS = 129;  // tiles per partition <= 128

// Warp-wide inclusive prefix sum.
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(FULL_MASK, v, o);
        if (lane >= o) v += t;
    }
    return v;
}

// The plain plan runs as ONE warp limited to 32 registers a thread, so that it
// fits beside a persistent attention CTA on the SM it lands on (the attention
// kernels leave at least 1024 registers of an SM free) and no attention CTA
// waits for it to finish. The attention warps only need its results (work-list
// tail order, zeroed cursor and merge counters) from their first dynamic claim
// or first finished partition on; their first units come from the full
// partitions, whose order they compute themselves (UnitSource::init).
//
// Work-list order: every sequence's full partitions in sequence order, then
// the last, partial partitions, longest first.
constexpr int PLAN_WARP_THREADS = 32;

__global__ void __maxnreg__(32) pa_plan_kernel(const DecodeParams p) {
    __shared__ int s_bin_count[PLAN_MAX_BINS];
    __shared__ int s_bin_next[PLAN_MAX_BINS];
    // Let the attention kernel launch now; it waits for this grid's results.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int lane = threadIdx.x;
    const int B = p.num_seqs, P = p.partition, tiles = P / 16;
    for (int i = lane; i < PLAN_MAX_BINS; i += 32) s_bin_count[i] = 0;
    {
        // Merge and chunk counters (one region): 16-byte stores (it is 256-byte aligned).
        const int n = B * p.num_kv_heads * (1 + p.max_chunks);
        int4 *c4 = reinterpret_cast<int4 *>(p.merge_count);
        for (int i = lane; i < n / 4; i += 32) c4[i] = make_int4(0, 0, 0, 0);
        for (int i = (n / 4) * 4 + lane; i < n; i += 32) p.merge_count[i] = 0;
    }
    __syncwarp();

    // Pass 1: full partitions in sequence order; histogram of the tails.
    int carry = 0;
    for (int base = 0; base < B; base += 32) {
        const int s = base + lane;
        const int ctx = s < B ? clamped_context(p, s, true) : 0;
        const int full = ctx / P, tail = ctx - full * P;
        if (tail > 0) atomicAdd(&s_bin_count[(tail + 15) >> 4], 1);
        const int incl = warp_incl_scan(full, lane);
        const int off = carry + incl - full;
        const int nparts = full + (tail > 0);
        for (int j = 0; j < full; ++j) p.entries[off + j] = make_int4(s, j, P, nparts);
        carry += __shfl_sync(FULL_MASK, incl, 31);
    }
    __syncwarp();
    // Tails after the full partitions, longest first: start of each bin by a
    // scan over the bins in descending order.
    int pos = carry;
    for (int b0 = tiles; b0 >= 1; b0 -= 32) {
        const int b = b0 - lane;
        const int cnt = b >= 1 ? s_bin_count[b] : 0;
        const int incl = warp_incl_scan(cnt, lane);
        if (b >= 1) s_bin_next[b] = pos + incl - cnt;
        pos += __shfl_sync(FULL_MASK, incl, 31);
    }
    if (lane == 0) {
        *p.num_entries = pos;
        *p.counter = 0;
    }
    __syncwarp();
    // Pass 2: each sequence's last, partial partition. An empty sequence gets
    // no work; the warp zeroes its output rows here.
    for (int base = 0; base < B; base += 32) {
        const int s = base + lane;
        const int ctx = s < B ? clamped_context(p, s, false) : -1;
        const int full = ctx / P, tail = ctx - full * P;
        if (s < B && tail > 0) {
            const int at = atomicAdd(&s_bin_next[(tail + 15) >> 4], 1);
            p.entries[at] = make_int4(s, full, tail, full + 1);
        }
        unsigned empty = __ballot_sync(FULL_MASK, ctx == 0);
        const int nvec = p.num_heads * p.head_dim / 8;
        while (empty) {
            const int e = __ffs(empty) - 1;
            empty &= empty - 1;
            uint4 *row = static_cast<uint4 *>(p.out) + (size_t)(base + e) * nvec;
            for (int i = lane; i < nvec; i += 32) row[i] = make_uint4(0, 0, 0, 0);
        }
    }
}

// ---- 1b. work list with shared-prefix units ------------------------------------
// Sequences forked from one another (beam search, parallel sampling) hold the
// same physical blocks at the start of their tables ("vLLM架构深度解析：
// PagedAttention如何实现高吞吐LLM推理", section KV Cache内存共享). Their
// attention over those blocks is the same product with different queries, so
// one unit can stream the shared tiles once for up to 16 / G sequences: their
// G query rows each fill columns of the MMA tile (two halves of 8). Each member's own
// blocks run as ordinary units, and the partitions merge by the usual
// log-sum-exp identity (the definition's sum over all tokens, regrouped).
//
// Grouping: sequences are sorted by their first block; within a run of equal
// first blocks, consecutive members form sub-groups of up to 16 / G. A
// sub-group shares the leading full blocks that every member has in common
// with its first member (a block is shared only below each member's context;
// with append_guard, only below the block of the member's last position, so
// the row a fused append writes is never in a shared unit). The shared tokens
// are cut into partitions 0 .. pp-1 written for every member, the rest of each
// member into pp, pp+1, ...
constexpr int SHARE_MAX_SEQS = PLAN_THREADS;  // one sequence per plan thread
constexpr int SHARE_RANK_MAX = 256;           // batches sorted by rank rather than bitonically
constexpr int NO_SHARE = 0x7fffffff;

__device__ __forceinline__ int shared_full_blocks(const DecodeParams &p, int ctx) {
    const int pos = p.append_guard ? ctx - 1 : ctx;
    return pos > 0 ? pos / p.block_size : 0;
}

__global__ void __launch_bounds__(PLAN_THREADS) pa_plan_shared_kernel(const DecodeParams p) {
    __shared__ unsigned long long s_key[SHARE_MAX_SEQS];  // (first block << 32) | sequence, sorted
    __shared__ unsigned long long s_in[SHARE_RANK_MAX];   // keys before sorting (rank sort)
    __shared__ int s_ctx[SHARE_MAX_SEQS];                 // clamped context of each sequence
    __shared__ int s_grp[SHARE_MAX_SEQS];                 // sub-group of a position: first | count << 16
    __shared__ int s_lcp[SHARE_MAX_SEQS];                 // leading blocks shared with the sub-group's first
    __shared__ int s_bin_count[PLAN_MAX_BINS];
    __shared__ int s_bin_next[PLAN_MAX_BINS];
    __shared__ int s_warp[32];
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int B = p.num_seqs, P = p.partition, tiles = P / 16, bs = p.block_size, W = p.max_blocks_per_seq;
    const int cap = 16 / (p.num_heads / p.num_kv_heads);  // sequences per shared unit (16 query rows)
    int n = 1;
    while (n < B) n <<= 1;
    for (int i = tid; i < PLAN_MAX_BINS; i += PLAN_THREADS) s_bin_count[i] = 0;
    for (int i = tid; i < B * p.num_kv_heads; i += PLAN_THREADS) p.merge_count[i] = 0;

    // Key of this thread's sequence; padding keys sort last.
    unsigned long long key = ~0ull;
    if (tid < B) {
        const int first = p.block_tables[(size_t)tid * W];  // loaded alongside the context
        const int ctx = clamped_context(p, tid, true);
        s_ctx[tid] = ctx;
        const int b0 = shared_full_blocks(p, ctx) > 0 && first >= 0 && first < p.num_blocks ? first : NO_SHARE;
        key = ((unsigned long long)(unsigned)b0 << 32) | (unsigned)tid;
    }
    // Up to SHARE_RANK_MAX sequences: rank sort (keys are distinct, so each
    // key's rank, the number of smaller keys, is its position). Beyond:
    // bitonic sort, one key per thread: strides below 32 by shuffles within
    // the warp (only the warps that hold keys), larger ones through shared
    // memory (every thread takes the block barriers).
    const bool keyed_warp = warp * 32 < n;
    if (B <= SHARE_RANK_MAX) {
        if (tid < B) s_in[tid] = key;
        __syncthreads();
        if (tid < B) {
            int rank = 0;
#pragma unroll 8
            for (int j = 0; j < B; ++j) rank += s_in[j] < key;
            s_key[rank] = key;
        }
        __syncthreads();
        if (tid < B) key = s_key[tid];
        n = 0;  // skips the bitonic steps
    }
    for (int k = 2; k <= n; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            unsigned long long other = key;
            if (j >= 32) {
                __syncthreads();
                if (tid < n) s_key[tid] = key;
                __syncthreads();
                if (tid < n) other = s_key[tid ^ j];
            } else if (keyed_warp) {
                other = __shfl_xor_sync(FULL_MASK, key, j);
            }
            const bool up = (tid & k) == 0, lower = (tid & j) == 0;
            if (tid < n) key = (lower == up) ? (key < other ? key : other) : (key < other ? other : key);
        }
    }
    __syncthreads();
    if (tid < n) s_key[tid] = key;
    __syncthreads();
    // Run of equal first blocks around this position, and its sub-group.
    if (tid < B) {
        const unsigned b0 = (unsigned)(key >> 32);
        int lead = tid, cnt = 1;
        if (b0 != (unsigned)NO_SHARE) {
            int lo = 0, hi = tid;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if ((unsigned)(s_key[mid] >> 32) < b0) lo = mid + 1; else hi = mid;
            }
            const int start = lo;
            lo = tid + 1;
            hi = B;
            while (lo < hi) {
                const int mid = (lo + hi) >> 1;
                if ((unsigned)(s_key[mid] >> 32) <= b0) lo = mid + 1; else hi = mid;
            }
            lead = start + (tid - start) / cap * cap;
            cnt = min(cap, lo - lead);
        }
        s_grp[tid] = lead | (cnt << 16);
    }
    __syncthreads();
    // Leading blocks each position shares with its sub-group's first member:
    // one warp per position, two positions per round (positions i and i + 32
    // of a warp's stripe), 4 x 32 table entries of each row per load batch,
    // so that B <= 64 with shared prefixes up to 128 blocks costs one
    // dependent round trip.
    for (int i0 = warp; i0 < B; i0 += 2 * (PLAN_THREADS / 32)) {
        int lcp[2], lim[2];
        const int *tm[2], *tl[2];
        bool todo[2];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int i = i0 + h * (PLAN_THREADS / 32);
            const int ii = i < B ? i : i0;
            const int lead = s_grp[ii] & 0xffff;
            const int m = (int)(s_key[ii] & 0xffffffffu), l = (int)(s_key[lead] & 0xffffffffu);
            const int nm = shared_full_blocks(p, s_ctx[m]);
            todo[h] = i < B && ii != lead;
            lim[h] = todo[h] ? min(nm, shared_full_blocks(p, s_ctx[l])) : 0;
            lcp[h] = todo[h] ? lim[h] : nm;
            tm[h] = p.block_tables + (size_t)m * W;
            tl[h] = p.block_tables + (size_t)l * W;
        }
        for (int j0 = 0; j0 < max(lim[0], lim[1]); j0 += 128) {
            int a[2][4], b[2][4];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int j = j0 + 32 * r + lane;
                    const bool in = j < lim[h] && lcp[h] == lim[h];
                    a[h][r] = in ? tm[h][j] : 0;
                    b[h][r] = in ? tl[h][j] : 0;
                }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                if (lcp[h] != lim[h] || !todo[h]) continue;  // decided (uniform across the warp)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const unsigned d = __ballot_sync(FULL_MASK, a[h][r] != b[h][r]);
                    if (d && lcp[h] == lim[h]) lcp[h] = j0 + 32 * r + __ffs(d) - 1;
                }
            }
            if ((lcp[0] != lim[0] || !todo[0]) && (lcp[1] != lim[1] || !todo[1])) break;
        }
        if (lane == 0) {
            s_lcp[i0] = lcp[0];
            if (i0 + PLAN_THREADS / 32 < B) s_lcp[i0 + PLAN_THREADS / 32] = lcp[1];
        }
    }
    __syncthreads();

    // Per position: shared tokens S of its sub-group, its partitions, and
    // (at a sub-group's first position) the shared partitions.
    int m = 0, ctx = 0, S = 0, pp = 0, sfull = 0, stail = 0, nparts = 0, pfull = 0, ptail = 0, cnt = 1;
    if (tid < B) {
        const int lead = s_grp[tid] & 0xffff;
        cnt = s_grp[tid] >> 16;
        int sh = 0;
        if (cnt >= 2) {
            sh = s_lcp[lead];
            for (int j = 1; j < cnt; ++j) sh = min(sh, s_lcp[lead + j]);
        }
        m = (int)(key & 0xffffffffu);
        ctx = s_ctx[m];
        S = sh * bs;
        pp = (S + P - 1) / P;
        sfull = (ctx - S) / P;
        stail = (ctx - S) - sfull * P;
        nparts = pp + sfull + (stail > 0);
        if (S > 0 && lead == tid) {
            pfull = S / P;
            ptail = S - pfull * P;
        }
        p.members[tid] = m;
        // A sequence with one partition and no shared blocks has its output
        // written by the attention kernel: 0 tells the merge launch to skip
        // it. With shared blocks, even one partition (its whole context in a
        // shared unit) is a partial that the merge normalises.
        p.member_nparts[tid] = S == 0 && nparts == 1 ? 0 : nparts;
        if (stail > 0) atomicAdd(&s_bin_count[(stail + 15) >> 4], 1);
        if (ptail > 0) atomicAdd(&s_bin_count[(ptail + 15) >> 4], 1);
    }
    // Pass 1: full partitions at offsets from a block-wide scan.
    const int full = pfull + sfull;
    int incl = full;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(FULL_MASK, incl, o);
        if (lane >= o) incl += v;
    }
    if (lane == 31) s_warp[warp] = incl;
    __syncthreads();
    if (warp == 0) {
        const int w = lane < PLAN_THREADS / 32 ? s_warp[lane] : 0;  // warps of the block only
        int wi = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(FULL_MASK, wi, o);
            if (lane >= o) wi += v;
        }
        s_warp[lane] = wi - w;
        if (lane == 31) {  // tails after all full partitions, longest first
            int pos = wi;
            for (int b = tiles; b >= 1; --b) {
                s_bin_next[b] = pos;
                pos += s_bin_count[b];
            }
            *p.num_entries = pos;
            *p.counter = 0;
        }
    }
    __syncthreads();
    int off = s_warp[warp] + incl - full;
    for (int j = 0; j < pfull; ++j, ++off) {
        p.entries[off] = make_int4(m, j, P, 0);
        p.entries_b[off] = make_int4(j * P, tid, cnt, 0);
    }
    for (int j = 0; j < sfull; ++j, ++off) {
        p.entries[off] = make_int4(m, pp + j, P, nparts);
        p.entries_b[off] = make_int4(S + j * P, 0, 0, 0);
    }
    // Pass 2: tails; empty sequences get zero output rows.
    if (tid < B) {
        if (stail > 0) {
            const int pos = atomicAdd(&s_bin_next[(stail + 15) >> 4], 1);
            p.entries[pos] = make_int4(m, pp + sfull, stail, nparts);
            p.entries_b[pos] = make_int4(S + sfull * P, 0, 0, 0);
        }
        if (ptail > 0) {
            const int pos = atomicAdd(&s_bin_next[(ptail + 15) >> 4], 1);
            p.entries[pos] = make_int4(m, pfull, ptail, 0);
            p.entries_b[pos] = make_int4(pfull * P, tid, cnt, 0);
        }
        if (ctx == 0) {
            const int nvec = p.num_heads * p.head_dim / 8;
            uint4 *row = static_cast<uint4 *>(p.out) + (size_t)m * nvec;
            for (int v = 0; v < nvec; ++v) row[v] = make_uint4(0, 0, 0, 0);
        }
    }
}

// ---- append (used with the CUDA-core kernel) ---------------------------------
// Writes k_new/v_new[s][h] into the slot of sequence s's last position
// (context_len - 1): slot = table[s][pos / bs] * bs + pos % bs. One thread per
// 16-byte vector of K and the matching vector of V.
__global__ void __launch_bounds__(256) pa_append_kernel(const DecodeParams p) {
    const int vpr = p.head_dim / 8;
    const long long total = (long long)p.num_seqs * p.num_kv_heads * vpr;
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += stride) {
        const long long row = i / vpr;
        const int vec = (int)(i - row * vpr);
        const int s = (int)(row / p.num_kv_heads);
        const int h = (int)(row - (long long)s * p.num_kv_heads);
        const int ctx = clamped_context(p, s, false);
        if (ctx == 0) continue;
        const int pos = ctx - 1;
        const int pb = p.block_tables[(size_t)s * p.max_blocks_per_seq + pos / p.block_size];
        if ((unsigned)pb >= (unsigned)p.num_blocks) {
            raise_error(PA_DEVERR_BLOCK_ID);
            continue;
        }
        const size_t dst = (((size_t)pb * p.num_kv_heads + h) * p.block_size + pos % p.block_size) * vpr + vec;
        static_cast<uint4 *>(const_cast<void *>(p.k_pool))[dst] = static_cast<const uint4 *>(p.k_new)[i];
        static_cast<uint4 *>(const_cast<void *>(p.v_pool))[dst] = static_cast<const uint4 *>(p.v_new)[i];
    }
}

// ---- 2. attention -------------------------------------------------------------
// Lane geometry of the score computation. A 16-token tile row is D elements =
// NV vectors of 16 bytes. Each lane holds VPL vectors of the row (so
// G*VPL*8 = 64 query values in registers) for TPL tokens; DG lanes share a
// token and their partial dot products are summed through a small
// shared-memory transpose, after which each lane owns R = G/2 (token, head)
// scores (G = 1: one score, shared by a lane pair). DG < 8 rotates each lane's
// vector order by its token group so that the 8 lanes of a shared-memory phase
// hit distinct banks. The weighted sum uses another mapping: lane l owns row
// elements [l*EPL, (l+1)*EPL) of every head, for all 16 tokens of the tile, so
// no cross-lane reduction is needed at the end.
template <int D, int G>
struct Geo {
    static constexpr int NV = D / 8;
    static constexpr int VPL = (8 / G < NV / 2) ? 8 / G : NV / 2;
    static constexpr int DG = NV / VPL;
    static constexpr int TG = 32 / DG;
    static constexpr int TPL = 16 / TG;
    static constexpr int V = TPL * G;
    static constexpr int R = G >= 2 ? G / 2 : 1;
    static constexpr bool ROT = DG < 8;
    static constexpr int NACC = TPL * G >= 4 ? 1 : 4 / (TPL * G);  // independent FMA chains
    static constexpr int EPL = D / 32;
    static constexpr int TILE_BYTES = 16 * D * 2;
    static constexpr int Q_BYTES = G * D * 2;
    static constexpr int XROW = (V % 4 == 0) ? V + 4 : V + 1;
    static constexpr int XTG = DG * XROW + ((V % 4 == 0) ? 16 : 0);
    static constexpr int XB_BYTES = G >= 2 ? ((TG * XTG * 4 + 15) & ~15) : 0;
    static constexpr int SC_BYTES = G * 16 * 4;  // probabilities of one tile, [head][token]
    static constexpr int BAR_BYTES = 16;         // up to 2 mbarriers per 16 bytes, see warp_smem_bytes
    static_assert(TG * DG == 32 && TPL * TG == 16, "lane geometry");
    static_assert(G == 1 || V == DG * R, "reduction geometry");
};

template <int D, int G, int NS>
__host__ __device__ constexpr int warp_smem_bytes() {
    return NS * Geo<D, G>::TILE_BYTES + 2 * Geo<D, G>::Q_BYTES + Geo<D, G>::XB_BYTES + Geo<D, G>::SC_BYTES +
           16 * ((NS * 8 + 15) / 16);
}

// Build-time tuning: stages of the per-warp ring and the warp cap per CTA.
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 4
#endif
#ifndef PA_DECODE_MAX_WARPS
#define PA_DECODE_MAX_WARPS 12
#endif
// Ring stages (each one 16-token K+V tile) of the tensor-core kernel, and the
// smallest head group that uses it; smaller groups use the CUDA-core kernel
// (by default every group uses the tensor-core kernel; building with
// -DPA_DECODE_TENSOR_MIN_GROUP=16 selects the CUDA-core kernel everywhere).
#ifndef PA_DECODE_MMA_STAGES
#define PA_DECODE_MMA_STAGES 2
#endif
#ifndef PA_DECODE_TENSOR_MIN_GROUP
#define PA_DECODE_TENSOR_MIN_GROUP 1
#endif
// Stages of the fp8-cache ring (its stages are half the bytes of a 16-bit one).
#ifndef PA_DECODE_MMA_STAGES_FP8
#define PA_DECODE_MMA_STAGES_FP8 2
#endif
// Warps per CTA of the fp8-cache kernel for small head groups.
#ifndef PA_DECODE_MAX_WARPS_FP8
#define PA_DECODE_MAX_WARPS_FP8 16
#endif
constexpr int DECODE_STAGES = PA_DECODE_STAGES;
constexpr int DECODE_MAX_WARPS = PA_DECODE_MAX_WARPS;
constexpr int DECODE_MMA_STAGES = PA_DECODE_MMA_STAGES;
constexpr int DECODE_MMA_STAGES_FP8 = PA_DECODE_MMA_STAGES_FP8;
constexpr int DECODE_MAX_WARPS_FP8 = PA_DECODE_MAX_WARPS_FP8;
constexpr int DECODE_TENSOR_MIN_GROUP = PA_DECODE_TENSOR_MIN_GROUP;
constexpr uint64_t WAIT_LIMIT_NS = 1000000000ull;  // 1 s
// Items of a unit over which the tensor-core kernel claims the next unit
// (the claim is three dependent global accesses, one per issued item).
constexpr int CLAIM_AHEAD = 3;
// The running maximum of a head is only raised when a score exceeds it by more
// than this many log2 units, so exponentials stay <= 2^8 and rescaling of the
// accumulators is rare. The final normalisation uses the same reference, so the
// result is the exact softmax in real arithmetic.
constexpr float LAZY_MAX_LOG2 = 8.0f;

struct Unit {
    int s, kvh, part, ntok, nparts, ntiles, tbl, slot;
    int tok0;       // first token of the unit
    int mcnt;       // shared-prefix unit: member sequences (0: sequence s alone)
    int mseq, mnp;  // lane j < mcnt: member j's sequence and its partition count
    bool valid;
};

// Hands out work-list units to one warp. Claiming a unit is a chain of three
// dependent global accesses (atomic cursor -> work-list entry -> the unit's
// block-table slice, one entry per lane); step() advances the chain for the
// next unit by one link, so that called once per issued tile (the CUDA-core
// kernel) or over a unit's last tiles (the tensor-core kernel) it has the
// next unit ready before the warp needs it; take() only finishes what is left.
// The first claims of a launch arrive about in CTA order, all at once, so
// in a longest-first list the first CTAs would take only long units and the
// last ones only short ones. Claims below `wave1` (a multiple of the warps
// per CTA, at most the number of warps) are therefore spread: claim c takes
// unit (c % K) * (wave1 / K) + c / K, K warps per CTA, so each CTA's first
// units come from every part of the list; later claims go in list order.
//
// Early start (init_early, the tensor-core kernels with the one-warp plan):
// the first wave is assigned statically instead — warp w of CTA b takes unit
// w * (number of CTAs) + b, a spread over every CTA — and the warp computes that unit's
// work-list entry itself when it is a full partition (the list starts with
// every sequence's full partitions in sequence order, a prefix sum over the
// context lengths). Later claims take wave1 + the cursor. The warp waits for
// the plan kernel (griddepcontrol.wait) only before it first needs its
// results: the cursor, a tail entry, or a merge counter.
struct UnitSource {
    const DecodeParams *p;
    int lane, total_units, Hkv, bs, blocks_per_part;
    int k, wave1;  // warps per CTA; claims spread over the first wave
    bool shared;   // entries carry a second int4 (first token, members)
    bool early;    // static first wave; cursor claims start at wave1
    bool planned;  // the plan kernel's results are visible to this warp
    bool claimed;  // u holds lane 0's raw cursor value, to be broadcast and mapped
    int state;    // 0 idle, 1 cursor claimed, 2 entry loaded, 3 table loaded, 4 list exhausted
    int u, tbl, mseq, mnp;
    int4 ent, entb;

    __device__ void init(const DecodeParams &params, int lane_id, int total, bool shared_units = false,
                         int warps_per_cta = 1, int warps_total = 0) {
        p = &params;
        lane = lane_id;
        total_units = total;
        k = warps_per_cta;
        wave1 = min(warps_total, total) / warps_per_cta * warps_per_cta;
        Hkv = params.num_kv_heads;
        bs = params.block_size;
        blocks_per_part = params.partition / params.block_size;
        shared = shared_units;
        early = false;
        planned = true;
        claimed = false;
        state = 0;
        u = 0;
        tbl = 0;
        mseq = mnp = 0;
        ent = entb = make_int4(0, 0, 0, 0);
    }

    // Early start: sets total_units from the context lengths and the warp's
    // static first claim (warp `warp` of CTA `cta`); nothing here reads what
    // the plan kernel writes. Returns total_units.
    __device__ int init_early(const DecodeParams &params, int lane_id, int warps_per_cta, int warps_total, int cta,
                              int warp) {
        init(params, lane_id, 0, false, warps_per_cta, warps_total);
        early = true;
        planned = false;
        const int B = params.num_seqs, P = params.partition;
        int tfull = 0, ntail = 0;
        for (int base = 0; base < B; base += 32) {
            const int s = base + lane;
            const int ctx = s < B ? clamped_context(params, s, false) : 0;
            int f = ctx / P;
#pragma unroll
            for (int o = 16; o >= 1; o >>= 1) f += __shfl_xor_sync(FULL_MASK, f, o);
            tfull += f;
            ntail += __popc(__ballot_sync(FULL_MASK, ctx % P != 0));
        }
        total_units = (tfull + ntail) * Hkv;
        // Warp-major over the CTAs: every CTA gets first units, from every part
        // of the longest-first list, even when there are fewer units than warps.
        wave1 = min(warps_total, total_units);
        u = warp * (warps_total / k) + cta;
        if (u >= wave1) return total_units;  // no static claim: the cursor from the start
        const int e = u / Hkv;
        state = 1;  // a tail entry: read from the plan's list (step() waits for it)
        if (e < tfull) {
            // The full partition e: sequence s with pre(s) <= e < pre(s) + full(s).
            int carry = 0;
            for (int base = 0; base < B; base += 32) {
                const int s = base + lane;
                const int ctx = s < B ? clamped_context(params, s, false) : 0;
                const int f = ctx / P;
                int incl = f;
#pragma unroll
                for (int o = 1; o < 32; o <<= 1) {
                    const int t = __shfl_up_sync(FULL_MASK, incl, o);
                    if (lane >= o) incl += t;
                }
                const unsigned hit = __ballot_sync(FULL_MASK, carry + incl - f <= e && e < carry + incl);
                if (hit) {
                    const int src = __ffs(hit) - 1;
                    const int j = __shfl_sync(FULL_MASK, e - (carry + incl - f), src);
                    const int np = __shfl_sync(FULL_MASK, f + (ctx % P != 0), src);
                    ent = make_int4(base + src, j, P, np);
                    state = 2;
                    break;
                }
                carry += __shfl_sync(FULL_MASK, incl, 31);
            }
        }
        return total_units;
    }

    // Makes the plan kernel's results visible to this warp (once).
    __device__ __forceinline__ void wait_plan() {
        if (!planned) {
            asm volatile("griddepcontrol.wait;" ::: "memory");
            planned = true;
        }
    }

    __device__ __forceinline__ void step() {
        if (state == 0) {
            wait_plan();
            int v = 0;
            if (lane == 0) v = atomicAdd(p->counter, 1);
            u = v;  // lane 0 only; broadcast in the next link
            claimed = true;
            state = 1;
        } else if (state == 1) {
            if (claimed) {
                u = __shfl_sync(FULL_MASK, u, 0);
                if (early)
                    u += wave1;
                else if (u < wave1)
                    u = (u % k) * (wave1 / k) + u / k;
                claimed = false;
            }
            if (u >= total_units) {
                state = 4;
                return;
            }
            wait_plan();
            ent = p->entries[u / Hkv];
            if (shared) entb = p->entries_b[u / Hkv];
            state = 2;
        } else if (state == 2) {
            const int nblk = (ent.z + bs - 1) / bs;
            const int blk0 = shared ? entb.x / bs : ent.y * blocks_per_part;
            tbl = lane < nblk ? p->block_tables[(size_t)ent.x * p->max_blocks_per_seq + blk0 + lane] : 0;
            if (shared && lane < entb.z) {
                mseq = p->members[entb.y + lane];
                mnp = p->member_nparts[entb.y + lane];
            }
            state = 3;
        }
    }

    // Finishes claiming the next unit; x.valid is false once the list is done.
    __device__ __forceinline__ void take(Unit &x) {
        while (state < 3) step();
        x.valid = state == 3;
        if (!x.valid) return;
        const int e = u / Hkv;
        x.kvh = u - e * Hkv;
        x.s = ent.x;
        x.part = ent.y;
        x.ntok = ent.z;
        x.nparts = ent.w;
        x.ntiles = (ent.z + 15) >> 4;
        x.tbl = tbl;
        x.tok0 = shared ? entb.x : ent.y * p->partition;
        x.mcnt = shared ? entb.z : 0;
        x.mseq = mseq;
        x.mnp = mnp;
        state = 0;
    }
};

__device__ __forceinline__ float2 f2(float a, float b) { return make_float2(a, b); }

// Merge of the partitions of one head by the log-sum-exp identity:
//   out = sum_j 2^(m_j - M) acc_j / sum_j 2^(m_j - M) l_j,  M = max_j m_j.
// ml(j) returns partition j's (m, l); acc(j) points at this lane's EPL floats
// of partition j's unnormalised output. Lane j computes partition j's weight
// (32 partitions per round) and the weights reach the other lanes by shuffle,
// so the output loop only waits on its own independent loads.
template <int EPL, typename ML, typename ACC>
__device__ __forceinline__ void merge_head(int nparts, int lane, ML ml, ACC acc, float (&o)[EPL]) {
    float M = -INFINITY;
    for (int j = lane; j < nparts; j += 32) M = fmaxf(M, ml(j).x);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL_MASK, M, off));
    float L = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
    for (int base = 0; base < nparts; base += 32) {
        float w = 0.f;
        if (base + lane < nparts) {
            const float2 v = ml(base + lane);
            w = exp2f(v.x - M);
            L = fmaf(w, v.y, L);
        }
        const int n = min(32, nparts - base);
#pragma unroll 8
        for (int jj = 0; jj < n; ++jj) {
            const float wj = __shfl_sync(FULL_MASK, w, jj);
            const float *a = acc(base + jj);
            if constexpr (EPL == 4) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(a));
                o[0] = fmaf(wj, v.x, o[0]); o[1] = fmaf(wj, v.y, o[1]);
                o[2] = fmaf(wj, v.z, o[2]); o[3] = fmaf(wj, v.w, o[3]);
            } else {
                const float2 v = __ldcg(reinterpret_cast<const float2 *>(a));
                o[0] = fmaf(wj, v.x, o[0]); o[1] = fmaf(wj, v.y, o[1]);
            }
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) L += __shfl_xor_sync(FULL_MASK, L, off);
    const float inv = 1.f / L;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] *= inv;
}

template <int EPL, typename T>
__device__ __forceinline__ void store_row(T *dst, const float (&o)[EPL]) {
    if constexpr (EPL == 4) {
        uint2 w;
        w.x = Elem<T>::pack(o[0], o[1]);
        w.y = Elem<T>::pack(o[2], o[3]);
        *reinterpret_cast<uint2 *>(dst) = w;
    } else {
        *reinterpret_cast<uint32_t *>(dst) = Elem<T>::pack(o[0], o[1]);
    }
}

// Merge for the CUDA-core kernel's partial layout: [head][part][D] floats,
// [head][part] (max, sum) pairs.
template <int D, int G, typename T>
__device__ __forceinline__ void merge_partitions(const DecodeParams &p, size_t head0, int nparts, int lane) {
    constexpr int EPL = D / 32;
    T *out = static_cast<T *>(p.out);
#pragma unroll 1
    for (int g = 0; g < G; ++g) {
        const size_t row0 = (head0 + g) * p.max_parts;
        float o[EPL];
        merge_head<EPL>(
            nparts, lane, [&](int j) { return __ldcg(&p.ml[row0 + j]); },
            [&](int j) { return p.part_acc + (row0 + j) * D + lane * EPL; }, o);
        store_row<EPL>(out + (head0 + g) * D + lane * EPL, o);
    }
}

template <int D, int G, typename T, int NS>
__global__ void __launch_bounds__(DECODE_MAX_WARPS * 32, 1) pa_decode_kernel(const DecodeParams p) {
    using Gm = Geo<D, G>;
    extern __shared__ __align__(128) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int Hkv = p.num_kv_heads, H = p.num_heads, bs = p.block_size;

    uint8_t *ring = smem + (size_t)warp * warp_smem_bytes<D, G, NS>();
    uint8_t *qbuf = ring + NS * Gm::TILE_BYTES;
    float *xb = reinterpret_cast<float *>(qbuf + 2 * Gm::Q_BYTES);
    float *sc = reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(xb) + Gm::XB_BYTES);
    uint64_t *bars = reinterpret_cast<uint64_t *>(reinterpret_cast<uint8_t *>(sc) + Gm::SC_BYTES);
    const uint32_t ring_s = smem_u32(ring), qbuf_s = smem_u32(qbuf), bar_s = smem_u32(bars);

    if (lane == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(bar_s + 8 * i, 1);
        fence_barrier_init();
    }
    __syncwarp();
    const uint64_t policy = l2_policy_evict_first();
    // The work list is written by the plan kernel that precedes this one.
    asm volatile("griddepcontrol.wait;" ::: "memory");

    const T *kpool = static_cast<const T *>(p.k_pool);
    const T *vpool = static_cast<const T *>(p.v_pool);
    const T *qg = static_cast<const T *>(p.q);
    const int total_units = *p.num_entries * Hkv;

    // Score-phase lane geometry.
    const int tg = lane / Gm::DG, dg = lane % Gm::DG;
    int voff[Gm::VPL];
#pragma unroll
    for (int c = 0; c < Gm::VPL; ++c)
        voff[c] = 16 * (dg + Gm::DG * (Gm::ROT ? ((c + tg) % Gm::VPL) : c));
    const int i_own = G >= 2 ? dg / 2 : 0;
    const int t_own = tg + Gm::TG * i_own;
    const int g0 = G >= 2 ? (dg & 1) * Gm::R : 0;
    const bool owner = G >= 2 || dg == 0;

    UnitSource src;
    src.init(p, lane, total_units);
    auto fetch = [&](Unit &x) { src.take(x); };

    // Item `it` of a unit: even items are K tiles, odd items V tiles (tile it/2);
    // item 0 also brings the unit's G query rows.
    auto issue = [&](int s, int kvh, int tbl, int qslot, int it, uint32_t stage) {
        const bool is_v = it & 1;
        const int tok = 16 * (it >> 1);
        const int bi = tok / bs;
        const int pb = __shfl_sync(FULL_MASK, tbl, bi);
        if (lane == 0) {
            const uint32_t bar = bar_s + 8 * stage;
            const bool ok = (unsigned)pb < (unsigned)p.num_blocks;
            if (!ok) raise_error(PA_DEVERR_BLOCK_ID);
            const uint32_t bytes = (ok ? Gm::TILE_BYTES : 0) + (it == 0 ? Gm::Q_BYTES : 0);
            fence_proxy_async_smem();
            if (bytes) {
                mbar_arrive_expect_tx(bar, bytes);
                if (ok) {
                    const T *pool = is_v ? vpool : kpool;
                    const T *src = pool + (((size_t)pb * Hkv + kvh) * bs + (tok - bi * bs)) * D;
                    bulk_load(ring_s + stage * Gm::TILE_BYTES, src, Gm::TILE_BYTES, bar, policy);
                }
                if (it == 0)
                    bulk_load(qbuf_s + qslot * Gm::Q_BYTES, qg + ((size_t)s * H + kvh * G) * D, Gm::Q_BYTES, bar,
                              policy);
            } else {
                mbar_arrive(bar);
            }
        }
    };

    Unit cur, nxt;
    fetch(cur);
    if (!cur.valid) return;
    cur.slot = 0;
    nxt.valid = false;
    int next_slot = 1;
    bool prod_on_nxt = false, exhausted = false;
    int pitem = 0;
    uint32_t issued = 0, consumed = 0;

    // Issue the producer's next item; open the next unit when the current one
    // is fully issued (never more than one unit ahead of the consumer).
    auto produce = [&]() {
        if (exhausted) return;
        if (pitem >= 2 * (prod_on_nxt ? nxt.ntiles : cur.ntiles)) {
            if (prod_on_nxt) return;
            fetch(nxt);
            if (!nxt.valid) {
                exhausted = true;
                return;
            }
            nxt.slot = next_slot;
            next_slot ^= 1;
            prod_on_nxt = true;
            pitem = 0;
        }
        if (prod_on_nxt)
            issue(nxt.s, nxt.kvh, nxt.tbl, nxt.slot, pitem, issued % NS);
        else
            issue(cur.s, cur.kvh, cur.tbl, cur.slot, pitem, issued % NS);
        ++pitem;
        ++issued;
        src.step();  // one link of the next unit's claim per issued item
    };

    // Wait for the consumer's next item; on a timeout flag it, wait (bounded)
    // for the copies still in flight, and report failure.
    auto wait_item = [&]() -> bool {
        const uint32_t stage = consumed % NS, parity = (consumed / NS) & 1;
        bool ok = mbar_wait_bounded(bar_s + 8 * stage, parity, WAIT_LIMIT_NS);
        ok = __all_sync(FULL_MASK, ok);
        if (!ok) {
            if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
            for (uint32_t c = consumed; c < issued; ++c)
                mbar_wait_bounded(bar_s + 8 * (c % NS), (c / NS) & 1, WAIT_LIMIT_NS);
        }
        return ok;
    };

    for (int i = 0; i < NS; ++i) produce();

    float2 qf[G][Gm::VPL * 4];     // query pairs, pre-scaled by scale*log2(e)
    float2 acc[G][Gm::EPL];        // (even-token, odd-token) partial sums of p*v

    for (;;) {
        float Mg[G];               // reference maximum per head (log2 units)
        float ls[Gm::R];           // this lane's sum of its owned probabilities
#pragma unroll
        for (int g = 0; g < G; ++g) {
            Mg[g] = -INFINITY;
#pragma unroll
            for (int e = 0; e < Gm::EPL; ++e) acc[g][e] = f2(0.f, 0.f);
        }
#pragma unroll
        for (int r = 0; r < Gm::R; ++r) ls[r] = 0.f;

        for (int k = 0; k < cur.ntiles; ++k) {
            // ------------------------------ scores of tile k ----------------
            if (!wait_item()) return;
            const uint8_t *tile = ring + (consumed % NS) * Gm::TILE_BYTES;
            if (k == 0) {
                const uint8_t *qs = qbuf + cur.slot * Gm::Q_BYTES;
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int c = 0; c < Gm::VPL; ++c) {
                        const uint4 raw = *reinterpret_cast<const uint4 *>(qs + g * D * 2 + voff[c]);
                        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const float2 v = Elem<T>::pair(w[j]);
                            qf[g][c * 4 + j] = f2(v.x * p.qscale, v.y * p.qscale);
                        }
                    }
            }
            const int valid = min(16, cur.ntok - 16 * k);
            float part[Gm::TPL][G];
#pragma unroll
            for (int i = 0; i < Gm::TPL; ++i) {
                const uint8_t *row = tile + (tg + Gm::TG * i) * (D * 2);
                float2 a2[G][Gm::NACC];
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int n = 0; n < Gm::NACC; ++n) a2[g][n] = f2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < Gm::VPL; ++c) {
                    const uint4 raw = *reinterpret_cast<const uint4 *>(row + voff[c]);
                    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 kv = Elem<T>::pair(w[j]);
#pragma unroll
                        for (int g = 0; g < G; ++g) {
                            float2 &a = a2[g][(c * 4 + j) % Gm::NACC];
                            a = __ffma2_rn(qf[g][c * 4 + j], kv, a);
                        }
                    }
                }
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    float sum = 0.f;
#pragma unroll
                    for (int n = 0; n < Gm::NACC; ++n) sum += a2[g][n].x + a2[g][n].y;
                    part[i][g] = sum;
                }
            }
            float sred[Gm::R];
            if constexpr (G == 1) {
                float v = part[0][0];
                v += __shfl_xor_sync(FULL_MASK, v, 1);
                sred[0] = v;
            } else {
                float *xrow = xb + tg * Gm::XTG + dg * Gm::XROW;
                if constexpr (Gm::V % 4 == 0) {
#pragma unroll
                    for (int j = 0; j < Gm::V; j += 4)
                        *reinterpret_cast<float4 *>(xrow + j) =
                            make_float4(part[j / G][j % G], part[(j + 1) / G][(j + 1) % G],
                                        part[(j + 2) / G][(j + 2) % G], part[(j + 3) / G][(j + 3) % G]);
                } else {
#pragma unroll
                    for (int j = 0; j < Gm::V; ++j) xrow[j] = part[j / G][j % G];
                }
                __syncwarp();
#pragma unroll
                for (int r = 0; r < Gm::R; ++r) sred[r] = 0.f;
#pragma unroll
                for (int d2 = 0; d2 < Gm::DG; ++d2) {
                    const float *src = xb + tg * Gm::XTG + d2 * Gm::XROW + dg * Gm::R;
                    if constexpr (Gm::R == 4) {
                        const float4 v = *reinterpret_cast<const float4 *>(src);
                        sred[0] += v.x; sred[1] += v.y; sred[2] += v.z; sred[3] += v.w;
                    } else if constexpr (Gm::R == 2) {
                        const float2 v = *reinterpret_cast<const float2 *>(src);
                        sred[0] += v.x; sred[1] += v.y;
                    } else {
                        sred[0] += src[0];
                    }
                }
            }
            // Tokens past the context (stale or never-written slots) get -inf.
            const bool tvalid = t_own < valid;
            float mown[Gm::R];
            bool raise = false;
#pragma unroll
            for (int r = 0; r < Gm::R; ++r) {
                sred[r] = tvalid ? sred[r] : -INFINITY;
                mown[r] = 0.f;
#pragma unroll
                for (int g = 0; g < G; ++g)
                    if (g == g0 + r) mown[r] = Mg[g];
                raise |= !(sred[r] <= mown[r] + LAZY_MAX_LOG2);
            }
            // ------------------------------ online softmax ------------------
            if (__any_sync(FULL_MASK, raise)) {
                float tm[G];
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    tm[g] = -INFINITY;
#pragma unroll
                    for (int r = 0; r < Gm::R; ++r)
                        if (g == g0 + r) tm[g] = fmaxf(tm[g], sred[r]);
                }
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
                    for (int g = 0; g < G; ++g) tm[g] = fmaxf(tm[g], __shfl_xor_sync(FULL_MASK, tm[g], o));
#pragma unroll
                for (int g = 0; g < G; ++g) {
                    const float mn = fmaxf(Mg[g], tm[g]);
                    const float alpha = exp2f(Mg[g] - mn);  // 0 on the first tile (Mg = -inf)
                    Mg[g] = mn;
#pragma unroll
                    for (int e = 0; e < Gm::EPL; ++e) acc[g][e] = __fmul2_rn(acc[g][e], f2(alpha, alpha));
#pragma unroll
                    for (int r = 0; r < Gm::R; ++r)
                        if (g == g0 + r) {
                            ls[r] *= alpha;
                            mown[r] = mn;
                        }
                }
            }
#pragma unroll
            for (int r = 0; r < Gm::R; ++r) {
                const float e = exp2f(sred[r] - mown[r]);
                ls[r] += e;
                if (owner) sc[(g0 + r) * 16 + t_own] = e;
            }
            ++consumed;
            __syncwarp();
            produce();

            // ------------------------------ values of tile k ----------------
            if (!wait_item()) return;
            tile = ring + (consumed % NS) * Gm::TILE_BYTES;
#pragma unroll
            for (int t4 = 0; t4 < 4; ++t4) {
                float4 pq[G];
#pragma unroll
                for (int g = 0; g < G; ++g) pq[g] = *reinterpret_cast<const float4 *>(sc + g * 16 + 4 * t4);
#pragma unroll
                for (int h2 = 0; h2 < 2; ++h2) {
                    const int t = 4 * t4 + 2 * h2;
                    const uint8_t *src = tile + t * (D * 2) + lane * (Gm::EPL * 2);
                    float2 vp[Gm::EPL];  // (token t, token t+1) of each owned element
                    if constexpr (Gm::EPL == 4) {
                        uint2 r0 = *reinterpret_cast<const uint2 *>(src);
                        uint2 r1 = *reinterpret_cast<const uint2 *>(src + D * 2);
                        if (t >= valid) r0 = make_uint2(0, 0);       // never multiply stale slots
                        if (t + 1 >= valid) r1 = make_uint2(0, 0);
                        const float2 a = Elem<T>::pair(r0.x), b = Elem<T>::pair(r0.y);
                        const float2 c = Elem<T>::pair(r1.x), d = Elem<T>::pair(r1.y);
                        vp[0] = f2(a.x, c.x); vp[1] = f2(a.y, c.y);
                        vp[2] = f2(b.x, d.x); vp[3] = f2(b.y, d.y);
                    } else {
                        uint32_t r0 = *reinterpret_cast<const uint32_t *>(src);
                        uint32_t r1 = *reinterpret_cast<const uint32_t *>(src + D * 2);
                        if (t >= valid) r0 = 0;
                        if (t + 1 >= valid) r1 = 0;
                        const float2 a = Elem<T>::pair(r0), c = Elem<T>::pair(r1);
                        vp[0] = f2(a.x, c.x); vp[1] = f2(a.y, c.y);
                    }
#pragma unroll
                    for (int g = 0; g < G; ++g) {
                        const float2 pp = h2 ? f2(pq[g].z, pq[g].w) : f2(pq[g].x, pq[g].y);
#pragma unroll
                        for (int e = 0; e < Gm::EPL; ++e) acc[g][e] = __ffma2_rn(pp, vp[e], acc[g][e]);
                    }
                }
            }
            ++consumed;
            __syncwarp();
            produce();
        }

        // ---------------- totals and store -------------------------------------
        float Lg[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float l = 0.f;
#pragma unroll
            for (int r = 0; r < Gm::R; ++r)
                if (owner && g == g0 + r) l = ls[r];
            Lg[g] = l;
        }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
            for (int g = 0; g < G; ++g) Lg[g] += __shfl_xor_sync(FULL_MASK, Lg[g], o);

        const size_t head0 = (size_t)cur.s * H + (size_t)cur.kvh * G;
        if (cur.nparts == 1) {
            T *out = static_cast<T *>(p.out);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const float inv = 1.f / Lg[g];
                T *dst = out + (head0 + g) * D + lane * Gm::EPL;
                if constexpr (Gm::EPL == 4) {
                    uint2 w;
                    w.x = Elem<T>::pack((acc[g][0].x + acc[g][0].y) * inv, (acc[g][1].x + acc[g][1].y) * inv);
                    w.y = Elem<T>::pack((acc[g][2].x + acc[g][2].y) * inv, (acc[g][3].x + acc[g][3].y) * inv);
                    *reinterpret_cast<uint2 *>(dst) = w;
                } else {
                    *reinterpret_cast<uint32_t *>(dst) =
                        Elem<T>::pack((acc[g][0].x + acc[g][0].y) * inv, (acc[g][1].x + acc[g][1].y) * inv);
                }
            }
        } else {
#pragma unroll
            for (int g = 0; g < G; ++g) {
                const size_t row = (head0 + g) * p.max_parts + cur.part;
                float *dst = p.part_acc + row * D + lane * Gm::EPL;
                if constexpr (Gm::EPL == 4)
                    *reinterpret_cast<float4 *>(dst) =
                        make_float4(acc[g][0].x + acc[g][0].y, acc[g][1].x + acc[g][1].y,
                                    acc[g][2].x + acc[g][2].y, acc[g][3].x + acc[g][3].y);
                else
                    *reinterpret_cast<float2 *>(dst) = f2(acc[g][0].x + acc[g][0].y, acc[g][1].x + acc[g][1].y);
                if (lane == g) p.ml[row] = f2(Mg[g], Lg[g]);
            }
            // The last partition of this (sequence, KV head) to finish merges all.
            const bool last = count_partition(&p.merge_count[(size_t)cur.s * Hkv + cur.kvh], cur.nparts, lane == 0);
            if (__shfl_sync(FULL_MASK, last, 0)) merge_partitions<D, G, T>(p, head0, cur.nparts, lane);
        }

        // ---------------- next unit -------------------------------------------
        while (!prod_on_nxt && !exhausted) produce();
        if (!prod_on_nxt) break;
        cur = nxt;
        prod_on_nxt = false;
    }
}

}  // namespace pa
