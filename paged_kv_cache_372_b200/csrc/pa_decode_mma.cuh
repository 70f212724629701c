// Paged decode attention on tensor cores (the default kernel, any head group).
//
// Same work list, unit scheduling, online softmax and split merge as
// pa_decode_kernel (pa_decode.cuh); the per-tile arithmetic differs. With G
// query heads per KV head, one 16-token tile gives two small dense products
// per warp, each a single mma.sync m16n8k16 per 16-wide slice:
//
//   S^T[16 tokens x 8 heads]  = K_tile[16 x D] . Q^T[D x 8]       (D/16 MMAs)
//   O^T[D x 8 heads]         += V_tile^T[D x 16] . P^T[16 x 8]    (D/16 MMAs)
//
// heads padded to N = 8 with zero query rows. K and V tiles arrive by tiled
// TMA (cp.async.bulk.tensor, 128-byte swizzle) so the ldmatrix fragment loads
// are bank-conflict free; the probabilities P go from the S accumulators to
// the B operand of the second product by an in-register 8x8 transpose
// (movmatrix). Scores, softmax state and O^T stay in fp32; P is rounded to the
// input type for the second product and the softmax denominator sums the
// same rounded values.
//
// An item (one ring stage) is one such tile, or two (32 tokens) where a
// 16-token tile is at most 4 KB (mma_tile_rows).
//
// Variants (template flags): KV8 reads an 8-bit cache (byte tiles widened to
// f16 in registers), I8 with INT8 codes, HS the scales' granularity (0: one
// per tensor, 1: one per KV head, 2: one per (physical block, KV head));
// SHARED lets a unit serve up to 16 / G sequences that share the unit's
// blocks, their G query rows each filling columns of two 8-column MMA tiles
// (pa_decode_shared and pa_decode_shared_quant, 8 warps per CTA).
#pragma once

#include <cuda.h>
#include <cuda_fp8.h>

#include <type_traits>

#include "pa_decode.cuh"

namespace pa {

// KV8: the pools hold 8-bit codes (E4M3, or INT8 with I8), one byte per
// element, dequantised with per-tensor or (HS) per-KV-head scales: the key
// scale folded into the score scale, the value scale into the output scale.
//
// A tile row is D * EB bytes: 256 or 128 (loaded in 128-byte boxes with the
// 128-byte swizzle) or 64 (an 8-bit cache at head_dim 64: one 64-byte box
// with the 64-byte swizzle).
template <int D, int G, bool KV8 = false, int TR_ = 16>
struct MmaGeo {
    static_assert(G == 1 || G == 2 || G == 4 || G == 8, "head group size");
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static constexpr int TR = TR_;                        // tokens (rows) of one item
    static constexpr int EB = KV8 ? 1 : 2;                // bytes per pool element
    static constexpr int KS = D / 16;                     // 16-wide slices of a row
    static constexpr int ROW_BYTES = D * EB;
    static constexpr int BOX_ROW = ROW_BYTES < 128 ? ROW_BYTES : 128;  // bytes of a box row
    static constexpr int BOX_ELEMS = BOX_ROW / EB;        // elements of a box row (TMA box width)
    static constexpr int NBOX = ROW_BYTES / BOX_ROW;      // TMA boxes per row
    static constexpr int BOX_BYTES = 16 * BOX_ROW;        // one box of a 16-row tile
    static constexpr int CHUNKS = ROW_BYTES / 16;         // 16-byte chunks of a row
    static constexpr int HALF_BYTES = TR * D * EB;        // one K (or V) tile
    static constexpr int STAGE_BYTES = 2 * HALF_BYTES;    // K then V of one tile
    static constexpr int SUB_BYTES = 2 * 16 * D * EB;     // K and V rows of one 16-row sub-tile
    static_assert(TR == 16 || (TR == 32 && NBOX == 1), "32-row tiles take one box per row");
    // Byte offset of 16-byte chunk `chunk` of row `row` of a tile.
    static __device__ __forceinline__ uint32_t addr(int row, int chunk);
};

// Tokens per item (stage): 32 where a 16-token tile of K and V is at most
// 4 KB (an 8-bit cache, or head_dim 64) and the units are not shared: two
// 16-token MMA sub-tiles behind one wait, one softmax update and one issue,
// which halves the per-token share of that fixed work. 16 otherwise.
template <int D, bool KV8, bool SHARED>
__host__ __device__ constexpr int mma_tile_rows() {
    return !SHARED && (KV8 || D == 64) ? 32 : 16;
}

// Query rows of a unit shared by several sequences: two n8 column halves of
// the MMA tile, the G rows of each of up to 16 / G member sequences.
constexpr int SHARE_ROWS = 16;

// Query slots of a warp: the G rows of one sequence, double-buffered (the
// next unit's rows arrive while the current unit runs), or for units shared
// by several sequences one slot of SHARE_ROWS rows that the next unit's rows
// may fill once the current unit has read its own.
template <int D, int G, bool SHARED>
__host__ __device__ constexpr int mma_q_slot_bytes() {
    return (SHARED ? SHARE_ROWS : G) * D * 2;
}
template <bool SHARED>
__host__ __device__ constexpr int mma_q_slots() {
    return SHARED ? 1 : 2;
}

template <int D, int G, int NS, bool KV8 = false, bool SHARED = false>
__host__ __device__ constexpr int mma_warp_bytes() {
    return NS * MmaGeo<D, G, KV8, mma_tile_rows<D, KV8, SHARED>()>::STAGE_BYTES +
           mma_q_slots<SHARED>() * mma_q_slot_bytes<D, G, SHARED>() + NS * 8;
}

template <int D, int G, int NS, bool KV8 = false, bool SHARED = false>
__host__ __device__ constexpr int mma_smem_bytes(int warps) {
    // 1024 bytes of slack re-align the base for the 128-byte swizzle pattern.
    return 1024 + warps * mma_warp_bytes<D, G, NS, KV8, SHARED>();
}

// Warps per CTA: the 8-bit kernel at head_dim 64 runs DECODE_MAX_WARPS_FP8
// warps for small head groups (up to 4 query heads per KV head, where it fits
// 128 registers a thread); at head_dim 128 its 32-token stages leave shared
// memory for DECODE_MAX_WARPS (up to 170 registers a thread).
#ifndef PA_FP8_WIDE_MAX_GROUP
#define PA_FP8_WIDE_MAX_GROUP 4
#endif
// Shared-prefix units keep a second half of query columns (accumulators and
// query fragments): 8 warps per CTA, so each thread has up to 255 registers.
constexpr int SHARE_MAX_WARPS = 8;
// 8 query heads per KV head at head_dim 128: a full 8-column MMA tile of
// accumulators per slice; 8 warps per CTA give each thread 255 registers.
#ifndef PA_G8_MAX_WARPS
#define PA_G8_MAX_WARPS 8
#endif
constexpr int G8_MAX_WARPS = PA_G8_MAX_WARPS;
template <int D, int G, bool KV8, bool SHARED = false>
__host__ __device__ constexpr int mma_max_warps() {
    return SHARED ? SHARE_MAX_WARPS
                  : KV8 && D == 64 && G <= PA_FP8_WIDE_MAX_GROUP ? DECODE_MAX_WARPS_FP8
                  : G == 8 && D == 128 ? G8_MAX_WARPS : DECODE_MAX_WARPS;
}

// E4M3 -> f16 widening: every E4M3 value is exactly an f16. One cvt converts
// the two codes of one 16-bit half of a register; taking the half through a
// register split (rather than a shift) keeps it to one instruction.
// Codes in bytes 0 and 1 (low byte first) -> two f16.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t codes) {
    uint32_t r;
    asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n cvt.rn.f16x2.e4m3x2 %0, lo;\n}" : "=r"(r) : "r"(codes));
    return r;
}
// Codes in bytes 2 and 3 -> two f16.
__device__ __forceinline__ uint32_t e4m3x2_hi_to_f16x2(uint32_t codes) {
    uint32_t r;
    asm("{\n .reg .b16 lo, hi;\n mov.b32 {lo, hi}, %1;\n cvt.rn.f16x2.e4m3x2 %0, hi;\n}" : "=r"(r) : "r"(codes));
    return r;
}

// INT8 cache, stored excess-128 (byte u holds u - 128): the f16 number with
// high byte 0x64 and low byte u is exactly 1024 + u, so one byte permute per
// pair of codes makes the MMA operand. For keys the constant 1152 = 1024 + 128
// is taken off the scores afterwards (one correction per query row). Values
// take it off in f16 before their product (i8_unbias, exact), since the
// output sums grow over a whole partition and 1152 * (sum of the weights) in
// fp32 would cost them about ten bits.
// Codes in bytes 0 and 1 (low byte first) -> two f16.
__device__ __forceinline__ uint32_t i8x2_to_f16x2(uint32_t codes) { return __byte_perm(codes, 0x64646464u, 0x4140); }
// Codes in bytes 2 and 3 -> two f16.
__device__ __forceinline__ uint32_t i8x2_hi_to_f16x2(uint32_t codes) {
    return __byte_perm(codes, 0x64646464u, 0x4342);
}
constexpr float I8_OFFSET = 1152.f;
// (1024 + u) - 1152 = u - 128, the signed code, exactly (two f16 at once).
__device__ __forceinline__ uint32_t i8_unbias(uint32_t w) {
    uint32_t r;
    asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(r) : "r"(w), "r"(0x64806480u));  // f16 1152 = 0x6480
    return r;
}

// Two 16-bit query elements of type T -> f16x2 (bf16 -> f16 is exact in f16's
// normal range). A bf16 element above f16's largest finite value (65504)
// would become infinite: `big` is set so that the caller can flag it.
template <typename T>
__device__ __forceinline__ uint32_t to_f16x2(uint32_t w, bool &big) {
    if constexpr (std::is_same<T, __half>::value) {
        return w;
    } else {
        const float2 f = Elem<T>::pair(w);
        big |= fabsf(f.x) > 65504.f || fabsf(f.y) > 65504.f;
        return Elem<__half>::pack(f.x, f.y);
    }
}

template <typename T>
struct MmaType;
template <>
struct MmaType<__nv_bfloat16> {
    static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    static constexpr CUtensorMapDataType tma_type = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
};
template <>
struct MmaType<__half> {
    static __device__ __forceinline__ void mma(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    static constexpr CUtensorMapDataType tma_type = CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
};

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

// Tiled 2-D TMA load of one box {x = column, y = row} into this CTA's shared memory.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap *map, int x, int y, uint32_t bar,
                                            uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

// Byte offset of 16-byte chunk `chunk` of row `row` inside a tile loaded as
// NBOX boxes of [16 rows][128 bytes] with the 128-byte swizzle: within each
// 1024-byte group of 8 rows the chunk index is XORed with the row index.
__device__ __forceinline__ uint32_t swz(int row, int chunk) {
    return (uint32_t)((chunk >> 3) * 2048 + row * 128 + (((chunk & 7) ^ (row & 7)) << 4));
}

// The same for one box of [16 rows][64 bytes] with the 64-byte swizzle: the
// chunk index (0..3) is XORed with bits 1..2 of the row index, so the 8 rows
// an ldmatrix phase reads fall in distinct banks.
__device__ __forceinline__ uint32_t swz64(int row, int chunk) {
    return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

template <int D, int G, bool KV8, int TR_>
__device__ __forceinline__ uint32_t MmaGeo<D, G, KV8, TR_>::addr(int row, int chunk) {
    if constexpr (BOX_ROW == 64)
        return swz64(row, chunk);
    else
        return swz(row, chunk);
}

// Merge of partial slots [first, first + nparts) of one (sequence, KV head)
// for this kernel's partial layout: [slot][D][G] floats and [slot][G] (max,
// sum) pairs (head-innermost, so the accumulator fragments store as pairs).
// All G heads in one pass: lane j computes slot j's G weights (32 slots per
// round), the weights reach the other lanes by shuffle, and each lane reads
// its EPL x G contiguous floats of every slot with vector loads. With
// dst_slot < 0 the result is normalised into the output rows; otherwise it is
// written, unnormalised with its (max, sum), to partial slot dst_slot (a chunk
// merge, see MERGE_FANIN).
// LEAN (where registers are scarce: the 8-bit kernels, and 8 query heads at
// head_dim 128) keeps fewer values live: the
// (max, sum) pairs are read twice and no partials are loaded ahead.
template <int D, int G, typename T, bool LEAN = false>
__device__ __forceinline__ void mma_merge(const DecodeParams &p, size_t group, size_t head0, int first, int nparts,
                                          int lane, int dst_slot = -1) {
    constexpr int EPL = D / 32;
    constexpr int F = EPL * G;                             // floats of one partition per lane
    constexpr int VW = F >= 4 ? 4 : F;                     // floats per vector load (4 or 2)
    constexpr int NV4 = F / VW;                            // vector loads per partition per lane
    // partitions whose partials load up front, and in flight in the loop
    constexpr int PF = LEAN ? 0 : (F <= 8 ? 4 : (F <= 16 ? 1 : 0));
    constexpr int MERGE_UNROLL = F >= 32 ? 2 : 4;
    const float2 *ml = p.ml + (group * p.max_parts + first) * G;
    const float *acc = p.part_acc + (group * p.max_parts + first) * (size_t)(D * G);
    auto load = [&](int j, float (&f)[F]) {
        const float *a = acc + (size_t)j * D * G + lane * F;
#pragma unroll
        for (int i = 0; i < NV4; ++i) {
            if constexpr (VW == 4) {
                const float4 v = __ldcg(reinterpret_cast<const float4 *>(a) + i);
                f[4 * i] = v.x; f[4 * i + 1] = v.y; f[4 * i + 2] = v.z; f[4 * i + 3] = v.w;
            } else {
                const float2 v = __ldcg(reinterpret_cast<const float2 *>(a) + i);
                f[2 * i] = v.x; f[2 * i + 1] = v.y;
            }
        }
    };
    // The first partitions' partials are requested together with the (max,
    // sum) pairs, which each lane reads once (lane j: partition j), so the
    // usual few-partition merge waits on one round of loads.
    float pre[PF > 0 ? PF : 1][F];
#pragma unroll
    for (int q = 0; q < PF; ++q) {
        if (q < nparts) {
            load(q, pre[q]);
        } else {
#pragma unroll
            for (int c = 0; c < F; ++c) pre[q][c] = 0.f;
        }
    }
    float2 mine[LEAN ? 1 : G];
    float M[G], L[G], o[F];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float2 v = lane < nparts ? __ldcg(&ml[lane * G + g]) : make_float2(-INFINITY, 0.f);
        if constexpr (!LEAN) mine[g] = v;
        M[g] = v.x;
        L[g] = 0.f;
    }
    for (int j = lane + 32; j < nparts; j += 32)
#pragma unroll
        for (int g = 0; g < G; ++g) M[g] = fmaxf(M[g], __ldcg(&ml[j * G + g].x));
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) M[g] = fmaxf(M[g], __shfl_xor_sync(FULL_MASK, M[g], off));
#pragma unroll
    for (int c = 0; c < F; ++c) o[c] = 0.f;
    for (int base = 0; base < nparts; base += 32) {
        float w[G];
#pragma unroll
        for (int g = 0; g < G; ++g) {
            float2 v;
            if (!LEAN && base == 0)
                v = mine[LEAN ? 0 : g];
            else
                v = base + lane < nparts ? __ldcg(&ml[(base + lane) * G + g]) : make_float2(-INFINITY, 0.f);
            w[g] = base + lane < nparts ? exp2f(v.x - M[g]) : 0.f;
            L[g] = fmaf(w[g], v.y, L[g]);
        }
        const int n = min(32, nparts - base);
        int jj = 0;
        if (PF > 0 && base == 0) {
#pragma unroll
            for (int q = 0; q < PF; ++q) {
                float wj[G];
#pragma unroll
                for (int g = 0; g < G; ++g) wj[g] = __shfl_sync(FULL_MASK, w[g], q);  // 0 past nparts
#pragma unroll
                for (int c = 0; c < F; ++c) o[c] = fmaf(wj[c % G], pre[q][c], o[c]);
            }
            jj = PF;
        }
#pragma unroll MERGE_UNROLL
        for (; jj < n; ++jj) {
            float f[F];
            load(base + jj, f);
            float wj[G];
#pragma unroll
            for (int g = 0; g < G; ++g) wj[g] = __shfl_sync(FULL_MASK, w[g], jj);
#pragma unroll
            for (int c = 0; c < F; ++c) o[c] = fmaf(wj[c % G], f[c], o[c]);
        }
    }
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1)
#pragma unroll
        for (int g = 0; g < G; ++g) L[g] += __shfl_xor_sync(FULL_MASK, L[g], off);
    if (dst_slot >= 0) {
        const size_t slot = group * p.max_parts + dst_slot;
        float *dst = p.part_acc + slot * (size_t)(D * G) + lane * F;
#pragma unroll
        for (int i = 0; i < NV4; ++i) {
            if constexpr (VW == 4)
                __stcg(reinterpret_cast<float4 *>(dst) + i,
                       make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]));
            else
                __stcg(reinterpret_cast<float2 *>(dst) + i, make_float2(o[2 * i], o[2 * i + 1]));
        }
#pragma unroll
        for (int g = 0; g < G; ++g)
            if (lane == g) p.ml[slot * G + g] = make_float2(M[g], L[g]);
        return;
    }
    T *out = static_cast<T *>(p.out);
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const float inv = 1.f / L[g];
        float r[EPL];
#pragma unroll
        for (int e = 0; e < EPL; ++e) r[e] = o[e * G + g] * inv;
        store_row<EPL>(out + (head0 + g) * D + lane * EPL, r);
    }
}

// The split-context merge as its own launch (DecodeParams::reduce_launch, for
// sequences of many partitions; see REDUCE_LAUNCH_MIN_PARTS): one CTA
// per (sequence, KV head), REDUCE_GROUPS thread groups of D*G/4 threads, each
// thread one float4 of the [D][G] partial row of every partition in its
// group's share (partitions r, r + REDUCE_GROUPS, ...); the groups' sums
// combine in shared memory. The arithmetic of mma_merge:
// out = sum_j 2^(m_j - M) acc_j / sum_j 2^(m_j - M) l_j.
constexpr int REDUCE_GROUPS = 4;

// Partitions above which a sequence's split merge runs in the merge launch
// (pa_reduce_kernel, one CTA per (sequence, KV head), its partitions shared
// by four thread groups) instead of in the attention kernel's last-arriving
// warps; the launch happens when some sequence has more, and the others still
// merge in the attention kernel. Measured: long32k with 64 partitions per
// sequence 189.3 -> 178.1 us (fp8 cache 119.3 -> 107.9 us); llama3_8b, where
// the few long sequences have up to 11, 146.2 -> 149.5 us with every merge
// moved (the launch costs more than the merges it moves).
constexpr int REDUCE_LAUNCH_MIN_PARTS = 16;

// The merge launch of shared-prefix decode: a member has few partitions (its
// shared ones and its own), so one warp merges one (grouping position, KV
// head) with mma_merge, 8 per CTA; the sequence and its partition count come
// from the grouping plan's members / member_nparts.
template <int D, int G, typename T>
__global__ void __launch_bounds__(256) pa_reduce_members_kernel(const DecodeParams p) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int lane = threadIdx.x & 31;
    const int item = blockIdx.x * 8 + (threadIdx.x >> 5);
    if (item >= p.num_seqs * p.num_kv_heads) return;
    const int pos = item / p.num_kv_heads, kvh = item - pos * p.num_kv_heads;
    const int s = p.members[pos], nparts = p.member_nparts[pos];
    if (nparts < 1) return;  // empty, or written by the attention kernel (member_nparts 0)
    mma_merge<D, G, T>(p, (size_t)s * p.num_kv_heads + kvh, (size_t)s * p.num_heads + (size_t)kvh * G, 0, nparts,
                       lane);
}

// CTA = (sequence, KV head).
template <int D, int G, typename T>
__global__ void pa_reduce_kernel(const DecodeParams p) {
    constexpr int V4 = D * G / 4;
    extern __shared__ float4 s_red[];  // [REDUCE_GROUPS][V4] sums, [REDUCE_GROUPS][V4] weight sums, (max, sum)s
    float2 *s_ml = reinterpret_cast<float2 *>(s_red + 2 * REDUCE_GROUPS * V4);  // [nparts][G]
    asm volatile("griddepcontrol.wait;" ::: "memory");
    const int s = blockIdx.x / p.num_kv_heads, kvh = blockIdx.x - s * p.num_kv_heads;
    const int nparts = (clamped_context(p, s, false) + p.partition - 1) / p.partition;
    if (nparts <= REDUCE_LAUNCH_MIN_PARTS) return;  // merged or written by the attention kernel
    const size_t group = (size_t)s * p.num_kv_heads + kvh;
    const float2 *ml = p.ml + group * p.max_parts * G;
    for (int i = threadIdx.x; i < nparts * G; i += blockDim.x) s_ml[i] = __ldcg(ml + i);
    __syncthreads();
    const int v = threadIdx.x % V4, r = threadIdx.x / V4;
    float M[4], acc[4] = {0.f, 0.f, 0.f, 0.f}, L[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int g = (4 * v + c) % G;
        M[c] = -INFINITY;
        for (int j = 0; j < nparts; ++j) M[c] = fmaxf(M[c], s_ml[j * G + g].x);
    }
    const float4 *part = reinterpret_cast<const float4 *>(p.part_acc + group * p.max_parts * (D * G));
#pragma unroll 4
    for (int j = r; j < nparts; j += REDUCE_GROUPS) {
        const float4 a = __ldcg(part + (size_t)j * V4 + v);
        const float f[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            const float2 m = s_ml[j * G + (4 * v + c) % G];
            const float w = exp2f(m.x - M[c]);
            acc[c] = fmaf(w, f[c], acc[c]);
            L[c] = fmaf(w, m.y, L[c]);
        }
    }
    s_red[r * V4 + v] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    s_red[(REDUCE_GROUPS + r) * V4 + v] = make_float4(L[0], L[1], L[2], L[3]);
    __syncthreads();
    if (r != 0) return;
    float o[4] = {0.f, 0.f, 0.f, 0.f}, l[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int q = 0; q < REDUCE_GROUPS; ++q) {
        const float4 a = s_red[q * V4 + v], b = s_red[(REDUCE_GROUPS + q) * V4 + v];
        o[0] += a.x; o[1] += a.y; o[2] += a.z; o[3] += a.w;
        l[0] += b.x; l[1] += b.y; l[2] += b.z; l[3] += b.w;
    }
    T *out = static_cast<T *>(p.out);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const int e = 4 * v + c, d = e / G, g = e % G;
        out[((size_t)s * p.num_heads + (size_t)kvh * G + g) * D + d] = static_cast<T>(o[c] / l[c]);
    }
}

template <int D, int G, typename T, int NS, bool KV8 = false, bool SHARED = false, bool I8 = false, int HS = 0>
__global__ void __launch_bounds__(mma_max_warps<D, G, KV8, SHARED>() * 32, 1)
    pa_decode_mma_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tm_k,
                         const __grid_constant__ CUtensorMap tm_v) {
    static_assert(!I8 || KV8, "INT8 codes are an 8-bit cache");
    static_assert(!HS || KV8, "per-head and per-block scales are an 8-bit cache's");
    using Gm = MmaGeo<D, G, KV8, mma_tile_rows<D, KV8, SHARED>()>;
    constexpr int TR = Gm::TR;   // tokens of an item
    constexpr int NT = TR / 16;  // its 16-token MMA sub-tiles
    static_assert(!SHARED || NT == 1, "shared units keep 16-token items");
    // The merge's two-pass form (no partials requested up front) where
    // registers are scarce: the 8-bit kernels, and 8 query heads at head_dim 128.
    constexpr bool LEAN_MERGE = KV8 || (G == 8 && D == 128);
    constexpr int QB = mma_q_slot_bytes<D, G, SHARED>();  // bytes of one query slot
    constexpr int QS = mma_q_slots<SHARED>();              // query slots per warp
    constexpr int QG = G * D * 2;                          // query rows of one sequence
    using MT = typename std::conditional<KV8, __half, T>::type;  // MMA operand type
    extern __shared__ uint8_t smem_raw[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int warps = blockDim.x >> 5;
    const int Hkv = p.num_kv_heads, H = p.num_heads, bs = p.block_size;
    const int g8 = lane >> 2, t4 = lane & 3;  // mma fragment row / column-pair index

    // Shared memory: [rings of all warps][query buffers][mbarriers], base 1024-aligned.
    const uint32_t raw_s = smem_u32(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t *base = smem_raw + (base_s - raw_s);
    const uint32_t ring_s = base_s + warp * NS * Gm::STAGE_BYTES;
    uint8_t *ring = base + warp * NS * Gm::STAGE_BYTES;
    const uint32_t qbuf_s = base_s + warps * NS * Gm::STAGE_BYTES + warp * QS * QB;
    const uint8_t *qbuf = base + warps * NS * Gm::STAGE_BYTES + warp * QS * QB;
    const uint32_t bar_s = base_s + warps * (NS * Gm::STAGE_BYTES + QS * QB) + warp * NS * 8;

    if (lane == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(bar_s + 8 * i, 1);
        fence_barrier_init();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tm_v)) : "memory");
    }
    __syncwarp();
    const uint64_t policy = l2_policy_evict_first();
    const T *qg = static_cast<const T *>(p.q);

    UnitSource src;
    if (!SHARED && p.early) {
        // The plan kernel runs alongside: first units from the contexts alone.
        src.init_early(p, lane, warps, warps * (int)gridDim.x, blockIdx.x, warp);
    } else {
        asm volatile("griddepcontrol.wait;" ::: "memory");
        src.init(p, lane, *p.num_entries * Hkv, SHARED, warps, warps * (int)gridDim.x);
    }
    auto fetch = [&](Unit &x) {
        src.take(x);
        if constexpr (NT > 1) x.ntiles = (x.ntok + TR - 1) / TR;  // items of TR tokens
    };

    // Item `it` of a unit is its tile `it`: the K and V rows of TR tokens (one
    // 16-row box per sub-tile; a sub-tile past the unit's end is not loaded);
    // item 0 also brings the unit's query rows (G per member sequence; mseq
    // is lane j's member sequence for a unit of mcnt > 0 members).
    auto issue = [&](int s, int kvh, int tbl, int ntok, int qslot, int mcnt, int mseq, int it, uint32_t stage) {
        const int tok = TR * it;
        const int bi = tok / bs;
        const int pb = __shfl_sync(FULL_MASK, tbl, bi);
        // Second sub-tile (TR = 32): its block, if it holds tokens of the unit.
        const bool sub1 = NT > 1 && tok + 16 < ntok;
        const int bi1 = (tok + 16) / bs;
        const int pb1 = NT > 1 ? __shfl_sync(FULL_MASK, tbl, bi1 & 31) : 0;
        // Member sequences of a shared unit reach the issuing lane by shuffle.
        int mid[SHARED ? SHARE_ROWS : 1];
        if constexpr (SHARED) {
#pragma unroll
            for (int j = 0; j < SHARE_ROWS; ++j) mid[j] = __shfl_sync(FULL_MASK, mseq, j);
        }
        if (lane == 0) {
            const uint32_t bar = bar_s + 8 * stage;
            const bool ok = (unsigned)pb < (unsigned)p.num_blocks;
            const bool ok1 = sub1 && (unsigned)pb1 < (unsigned)p.num_blocks;
            if (!ok || sub1 != ok1) raise_error(PA_DEVERR_BLOCK_ID);
            const int qrows_bytes = it != 0 ? 0 : (SHARED && mcnt > 0 ? mcnt * QG : QG);
            const uint32_t bytes = (ok ? Gm::SUB_BYTES : 0) + (ok1 ? Gm::SUB_BYTES : 0) + qrows_bytes;
            fence_proxy_async_smem();
            if (bytes) {
                mbar_arrive_expect_tx(bar, bytes);
                const uint32_t dst = ring_s + stage * Gm::STAGE_BYTES;
                if (ok) {
                    const int row = (pb * Hkv + kvh) * bs + (tok - bi * bs);
#pragma unroll
                    for (int b = 0; b < Gm::NBOX; ++b) {
                        tma_load_2d(dst + b * Gm::BOX_BYTES, &tm_k, Gm::BOX_ELEMS * b, row, bar, policy);
                        tma_load_2d(dst + Gm::HALF_BYTES + b * Gm::BOX_BYTES, &tm_v, Gm::BOX_ELEMS * b, row, bar,
                                    policy);
                    }
                }
                if constexpr (NT > 1) {
                    if (ok1) {  // rows 16..31 of the tile (one box per row)
                        const int row1 = (pb1 * Hkv + kvh) * bs + (tok + 16 - bi1 * bs);
                        tma_load_2d(dst + Gm::BOX_BYTES, &tm_k, 0, row1, bar, policy);
                        tma_load_2d(dst + Gm::HALF_BYTES + Gm::BOX_BYTES, &tm_v, 0, row1, bar, policy);
                    }
                }
                if (it == 0) {
                    if constexpr (SHARED) {
                        if (mcnt > 0) {
#pragma unroll
                            for (int j = 0; j < SHARE_ROWS; ++j)
                                if (j < mcnt)
                                    bulk_load(qbuf_s + qslot * QB + j * QG,
                                              qg + ((size_t)mid[j] * H + kvh * G) * D, QG, bar, policy);
                        } else {
                            bulk_load(qbuf_s + qslot * QB, qg + ((size_t)s * H + kvh * G) * D, QG, bar, policy);
                        }
                    } else {
                        bulk_load(qbuf_s + qslot * QB, qg + ((size_t)s * H + kvh * G) * D, QG, bar, policy);
                    }
                }
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
    uint32_t cur_q_item = 0, nxt_q_item = 0;  // issue index of a unit's item 0 (its query rows)

    // Issues the next item if it may go now; returns whether it did.
    auto produce = [&]() -> bool {
        if (exhausted) return false;
        if (pitem >= (prod_on_nxt ? nxt.ntiles : cur.ntiles)) {
            if (prod_on_nxt) return false;
            fetch(nxt);
            if (!nxt.valid) {
                exhausted = true;
                return false;
            }
            nxt.slot = QS == 1 ? 0 : next_slot;
            next_slot ^= 1;
            prod_on_nxt = true;
            pitem = 0;
        }
        // One query slot: the next unit's rows wait until the current unit
        // has read its own (at its first tile).
        if (QS == 1 && prod_on_nxt && pitem == 0 && consumed <= cur_q_item) return false;
        if (pitem == 0) {
            if (prod_on_nxt)
                nxt_q_item = issued;
            else
                cur_q_item = issued;
        }
        if (prod_on_nxt)
            issue(nxt.s, nxt.kvh, nxt.tbl, nxt.ntok, nxt.slot, nxt.mcnt, nxt.mseq, pitem, issued % NS);
        else
            issue(cur.s, cur.kvh, cur.tbl, cur.ntok, cur.slot, cur.mcnt, cur.mseq, pitem, issued % NS);
        ++pitem;
        ++issued;
        // One link of the next unit's claim per issued item, over the unit's
        // last CLAIM_AHEAD items only: claimed earlier, a unit would wait on
        // a busy warp while others that finish sooner could start it.
        if ((prod_on_nxt ? nxt.ntiles : cur.ntiles) - pitem < CLAIM_AHEAD) src.step();
        return true;
    };
    // Keeps NS items in flight while there is work that may be issued.
    auto fill = [&]() {
        while (issued - consumed < (uint32_t)NS && produce()) {
        }
    };

    // Waits for the next item to consume; on a timeout it flags it, waits
    // (bounded) for every copy still in flight, and reports failure.
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

    // With two query slots nothing is ever held back: NS items now, then one
    // per freed stage keeps the ring full. With one slot, refill to NS.
    if constexpr (QS == 1)
        fill();
    else
        for (int i = 0; i < NS; ++i) produce();

    // Query rows (MMA columns) of this lane's accumulators.
    const int h0 = 2 * t4, h1 = 2 * t4 + 1;
    // Fused append: the unit that holds a sequence's last token writes the new
    // K/V row into the pool and uses it in place of the tile's old contents.
    constexpr int NVR = D / 8;  // 16-byte vectors per row
    const bool append = !KV8 && p.k_new != nullptr;  // the fp8 cache has no fused append

    for (;;) {
        // Query rows of the unit (G per member sequence) and whether this
        // lane's two accumulator columns are among them.
        const int nrows = SHARED && cur.mcnt > 0 ? cur.mcnt * G : G;
        const bool hv0 = h0 < nrows, hv1 = h1 < nrows;
        uint32_t qb[Gm::KS][2];  // B fragments of Q^T: query row g8, 2 columns
        float o[Gm::KS][4];      // O^T fragments: rows d = 16*i + g8 (+8), heads h0, h1
        float M0 = -INFINITY, M1 = -INFINITY, l0 = 0.f, l1 = 0.f;
#pragma unroll
        for (int i = 0; i < Gm::KS; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) o[i][j] = 0.f;
        // Shared units with more than 8 query rows: the second column half
        // (rows 8 + h0, 8 + h1), with its own fragments, maxima, sums and
        // accumulators.
        constexpr int K2 = SHARED ? Gm::KS : 1;
        const bool two = SHARED && nrows > 8;
        const bool hw0 = 8 + h0 < nrows, hw1 = 8 + h1 < nrows;
        uint32_t qc[K2][2];
        float o2[K2][4];
        float N0 = -INFINITY, N1 = -INFINITY, m0s = 0.f, m1s = 0.f;  // maxima and sums of the second half
#pragma unroll
        for (int i = 0; i < K2; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) o2[i][j] = 0.f;
        // Lanes [0, NVR) hold one 16-byte vector of the new K row, lanes
        // [NVR, 2*NVR) of the new V row; loaded now, used at the last tile.
        const bool app_unit = append && cur.part == cur.nparts - 1;
        // Dequantisation of an 8-bit cache: the key scale folds into the
        // score scale uq, the value scale uv applies at the store (per unit
        // with per-head scales, HS == 1; kernel parameters otherwise). kc0 /
        // kc1 take the INT8 offset off the scores of query rows h0 / h1.
        // Per-block scales (HS == 2): lane j holds the scales of the unit's
        // block j (the table slice it holds); a sub-tile's key scale joins uq
        // and the INT8 offsets, its value scale, relative to the unit's
        // largest (uv), weights the probabilities of the value product.
        float uq = p.qscale, uv = p.v_scale, kc0 = 0.f, kc1 = 0.f, kd0 = 0.f, kd1 = 0.f;
        float kbl = 1.f, vbl = 1.f, ivmax = 1.f;
        if constexpr (HS == 1) {
            uq = p.qscale * __ldg(p.k_scales + cur.kvh);
            uv = __ldg(p.v_scales + cur.kvh);
        } else if constexpr (HS == 2) {
            float vmax = 0.f;
            if (lane < (cur.ntok + bs - 1) / bs && (unsigned)cur.tbl < (unsigned)p.num_blocks) {
                const size_t si = (size_t)cur.tbl * Hkv + cur.kvh;
                kbl = __ldg(p.k_scales + si);
                vbl = __ldg(p.v_scales + si);
                vmax = vbl;
            }
#pragma unroll
            for (int off = 16; off >= 1; off >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(FULL_MASK, vmax, off));
            uv = vmax;
            ivmax = vmax > 0.f ? 1.f / vmax : 0.f;
        }
        uint4 newrow = make_uint4(0, 0, 0, 0);
        if (app_unit && lane < 2 * NVR) {
            const size_t rowoff = ((size_t)cur.s * Hkv + cur.kvh) * D;
            const T *src = static_cast<const T *>(lane < NVR ? p.k_new : p.v_new);
            newrow = *reinterpret_cast<const uint4 *>(src + rowoff + (lane % NVR) * 8);
        }

        for (int k = 0; k < cur.ntiles; ++k) {
            if (!wait_item()) return;
            const uint32_t stage = consumed % NS;
            const uint32_t ks_s = ring_s + stage * Gm::STAGE_BYTES;
            const uint32_t vs_s = ks_s + Gm::HALF_BYTES;
            if (k == 0) {
                const uint8_t *qs = qbuf + cur.slot * QB;
                bool qbig = false;  // a bf16 query element outside f16's range (fp8 cache)
#pragma unroll
                for (int i = 0; i < Gm::KS; ++i) {
                    if constexpr (KV8) {
                        // Slice i pairs K elements 16i + 4*t4 + {0,1} and + {2,3}
                        // (the order the byte-wise fragments arrive in); the
                        // query fragment follows the same order.
                        const int d = 16 * i + 4 * t4;
                        qb[i][0] = g8 < nrows
                                       ? to_f16x2<T>(*reinterpret_cast<const uint32_t *>(qs + (g8 * D + d) * 2), qbig)
                                       : 0u;
                        qb[i][1] = g8 < nrows ? to_f16x2<T>(
                                                    *reinterpret_cast<const uint32_t *>(qs + (g8 * D + d + 2) * 2), qbig)
                                              : 0u;
                        if constexpr (SHARED) {
                            const int r = 8 + g8;
                            qc[i][0] = r < nrows
                                           ? to_f16x2<T>(*reinterpret_cast<const uint32_t *>(qs + (r * D + d) * 2), qbig)
                                           : 0u;
                            qc[i][1] = r < nrows ? to_f16x2<T>(
                                                       *reinterpret_cast<const uint32_t *>(qs + (r * D + d + 2) * 2), qbig)
                                                 : 0u;
                        }
                    } else {
                        const int d = 16 * i + 2 * t4;
                        qb[i][0] = g8 < nrows ? *reinterpret_cast<const uint32_t *>(qs + (g8 * D + d) * 2) : 0u;
                        qb[i][1] = g8 < nrows ? *reinterpret_cast<const uint32_t *>(qs + (g8 * D + d + 8) * 2) : 0u;
                        if constexpr (SHARED) {
                            const int r = 8 + g8;
                            qc[i][0] = r < nrows ? *reinterpret_cast<const uint32_t *>(qs + (r * D + d) * 2) : 0u;
                            qc[i][1] = r < nrows ? *reinterpret_cast<const uint32_t *>(qs + (r * D + d + 8) * 2) : 0u;
                        }
                    }
                }
                if constexpr (KV8 && !std::is_same<T, __half>::value) {
                    if (__any_sync(FULL_MASK, qbig) && lane == 0) raise_error(PA_DEVERR_QRANGE);
                }
                if constexpr (I8) {
                    // Sum of query row g8 (the f16 values the MMA multiplies),
                    // over the quad's lanes, then rows h0 and h1 of this lane.
                    float qs = 0.f;
#pragma unroll
                    for (int i = 0; i < Gm::KS; ++i) {
                        const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&qb[i][0]));
                        const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&qb[i][1]));
                        qs += (a.x + a.y) + (b.x + b.y);
                    }
                    qs += __shfl_xor_sync(FULL_MASK, qs, 1);
                    qs += __shfl_xor_sync(FULL_MASK, qs, 2);
                    kc0 = -I8_OFFSET * uq * __shfl_sync(FULL_MASK, qs, 8 * t4);
                    kc1 = -I8_OFFSET * uq * __shfl_sync(FULL_MASK, qs, 8 * t4 + 4);
                    if constexpr (SHARED) {
                        float qt = 0.f;  // the same for rows 8 + g8 (second half)
#pragma unroll
                        for (int i = 0; i < Gm::KS; ++i) {
                            const float2 a = __half22float2(*reinterpret_cast<const __half2 *>(&qc[i][0]));
                            const float2 b = __half22float2(*reinterpret_cast<const __half2 *>(&qc[i][1]));
                            qt += (a.x + a.y) + (b.x + b.y);
                        }
                        qt += __shfl_xor_sync(FULL_MASK, qt, 1);
                        qt += __shfl_xor_sync(FULL_MASK, qt, 2);
                        kd0 = -I8_OFFSET * uq * __shfl_sync(FULL_MASK, qt, 8 * t4);
                        kd1 = -I8_OFFSET * uq * __shfl_sync(FULL_MASK, qt, 8 * t4 + 4);
                    }
                }
            }
            const int valid = min(TR, cur.ntok - TR * k);  // tokens of the item
            if (app_unit && k == cur.ntiles - 1) {
                const int tok = cur.ntok - 1;  // the sequence's last position, in this tile
                const int pb = __shfl_sync(FULL_MASK, cur.tbl, tok / bs);
                if (lane < 2 * NVR) {
                    const int half = lane / NVR, c = lane % NVR;
                    uint8_t *st = ring + stage * Gm::STAGE_BYTES + half * Gm::HALF_BYTES;
                    *reinterpret_cast<uint4 *>(st + Gm::addr(tok % TR, c)) = newrow;
                    if ((unsigned)pb < (unsigned)p.num_blocks) {
                        T *pool = static_cast<T *>(const_cast<void *>(half ? p.v_pool : p.k_pool));
                        *reinterpret_cast<uint4 *>(pool + (((size_t)pb * Hkv + cur.kvh) * bs + tok % bs) * D + c * 8) =
                            newrow;
                    } else if (lane == 0) {
                        raise_error(PA_DEVERR_BLOCK_ID);
                    }
                }
                fence_proxy_async_smem();  // these writes precede the stage's next TMA fill
                __syncwarp();
            }

            // ---------------- S^T = K . Q^T ------------------------------------
            // Per 16-token sub-tile j of the item: two accumulators (even / odd
            // slices) halve the chain of dependent MMAs, and the sub-tiles'
            // chains are independent of each other. A sub-tile with no token of
            // the unit was not loaded and is skipped (warp-uniform).
            float s[NT][4], s2[NT][4];
#pragma unroll
            for (int j = 0; j < NT; ++j)
#pragma unroll
                for (int c = 0; c < 4; ++c) s[j][c] = s2[j][c] = 0.f;
            float u[4] = {0.f, 0.f, 0.f, 0.f}, u2[4] = {0.f, 0.f, 0.f, 0.f};  // second half
            if constexpr (KV8) {
                // A 16-byte chunk holds 16 codes of a row; ldmatrix on byte pairs
                // gives each thread codes 4*t4 .. 4*t4+3 of rows g8 and g8+8.
                const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
                const int csel = lane >> 4;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j > 0 && valid <= 16 * j) break;
#pragma unroll
                    for (int i = 0; i < Gm::KS; i += 2) {
                        uint32_t r[4];
                        ldsm_x4(r, ks_s + Gm::addr(16 * j + row, i + csel));
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            const uint32_t lo = r[2 * h], hi = r[2 * h + 1];
                            uint32_t a[4];
                            if constexpr (I8) {
                                a[0] = i8x2_to_f16x2(lo); a[1] = i8x2_to_f16x2(hi);
                                a[2] = i8x2_hi_to_f16x2(lo); a[3] = i8x2_hi_to_f16x2(hi);
                            } else {
                                a[0] = e4m3x2_to_f16x2(lo); a[1] = e4m3x2_to_f16x2(hi);
                                a[2] = e4m3x2_hi_to_f16x2(lo); a[3] = e4m3x2_hi_to_f16x2(hi);
                            }
                            MmaType<__half>::mma(h ? s2[j] : s[j], a, qb[i + h][0], qb[i + h][1]);
                            if constexpr (SHARED) {
                                if (two) MmaType<__half>::mma(h ? u2 : u, a, qc[i + h][0], qc[i + h][1]);
                            }
                        }
                    }
                }
            } else {
                const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
                const int csel = lane >> 4;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j > 0 && valid <= 16 * j) break;
#pragma unroll
                    for (int i = 0; i < Gm::KS; ++i) {
                        uint32_t a[4];
                        ldsm_x4(a, ks_s + Gm::addr(16 * j + row, 2 * i + csel));
                        MmaType<T>::mma((i & 1) ? s2[j] : s[j], a, qb[i][0], qb[i][1]);
                        if constexpr (SHARED) {
                            if (two) MmaType<T>::mma((i & 1) ? u2 : u, a, qc[i][0], qc[i][1]);
                        }
                    }
                }
            }
            // s[j][0], s[j][1]: token 16j + g8, heads h0, h1; s[j][2], s[j][3]: token 16j + g8 + 8.
            float x[NT][4], vr[NT], ksc[NT];
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                float uqj = uq, kcj0 = kc0, kcj1 = kc1;
                vr[j] = 1.f;
                ksc[j] = 1.f;
                if constexpr (HS == 2) {  // the scales of the sub-tile's block
                    const int bj = (TR * k + 16 * j) / bs;
                    ksc[j] = __shfl_sync(FULL_MASK, kbl, bj & 31);
                    vr[j] = __shfl_sync(FULL_MASK, vbl, bj & 31) * ivmax;
                    uqj = uq * ksc[j];
                    kcj0 = kc0 * ksc[j];
                    kcj1 = kc1 * ksc[j];
                }
                const bool lo_in = 16 * j + g8 < valid, hi_in = 16 * j + g8 + 8 < valid;
                x[j][0] = lo_in ? fmaf(s[j][0] + s2[j][0], uqj, kcj0) : -INFINITY;
                x[j][1] = lo_in ? fmaf(s[j][1] + s2[j][1], uqj, kcj1) : -INFINITY;
                x[j][2] = hi_in ? fmaf(s[j][2] + s2[j][2], uqj, kcj0) : -INFINITY;
                x[j][3] = hi_in ? fmaf(s[j][3] + s2[j][3], uqj, kcj1) : -INFINITY;
                mx0 = fmaxf(mx0, fmaxf(x[j][0], x[j][2]));
                mx1 = fmaxf(mx1, fmaxf(x[j][1], x[j][3]));
            }
            bool raise = (hv0 && !(mx0 <= M0 + LAZY_MAX_LOG2)) || (hv1 && !(mx1 <= M1 + LAZY_MAX_LOG2));
            if (__any_sync(FULL_MASK, raise)) {
                float m0 = mx0, m1 = mx1;
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    m0 = fmaxf(m0, __shfl_xor_sync(FULL_MASK, m0, off));
                    m1 = fmaxf(m1, __shfl_xor_sync(FULL_MASK, m1, off));
                }
                const float n0 = fmaxf(M0, m0), n1 = fmaxf(M1, m1);
                const float a0 = exp2f(M0 - n0), a1 = exp2f(M1 - n1);
                M0 = n0;
                M1 = n1;
                l0 *= a0;
                l1 *= a1;
#pragma unroll
                for (int i = 0; i < Gm::KS; ++i) {
                    o[i][0] *= a0; o[i][1] *= a1;
                    o[i][2] *= a0; o[i][3] *= a1;
                }
            }
            // P^T B fragments per sub-tile: head g8, tokens 2*t4 (+1) and 8 + 2*t4 (+1).
            // Padding heads (>= G) carry zero scores; give them weight 0.
            uint32_t pb[NT][2];
#pragma unroll
            for (int j = 0; j < NT; ++j) {
                const float p0 = hv0 ? exp2f(x[j][0] - M0) : 0.f, p1 = hv1 ? exp2f(x[j][1] - M1) : 0.f;
                const float p2 = hv0 ? exp2f(x[j][2] - M0) : 0.f, p3 = hv1 ? exp2f(x[j][3] - M1) : 0.f;
                uint32_t w_lo, w_hi;
                if constexpr (HS == 2) {
                    // The value product weighs each token by its block's value
                    // scale (relative to uv); the denominator sums the weights.
                    w_lo = Elem<MT>::pack(p0 * vr[j], p1 * vr[j]);
                    w_hi = Elem<MT>::pack(p2 * vr[j], p3 * vr[j]);
                    l0 += p0 + p2;
                    l1 += p1 + p3;
                } else {
                    w_lo = Elem<MT>::pack(p0, p1);
                    w_hi = Elem<MT>::pack(p2, p3);
                    const float2 r_lo = Elem<MT>::pair(w_lo), r_hi = Elem<MT>::pair(w_hi);
                    l0 += r_lo.x + r_hi.x;
                    l1 += r_lo.y + r_hi.y;
                }
                pb[j][0] = movmatrix_trans(w_lo);
                pb[j][1] = movmatrix_trans(w_hi);
            }
            // The same for the second column half of a wide shared unit.
            uint32_t pc0 = 0u, pc1 = 0u;
            if constexpr (SHARED) {
                if (two) {
                    const bool v_lo = g8 < valid, v_hi = g8 + 8 < valid;
                    // (per-block scales: the tile's key scale, as for the first half)
                    const float uqb = uq * ksc[0], kdb0 = kd0 * ksc[0], kdb1 = kd1 * ksc[0];
                    const float y0 = v_lo ? fmaf(u[0] + u2[0], uqb, kdb0) : -INFINITY;
                    const float y1 = v_lo ? fmaf(u[1] + u2[1], uqb, kdb1) : -INFINITY;
                    const float y2 = v_hi ? fmaf(u[2] + u2[2], uqb, kdb0) : -INFINITY;
                    const float y3 = v_hi ? fmaf(u[3] + u2[3], uqb, kdb1) : -INFINITY;
                    const bool raise2 = (hw0 && !(fmaxf(y0, y2) <= N0 + LAZY_MAX_LOG2)) ||
                                        (hw1 && !(fmaxf(y1, y3) <= N1 + LAZY_MAX_LOG2));
                    if (__any_sync(FULL_MASK, raise2)) {
                        float n0 = fmaxf(y0, y2), n1 = fmaxf(y1, y3);
#pragma unroll
                        for (int off = 4; off < 32; off <<= 1) {
                            n0 = fmaxf(n0, __shfl_xor_sync(FULL_MASK, n0, off));
                            n1 = fmaxf(n1, __shfl_xor_sync(FULL_MASK, n1, off));
                        }
                        n0 = fmaxf(N0, n0);
                        n1 = fmaxf(N1, n1);
                        const float a0 = exp2f(N0 - n0), a1 = exp2f(N1 - n1);
                        N0 = n0;
                        N1 = n1;
                        m0s *= a0;
                        m1s *= a1;
#pragma unroll
                        for (int i = 0; i < K2; ++i) {
                            o2[i][0] *= a0; o2[i][1] *= a1;
                            o2[i][2] *= a0; o2[i][3] *= a1;
                        }
                    }
                    const float q0 = hw0 ? exp2f(y0 - N0) : 0.f, q1 = hw1 ? exp2f(y1 - N1) : 0.f;
                    const float q2 = hw0 ? exp2f(y2 - N0) : 0.f, q3 = hw1 ? exp2f(y3 - N1) : 0.f;
                    uint32_t z_lo, z_hi;
                    if constexpr (HS == 2) {  // weighted by the tile's value scale, as for the first half
                        z_lo = Elem<MT>::pack(q0 * vr[0], q1 * vr[0]);
                        z_hi = Elem<MT>::pack(q2 * vr[0], q3 * vr[0]);
                        m0s += q0 + q2;
                        m1s += q1 + q3;
                    } else {
                        z_lo = Elem<MT>::pack(q0, q1);
                        z_hi = Elem<MT>::pack(q2, q3);
                        const float2 r_lo = Elem<MT>::pair(z_lo), r_hi = Elem<MT>::pair(z_hi);
                        m0s += r_lo.x + r_hi.x;
                        m1s += r_lo.y + r_hi.y;
                    }
                    pc0 = movmatrix_trans(z_lo);
                    pc1 = movmatrix_trans(z_hi);
                }
            }

            // ---------------- O^T += V^T . P^T ----------------------------------
            if (valid < TR) {
                // Stale or never-written slots past the context in a loaded
                // sub-tile must not reach the product (their weight is 0 but
                // 0 * NaN is NaN): zero them. A sub-tile that was not loaded is
                // not multiplied at all.
                const int end = (valid + 15) & ~15;
                uint8_t *vt = ring + stage * Gm::STAGE_BYTES + Gm::HALF_BYTES;
                for (int idx = lane; idx < (end - valid) * Gm::CHUNKS; idx += 32) {
                    const int r = valid + idx / Gm::CHUNKS;
                    const int c = idx % Gm::CHUNKS;
                    *reinterpret_cast<uint4 *>(vt + Gm::addr(r, c)) = make_uint4(0, 0, 0, 0);
                }
                fence_proxy_async_smem();  // these writes precede the stage's next TMA fill
                __syncwarp();
            }
            if constexpr (KV8) {
                // Transposed ldmatrix on byte pairs gives each thread, for tokens
                // 2*t4 and 2*t4+1, the codes of elements 2*g8 and 2*g8+1 of a
                // 16-element slice; a byte permute regroups them by element, so
                // accumulator rows g8 / g8+8 hold elements 16i + 2*g8 / + 1.
                const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
                const int csel = lane >> 4;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j > 0 && valid <= 16 * j) break;
#pragma unroll
                    for (int i = 0; i < Gm::KS; i += 2) {
                        uint32_t r[4];
                        ldsm_x4_trans(r, vs_s + Gm::addr(16 * j + row, i + csel));
#pragma unroll
                        for (int h = 0; h < 2; ++h) {
                            uint32_t a[4];
                            if constexpr (I8) {
                                // Bytes 0 / 2 are element 2*g8 of the two tokens, 1 / 3 element 2*g8+1.
                                a[0] = i8_unbias(__byte_perm(r[2 * h], 0x64646464u, 0x4240));
                                a[1] = i8_unbias(__byte_perm(r[2 * h], 0x64646464u, 0x4341));
                                a[2] = i8_unbias(__byte_perm(r[2 * h + 1], 0x64646464u, 0x4240));
                                a[3] = i8_unbias(__byte_perm(r[2 * h + 1], 0x64646464u, 0x4341));
                            } else {
                                const uint32_t x8 = __byte_perm(r[2 * h], 0, 0x3120);      // tokens 0-7
                                const uint32_t y8 = __byte_perm(r[2 * h + 1], 0, 0x3120);  // tokens 8-15
                                a[0] = e4m3x2_to_f16x2(x8); a[1] = e4m3x2_hi_to_f16x2(x8);
                                a[2] = e4m3x2_to_f16x2(y8); a[3] = e4m3x2_hi_to_f16x2(y8);
                            }
                            MmaType<__half>::mma(o[i + h], a, pb[j][0], pb[j][1]);
                            if constexpr (SHARED) {
                                if (two) MmaType<__half>::mma(o2[i + h], a, pc0, pc1);
                            }
                        }
                    }
                }
            } else {
                const int row = (lane & 7) + 8 * (lane >> 4);
                const int csel = (lane >> 3) & 1;
#pragma unroll
                for (int j = 0; j < NT; ++j) {
                    if (j > 0 && valid <= 16 * j) break;
#pragma unroll
                    for (int i = 0; i < Gm::KS; ++i) {
                        uint32_t a[4];
                        ldsm_x4_trans(a, vs_s + Gm::addr(16 * j + row, 2 * i + csel));
                        MmaType<T>::mma(o[i], a, pb[j][0], pb[j][1]);
                        if constexpr (SHARED) {
                            if (two) MmaType<T>::mma(o2[i], a, pc0, pc1);
                        }
                    }
                }
            }
            ++consumed;
            __syncwarp();
            if constexpr (QS == 1)
                fill();
            else
                produce();
        }

        // ---------------- totals and store -------------------------------------
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
            l0 += __shfl_xor_sync(FULL_MASK, l0, off);
            l1 += __shfl_xor_sync(FULL_MASK, l1, off);
            if constexpr (SHARED) {
                m0s += __shfl_xor_sync(FULL_MASK, m0s, off);
                m1s += __shfl_xor_sync(FULL_MASK, m1s, off);
            }
        }
        const size_t head0 = (size_t)cur.s * H + (size_t)cur.kvh * G;
        if (SHARED && cur.mcnt > 0) {
            // Partials of every member: query row r (column r of the first
            // half, or r - 8 of the second) is head r % G of member r / G.
            const float vs = KV8 ? uv : 1.f;
            auto store_half = [&](const float (&oo)[Gm::KS][4], int r0, int r1, bool va, bool vb, float Ma, float Mb,
                                  float la, float lb) {
                const int seq0 = __shfl_sync(FULL_MASK, cur.mseq, (r0 / G) & (SHARE_ROWS - 1));
                const int seq1 = __shfl_sync(FULL_MASK, cur.mseq, (r1 / G) & (SHARE_ROWS - 1));
                const size_t row0 = ((size_t)seq0 * Hkv + cur.kvh) * p.max_parts + cur.part;
                const size_t row1 = ((size_t)seq1 * Hkv + cur.kvh) * p.max_parts + cur.part;
                float *acc0 = p.part_acc + row0 * (size_t)(D * G);
                float *acc1 = p.part_acc + row1 * (size_t)(D * G);
                const int g0 = r0 % G, g1 = r1 % G;
#pragma unroll
                for (int i = 0; i < Gm::KS; ++i) {
                    const int d = KV8 ? 16 * i + 2 * g8 : 16 * i + g8;
                    const int d2 = KV8 ? d + 1 : d + 8;
                    if constexpr (G == 1) {
                        if (va) {
                            acc0[d] = oo[i][0] * vs;
                            acc0[d2] = oo[i][2] * vs;
                        }
                        if (vb) {
                            acc1[d] = oo[i][1] * vs;
                            acc1[d2] = oo[i][3] * vs;
                        }
                    } else if (vb) {  // G even: rows r0, r0 + 1 are heads g0, g0 + 1 of one member
                        *reinterpret_cast<float2 *>(acc0 + d * G + g0) = make_float2(oo[i][0] * vs, oo[i][1] * vs);
                        *reinterpret_cast<float2 *>(acc0 + d2 * G + g0) = make_float2(oo[i][2] * vs, oo[i][3] * vs);
                    }
                }
                if (g8 == 0 && va) p.ml[row0 * G + g0] = make_float2(Ma, la);
                if (g8 == 0 && vb) p.ml[row1 * G + g1] = make_float2(Mb, lb);
            };
            store_half(o, h0, h1, hv0, hv1, M0, M1, l0, l1);
            if constexpr (SHARED) {
                if (two) store_half(o2, 8 + h0, 8 + h1, hw0, hw1, N0, N1, m0s, m1s);
            }
            if (p.reduce_launch) goto next_unit;  // merged by pa_reduce_kernel
            // Lane j counts member j's partition.
            src.wait_plan();  // the merge counters are zeroed by the plan kernel
            const bool last = count_partition(&p.merge_count[(size_t)cur.mseq * Hkv + cur.kvh], cur.mnp,
                                              lane < cur.mcnt);
            // Members whose last partition this was, merged one after another
            // (merging them together, with all members' loads in flight at
            // once, was measured slower: it needs more registers).
            unsigned lm = __ballot_sync(FULL_MASK, last);
            while (lm) {
                const int j = __ffs(lm) - 1;
                lm &= lm - 1;
                const int sj = __shfl_sync(FULL_MASK, cur.mseq, j);
                const int nj = __shfl_sync(FULL_MASK, cur.mnp, j);
                mma_merge<D, G, T, LEAN_MERGE>(p, (size_t)sj * Hkv + cur.kvh, (size_t)sj * H + (size_t)cur.kvh * G, 0, nj,
                                        lane);
            }
        } else if (KV8 && cur.nparts == 1) {
            // Accumulator rows g8 / g8+8 of slice i are elements 16i + 2*g8 / + 1:
            // pairs of adjacent elements per head, stored directly.
            const float i0 = hv0 ? uv / l0 : 0.f, i1 = hv1 ? uv / l1 : 0.f;
            T *out = static_cast<T *>(p.out) + head0 * D;
#pragma unroll
            for (int i = 0; i < Gm::KS; ++i) {
                const int d = 16 * i + 2 * g8;
                if (hv0) *reinterpret_cast<uint32_t *>(out + h0 * D + d) = Elem<T>::pack(o[i][0] * i0, o[i][2] * i0);
                if (hv1) *reinterpret_cast<uint32_t *>(out + h1 * D + d) = Elem<T>::pack(o[i][1] * i1, o[i][3] * i1);
            }
        } else if (cur.nparts == 1) {
            const float i0 = hv0 ? 1.f / l0 : 0.f, i1 = hv1 ? 1.f / l1 : 0.f;
            T *out = static_cast<T *>(p.out) + head0 * D;
#pragma unroll
            for (int i = 0; i < Gm::KS; ++i) {
                // [d][head] pairs -> transpose -> [head g8][d = 2*t4, 2*t4 + 1]
                const uint32_t lo = movmatrix_trans(Elem<T>::pack(o[i][0] * i0, o[i][1] * i1));
                const uint32_t hi = movmatrix_trans(Elem<T>::pack(o[i][2] * i0, o[i][3] * i1));
                if (g8 < G) {
                    *reinterpret_cast<uint32_t *>(out + g8 * D + 16 * i + 2 * t4) = lo;
                    *reinterpret_cast<uint32_t *>(out + g8 * D + 16 * i + 8 + 2 * t4) = hi;
                }
            }
        } else {
            const size_t group = (size_t)cur.s * Hkv + cur.kvh;
            const size_t row = group * p.max_parts + cur.part;
            float *acc = p.part_acc + row * (size_t)(D * G);
            // Rows g8 / g8+8 of slice i: elements 16i + g8 / + 8 (16-bit cache)
            // or 16i + 2*g8 / + 1 (fp8 cache, values scaled by v_scale).
            const float vs = KV8 ? uv : 1.f;
#pragma unroll
            for (int i = 0; i < Gm::KS; ++i) {
                const int d = KV8 ? 16 * i + 2 * g8 : 16 * i + g8;
                const int d2 = KV8 ? d + 1 : d + 8;
                if constexpr (G == 1) {
                    if (hv0) {
                        acc[d] = o[i][0] * vs;
                        acc[d2] = o[i][2] * vs;
                    }
                } else if (hv1) {
                    *reinterpret_cast<float2 *>(acc + d * G + h0) = make_float2(o[i][0] * vs, o[i][1] * vs);
                    *reinterpret_cast<float2 *>(acc + d2 * G + h0) = make_float2(o[i][2] * vs, o[i][3] * vs);
                }
            }
            if (g8 == 0 && hv0) p.ml[row * G + h0] = make_float2(M0, l0);
            if (g8 == 0 && hv1) p.ml[row * G + h1] = make_float2(M1, l1);
            // Merged by the merge launch: shared mode's every sequence, else
            // the sequences with more than REDUCE_LAUNCH_MIN_PARTS partitions.
            if (p.reduce_launch && (SHARED || cur.nparts > REDUCE_LAUNCH_MIN_PARTS)) goto next_unit;
            src.wait_plan();  // the merge counters are zeroed by the plan kernel
            // One level (at most MERGE_FANIN partitions, or shared-prefix units'
            // workspace), or two: this partition's chunk into its chunk
            // partial, then the chunk partials. One merge call site in a loop
            // keeps the merge inlined once. The 8-bit kernels keep one level,
            // for registers (beyond REDUCE_LAUNCH_MIN_PARTS partitions their
            // merges run in the separate launch anyway).
            const bool chunked = !KV8 && cur.nparts > MERGE_FANIN && p.max_chunks > 0;
            const int nch = (cur.nparts + MERGE_FANIN - 1) / MERGE_FANIN;
            int first = 0, n = cur.nparts, dst = -1;
            bool go;
            if (chunked) {
                const int c = cur.part / MERGE_FANIN;
                first = c * MERGE_FANIN;
                n = min(MERGE_FANIN, cur.nparts - first);
                dst = p.l1_base + c;
                go = count_partition(&p.chunk_count[group * p.max_chunks + c], n, lane == 0);
            } else {
                go = count_partition(&p.merge_count[group], cur.nparts, lane == 0);
            }
#pragma unroll 1
            while (__shfl_sync(FULL_MASK, go, 0)) {
                mma_merge<D, G, T, LEAN_MERGE>(p, group, head0, first, n, lane, dst);
                if (dst < 0) break;
                go = count_partition(&p.merge_count[group], nch, lane == 0);
                first = p.l1_base;
                n = nch;
                dst = -1;
            }
        }

    next_unit:
        while (!prod_on_nxt && !exhausted) produce();
        if (!prod_on_nxt) break;
        cur = nxt;
        cur_q_item = nxt_q_item;
        prod_on_nxt = false;
        if constexpr (QS == 1) fill();
    }
}

}  // namespace pa
