// The two data movers of the paged cache, as 16-byte vector copies.
//
//  pa_reshape_kernel     writes each new token's K and V rows into the pool
//                        slot its slot_mapping entry names (the append of the
//                        m.nxbn.cn VLLM explainer, section 一).
//  pa_copy_blocks_kernel copy-on-write copies of whole blocks across a list
//                        of pools ("vLLM架构深度解析：PagedAttention如何实现高吞吐LLM推理",
//                        section KV Cache内存共享).
// Both are bit copies. Out-of-range indices are skipped and flagged.
#pragma once

#include <cuda_fp8.h>

#include "pa_common.cuh"

namespace pa {

// One thread moves one 16-byte vector of K and the matching vector of V.
// The flat vector index i over [T][Hkv][D/8] is both the source index and,
// through the slot, the row and column of the destination.
__global__ void __launch_bounds__(256) pa_reshape_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                                         uint4 *__restrict__ k_pool, uint4 *__restrict__ v_pool,
                                                         const int64_t *__restrict__ slot_mapping,
                                                         long long total_vectors, int vec_per_row, int num_kv_heads,
                                                         int block_size, long long num_slots) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total_vectors; i += stride) {
        const long long row = i / vec_per_row;  // (token, head)
        const int vec = (int)(i - row * vec_per_row);
        const long long t = row / num_kv_heads;
        const int h = (int)(row - t * num_kv_heads);
        const int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_slots) {
            raise_error(PA_DEVERR_SLOT);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int64_t off = slot - blk * block_size;
        const size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + off) * vec_per_row + vec;
        const uint4 kv = k[i];
        const uint4 vv = v[i];
        k_pool[dst] = kv;
        v_pool[dst] = vv;
    }
}

// Two INT8 codes (excess-128) of two fp32 values already divided by their
// scale: round to nearest even, clamp to [-127, 127], NaN stores zero.
__device__ __forceinline__ uint32_t int8x2_encode(float2 y) {
    const int a = isnan(y.x) ? 0 : min(127, max(-127, __float2int_rn(y.x)));
    const int b = isnan(y.y) ? 0 : min(127, max(-127, __float2int_rn(y.y)));
    return (uint32_t)(a + 128) | ((uint32_t)(b + 128) << 8);
}

// Quantising cache write for an 8-bit cache: code = encode(x / scale), the
// division in fp32 (IEEE, round to nearest). E4M3 (I8 false): the conversion
// rounds to nearest even and saturates at +-448; INT8 (I8 true): round to
// nearest even, clamp to [-127, 127], stored excess-128. The scale is k_scale /
// v_scale, or with k_scales / v_scales the entry of the row's KV head. One
// thread turns one 16-byte vector of K (8 elements) into 8 codes, and the same
// for V.
template <typename T, bool I8>
__global__ void __launch_bounds__(256) pa_reshape_kv8_kernel(const uint4 *__restrict__ k, const uint4 *__restrict__ v,
                                                             uint2 *__restrict__ k_pool, uint2 *__restrict__ v_pool,
                                                             const int64_t *__restrict__ slot_mapping,
                                                             long long total_vectors, int vec_per_row,
                                                             int num_kv_heads, int block_size, long long num_slots,
                                                             float k_scale, float v_scale,
                                                             const float *__restrict__ k_scales,
                                                             const float *__restrict__ v_scales,
                                                             int scales_per_block) {
    const long long stride = (long long)gridDim.x * blockDim.x;
    for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total_vectors; i += stride) {
        const long long row = i / vec_per_row;
        const int vec = (int)(i - row * vec_per_row);
        const long long t = row / num_kv_heads;
        const int h = (int)(row - t * num_kv_heads);
        const int64_t slot = slot_mapping[t];
        if (slot < 0) continue;
        if (slot >= num_slots) {
            raise_error(PA_DEVERR_SLOT);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int64_t off = slot - blk * block_size;
        const size_t dst = (((size_t)blk * num_kv_heads + h) * block_size + off) * vec_per_row + vec;
        const uint4 src[2] = {k[i], v[i]};
        // One scale per KV head, or per (block, KV head) with scales_per_block.
        const size_t si = scales_per_block ? (size_t)blk * num_kv_heads + h : (size_t)h;
        const float sc[2] = {k_scales ? k_scales[si] : k_scale, v_scales ? v_scales[si] : v_scale};
        uint2 codes[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const uint32_t w[4] = {src[j].x, src[j].y, src[j].z, src[j].w};
            uint32_t c[2] = {0u, 0u};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const float2 f = Elem<T>::pair(w[q]);
                const float2 y = make_float2(__fdiv_rn(f.x, sc[j]), __fdiv_rn(f.y, sc[j]));
                uint32_t two;
                if constexpr (I8)
                    two = int8x2_encode(y);
                else
                    two = (uint32_t)__nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, __NV_E4M3);
                c[q >> 1] |= two << (16 * (q & 1));
            }
            codes[j] = make_uint2(c[0], c[1]);
        }
        k_pool[dst] = codes[0];
        v_pool[dst] = codes[1];
    }
}

constexpr int COPY_MAX_POOLS = 64;

struct PoolList {
    uint4 *ptr[COPY_MAX_POOLS];
};

// blockIdx.x = pair, blockIdx.y = pool; the CTA copies one whole block.
__global__ void __launch_bounds__(256) pa_copy_blocks_kernel(PoolList pools, const int64_t *__restrict__ pairs,
                                                             long long vec_per_block, long long num_blocks) {
    const int64_t src = pairs[2 * (size_t)blockIdx.x];
    const int64_t dst = pairs[2 * (size_t)blockIdx.x + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0) raise_error(PA_DEVERR_PAIR);
        return;
    }
    uint4 *base = pools.ptr[blockIdx.y];
    const uint4 *from = base + (size_t)src * vec_per_block;
    uint4 *to = base + (size_t)dst * vec_per_block;
    long long i = threadIdx.x;
    for (; i + 3 * 256 < vec_per_block; i += 4 * 256) {
        const uint4 a = from[i], b = from[i + 256], c = from[i + 512], d = from[i + 768];
        to[i] = a;
        to[i + 256] = b;
        to[i + 512] = c;
        to[i + 768] = d;
    }
    for (; i < vec_per_block; i += 256) to[i] = from[i];
}

// Cross-pool block copies for swapping: blockIdx.x = pair, blockIdx.y = pool
// index; the CTA copies block src of src[pool] to block dst of dst[pool].
// Either side may be page-locked host memory reached through unified
// addressing, so each thread keeps four 16-byte loads in flight.
struct ConstPoolList {
    const uint4 *ptr[COPY_MAX_POOLS];
};

__global__ void __launch_bounds__(256) pa_swap_blocks_kernel(PoolList dst, ConstPoolList src,
                                                             const int64_t *__restrict__ pairs,
                                                             long long vec_per_block, long long num_src_blocks,
                                                             long long num_dst_blocks) {
    const int64_t s = pairs[2 * (size_t)blockIdx.x];
    const int64_t d = pairs[2 * (size_t)blockIdx.x + 1];
    if (s < 0 || s >= num_src_blocks || d < 0 || d >= num_dst_blocks) {
        if (threadIdx.x == 0) raise_error(PA_DEVERR_PAIR);
        return;
    }
    const uint4 *from = src.ptr[blockIdx.y] + (size_t)s * vec_per_block;
    uint4 *to = dst.ptr[blockIdx.y] + (size_t)d * vec_per_block;
    long long i = threadIdx.x;
    for (; i + 3 * 256 < vec_per_block; i += 4 * 256) {
        const uint4 a = from[i], b = from[i + 256], c = from[i + 512], e = from[i + 768];
        to[i] = a;
        to[i + 256] = b;
        to[i + 512] = c;
        to[i + 768] = e;
    }
    for (; i < vec_per_block; i += 256) to[i] = from[i];
}

}  // namespace pa
