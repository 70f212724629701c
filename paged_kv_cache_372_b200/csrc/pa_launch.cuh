// Launch side of pa_decode: partition choice, tensor maps, kernel selection
// and launch configuration. Included by pa_api.cu after its host helpers
// (fail, cuda_fail, device_info, ceil_div).
#pragma once

#include <cudaTypedefs.h>

#include <algorithm>

#include "pa_decode.cuh"
#include "pa_decode_mma.cuh"

namespace {

// Largest partition the attention kernels take: the unit's block-table slice
// fits one register per lane (<= 32 blocks).
int partition_cap(int block_size) { return 32 * block_size; }

// Partition used when the caller passes 0 (a whole sequence when every
// context fits in it): 32 blocks for grouped heads, 256 tokens for one query
// head per KV head (measured best on the benchmark workloads).
// Which entry point a partition is chosen for.
enum class PartMode { plain, shared, fp8 };

// With shared-prefix units (which always merge) 16 blocks for grouped heads:
// the shared tiles are streamed once per group, so the remaining work is
// spread better over the warps in smaller units. The 8-bit kernels: 512
// tokens at every group size (measured on the Llama-3-8B-shaped batch: 84.8 us
// against 93.8 at 256, whose longest sequences needed the merge launch; at
// head_dim 64, 64.6 against 70.5 us on the LLaMA-7B-shaped batch).
int auto_partition(int group, int block_size, PartMode mode = PartMode::plain) {
    switch (mode) {
        case PartMode::shared: return group >= 2 ? 16 * block_size : 256;
        case PartMode::fp8: return 512;
        default: return group >= 2 ? 32 * block_size : 256;
    }
}

bool shape_supported(int num_heads, int num_kv_heads, int head_dim, int block_size) {
    if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads) return false;
    const int g = num_heads / num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return false;
    if (head_dim != 64 && head_dim != 128) return false;
    return block_size == 16 || block_size == 32 || block_size == 64;
}

// Resolves partition_size (0 = auto). Returns 0 for an invalid request.
int resolve_partition(int group, int block_size, int max_context_len, int requested,
                      PartMode mode = PartMode::plain) {
    if (requested > 0) {
        if (requested % 16 || requested % block_size || requested > partition_cap(block_size)) return 0;
        return requested;
    }
    const int auto_p = auto_partition(group, block_size, mode);
    if (max_context_len <= auto_p) {
        const int need = max_context_len > 0 ? max_context_len : 1;
        return ((need + block_size - 1) / block_size) * block_size;
    }
    return auto_p;
}

// Raises kernel Kernel's dynamic shared-memory limit on this device, once per
// (kernel, device, size): one flag array per kernel function, not per type.
template <auto Kernel>
cudaError_t set_dynamic_smem(int dev, int smem) {
    static std::atomic<int> done[kMaxDevices];
    if (done[dev].load(std::memory_order_acquire) == smem) return cudaSuccess;
    const cudaError_t e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e == cudaSuccess) done[dev].store(smem, std::memory_order_release);
    return e;
}

template <int D, int G, typename T>
pa_status launch_decode(pa::DecodeParams &p, cudaStream_t stream) {
    constexpr int NS = pa::DECODE_STAGES;
    DeviceInfo info;
    pa_status st = device_info(&info);
    if (st != PA_OK) return st;
    const int per_warp = pa::warp_smem_bytes<D, G, NS>();
    int warps = info.smem_optin / per_warp;
    if (warps > pa::DECODE_MAX_WARPS) warps = pa::DECODE_MAX_WARPS;
    if (warps < 1) return fail(PA_ERR_UNSUPPORTED, "%d bytes of shared memory per warp", per_warp);
    const int smem = warps * per_warp;
    auto kernel = pa::pa_decode_kernel<D, G, T, NS>;
    cudaError_t e = set_dynamic_smem<pa::pa_decode_kernel<D, G, T, NS>>(info.dev, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");

    if (p.k_new) {
        // The CUDA-core kernel has no fused append: write the new rows first.
        const long long total = (long long)p.num_seqs * p.num_kv_heads * (D / 8);
        long long blocks = (total + 255) / 256;
        if (blocks > (long long)info.sms * 16) blocks = (long long)info.sms * 16;
        pa::pa_append_kernel<<<(unsigned)blocks, 256, 0, stream>>>(p);
        ++g_launches;
    }
    pa::pa_plan_kernel<<<1, pa::PLAN_WARP_THREADS, 0, stream>>>(p);
    ++g_launches;
    // Programmatic dependent launch: the attention CTAs start their set-up
    // while the plan kernel runs and wait for its results in-kernel.
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(info.sms);
    cfg.blockDim = dim3(warps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, p);
    if (e != cudaSuccess) return cuda_fail(e, "pa_decode launch");
    ++g_launches;
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pa_decode launch");
    return PA_OK;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
pa_status tensor_map_encoder(PFN_cuTensorMapEncodeTiled *out) {
    static std::mutex mu;
    static PFN_cuTensorMapEncodeTiled fn = nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !ptr)
            return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled entry point unavailable");
        fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled>(ptr);
    }
    *out = fn;
    return PA_OK;
}

// A pool [num_blocks][num_kv_heads][block_size][D] as a 2-D tensor of
// rows x D elements, read in boxes of 16 rows x 128 bytes (64 16-bit or 128
// 8-bit elements) with the 128-byte shared-memory swizzle. Encoded maps are
// kept (the last kMapCache distinct pools), since a serving loop decodes over
// the same pools call after call.
constexpr int kMapCache = 16;

pa_status encode_pool_map(CUtensorMap *map, const void *pool, long long rows, int D, int elem_bytes,
                          CUtensorMapDataType type, int dev) {
    struct Entry {
        const void *pool;
        long long rows;
        int D, elem_bytes, type, dev;
        CUtensorMap map;
    };
    static std::mutex mu;
    static Entry cache[kMapCache];
    static int filled = 0, next = 0;
    {
        std::lock_guard<std::mutex> lock(mu);
        for (int i = 0; i < filled; ++i) {
            const Entry &c = cache[i];
            if (c.pool == pool && c.rows == rows && c.D == D && c.elem_bytes == elem_bytes && c.type == (int)type &&
                c.dev == dev) {
                *map = c.map;
                return PA_OK;
            }
        }
    }
    PFN_cuTensorMapEncodeTiled enc;
    pa_status st = tensor_map_encoder(&enc);
    if (st != PA_OK) return st;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * elem_bytes};
    // Box rows of 128 bytes with the 128-byte swizzle, or (an 8-bit cache at
    // head_dim 64) one 64-byte box with the 64-byte swizzle.
    const int box_row = D * elem_bytes < 128 ? D * elem_bytes : 128;
    const cuuint32_t box[2] = {(cuuint32_t)(box_row / elem_bytes), 16};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, type, 2, const_cast<void *>(pool), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     box_row == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    std::lock_guard<std::mutex> lock(mu);
    Entry &c = cache[next];
    c.pool = pool;
    c.rows = rows;
    c.D = D;
    c.elem_bytes = elem_bytes;
    c.type = (int)type;
    c.dev = dev;
    c.map = *map;
    next = (next + 1) % kMapCache;
    if (filled < kMapCache) ++filled;
    return PA_OK;
}

// Sequences up to which the tensor-core kernels start without waiting for the
// plan (each warp passes over the context lengths once or twice at start).
constexpr int EARLY_MAX_SEQS = 512;

// pa::REDUCE_LAUNCH_MIN_PARTS (the kernel header) decides which sequences'
// split merges run in the merge launch.
using pa::REDUCE_LAUNCH_MIN_PARTS;
constexpr int REDUCE_SMEM_MAX = 200 * 1024;

// Dynamic shared memory of pa_reduce_kernel<D, G>: the thread groups' sums and
// the (max, sum) pairs of up to `parts` partitions.
template <int D, int G>
size_t reduce_smem_bytes(int parts) {
    return 2 * pa::REDUCE_GROUPS * (D * G / 4) * 16 + (size_t)parts * G * 8;
}

template <int D, int G, typename T, bool KV8 = false, bool SHARED = false, bool I8 = false, int HS = 0>
pa_status launch_decode_mma(pa::DecodeParams &p, cudaStream_t stream) {
    constexpr int NS = KV8 ? pa::DECODE_MMA_STAGES_FP8 : pa::DECODE_MMA_STAGES;
    DeviceInfo info;
    pa_status st = device_info(&info);
    if (st != PA_OK) return st;
    const long long rows = (long long)p.num_blocks * p.num_kv_heads * p.block_size;
    if (rows >= (1ll << 31)) return fail(PA_ERR_UNSUPPORTED, "pool has %lld rows, above 2^31", rows);
    CUtensorMap tmk, tmv;
    const CUtensorMapDataType type = KV8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : pa::MmaType<T>::tma_type;
    if ((st = encode_pool_map(&tmk, p.k_pool, rows, D, KV8 ? 1 : 2, type, info.dev)) != PA_OK) return st;
    if ((st = encode_pool_map(&tmv, p.v_pool, rows, D, KV8 ? 1 : 2, type, info.dev)) != PA_OK) return st;
    constexpr int max_warps = pa::mma_max_warps<D, G, KV8, SHARED>();
    int warps = (info.smem_optin - 1024) / pa::mma_warp_bytes<D, G, NS, KV8, SHARED>();
    if (warps > max_warps) warps = max_warps;
    if (warps < 1) return fail(PA_ERR_UNSUPPORTED, "not enough shared memory for one warp");
    const int smem = pa::mma_smem_bytes<D, G, NS, KV8, SHARED>(warps);
    auto kernel = pa::pa_decode_mma_kernel<D, G, T, NS, KV8, SHARED, I8, HS>;
    cudaError_t e = set_dynamic_smem<pa::pa_decode_mma_kernel<D, G, T, NS, KV8, SHARED, I8, HS>>(info.dev, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");

    if constexpr (SHARED) {
        // Shared units end with several members' merges; they run in the
        // merge launch, one CTA per (member, KV head), all at once.
        p.reduce_launch = p.max_parts > 1 && reduce_smem_bytes<D, G>(p.max_parts) <= REDUCE_SMEM_MAX;
        pa::pa_plan_shared_kernel<<<1, pa::PLAN_THREADS, 0, stream>>>(p);
        ++g_launches;
    } else {
        p.early = p.num_seqs <= EARLY_MAX_SEQS;
        // Sequences with many partitions merge in a launch of their own (while
        // its (max, sum) pairs fit the reduce kernel's shared memory), the
        // others in the attention kernel.
        p.reduce_launch = p.l1_base > REDUCE_LAUNCH_MIN_PARTS && reduce_smem_bytes<D, G>(p.l1_base) <= REDUCE_SMEM_MAX;
        pa::pa_plan_kernel<<<1, pa::PLAN_WARP_THREADS, 0, stream>>>(p);
        ++g_launches;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(info.sms);
    cfg.blockDim = dim3(warps * 32);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kernel, p, tmk, tmv);
    if (e != cudaSuccess) return cuda_fail(e, "pa_decode launch");
    ++g_launches;
    {
        if (p.reduce_launch) {
            constexpr int V4 = D * G / 4;
            cudaLaunchConfig_t rc = {};
            rc.gridDim = dim3((unsigned)(p.num_seqs * p.num_kv_heads));
            rc.blockDim = dim3(pa::REDUCE_GROUPS * V4);
            rc.dynamicSmemBytes = reduce_smem_bytes<D, G>(p.l1_base);
            rc.stream = stream;
            rc.attrs = attr;
            rc.numAttrs = 1;
            if constexpr (SHARED) {
                rc.gridDim = dim3((unsigned)((p.num_seqs * p.num_kv_heads + 7) / 8));
                rc.blockDim = dim3(256);
                rc.dynamicSmemBytes = 0;
                e = cudaLaunchKernelEx(&rc, pa::pa_reduce_members_kernel<D, G, T>, p);
            } else {
                e = set_dynamic_smem<pa::pa_reduce_kernel<D, G, T>>(info.dev, REDUCE_SMEM_MAX);
                if (e == cudaSuccess) e = cudaLaunchKernelEx(&rc, pa::pa_reduce_kernel<D, G, T>, p);
            }
            if (e != cudaSuccess) return cuda_fail(e, "pa_reduce_kernel launch");
            ++g_launches;
        }
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pa_decode launch");
    return PA_OK;
}

// 8-bit cache (E4M3, or INT8 with I8; HS: scales per tensor 0, per KV head 1,
// per (block, KV head) 2): tensor-core
// kernel, head_dim 64 or 128.
template <int D, typename T, bool I8 = false, int HS = 0>
pa_status dispatch_group_fp8(pa::DecodeParams &p, int group, cudaStream_t stream) {
    switch (group) {
        case 1: return launch_decode_mma<D, 1, T, true, false, I8, HS>(p, stream);
        case 2: return launch_decode_mma<D, 2, T, true, false, I8, HS>(p, stream);
        case 4: return launch_decode_mma<D, 4, T, true, false, I8, HS>(p, stream);
        case 8: return launch_decode_mma<D, 8, T, true, false, I8, HS>(p, stream);
    }
    return fail(PA_ERR_UNSUPPORTED, "group size %d", group);
}

// Shared-prefix units (pa_decode_shared): tensor-core kernel, 16-bit cache.
template <int D, typename T>
pa_status dispatch_group_shared(pa::DecodeParams &p, int group, cudaStream_t stream) {
    if (group < pa::DECODE_TENSOR_MIN_GROUP)
        return fail(PA_ERR_UNSUPPORTED, "shared-prefix units need the tensor-core kernel (group %d)", group);
    switch (group) {
        case 1: return launch_decode_mma<D, 1, T, false, true>(p, stream);
        case 2: return launch_decode_mma<D, 2, T, false, true>(p, stream);
        case 4: return launch_decode_mma<D, 4, T, false, true>(p, stream);
        case 8: return launch_decode_mma<D, 8, T, false, true>(p, stream);
    }
    return fail(PA_ERR_UNSUPPORTED, "group size %d", group);
}

// Shared-prefix units over an 8-bit cache (one scale per KV head, HS 1, or
// per (block, KV head), HS 2).
template <int D, typename T, bool I8, int HS = 1>
pa_status dispatch_group_shared_kv8(pa::DecodeParams &p, int group, cudaStream_t stream) {
    switch (group) {
        case 1: return launch_decode_mma<D, 1, T, true, true, I8, HS>(p, stream);
        case 2: return launch_decode_mma<D, 2, T, true, true, I8, HS>(p, stream);
        case 4: return launch_decode_mma<D, 4, T, true, true, I8, HS>(p, stream);
        case 8: return launch_decode_mma<D, 8, T, true, true, I8, HS>(p, stream);
    }
    return fail(PA_ERR_UNSUPPORTED, "group size %d", group);
}

template <int D, typename T>
pa_status dispatch_group(pa::DecodeParams &p, int group, cudaStream_t stream) {
    if (group >= pa::DECODE_TENSOR_MIN_GROUP) {
        switch (group) {
#if PA_DECODE_TENSOR_MIN_GROUP <= 1
            case 1: return launch_decode_mma<D, 1, T>(p, stream);
#endif
            case 2: return launch_decode_mma<D, 2, T>(p, stream);
            case 4: return launch_decode_mma<D, 4, T>(p, stream);
            case 8: return launch_decode_mma<D, 8, T>(p, stream);
        }
    }
    switch (group) {
#if PA_DECODE_TENSOR_MIN_GROUP > 1
        case 1: return launch_decode<D, 1, T>(p, stream);
#endif
#if PA_DECODE_TENSOR_MIN_GROUP > 2
        case 2: return launch_decode<D, 2, T>(p, stream);
#endif
#if PA_DECODE_TENSOR_MIN_GROUP > 4
        case 4: return launch_decode<D, 4, T>(p, stream);
#endif
#if PA_DECODE_TENSOR_MIN_GROUP > 8
        case 8: return launch_decode<D, 8, T>(p, stream);
#endif
    }
    return fail(PA_ERR_UNSUPPORTED, "group size %d", group);
}

}  // namespace
