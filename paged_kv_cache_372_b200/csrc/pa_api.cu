// Host side of the C ABI declared in include/pa.h: argument validation,
// partition choice, workspace carving and kernel launches on the caller's
// stream. Nothing here allocates device memory or synchronises (except
// pa_device_errors, which exists to do so).
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "pa.h"
#include "pa_cache.cuh"
#include "pa_common.cuh"
#include "pa_decode.cuh"
#include "pa_decode_mma.cuh"

#include <cudaTypedefs.h>

namespace {

thread_local std::string g_last_error;

pa_status fail(pa_status st, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return st;
}

pa_status cuda_fail(cudaError_t e, const char *what) {
    return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

struct DeviceInfo {
    int sms = 0;
    int smem_optin = 0;
};

constexpr int kMaxDevices = 64;

pa_status device_info(DeviceInfo *out) {
    static std::mutex mu;
    static DeviceInfo cache[kMaxDevices];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(PA_ERR_CUDA, "device index %d out of range", dev);
    std::lock_guard<std::mutex> lock(mu);
    if (cache[dev].sms == 0) {
        int sms = 0, smem = 0;
        e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
        e = cudaDeviceGetAttribute(&smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(shared memory)");
        cache[dev].sms = sms;
        cache[dev].smem_optin = smem;
    }
    *out = cache[dev];
    return PA_OK;
}

// Largest partition the attention kernels take: the unit's block-table slice
// fits one register per lane (<= 32 blocks).
int partition_cap(int block_size) { return 32 * block_size; }

// Partition used when the caller passes 0 (a whole sequence when every
// context fits in it). The tensor-core kernel streams fast enough per warp
// that long units (32 blocks) are best; the CUDA-core kernel (one query head
// per KV head) needs more, shorter units to keep every warp busy.
int auto_partition(int group, int block_size) { return group >= pa::DECODE_TENSOR_MIN_GROUP ? 32 * block_size : 256; }

bool shape_supported(int num_heads, int num_kv_heads, int head_dim, int block_size) {
    if (num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads) return false;
    const int g = num_heads / num_kv_heads;
    if (g != 1 && g != 2 && g != 4 && g != 8) return false;
    if (head_dim != 64 && head_dim != 128) return false;
    return block_size == 16 || block_size == 32 || block_size == 64;
}

// Resolves partition_size (0 = auto). Returns 0 for an invalid request.
int resolve_partition(int group, int block_size, int max_context_len, int requested) {
    if (requested > 0) {
        if (requested % 16 || requested % block_size || requested > partition_cap(block_size)) return 0;
        return requested;
    }
    const int auto_p = auto_partition(group, block_size);
    if (max_context_len <= auto_p) {
        const int need = max_context_len > 0 ? max_context_len : 1;
        return ((need + block_size - 1) / block_size) * block_size;
    }
    return auto_p;
}

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

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
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");

    pa::pa_plan_kernel<<<1, pa::PLAN_THREADS, 0, stream>>>(p);
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
// rows x D elements, read in boxes of 16 rows x 64 columns (128 bytes) with
// the 128-byte shared-memory swizzle.
template <typename T>
pa_status encode_pool_map(CUtensorMap *map, const void *pool, long long rows, int D) {
    PFN_cuTensorMapEncodeTiled enc;
    pa_status st = tensor_map_encoder(&enc);
    if (st != PA_OK) return st;
    const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
    const cuuint32_t box[2] = {64, 16};
    const cuuint32_t estr[2] = {1, 1};
    CUresult r = enc(map, pa::MmaType<T>::tma_type, 2, const_cast<void *>(pool), dims, strides, box, estr,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
    return PA_OK;
}

template <int D, int G, typename T>
pa_status launch_decode_mma(pa::DecodeParams &p, cudaStream_t stream) {
    constexpr int NS = pa::DECODE_MMA_STAGES;
    DeviceInfo info;
    pa_status st = device_info(&info);
    if (st != PA_OK) return st;
    const long long rows = (long long)p.num_blocks * p.num_kv_heads * p.block_size;
    if (rows >= (1ll << 31)) return fail(PA_ERR_UNSUPPORTED, "pool has %lld rows, above 2^31", rows);
    CUtensorMap tmk, tmv;
    if ((st = encode_pool_map<T>(&tmk, p.k_pool, rows, D)) != PA_OK) return st;
    if ((st = encode_pool_map<T>(&tmv, p.v_pool, rows, D)) != PA_OK) return st;
    int warps = (info.smem_optin - 1024) / pa::mma_warp_bytes<D, G, NS>();
    if (warps > pa::DECODE_MAX_WARPS) warps = pa::DECODE_MAX_WARPS;
    if (warps < 1) return fail(PA_ERR_UNSUPPORTED, "not enough shared memory for one warp");
    const int smem = pa::mma_smem_bytes<D, G, NS>(warps);
    auto kernel = pa::pa_decode_mma_kernel<D, G, T, NS>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute");

    pa::pa_plan_kernel<<<1, pa::PLAN_THREADS, 0, stream>>>(p);
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
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pa_decode launch");
    return PA_OK;
}

template <int D, typename T>
pa_status dispatch_group(pa::DecodeParams &p, int group, cudaStream_t stream) {
    if (group >= pa::DECODE_TENSOR_MIN_GROUP) {
        switch (group) {
            case 2: return launch_decode_mma<D, 2, T>(p, stream);
            case 4: return launch_decode_mma<D, 4, T>(p, stream);
            case 8: return launch_decode_mma<D, 8, T>(p, stream);
        }
    }
    switch (group) {
        case 1: return launch_decode<D, 1, T>(p, stream);
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

// Lets other translation units of the library record pa_last_error() text.
void pa_internal_set_last_error(const char *msg) { g_last_error = msg ? msg : ""; }

extern "C" {

const char *pa_status_string(int status) {
    switch (status) {
        case PA_OK: return "PA_OK";
        case PA_ERR_INVALID: return "PA_ERR_INVALID";
        case PA_ERR_UNSUPPORTED: return "PA_ERR_UNSUPPORTED";
        case PA_ERR_CUDA: return "PA_ERR_CUDA";
        case PA_ERR_DEVICE_CHECK: return "PA_ERR_DEVICE_CHECK";
    }
    return "PA_ERR_UNKNOWN";
}

const char *pa_last_error(void) { return g_last_error.c_str(); }

int pa_decode_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                             int max_context_len, int partition_size) {
    if (num_seqs < 0 || max_context_len < 0 || partition_size < 0) return 0;
    if (!shape_supported(num_heads, num_kv_heads, head_dim, block_size)) return 0;
    return resolve_partition(num_heads / num_kv_heads, block_size, max_context_len, partition_size);
}

size_t pa_decode_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                int max_context_len, int partition_size) {
    const int P = pa_decode_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                           max_context_len, partition_size);
    if (P == 0) return 0;
    const int max_parts = max_context_len > 0 ? ceil_div(max_context_len, P) : 1;
    return pa::ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_parts).total;
}

pa_status pa_decode(void *out, const void *q, const void *k_pool, const void *v_pool, const int32_t *block_tables,
                    const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                    int block_size, int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                    int dtype, int partition_size, void *workspace, size_t workspace_bytes, pa_stream_t stream) {
    g_last_error.clear();
    if (num_seqs < 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 || max_context_len < 0 || partition_size < 0)
        return fail(PA_ERR_INVALID, "negative or zero size argument");
    if (dtype != PA_F16 && dtype != PA_BF16) return fail(PA_ERR_INVALID, "dtype %d", dtype);
    if (!shape_supported(num_heads, num_kv_heads, head_dim, block_size))
        return fail(PA_ERR_UNSUPPORTED, "heads %d/%d, head_dim %d, block_size %d", num_heads, num_kv_heads,
                    head_dim, block_size);
    if (!(scale == scale)) return fail(PA_ERR_INVALID, "scale is NaN");
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_pool || !v_pool || !block_tables || !context_lens || !workspace)
        return fail(PA_ERR_INVALID, "null pointer");
    if (!aligned(out, 16) || !aligned(q, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
        !aligned(block_tables, 4) || !aligned(context_lens, 4) || !aligned(workspace, 256))
        return fail(PA_ERR_INVALID, "misaligned pointer (16 B tensors, 4 B int arrays, 256 B workspace)");
    const int P = resolve_partition(num_heads / num_kv_heads, block_size, max_context_len, partition_size);
    if (P == 0)
        return fail(PA_ERR_INVALID, "partition_size %d (multiple of 16 and of block_size, at most %d)",
                    partition_size, partition_cap(block_size));
    const long long table_tokens = (long long)max_blocks_per_seq * block_size;
    const int ctx_limit = (int)(table_tokens < max_context_len ? table_tokens : max_context_len);
    const int max_parts = max_context_len > 0 ? ceil_div(max_context_len, P) : 1;
    if ((long long)num_seqs * max_parts * num_kv_heads >= (1ll << 31))
        return fail(PA_ERR_UNSUPPORTED, "too many work units");
    const pa::WsLayout L = pa::ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_parts);
    if (workspace_bytes < L.total)
        return fail(PA_ERR_INVALID, "workspace %zu bytes < %zu needed", workspace_bytes, L.total);

    pa::DecodeParams p;
    p.out = out;
    p.q = q;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.block_tables = block_tables;
    p.context_lens = context_lens;
    p.num_seqs = num_seqs;
    p.num_heads = num_heads;
    p.num_kv_heads = num_kv_heads;
    p.head_dim = head_dim;
    p.block_size = block_size;
    p.max_blocks_per_seq = max_blocks_per_seq;
    p.num_blocks = num_blocks;
    p.ctx_limit = ctx_limit;
    p.partition = P;
    p.max_parts = max_parts;
    p.qscale = scale * 1.4426950408889634f;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    p.counter = reinterpret_cast<int *>(ws);
    p.num_entries = reinterpret_cast<int *>(ws) + 1;
    p.entries = reinterpret_cast<int4 *>(ws + L.entries);
    p.ml = reinterpret_cast<float2 *>(ws + L.ml);
    p.part_acc = reinterpret_cast<float *>(ws + L.acc);
    p.merge_count = reinterpret_cast<int *>(ws + L.count);

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int group = num_heads / num_kv_heads;
    if (head_dim == 128)
        return dtype == PA_F16 ? dispatch_group<128, __half>(p, group, s)
                               : dispatch_group<128, __nv_bfloat16>(p, group, s);
    return dtype == PA_F16 ? dispatch_group<64, __half>(p, group, s) : dispatch_group<64, __nv_bfloat16>(p, group, s);
}

pa_status pa_reshape_and_cache(const void *k, const void *v, void *k_pool, void *v_pool, const int64_t *slot_mapping,
                               int num_tokens, int num_kv_heads, int head_dim, int block_size, int num_blocks,
                               int dtype, pa_stream_t stream) {
    g_last_error.clear();
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return fail(PA_ERR_INVALID, "size argument");
    if (dtype != PA_F16 && dtype != PA_BF16) return fail(PA_ERR_INVALID, "dtype %d", dtype);
    if (head_dim != 64 && head_dim != 128) return fail(PA_ERR_UNSUPPORTED, "head_dim %d", head_dim);
    if (block_size != 16 && block_size != 32 && block_size != 64)
        return fail(PA_ERR_UNSUPPORTED, "block_size %d", block_size);
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !k_pool || !v_pool || !slot_mapping) return fail(PA_ERR_INVALID, "null pointer");
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_pool, 16) || !aligned(v_pool, 16) ||
        !aligned(slot_mapping, 8))
        return fail(PA_ERR_INVALID, "misaligned pointer");
    DeviceInfo info;
    pa_status st = device_info(&info);
    if (st != PA_OK) return st;
    const int vec_per_row = head_dim / 8;
    const long long total = (long long)num_tokens * num_kv_heads * vec_per_row;
    long long blocks = (total + 255) / 256;
    const long long cap = (long long)info.sms * 16;
    if (blocks > cap) blocks = cap;
    pa::pa_reshape_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<uint4 *>(k_pool),
        static_cast<uint4 *>(v_pool), slot_mapping, total, vec_per_row, num_kv_heads, block_size,
        (long long)num_blocks * block_size);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pa_reshape_and_cache launch");
    return PA_OK;
}

pa_status pa_copy_blocks(void *const *pools, int num_pools, const int64_t *src_dst_pairs, int num_pairs,
                         size_t block_bytes, int num_blocks, pa_stream_t stream) {
    g_last_error.clear();
    if (num_pools < 0 || num_pairs < 0 || num_blocks <= 0) return fail(PA_ERR_INVALID, "size argument");
    if (num_pairs == 0 || num_pools == 0) return PA_OK;
    if (num_pairs > 2147483647 / 2) return fail(PA_ERR_UNSUPPORTED, "too many pairs");
    if (!pools || !src_dst_pairs) return fail(PA_ERR_INVALID, "null pointer");
    if (block_bytes == 0 || block_bytes % 16) return fail(PA_ERR_INVALID, "block_bytes %zu not a multiple of 16", block_bytes);
    if (!aligned(src_dst_pairs, 8)) return fail(PA_ERR_INVALID, "misaligned pairs");
    for (int i = 0; i < num_pools; ++i)
        if (!pools[i] || !aligned(pools[i], 16)) return fail(PA_ERR_INVALID, "pool %d null or misaligned", i);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int first = 0; first < num_pools; first += pa::COPY_MAX_POOLS) {
        const int n = num_pools - first < pa::COPY_MAX_POOLS ? num_pools - first : pa::COPY_MAX_POOLS;
        pa::PoolList list;
        for (int i = 0; i < pa::COPY_MAX_POOLS; ++i) list.ptr[i] = i < n ? static_cast<uint4 *>(pools[first + i]) : nullptr;
        const dim3 grid((unsigned)num_pairs, (unsigned)n);
        pa::pa_copy_blocks_kernel<<<grid, 256, 0, s>>>(list, src_dst_pairs, (long long)(block_bytes / 16),
                                                       (long long)num_blocks);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pa_copy_blocks launch");
    return PA_OK;
}

pa_status pa_device_errors(unsigned int *flags, int clear, pa_stream_t stream) {
    g_last_error.clear();
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned int v = 0;
    e = cudaMemcpyFromSymbol(&v, pa::g_device_errors, sizeof(v));
    if (e != cudaSuccess) return cuda_fail(e, "read error word");
    if (clear && v) {
        const unsigned int zero = 0;
        e = cudaMemcpyToSymbol(pa::g_device_errors, &zero, sizeof(zero));
        if (e != cudaSuccess) return cuda_fail(e, "clear error word");
    }
    if (flags) *flags = v;
    return v ? PA_ERR_DEVICE_CHECK : PA_OK;
}

int pa_num_sms(void) {
    DeviceInfo info;
    return device_info(&info) == PA_OK ? info.sms : 0;
}

}  // extern "C"
