// Host side of the C ABI declared in include/pa.h: argument validation,
// partition choice, workspace carving and kernel launches on the caller's
// stream. Nothing here allocates device memory or synchronises (except
// pa_device_errors, which exists to do so).
#include <cstdarg>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include "pa.h"
#include "pa_cache.cuh"
#include "pa_common.cuh"
#include "pa_decode.cuh"
#include "pa_decode_mma.cuh"

namespace {

thread_local std::string g_last_error;
// Kernels launched from this thread (every entry point; read by pa_launch_count).
thread_local unsigned long long g_launches = 0;

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
    int dev = 0;
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
        cache[dev].dev = dev;
        cache[dev].sms = sms;
        cache[dev].smem_optin = smem;
    }
    *out = cache[dev];
    return PA_OK;
}

int ceil_div(long long a, long long b) { return (int)((a + b - 1) / b); }

}  // namespace

#include "pa_launch.cuh"

namespace {

// One warp waits, with a limit, on an mbarrier that never completes.
__global__ void pa_bounded_wait_probe(unsigned long long limit_ns) {
    __shared__ __align__(8) uint64_t bar;
    const uint32_t bar_s = pa::smem_u32(&bar);
    if (threadIdx.x == 0) {
        pa::mbar_init(bar_s, 1);
        pa::fence_barrier_init();
    }
    __syncwarp();
    bool ok = pa::mbar_wait_bounded(bar_s, 0, limit_ns);
    ok = __all_sync(pa::FULL_MASK, ok);
    if (!ok && threadIdx.x == 0) pa::raise_error(PA_DEVERR_TIMEOUT);
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

unsigned long long pa_launch_count(void) { return g_launches; }

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

int pa_decode_shared_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                    int max_context_len, int partition_size) {
    if (num_seqs < 0 || max_context_len < 0 || partition_size < 0) return 0;
    if (!shape_supported(num_heads, num_kv_heads, head_dim, block_size)) return 0;
    return resolve_partition(num_heads / num_kv_heads, block_size, max_context_len, partition_size,
                             PartMode::shared);
}

int pa_decode_fp8_partition_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                 int max_context_len, int partition_size) {
    if (num_seqs < 0 || max_context_len < 0 || partition_size < 0) return 0;
    if (!shape_supported(num_heads, num_kv_heads, head_dim, block_size)) return 0;
    return resolve_partition(num_heads / num_kv_heads, block_size, max_context_len, partition_size, PartMode::fp8);
}

size_t pa_decode_fp8_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                    int max_context_len, int partition_size) {
    const int P = pa_decode_fp8_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                               max_context_len, partition_size);
    if (P == 0) return 0;
    const int max_parts = max_context_len > 0 ? ceil_div(max_context_len, P) : 1;
    return pa::ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_parts).total;
}

size_t pa_decode_shared_workspace_size(int num_seqs, int num_heads, int num_kv_heads, int head_dim, int block_size,
                                       int max_context_len, int partition_size) {
    const int P = pa_decode_shared_partition_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                  max_context_len, partition_size);
    if (P == 0) return 0;
    const int max_parts = (max_context_len > 0 ? ceil_div(max_context_len, P) : 1) + 1;
    return pa::ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_parts, true).total;
}

}  // extern "C"

namespace {

// 8-bit cache kernels by code format and scale granularity.
template <int D, typename T>
pa_status dispatch_kv8(pa::DecodeParams &p, int group, cudaStream_t s, bool int8, int hs) {
    if (int8)
        return hs == 2 ? dispatch_group_fp8<D, T, true, 2>(p, group, s) : dispatch_group_fp8<D, T, true, 1>(p, group, s);
    return hs == 2   ? dispatch_group_fp8<D, T, false, 2>(p, group, s)
           : hs == 1 ? dispatch_group_fp8<D, T, false, 1>(p, group, s)
                     : dispatch_group_fp8<D, T, false, 0>(p, group, s);
}

// Shared-prefix units over an 8-bit cache, by code format and scale granularity.
template <int D, typename T>
pa_status dispatch_shared_kv8(pa::DecodeParams &p, int group, cudaStream_t s, bool int8, bool block_scales) {
    if (int8)
        return block_scales ? dispatch_group_shared_kv8<D, T, true, 2>(p, group, s)
                            : dispatch_group_shared_kv8<D, T, true, 1>(p, group, s);
    return block_scales ? dispatch_group_shared_kv8<D, T, false, 2>(p, group, s)
                        : dispatch_group_shared_kv8<D, T, false, 1>(p, group, s);
}

pa_status decode_impl(void *out, const void *q, const void *k_new, const void *v_new, const void *k_pool,
                      const void *v_pool, const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                      int num_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                      int num_blocks, int max_context_len, float scale, int dtype, int partition_size,
                      void *workspace, size_t workspace_bytes, pa_stream_t stream, bool kv8 = false,
                      float k_scale = 1.f, float v_scale = 1.f, bool shared = false, bool int8 = false,
                      const float *k_scales = nullptr, const float *v_scales = nullptr, bool block_scales = false) {
    g_last_error.clear();
    if ((k_scales == nullptr) != (v_scales == nullptr) || (k_scales && (!aligned(k_scales, 4) || !aligned(v_scales, 4))))
        return fail(PA_ERR_INVALID, "k_scales and v_scales: both null or both 4-byte aligned device arrays");
    if (kv8 && (!(k_scale > 0.f) || !(v_scale > 0.f) || k_scale == INFINITY || v_scale == INFINITY))
        return fail(PA_ERR_INVALID, "k_scale and v_scale must be positive and finite");
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
    if (shared && num_seqs > pa::SHARE_MAX_SEQS) {
        // The grouping plan is one CTA: a larger batch runs as consecutive
        // chunks of SHARE_MAX_SEQS sequences, in stream order on the same
        // workspace; sequences share blocks' work only within their chunk.
        const size_t es = 2;  // bytes of a q / out / k_new / v_new element
        const size_t qrow = (size_t)num_heads * head_dim * es, kvrow = (size_t)num_kv_heads * head_dim * es;
        for (int c0 = 0; c0 < num_seqs; c0 += pa::SHARE_MAX_SEQS) {
            const int n = num_seqs - c0 < pa::SHARE_MAX_SEQS ? num_seqs - c0 : pa::SHARE_MAX_SEQS;
            const pa_status st = decode_impl(
                static_cast<uint8_t *>(out) + c0 * qrow, static_cast<const uint8_t *>(q) + c0 * qrow,
                k_new ? static_cast<const uint8_t *>(k_new) + c0 * kvrow : nullptr,
                v_new ? static_cast<const uint8_t *>(v_new) + c0 * kvrow : nullptr, k_pool, v_pool,
                block_tables + (size_t)c0 * max_blocks_per_seq, context_lens + c0, n, num_heads, num_kv_heads,
                head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale, dtype, partition_size,
                workspace, workspace_bytes, stream, kv8, k_scale, v_scale, shared, int8, k_scales, v_scales,
                block_scales);
            if (st != PA_OK) return st;
        }
        return PA_OK;
    }
    const int P = resolve_partition(num_heads / num_kv_heads, block_size, max_context_len, partition_size,
                                    shared ? PartMode::shared : kv8 ? PartMode::fp8 : PartMode::plain);
    if (P == 0)
        return fail(PA_ERR_INVALID, "partition_size %d (multiple of 16 and of block_size, at most %d)",
                    partition_size, partition_cap(block_size));
    const long long table_tokens = (long long)max_blocks_per_seq * block_size;
    const int ctx_limit = (int)(table_tokens < max_context_len ? table_tokens : max_context_len);
    // With shared prefixes a sequence's partitions are cut at the end of its
    // shared blocks too, so it can have one more.
    const int max_parts = (max_context_len > 0 ? ceil_div(max_context_len, P) : 1) + (shared ? 1 : 0);
    if ((long long)num_seqs * max_parts * num_kv_heads >= (1ll << 31))
        return fail(PA_ERR_UNSUPPORTED, "too many work units");
    const pa::WsLayout L = pa::ws_layout(num_seqs, num_heads, num_kv_heads, head_dim, max_parts, shared);
    if (workspace_bytes < L.total)
        return fail(PA_ERR_INVALID, "workspace %zu bytes < %zu needed", workspace_bytes, L.total);

    if ((k_new || v_new) && (!k_new || !v_new || !aligned(k_new, 16) || !aligned(v_new, 16)))
        return fail(PA_ERR_INVALID, "k_new/v_new null or misaligned");

    pa::DecodeParams p;
    p.out = out;
    p.q = q;
    p.k_pool = k_pool;
    p.v_pool = v_pool;
    p.k_new = k_new;
    p.v_new = v_new;
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
    p.max_parts = L.slots;
    p.l1_base = max_parts;
    p.max_chunks = L.chunks;
    p.qscale = scale * 1.4426950408889634f * k_scale;
    p.v_scale = v_scale;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    p.counter = reinterpret_cast<int *>(ws);
    p.num_entries = reinterpret_cast<int *>(ws) + 1;
    p.entries = reinterpret_cast<int4 *>(ws + L.entries);
    p.ml = reinterpret_cast<float2 *>(ws + L.ml);
    p.part_acc = reinterpret_cast<float *>(ws + L.acc);
    p.merge_count = reinterpret_cast<int *>(ws + L.count);
    p.chunk_count = reinterpret_cast<int *>(ws + L.chunk_count);
    p.entries_b = shared ? reinterpret_cast<int4 *>(ws + L.entries_b) : nullptr;
    p.members = shared ? reinterpret_cast<int *>(ws + L.members) : nullptr;
    p.member_nparts = shared ? reinterpret_cast<int *>(ws + L.member_nparts) : nullptr;
    p.append_guard = k_new != nullptr;
    p.early = 0;          // set by the launcher of the tensor-core kernels
    p.reduce_launch = 0;  // likewise
    p.k_scales = k_scales;
    p.v_scales = v_scales;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int group = num_heads / num_kv_heads;
    if (kv8 && shared) {
        if (head_dim == 128)
            return dtype == PA_F16 ? dispatch_shared_kv8<128, __half>(p, group, s, int8, block_scales)
                                   : dispatch_shared_kv8<128, __nv_bfloat16>(p, group, s, int8, block_scales);
        return dtype == PA_F16 ? dispatch_shared_kv8<64, __half>(p, group, s, int8, block_scales)
                               : dispatch_shared_kv8<64, __nv_bfloat16>(p, group, s, int8, block_scales);
    }
    if (kv8) {
        // Scales: per (block, KV head) 2, per KV head 1, per tensor 0 (E4M3 only).
        const int hs = block_scales ? 2 : k_scales ? 1 : 0;
        if (head_dim == 128)
            return dtype == PA_F16 ? dispatch_kv8<128, __half>(p, group, s, int8, hs)
                                   : dispatch_kv8<128, __nv_bfloat16>(p, group, s, int8, hs);
        return dtype == PA_F16 ? dispatch_kv8<64, __half>(p, group, s, int8, hs)
                               : dispatch_kv8<64, __nv_bfloat16>(p, group, s, int8, hs);
    }
    if (shared) {
        if (head_dim == 128)
            return dtype == PA_F16 ? dispatch_group_shared<128, __half>(p, group, s)
                                   : dispatch_group_shared<128, __nv_bfloat16>(p, group, s);
        return dtype == PA_F16 ? dispatch_group_shared<64, __half>(p, group, s)
                               : dispatch_group_shared<64, __nv_bfloat16>(p, group, s);
    }
    if (head_dim == 128)
        return dtype == PA_F16 ? dispatch_group<128, __half>(p, group, s)
                               : dispatch_group<128, __nv_bfloat16>(p, group, s);
    return dtype == PA_F16 ? dispatch_group<64, __half>(p, group, s) : dispatch_group<64, __nv_bfloat16>(p, group, s);
}

}  // namespace

extern "C" {

pa_status pa_decode(void *out, const void *q, const void *k_pool, const void *v_pool, const int32_t *block_tables,
                    const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                    int block_size, int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                    int dtype, int partition_size, void *workspace, size_t workspace_bytes, pa_stream_t stream) {
    return decode_impl(out, q, nullptr, nullptr, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale,
                       dtype, partition_size, workspace, workspace_bytes, stream);
}

pa_status pa_decode_fp8(void *out, const void *q, const void *k_pool, const void *v_pool, const int32_t *block_tables,
                        const int32_t *context_lens, int num_seqs, int num_heads, int num_kv_heads, int head_dim,
                        int block_size, int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                        int dtype, float k_scale, float v_scale, int partition_size, void *workspace,
                        size_t workspace_bytes, pa_stream_t stream) {
    return decode_impl(out, q, nullptr, nullptr, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale,
                       dtype, partition_size, workspace, workspace_bytes, stream, true, k_scale, v_scale);
}

pa_status pa_decode_append(void *out, const void *q, const void *k_new, const void *v_new, void *k_pool,
                           void *v_pool, const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                           int num_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                           int num_blocks, int max_context_len, float scale, int dtype, int partition_size,
                           void *workspace, size_t workspace_bytes, pa_stream_t stream) {
    if (num_seqs > 0 && (!k_new || !v_new)) {
        g_last_error = "k_new/v_new null";
        return PA_ERR_INVALID;
    }
    return decode_impl(out, q, k_new, v_new, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale,
                       dtype, partition_size, workspace, workspace_bytes, stream);
}

pa_status pa_decode_shared(void *out, const void *q, const void *k_new, const void *v_new, void *k_pool,
                           void *v_pool, const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                           int num_heads, int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq,
                           int num_blocks, int max_context_len, float scale, int dtype, int partition_size,
                           void *workspace, size_t workspace_bytes, pa_stream_t stream) {
    if ((k_new == nullptr) != (v_new == nullptr)) {
        g_last_error = "k_new and v_new must both be null or both be set";
        return PA_ERR_INVALID;
    }
    return decode_impl(out, q, k_new, v_new, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale,
                       dtype, partition_size, workspace, workspace_bytes, stream, false, 1.f, 1.f, true);
}

pa_status pa_decode_shared_quant(void *out, const void *q, const void *k_pool, const void *v_pool,
                                 const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                                 int num_heads, int num_kv_heads, int head_dim, int block_size,
                                 int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                                 int dtype, int kv_format, const float *k_scales, const float *v_scales,
                                 int partition_size, void *workspace, size_t workspace_bytes, pa_stream_t stream) {
    g_last_error.clear();
    if (kv_format != PA_KV_E4M3 && kv_format != PA_KV_INT8) return fail(PA_ERR_INVALID, "kv_format %d", kv_format);
    if (num_seqs > 0 && (!k_scales || !v_scales)) return fail(PA_ERR_INVALID, "null scale array");
    return decode_impl(out, q, nullptr, nullptr, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale,
                       dtype, partition_size, workspace, workspace_bytes, stream, true, 1.f, 1.f, true,
                       kv_format == PA_KV_INT8, k_scales, v_scales);
}

pa_status pa_decode_shared_quant_blocks(void *out, const void *q, const void *k_pool, const void *v_pool,
                                        const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                                        int num_heads, int num_kv_heads, int head_dim, int block_size,
                                        int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                                        int dtype, int kv_format, const float *k_scales, const float *v_scales,
                                        int partition_size, void *workspace, size_t workspace_bytes,
                                        pa_stream_t stream) {
    g_last_error.clear();
    if (kv_format != PA_KV_E4M3 && kv_format != PA_KV_INT8) return fail(PA_ERR_INVALID, "kv_format %d", kv_format);
    if (num_seqs > 0 && (!k_scales || !v_scales)) return fail(PA_ERR_INVALID, "null scale array");
    return decode_impl(out, q, nullptr, nullptr, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale,
                       dtype, partition_size, workspace, workspace_bytes, stream, true, 1.f, 1.f, true,
                       kv_format == PA_KV_INT8, k_scales, v_scales, true);
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
    ++g_launches;
    pa::pa_reshape_kernel<<<(unsigned)blocks, 256, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<uint4 *>(k_pool),
        static_cast<uint4 *>(v_pool), slot_mapping, total, vec_per_row, num_kv_heads, block_size,
        (long long)num_blocks * block_size);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pa_reshape_and_cache launch");
    return PA_OK;
}

}  // extern "C"

namespace {

// The 8-bit cache write: E4M3 or INT8 codes, one scale per tensor (k_scale,
// v_scale) or one per KV head (k_scales, v_scales, device arrays).
pa_status reshape_kv8_impl(const void *k, const void *v, void *k_pool, void *v_pool, const int64_t *slot_mapping,
                           int num_tokens, int num_kv_heads, int head_dim, int block_size, int num_blocks, int dtype,
                           bool int8, float k_scale, float v_scale, const float *k_scales, const float *v_scales,
                           pa_stream_t stream, bool scales_per_block = false) {
    DeviceInfo info;
    pa_status st = device_info(&info);
    if (st != PA_OK) return st;
    const int vec_per_row = head_dim / 8;
    const long long total = (long long)num_tokens * num_kv_heads * vec_per_row;
    long long blocks = (total + 255) / 256;
    if (blocks > (long long)info.sms * 16) blocks = (long long)info.sms * 16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto launch = [&](auto kernel) {
        ++g_launches;
        kernel<<<(unsigned)blocks, 256, 0, s>>>(static_cast<const uint4 *>(k), static_cast<const uint4 *>(v),
                                                 static_cast<uint2 *>(k_pool), static_cast<uint2 *>(v_pool),
                                                 slot_mapping, total, vec_per_row, num_kv_heads, block_size,
                                                 (long long)num_blocks * block_size, k_scale, v_scale, k_scales,
                                                 v_scales, scales_per_block ? 1 : 0);
    };
    if (dtype == PA_F16)
        int8 ? launch(pa::pa_reshape_kv8_kernel<__half, true>) : launch(pa::pa_reshape_kv8_kernel<__half, false>);
    else
        int8 ? launch(pa::pa_reshape_kv8_kernel<__nv_bfloat16, true>)
             : launch(pa::pa_reshape_kv8_kernel<__nv_bfloat16, false>);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "8-bit cache write launch");
    return PA_OK;
}

}  // namespace

extern "C" {

pa_status pa_reshape_and_cache_fp8(const void *k, const void *v, void *k_pool, void *v_pool,
                                   const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                   int block_size, int num_blocks, int dtype, float k_scale, float v_scale,
                                   pa_stream_t stream) {
    g_last_error.clear();
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return fail(PA_ERR_INVALID, "size argument");
    if (dtype != PA_F16 && dtype != PA_BF16) return fail(PA_ERR_INVALID, "dtype %d", dtype);
    if (head_dim != 64 && head_dim != 128) return fail(PA_ERR_UNSUPPORTED, "head_dim %d", head_dim);
    if (block_size != 16 && block_size != 32 && block_size != 64)
        return fail(PA_ERR_UNSUPPORTED, "block_size %d", block_size);
    if (!(k_scale > 0.f) || !(v_scale > 0.f) || k_scale == INFINITY || v_scale == INFINITY)
        return fail(PA_ERR_INVALID, "k_scale and v_scale must be positive and finite");
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !k_pool || !v_pool || !slot_mapping) return fail(PA_ERR_INVALID, "null pointer");
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_pool, 8) || !aligned(v_pool, 8) || !aligned(slot_mapping, 8))
        return fail(PA_ERR_INVALID, "misaligned pointer");
    return reshape_kv8_impl(k, v, k_pool, v_pool, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                            num_blocks, dtype, false, k_scale, v_scale, nullptr, nullptr, stream);
}

static pa_status reshape_quant_checked(const void *k, const void *v, void *k_pool, void *v_pool,
                                       const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                       int block_size, int num_blocks, int dtype, int kv_format,
                                       const float *k_scales, const float *v_scales, pa_stream_t stream,
                                       bool scales_per_block);

pa_status pa_reshape_and_cache_quant(const void *k, const void *v, void *k_pool, void *v_pool,
                                     const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                     int block_size, int num_blocks, int dtype, int kv_format, const float *k_scales,
                                     const float *v_scales, pa_stream_t stream) {
    return reshape_quant_checked(k, v, k_pool, v_pool, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                                 num_blocks, dtype, kv_format, k_scales, v_scales, stream, false);
}

pa_status pa_reshape_and_cache_quant_blocks(const void *k, const void *v, void *k_pool, void *v_pool,
                                            const int64_t *slot_mapping, int num_tokens, int num_kv_heads,
                                            int head_dim, int block_size, int num_blocks, int dtype, int kv_format,
                                            const float *k_scales, const float *v_scales, pa_stream_t stream) {
    return reshape_quant_checked(k, v, k_pool, v_pool, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                                 num_blocks, dtype, kv_format, k_scales, v_scales, stream, true);
}

static pa_status reshape_quant_checked(const void *k, const void *v, void *k_pool, void *v_pool,
                                       const int64_t *slot_mapping, int num_tokens, int num_kv_heads, int head_dim,
                                       int block_size, int num_blocks, int dtype, int kv_format,
                                       const float *k_scales, const float *v_scales, pa_stream_t stream,
                                       bool scales_per_block) {
    g_last_error.clear();
    if (num_tokens < 0 || num_kv_heads <= 0 || num_blocks <= 0) return fail(PA_ERR_INVALID, "size argument");
    if (dtype != PA_F16 && dtype != PA_BF16) return fail(PA_ERR_INVALID, "dtype %d", dtype);
    if (kv_format != PA_KV_E4M3 && kv_format != PA_KV_INT8) return fail(PA_ERR_INVALID, "kv_format %d", kv_format);
    if (head_dim != 64 && head_dim != 128) return fail(PA_ERR_UNSUPPORTED, "head_dim %d", head_dim);
    if (block_size != 16 && block_size != 32 && block_size != 64)
        return fail(PA_ERR_UNSUPPORTED, "block_size %d", block_size);
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !k_pool || !v_pool || !slot_mapping || !k_scales || !v_scales)
        return fail(PA_ERR_INVALID, "null pointer");
    if (!aligned(k, 16) || !aligned(v, 16) || !aligned(k_pool, 8) || !aligned(v_pool, 8) ||
        !aligned(slot_mapping, 8) || !aligned(k_scales, 4) || !aligned(v_scales, 4))
        return fail(PA_ERR_INVALID, "misaligned pointer");
    return reshape_kv8_impl(k, v, k_pool, v_pool, slot_mapping, num_tokens, num_kv_heads, head_dim, block_size,
                            num_blocks, dtype, kv_format == PA_KV_INT8, 1.f, 1.f, k_scales, v_scales, stream,
                            scales_per_block);
}

pa_status pa_decode_quant(void *out, const void *q, const void *k_pool, const void *v_pool,
                          const int32_t *block_tables, const int32_t *context_lens, int num_seqs, int num_heads,
                          int num_kv_heads, int head_dim, int block_size, int max_blocks_per_seq, int num_blocks,
                          int max_context_len, float scale, int dtype, int kv_format, const float *k_scales,
                          const float *v_scales, int partition_size, void *workspace, size_t workspace_bytes,
                          pa_stream_t stream) {
    g_last_error.clear();
    if (kv_format != PA_KV_E4M3 && kv_format != PA_KV_INT8) return fail(PA_ERR_INVALID, "kv_format %d", kv_format);
    if (num_seqs > 0 && (!k_scales || !v_scales)) return fail(PA_ERR_INVALID, "null scale array");
    return decode_impl(out, q, nullptr, nullptr, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale,
                       dtype, partition_size, workspace, workspace_bytes, stream, true, 1.f, 1.f, false,
                       kv_format == PA_KV_INT8, k_scales, v_scales);
}

pa_status pa_decode_quant_blocks(void *out, const void *q, const void *k_pool, const void *v_pool,
                                 const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                                 int num_heads, int num_kv_heads, int head_dim, int block_size,
                                 int max_blocks_per_seq, int num_blocks, int max_context_len, float scale, int dtype,
                                 int kv_format, const float *k_scales, const float *v_scales, int partition_size,
                                 void *workspace, size_t workspace_bytes, pa_stream_t stream) {
    g_last_error.clear();
    if (kv_format != PA_KV_E4M3 && kv_format != PA_KV_INT8) return fail(PA_ERR_INVALID, "kv_format %d", kv_format);
    if (num_seqs > 0 && (!k_scales || !v_scales)) return fail(PA_ERR_INVALID, "null scale array");
    return decode_impl(out, q, nullptr, nullptr, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads,
                       num_kv_heads, head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale,
                       dtype, partition_size, workspace, workspace_bytes, stream, true, 1.f, 1.f, false,
                       kv_format == PA_KV_INT8, k_scales, v_scales, true);
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
        ++g_launches;
        pa::pa_copy_blocks_kernel<<<grid, 256, 0, s>>>(list, src_dst_pairs, (long long)(block_bytes / 16),
                                                       (long long)num_blocks);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pa_copy_blocks launch");
    return PA_OK;
}

}  // extern "C"

namespace {

// Device-usable address of `p`: device memory as is, page-locked host memory
// through its mapped device pointer; anything else (pageable host memory,
// unknown pointers) is rejected so that no kernel touches an unmapped address.
pa_status device_address(const void *p, const void **out, const char *what) {
    cudaPointerAttributes a;
    cudaError_t e = cudaPointerGetAttributes(&a, p);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return fail(PA_ERR_INVALID, "%s: not a CUDA-visible pointer", what);
    }
    if (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) {
        *out = p;
        return PA_OK;
    }
    if (a.type == cudaMemoryTypeHost && a.devicePointer) {
        *out = a.devicePointer;
        return PA_OK;
    }
    return fail(PA_ERR_INVALID, "%s: pageable host memory (use page-locked memory)", what);
}

}  // namespace

extern "C" {

pa_status pa_swap_blocks(void *const *dst_pools, const void *const *src_pools, int num_pools,
                         const int64_t *src_dst_pairs, int num_pairs, size_t block_bytes, int num_src_blocks,
                         int num_dst_blocks, pa_stream_t stream) {
    g_last_error.clear();
    if (num_pools < 0 || num_pairs < 0 || num_src_blocks <= 0 || num_dst_blocks <= 0)
        return fail(PA_ERR_INVALID, "size argument");
    if (num_pairs == 0 || num_pools == 0) return PA_OK;
    if (num_pairs > 2147483647 / 2) return fail(PA_ERR_UNSUPPORTED, "too many pairs");
    if (!dst_pools || !src_pools || !src_dst_pairs) return fail(PA_ERR_INVALID, "null pointer");
    if (block_bytes == 0 || block_bytes % 16)
        return fail(PA_ERR_INVALID, "block_bytes %zu not a multiple of 16", block_bytes);
    if (!aligned(src_dst_pairs, 8)) return fail(PA_ERR_INVALID, "misaligned pairs");
    const void *pairs = nullptr;
    pa_status st = device_address(src_dst_pairs, &pairs, "src_dst_pairs");
    if (st != PA_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    for (int first = 0; first < num_pools; first += pa::COPY_MAX_POOLS) {
        const int n = num_pools - first < pa::COPY_MAX_POOLS ? num_pools - first : pa::COPY_MAX_POOLS;
        pa::PoolList dst;
        pa::ConstPoolList src;
        for (int i = 0; i < pa::COPY_MAX_POOLS; ++i) {
            dst.ptr[i] = nullptr;
            src.ptr[i] = nullptr;
        }
        for (int i = 0; i < n; ++i) {
            if (!dst_pools[first + i] || !src_pools[first + i] || !aligned(dst_pools[first + i], 16) ||
                !aligned(src_pools[first + i], 16))
                return fail(PA_ERR_INVALID, "pool %d null or misaligned", first + i);
            const void *d = nullptr, *sp = nullptr;
            if ((st = device_address(dst_pools[first + i], &d, "dst pool")) != PA_OK) return st;
            if ((st = device_address(src_pools[first + i], &sp, "src pool")) != PA_OK) return st;
            dst.ptr[i] = static_cast<uint4 *>(const_cast<void *>(d));
            src.ptr[i] = static_cast<const uint4 *>(sp);
        }
        const dim3 grid((unsigned)num_pairs, (unsigned)n);
        ++g_launches;
        pa::pa_swap_blocks_kernel<<<grid, 256, 0, s>>>(dst, src, static_cast<const int64_t *>(pairs),
                                                       (long long)(block_bytes / 16), (long long)num_src_blocks,
                                                       (long long)num_dst_blocks);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "pa_swap_blocks launch");
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

pa_status pa_selftest_bounded_wait(unsigned long long limit_ns, pa_stream_t stream) {
    g_last_error.clear();
    if (limit_ns < 1000000ull || limit_ns > 10000000000ull)
        return fail(PA_ERR_INVALID, "limit %llu ns outside [1 ms, 10 s]", limit_ns);
    ++g_launches;
    pa_bounded_wait_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "bounded-wait probe launch");
    return PA_OK;
}

int pa_num_sms(void) {
    DeviceInfo info;
    return device_info(&info) == PA_OK ? info.sms : 0;
}

}  // extern "C"
