// pa_decode_noalloc: pa_decode for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc when they decode: an inference plugin
// whose host owns and pre-partitions all device memory, a real-time serving
// loop that must not take the allocator's implicit device synchronisation,
// or a process with a hard memory budget fixed at start-up. This entry point
// takes the same inputs and output as pa_decode but keeps pa_decode's scratch
// (work list, merge counters, split-context partials) in a fixed array in
// device memory that the library itself declares, so the caller passes no
// workspace and nothing is allocated per call.
//
// The array is PA_NOALLOC_SCRATCH_BYTES (16 MiB). Every GPU that loads this
// library holds it until the process exits.
#include <cstdio>

#include <cuda_runtime.h>

#include "pa.h"

// Defined in pa_api.cu: records the text pa_last_error() returns.
void pa_internal_set_last_error(const char *msg);

namespace {

__device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

}  // namespace

extern "C" pa_status pa_decode_noalloc(void *out, const void *q, const void *k_pool, const void *v_pool,
                                       const int32_t *block_tables, const int32_t *context_lens, int num_seqs,
                                       int num_heads, int num_kv_heads, int head_dim, int block_size,
                                       int max_blocks_per_seq, int num_blocks, int max_context_len, float scale,
                                       int dtype, int partition_size, pa_stream_t stream) {
    const size_t need = pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, block_size,
                                                 max_context_len, partition_size);
    if (need > (size_t)PA_NOALLOC_SCRATCH_BYTES) {
        char msg[256];
        snprintf(msg, sizeof(msg),
                 "pa_decode_noalloc: these sizes need %zu bytes of scratch, above the fixed %zu-byte array; "
                 "use pa_decode with a caller-owned workspace",
                 need, (size_t)PA_NOALLOC_SCRATCH_BYTES);
        pa_internal_set_last_error(msg);
        return PA_ERR_UNSUPPORTED;
    }
    // The array's device address on the current device. Host code cannot use
    // the array's name as an address; only this lookup gives one. It runs on
    // every call rather than being cached, so that the address stays right
    // after a device reset or a new primary context (which reload the module
    // at another address); once the module is loaded it is a host-side lookup.
    void *scratch = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&scratch, g_noalloc_scratch);
    if (e != cudaSuccess || !scratch) {
        pa_internal_set_last_error(e != cudaSuccess ? cudaGetErrorString(e) : "cudaGetSymbolAddress returned null");
        return PA_ERR_CUDA;
    }
    // pa_decode's plan kernel re-initialises everything in the scratch that
    // must start from zero (work-list cursor, merge counters) on every call.
    return pa_decode(out, q, k_pool, v_pool, block_tables, context_lens, num_seqs, num_heads, num_kv_heads,
                     head_dim, block_size, max_blocks_per_seq, num_blocks, max_context_len, scale, dtype,
                     partition_size, scratch, (size_t)PA_NOALLOC_SCRATCH_BYTES, stream);
}
