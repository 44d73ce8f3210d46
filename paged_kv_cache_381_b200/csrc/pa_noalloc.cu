// pa_decode_noalloc: paged decode whose split-K scratch is a fixed array
// compiled into this library, for callers that cannot allocate device memory.
//
// Why: a serving engine usually hands almost all device memory to its KV
// block pool up front and then forbids further device allocations, and some
// latency-critical callers may not call cudaMalloc at all (it can synchronise
// the device).  Such callers cannot provide the workspace that pa_decode asks
// for when contexts are longer than one partition.  This entry point takes
// the same inputs and outputs as pa_decode and uses the array below instead.
//
// Cost and limits:
//  * the array is PA_NOALLOC_SCRATCH_BYTES; every GPU on which this library's
//    module is loaded holds it until the process exits;
//  * a batch whose scratch need (pa_decode_workspace_size) exceeds it is
//    rejected with PA_ERR_UNSUPPORTED before anything is launched;
//  * the first call on a device looks up the array's device address for that
//    device (cudaGetSymbolAddress); make that first call before any stream
//    capture;
//  * all calls share the one array, and it keeps the previous call's contents.
//    Nothing in it needs to start at zero: every call rewrites the partition
//    plan and every partial result before reading them.  Calls that overlap on
//    the GPU (different streams, no ordering between them) race on the array.
// No cudaMalloc, cudaFree or allocating library routine is called here.

#include <mutex>

#include <cuda_runtime.h>

#include "pa.h"

namespace {

constexpr int kMaxDevices = 64;

// Scratch for the partition plan and partial results of the split-K path.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, never a device address, so
// the address is looked up (once per device, with that device current).
pa_status scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, const int32_t* context_lens, float scale,
                                       int block_size, int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                                       int max_blocks_per_seq, int max_context_len, int num_blocks, pa_dtype dtype,
                                       int partition_size, void* stream) {
    const size_t need = pa_decode_workspace_size(num_seqs, num_heads, head_dim, max_context_len, partition_size);
    if (need > (size_t)PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    if (need > 0) {
        const pa_status st = scratch_on_current_device(&scratch);
        if (st != PA_OK) return st;
    }
    return pa_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, block_size, num_kv_heads, num_seqs,
                     num_heads, head_dim, max_blocks_per_seq, max_context_len, num_blocks, dtype, partition_size,
                     scratch, need > 0 ? (size_t)PA_NOALLOC_SCRATCH_BYTES : 0, stream);
}
