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
//    device (cudaGetSymbolAddress) and keeps it for the device's current
//    context; make that first call before any stream capture.  A later call
//    made in another context of the device (after cudaDeviceReset, say, or a
//    primary context destroyed and made again) looks the address up again
//    instead of using the old one;
//  * all calls share the one array, and it keeps the previous call's contents.
//    Nothing in it needs to start at zero: every call rewrites the partition
//    plan and every partial result before reading them.  Calls that overlap on
//    the GPU (different streams, no ordering between them) race on the array.
// No cudaMalloc, cudaFree or allocating library routine is called here.

#include <algorithm>
#include <mutex>

#include <cuda.h>          // CUcontext / CUresult types only; driver calls go through the runtime's entry points
#include <cuda_runtime.h>

#include "pa.h"

namespace {

constexpr int kMaxDevices = 64;

// Scratch for the partition plan and partial results of the split-K path.
static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

// The unique id (never reused within the process) of the context current on
// the calling thread, through the driver's cuCtxGetCurrent / cuCtxGetId as the
// runtime hands them out; false when there is none or the calls are missing.
bool current_context_id(unsigned long long* id) {
    using GetCurrent = CUresult (*)(CUcontext*);
    using GetId = CUresult (*)(CUcontext, unsigned long long*);
    static GetCurrent get_current = nullptr;
    static GetId get_id = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_current = reinterpret_cast<GetCurrent>(p);
        p = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            get_id = reinterpret_cast<GetId>(p);
    });
    if (!get_current || !get_id) return false;
    CUcontext ctx = nullptr;
    if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
    return get_id(ctx, id) == CUDA_SUCCESS;
}

struct ScratchSlot {
    void* ptr = nullptr;
    unsigned long long ctx_id = 0;
};

std::mutex g_scratch_mu;
ScratchSlot g_scratch[kMaxDevices];

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, never a device address, so
// the address is looked up with the device current, once per device and
// context; without a context id to compare, it is looked up on every call.
pa_status scratch_on_current_device(void** out) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return PA_ERR_UNSUPPORTED;
    unsigned long long id = 0;
    const bool have_id = current_context_id(&id);
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot& slot = g_scratch[dev];
    if (!slot.ptr || !have_id || slot.ctx_id != id) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
        // the lookup makes the device's context current if none was
        unsigned long long now = 0;
        slot.ptr = p;
        slot.ctx_id = current_context_id(&now) ? now : 0;
        if (!have_id && slot.ctx_id == 0) slot.ptr = nullptr;   // nothing to compare with: look up next time too
        *out = p;
        return PA_OK;
    }
    *out = slot.ptr;
    return PA_OK;
}

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, const void* q, const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, const int32_t* context_lens, float scale,
                                       int block_size, int num_kv_heads, int num_seqs, int num_heads, int head_dim,
                                       int max_blocks_per_seq, int max_context_len, int num_blocks, pa_dtype dtype,
                                       int partition_size, void* stream) {
    // the scratch pa_decode will lay out: contexts are bounded by max_context_len
    // and by the block table's capacity, whichever is smaller
    const int64_t table_cap = (int64_t)std::max(max_blocks_per_seq, 0) * std::max(block_size, 0);
    const int cap = (int)std::max<int64_t>(0, std::min<int64_t>(max_context_len, table_cap));
    const size_t need = pa_decode_workspace_size(num_seqs, num_heads, head_dim, cap, partition_size);
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
