// C ABI of the paged KV-cache decode library: argument checks, kernel
// dispatch, launch accounting, the host-buffer step and the device error word.
// Declarations and contracts: include/pa.h.

#include <algorithm>
#include <atomic>
#include <cudaTypedefs.h>
#include <cmath>
#include <cstring>
#include <mutex>
#include <utility>
#include <vector>

// this unit holds the device error word (device/common.cuh) and reads it
#define PA_ERROR_WORD_UNIT 1
#include "device/cache_ops.cuh"
#include "device/decode.cuh"
#include "device/split_merge.cuh"
#include "device/verify.cuh"
#include "device/verify_tc.cuh"
#include "pa.h"

namespace pa_dev {

// The bounded wait's expiry path on its own: one thread waits on a barrier
// that nothing arrives at.  The wait must give up after kWaitLimitNs and the
// CTA must flag PA_DEVERR_TIMEOUT and exit, leaving the context usable.
__global__ void wait_expiry_kernel() {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0 && !mbar_wait(&bar, 0, &abort_flag)) flag_error(PA_DEVERR_TIMEOUT);
}

}  // namespace pa_dev

namespace {

constexpr int kDefaultPartition = 512;
constexpr int kMaxDevices = 64;

// ---------------------------------------------------------------- accounting
std::atomic<int64_t> g_launches{0};
std::mutex g_prof_mu;
bool g_prof_on = false;
uint32_t g_prof_mask = 0;
struct ProfRecord {
    int kernel;
    cudaEvent_t start, stop;
};
std::vector<ProfRecord> g_prof_records;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
    if (!g_event_pool.empty()) {
        cudaEvent_t e = g_event_pool.back();
        g_event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Counts one launch and, while profiling, brackets it with an event pair on
// its stream.
class LaunchScope {
  public:
    LaunchScope(int kernel, cudaStream_t stream) : kernel_(kernel), stream_(stream) {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        std::lock_guard<std::mutex> lk(g_prof_mu);
        if (g_prof_on && (g_prof_mask & (1u << kernel))) {
            start_ = take_event();
            stop_ = take_event();
            if (start_ && stop_) cudaEventRecord(start_, stream_);
        }
    }
    ~LaunchScope() {
        if (!start_ || !stop_) return;
        std::lock_guard<std::mutex> lk(g_prof_mu);
        cudaEventRecord(stop_, stream_);
        g_prof_records.push_back({kernel_, start_, stop_});
    }

  private:
    int kernel_;
    cudaStream_t stream_;
    cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

pa_status launch_status() { return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

// Launch as a programmatic dependent of the previous kernel in the stream: the
// launch may overlap that kernel's tail.  Every kernel launched this way
// executes griddepcontrol.wait before it reads anything earlier kernels wrote
// (and before it exits), so completion stays ordered along the stream.
template <typename... Params, typename... Args>
pa_status launch_dependent(void (*kern)(Params...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                           Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...) == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

// ------------------------------------------------------------- device info
int device_sms(int dev) {
    static std::atomic<int> cache[kMaxDevices];
    if (dev < 0 || dev >= kMaxDevices) return 148;
    int v = cache[dev].load(std::memory_order_relaxed);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cache[dev].store(v, std::memory_order_relaxed);
    }
    return v;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t elem_bytes(pa_dtype t) { return t == PA_F32 ? 4 : 2; }

bool valid_dtype(int t) { return t == PA_F32 || t == PA_F16 || t == PA_BF16; }

bool supported_block_size(int bs) { return bs == 8 || bs == 16 || bs == 32; }

bool supported_head_dim(int d) { return d == 64 || d == 128; }

pa_status check_cache_desc(const pa_cache_desc* c) {
    if (!c || c->num_blocks <= 0 || c->num_kv_heads <= 0 || !valid_dtype(c->dtype)) return PA_ERR_INVALID_ARG;
    if (!supported_block_size(c->block_size) || !supported_head_dim(c->head_dim)) return PA_ERR_UNSUPPORTED;
    return PA_OK;
}

// ------------------------------------------------------------ cache write
// Checks of pa_cache_write (all before any launch); fills the kernel arguments.
pa_status write_args(const void* k, const void* v, void* k_cache, void* v_cache, const int64_t* slot_mapping,
                     int num_tokens, const pa_cache_desc* cache, pa_dev::WriteArgs* w) {
    pa_status st = check_cache_desc(cache);
    if (st != PA_OK) return st;
    if (num_tokens < 0) return PA_ERR_INVALID_ARG;
    if (num_tokens == 0) return PA_OK;
    if (!k || !v || !k_cache || !v_cache || !slot_mapping) return PA_ERR_INVALID_ARG;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    const int64_t row_bytes = (int64_t)cache->num_kv_heads * cache->head_dim * elem_bytes(cache->dtype);
    w->k = static_cast<const uint4*>(k);
    w->v = static_cast<const uint4*>(v);
    w->k_cache = static_cast<uint4*>(k_cache);
    w->v_cache = static_cast<uint4*>(v_cache);
    w->slot_mapping = slot_mapping;
    w->num_tokens = num_tokens;
    w->row_vecs = (int)(row_bytes / 16);
    w->num_slots = (int64_t)cache->num_blocks * cache->block_size;
    return PA_OK;
}

// CTAs of 256 threads for a cache write: one thread per 16-byte vector, at most 65,535 CTAs
unsigned write_grid(const pa_dev::WriteArgs& w) {
    const int64_t threads = (int64_t)w.num_tokens * w.row_vecs;
    return (unsigned)std::max<int64_t>(1, std::min<int64_t>((threads + 255) / 256, 65535));
}

// ------------------------------------------------------------ workspace
struct WsLayout {
    size_t plan, count, split, counters, m, l, o, total;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

WsLayout ws_layout(int64_t S, int64_t Hq, int64_t D, int64_t maxP) {
    WsLayout w{};
    size_t off = 0;
    w.plan = off;
    off = align256(off + (size_t)(S * maxP) * sizeof(int2));
    w.count = off;                                      // pairs in the plan, split sequences, items dealt
    off = align256(off + 3 * sizeof(int));
    w.split = off;                                      // the split sequences
    off = align256(off + (size_t)S * sizeof(int));
    w.counters = off;                                   // fused-merge counters, <= S * Hq of them
    off = align256(off + (size_t)(S * Hq) * sizeof(int));
    w.m = off;
    off = align256(off + (size_t)(S * Hq * maxP) * sizeof(float));
    w.l = off;
    off = align256(off + (size_t)(S * Hq * maxP) * sizeof(float));
    w.o = off;
    off = align256(off + (size_t)(S * Hq * maxP * D) * sizeof(float));
    w.total = off;
    return w;
}

int resolve_partition(int partition_size) { return partition_size == 0 ? kDefaultPartition : partition_size; }

bool valid_partition(int p) { return p >= 32 && p <= 1024 && p % 32 == 0; }
// The verification kernels walk one partition's block ids from a table of 128
// entries in shared memory, and the plan sorts partitions of up to 2048 tokens.
constexpr int kMaxVerifyPartition = 2048;
constexpr int kVerifyTableEntries = 128;
bool valid_verify_partition_size(int p) { return p >= 32 && p <= kMaxVerifyPartition && p % 32 == 0; }
bool valid_verify_partition(int p, int block_size) {
    return valid_verify_partition_size(p) && p / block_size <= kVerifyTableEntries;
}

int64_t partitions_for(int64_t ctx, int64_t P) { return ctx <= P ? 1 : (ctx + P - 1) / P; }

// ------------------------------------------------------------ decode launch
std::atomic<int> g_decode_math{PA_MATH_AUTO};
std::atomic<int> g_split_merge{PA_MERGE_KERNEL};
constexpr int kMaxPartitions = 4096;    // partitions per sequence

// ---------------------------------------------------------------- TMA maps
// cuTensorMapEncodeTiled is reached through the runtime's driver entry point,
// so no driver library is linked.  Encoding is pure host work.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

// The pool [num_blocks, block_size, num_kv_heads, head_dim] as the 3-D tensor
// (head_dim, num_kv_heads, num_blocks * block_size), innermost first; one box
// is one 128-byte slice of head_dim for one kv head and block_size rows,
// landing with the 128-byte swizzle.
bool encode_pool_map(CUtensorMap* map, const void* pool, pa_dtype dtype, int head_dim, int num_kv_heads,
                     int num_blocks, int block_size, int box_rows) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t elt = dtype == PA_F32 ? 4 : 2;
    const CUtensorMapDataType t = dtype == PA_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                  : dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_kv_heads,
                          (cuuint64_t)num_blocks * (cuuint64_t)block_size};
    cuuint64_t strides[2] = {(cuuint64_t)head_dim * elt, (cuuint64_t)num_kv_heads * head_dim * elt};
    cuuint32_t box[3] = {(cuuint32_t)(128 / elt), 1u, (cuuint32_t)box_rows};
    cuuint32_t estride[3] = {1u, 1u, 1u};
    CUresult r = enc(map, t, 3, const_cast<void*>(pool), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// The pool as the 4-D tensor (128-byte head_dim slice, token row, slice index,
// kv head), innermost first.  One box is one block of one kv head with every
// slice: the slices land one after another, each as block_size rows of 128
// bytes with the 128-byte swizzle (the decode kernel's stage layout).
bool encode_pool_map_blocks(CUtensorMap* map, const void* pool, pa_dtype dtype, int head_dim, int num_kv_heads,
                            int num_blocks, int block_size) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) return false;
    const cuuint64_t elt = dtype == PA_F32 ? 4 : 2;
    const CUtensorMapDataType t = dtype == PA_F32   ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                  : dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint32_t slices = (cuuint32_t)(head_dim * elt / 128);
    cuuint64_t dims[4] = {128 / elt, (cuuint64_t)num_blocks * (cuuint64_t)block_size, slices,
                          (cuuint64_t)num_kv_heads};
    cuuint64_t strides[3] = {(cuuint64_t)num_kv_heads * head_dim * elt, 128, (cuuint64_t)head_dim * elt};
    cuuint32_t box[4] = {(cuuint32_t)(128 / elt), (cuuint32_t)block_size, slices, 1u};
    cuuint32_t estride[4] = {1u, 1u, 1u, 1u};
    CUresult r = enc(map, t, 4, const_cast<void*>(pool), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

// q [num_seqs, num_queries, num_heads, head_dim] as the 3-D tensor (head_dim,
// num_heads, num_seqs * num_queries), innermost first.  One box is one 128-byte
// slice of head_dim x `group` heads x `num_queries` rows: the query rows of one
// (sequence, kv head), landing as row i * group + g with the 128-byte swizzle.
bool encode_q_map(CUtensorMap* map, const void* q, pa_dtype dtype, int head_dim, int num_heads, int rows,
                  int group, int num_queries) {
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc || dtype == PA_F32 || group > 256 || num_queries > 256) return false;
    const cuuint64_t elt = 2;
    const CUtensorMapDataType t = dtype == PA_F16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    cuuint64_t dims[3] = {(cuuint64_t)head_dim, (cuuint64_t)num_heads, (cuuint64_t)rows};
    cuuint64_t strides[2] = {(cuuint64_t)head_dim * elt, (cuuint64_t)num_heads * head_dim * elt};
    cuuint32_t box[3] = {(cuuint32_t)(128 / elt), (cuuint32_t)group, (cuuint32_t)num_queries};
    cuuint32_t estride[3] = {1u, 1u, 1u};
    CUresult r = enc(map, t, 3, const_cast<void*>(q), dims, strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE,
                     CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <typename T, int D, int GC, bool TENSOR>
pa_status launch_decode(const pa_dev::DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                        int64_t pair_upper, cudaStream_t stream) {
    using C = pa_dev::DecodeCfg<T, D, GC, TENSOR>;
    auto kern = pa_dev::decode_kernel<T, D, GC, TENSOR>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    static std::atomic<uint64_t> configured{0};
    const uint64_t bit = 1ull << (dev & 63);
    const size_t smem_max = C::smem_bytes(C::MAX_PARTITION);
    if (!(configured.load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_max) != cudaSuccess)
            return PA_ERR_CUDA;
        configured.fetch_or(bit);
    }
    const size_t smem = C::smem_bytes(a.partition_size);
    static std::atomic<int64_t> occ_cache{0};   // (dev << 40) | (smem << 8) | blocks
    int occ = 0;
    const int64_t key = ((int64_t)dev << 40) | ((int64_t)smem << 8);
    const int64_t cached = occ_cache.load();
    if ((cached & ~int64_t(255)) == key && (cached & 255) > 0) {
        occ = (int)(cached & 255);
    } else {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, C::THREADS, smem) != cudaSuccess || occ <= 0)
            return PA_ERR_CUDA;
        occ_cache.store(key | std::min(occ, 255));
    }
    const int64_t items_upper = pair_upper * a.num_kv_heads * a.n_gchunks;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items_upper, (int64_t)device_sms(dev) * occ));
    LaunchScope scope(PA_KERNEL_DECODE, stream);
    return launch_dependent(kern, dim3((unsigned)grid), dim3(C::THREADS), smem, stream, a, tk, tv);
}

template <typename T, int D>
pa_status dispatch_group(const pa_dev::DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, int gc,
                         bool tensor, int64_t pair_upper, cudaStream_t st) {
    if constexpr (sizeof(T) == 2) {
        if (tensor) return launch_decode<T, D, 8, true>(a, tk, tv, pair_upper, st);
    }
    switch (gc) {
        case 1: return launch_decode<T, D, 1, false>(a, tk, tv, pair_upper, st);
        case 2: return launch_decode<T, D, 2, false>(a, tk, tv, pair_upper, st);
        case 4: return launch_decode<T, D, 4, false>(a, tk, tv, pair_upper, st);
        case 8: return launch_decode<T, D, 8, false>(a, tk, tv, pair_upper, st);
        default: return PA_ERR_UNSUPPORTED;
    }
}

template <typename T>
pa_status dispatch_head_dim(const pa_dev::DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, int D, int gc,
                            bool tensor, int64_t pair_upper, cudaStream_t st) {
    return D == 64 ? dispatch_group<T, 64>(a, tk, tv, gc, tensor, pair_upper, st)
                   : dispatch_group<T, 128>(a, tk, tv, gc, tensor, pair_upper, st);
}

template <typename T, int D>
pa_status launch_reduce_d(const pa_dev::DecodeArgs& a, cudaStream_t stream) {
    // persistent, one CTA per resident slot: the number of split rows is known
    // only on the device (plan)
    auto kern = pa_dev::reduce_kernel<T, D>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    static std::atomic<int> occ_of[kMaxDevices];
    const int threads = pa_dev::kReduceWarps * 32;
    int occ = dev < kMaxDevices ? occ_of[dev].load() : 0;
    if (occ <= 0) {
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, threads, 0) != cudaSuccess || occ <= 0)
            return PA_ERR_CUDA;
        if (dev < kMaxDevices) occ_of[dev].store(occ);
    }
    const int64_t rows = (int64_t)a.num_seqs * a.num_heads;
    const int64_t blocks_needed = (rows + pa_dev::kReduceWarps - 1) / pa_dev::kReduceWarps;
    const unsigned grid =
        (unsigned)std::max<int64_t>(1, std::min<int64_t>(blocks_needed, (int64_t)device_sms(dev) * occ));
    LaunchScope scope(PA_KERNEL_REDUCE, stream);
    return launch_dependent(kern, dim3(grid), dim3(threads), 0, stream, a);
}

template <typename T>
pa_status launch_reduce(const pa_dev::DecodeArgs& a, int D, cudaStream_t stream) {
    return D == 64 ? launch_reduce_d<T, 64>(a, stream) : launch_reduce_d<T, 128>(a, stream);
}

template <typename T, int D>
pa_status launch_verify(const pa_dev::DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv, int64_t pair_upper,
                        cudaStream_t stream) {
    using C = pa_dev::VerifyCfg<T, D>;
    auto kern = pa_dev::verify_kernel<T, D>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    static std::atomic<uint64_t> configured{0};
    static std::atomic<int> occ_of[kMaxDevices];
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::SMEM) != cudaSuccess)
            return PA_ERR_CUDA;
        int occ = 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, C::THREADS, C::SMEM) != cudaSuccess || occ <= 0)
            return PA_ERR_CUDA;
        if (dev < kMaxDevices) occ_of[dev].store(occ);
        configured.fetch_or(bit);
    }
    const int occ = dev < kMaxDevices ? std::max(1, occ_of[dev].load()) : 1;
    const int64_t items_upper = pair_upper * a.num_kv_heads * a.n_gchunks;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items_upper, (int64_t)device_sms(dev) * occ));
    LaunchScope scope(PA_KERNEL_VERIFY, stream);
    return launch_dependent(kern, dim3((unsigned)grid), dim3(C::THREADS), C::SMEM, stream, a, tk, tv);
}

template <typename T, int D>
pa_status launch_verify_tc(const pa_dev::DecodeArgs& a, const CUtensorMap& tk, const CUtensorMap& tv,
                           const CUtensorMap& tq, int64_t pair_upper, cudaStream_t stream) {
    using C = pa_dev::VerifyTcCfg<T, D>;
    auto kern = pa_dev::verify_tc_kernel<T, D>;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return PA_ERR_CUDA;
    static std::atomic<uint64_t> configured{0};
    static std::atomic<int> occ_of[kMaxDevices];
    static std::atomic<int> smem_of[kMaxDevices];
    const uint64_t bit = 1ull << (dev & 63);
    if (!(configured.load() & bit)) {
        int smem_sm = 0;
        cudaFuncAttributes fa;
        if (cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev) != cudaSuccess ||
            cudaFuncGetAttributes(&fa, kern) != cudaSuccess)
            return PA_ERR_CUDA;
        // Each CTA holds 256 of the SM's 512 TMEM columns: a third CTA on an SM would
        // only wait in tcgen05.alloc.  The shared memory asked for is raised until a
        // third no longer fits (1 KB reserved per CTA); the kernel uses C::SMEM of it.
        const int smem = std::max((int)C::SMEM, smem_sm / 3 - 1024 + 16);
        // the whole unified L1 as shared memory, so that two CTAs fit
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess ||
            cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, 100) != cudaSuccess)
            return PA_ERR_CUDA;
        // CTAs per SM from the shared memory and the registers
        const int by_smem = smem_sm / (smem + 1024);
        const int by_regs = 65536 / std::max(1, fa.numRegs * C::THREADS);
        const int occ = std::max(1, std::min(by_smem, by_regs));
        if (dev < kMaxDevices) {
            occ_of[dev].store(occ);
            smem_of[dev].store(smem);
        }
        configured.fetch_or(bit);
    }
    const int occ = std::min(2, dev < kMaxDevices ? std::max(1, occ_of[dev].load()) : 1);
    const size_t smem = dev < kMaxDevices && smem_of[dev].load() > 0 ? (size_t)smem_of[dev].load() : C::SMEM;
    const int64_t items_upper = pair_upper * a.num_kv_heads * a.n_gchunks;
    const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(items_upper, (int64_t)device_sms(dev) * occ));
    LaunchScope scope(PA_KERNEL_VERIFY, stream);
    return launch_dependent(kern, dim3((unsigned)grid), dim3(C::THREADS), smem, stream, a, tk, tv, tq);
}

std::atomic<int> g_verify_kernel{PA_VERIFY_AUTO};

int query_chunk(int group, bool tensor) {
    if (tensor) return 8;                  // mma n = 8: one tile holds up to 8 queries
    int g = std::min(group, 8);
    int c = 1;
    while (c < g) c <<= 1;
    return c;
}

}  // namespace

namespace {

// pa_decode, optionally preceded by a cache write (`wr`, pa_write_decode): all
// checks first, then the launches -- the write and the plan in one kernel when
// the batch is split, the write kernel alone when it is not.
pa_status decode_impl(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                      const int32_t* context_lens, float scale, int block_size, int num_kv_heads, int num_seqs,
                      int num_heads, int head_dim, int max_blocks_per_seq, int max_context_len, int num_blocks,
                      pa_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes, void* stream,
                      const pa_dev::WriteArgs* wr) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
        max_context_len < 0 || !valid_dtype(dtype) || !std::isfinite(scale))
        return PA_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    const int P = resolve_partition(partition_size);
    if (!valid_partition(P)) return PA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    auto write_alone = [&]() -> pa_status {
        LaunchScope scope(PA_KERNEL_CACHE_WRITE, s);
        pa_dev::cache_write_kernel<<<write_grid(*wr), 256, 0, s>>>(*wr);
        return launch_status();
    };
    if (num_seqs == 0) return wr ? write_alone() : PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;

    if ((int64_t)num_blocks * block_size > INT32_MAX) return PA_ERR_UNSUPPORTED;
    const int64_t table_cap = (int64_t)max_blocks_per_seq * block_size;
    const int64_t cap = std::min<int64_t>(max_context_len, table_cap);
    if (cap > INT32_MAX / 2) return PA_ERR_INVALID_ARG;
    const int64_t maxP = partitions_for(cap, P);
    if (maxP > kMaxPartitions) return PA_ERR_UNSUPPORTED;
    const int group = num_heads / num_kv_heads;
    const int math = g_decode_math.load(std::memory_order_relaxed);
    const bool tensor = dtype != PA_F32 && math != PA_MATH_SIMT;
    const int gc = query_chunk(group, tensor);
    const int n_gchunks = (group + gc - 1) / gc;
    if ((int64_t)num_seqs * maxP * num_kv_heads * n_gchunks > INT32_MAX) return PA_ERR_INVALID_ARG;

    pa_dev::DecodeArgs a{};
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = num_kv_heads;
    a.group = group;
    a.n_gchunks = n_gchunks;
    a.log2_bs = block_size == 8 ? 3 : block_size == 16 ? 4 : 5;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.ctx_cap = (int)cap;
    a.num_blocks = num_blocks;
    a.partition_size = P;
    a.max_partitions = (int)maxP;
    a.num_queries = 1;

    CUtensorMap tk, tv;
#if PA_DECODE_BOX_BLOCK
    // one TMA box = one block of one kv head, every 128-byte slice of head_dim
    if (!encode_pool_map_blocks(&tk, k_cache, dtype, head_dim, num_kv_heads, num_blocks, block_size) ||
        !encode_pool_map_blocks(&tv, v_cache, dtype, head_dim, num_kv_heads, num_blocks, block_size))
        return PA_ERR_CUDA;
#else
    const int box_rows = block_size;          // one TMA box = one block of one kv head, one 128-byte slice
    if (!encode_pool_map(&tk, k_cache, dtype, head_dim, num_kv_heads, num_blocks, block_size, box_rows) ||
        !encode_pool_map(&tv, v_cache, dtype, head_dim, num_kv_heads, num_blocks, block_size, box_rows))
        return PA_ERR_CUDA;
#endif
    if (maxP > 1) {
        const WsLayout L = ws_layout(num_seqs, num_heads, head_dim, maxP);
        if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return PA_ERR_INVALID_ARG;
        char* ws = static_cast<char*>(workspace);
        a.plan = reinterpret_cast<const int2*>(ws + L.plan);
        a.plan_count = reinterpret_cast<const int*>(ws + L.count);
        a.split_seqs = reinterpret_cast<const int*>(ws + L.split);
        a.part_m = reinterpret_cast<float*>(ws + L.m);
        a.part_l = reinterpret_cast<float*>(ws + L.l);
        a.part_o = reinterpret_cast<float*>(ws + L.o);
        const bool fused = g_split_merge.load(std::memory_order_relaxed) == PA_MERGE_FUSED;
        int* counters = reinterpret_cast<int*>(ws + L.counters);
        a.merge_count = fused ? counters : nullptr;
        const int num_counters = fused ? num_seqs * num_kv_heads * n_gchunks : 0;
        int2* plan = reinterpret_cast<int2*>(ws + L.plan);
        int* count = reinterpret_cast<int*>(ws + L.count);
        int* split = reinterpret_cast<int*>(ws + L.split);
        a.work_counter = count + 2;
        if (wr) {
            LaunchScope scope(PA_KERNEL_WRITE_PLAN, s);
            const unsigned wb = write_grid(*wr);
            pa_dev::write_plan_kernel<<<wb + 1, 256, 0, s>>>(*wr, (int)wb, a, plan, count, split, counters,
                                                             num_counters);
            if (launch_status() != PA_OK) return PA_ERR_CUDA;
        } else {
            LaunchScope scope(PA_KERNEL_PLAN, s);
            const int threads = std::min(1024, std::max(32, (num_seqs + 31) / 32 * 32));
            if (launch_dependent(pa_dev::plan_kernel, dim3(1), dim3(threads), 0, s, a, plan, count, split, counters,
                                 num_counters) != PA_OK)
                return PA_ERR_CUDA;
        }
    } else if (wr && write_alone() != PA_OK) {
        return PA_ERR_CUDA;
    }
    const int64_t pair_upper = (int64_t)num_seqs * maxP;
    pa_status st;
    switch (dtype) {
        case PA_F32: st = dispatch_head_dim<float>(a, tk, tv, head_dim, gc, false, pair_upper, s); break;
        case PA_F16: st = dispatch_head_dim<__half>(a, tk, tv, head_dim, gc, tensor, pair_upper, s); break;
        default: st = dispatch_head_dim<__nv_bfloat16>(a, tk, tv, head_dim, gc, tensor, pair_upper, s); break;
    }
    if (st != PA_OK || maxP <= 1 || a.merge_count != nullptr) return st;
    switch (dtype) {
        case PA_F32: return launch_reduce<float>(a, head_dim, s);
        case PA_F16: return launch_reduce<__half>(a, head_dim, s);
        default: return launch_reduce<__nv_bfloat16>(a, head_dim, s);
    }
}


pa_status step_compute(const pa_step_device* d, void* k_cache, void* v_cache, const pa_step_shape* sh, void* stream) {
    pa_cache_desc cd{sh->num_blocks, sh->block_size, sh->num_kv_heads, sh->head_dim, sh->dtype};
    pa_status st = PA_OK;
    if (sh->num_cow > 0 && (st = pa_copy_blocks(k_cache, v_cache, d->cow_pairs, sh->num_cow, &cd, stream)) != PA_OK)
        return st;
    return pa_write_decode(d->k, d->v, d->slot_mapping, sh->num_tokens, d->out, d->q, k_cache, v_cache,
                           d->block_tables, d->context_lens, sh->scale, sh->block_size, sh->num_kv_heads,
                           sh->num_seqs, sh->num_heads, sh->head_dim, sh->max_blocks_per_seq, sh->max_context_len,
                           sh->num_blocks, sh->dtype, sh->partition_size, d->workspace, d->workspace_bytes, stream);
}

bool step_inputs(const pa_step_host* h, const pa_step_device* d, const pa_step_shape* sh, cudaStream_t s) {
    const size_t e = elem_bytes(sh->dtype);
    const size_t qbytes = (size_t)sh->num_seqs * sh->num_heads * sh->head_dim * e;
    const size_t kvbytes = (size_t)sh->num_tokens * sh->num_kv_heads * sh->head_dim * e;
    auto h2d = [&](void* dst, const void* src, size_t n) -> bool {
        if (n == 0) return true;
        if (!dst || !src) return false;
        return cudaMemcpyAsync(dst, src, n, cudaMemcpyHostToDevice, s) == cudaSuccess;
    };
    return h2d(d->q, h->q, qbytes) && h2d(d->k, h->k, kvbytes) && h2d(d->v, h->v, kvbytes) &&
           h2d(d->slot_mapping, h->slot_mapping, (size_t)sh->num_tokens * sizeof(int64_t)) &&
           h2d(d->block_tables, h->block_tables, (size_t)sh->num_seqs * sh->max_blocks_per_seq * sizeof(int32_t)) &&
           h2d(d->context_lens, h->context_lens, (size_t)sh->num_seqs * sizeof(int32_t)) &&
           h2d(d->cow_pairs, h->cow_pairs, (size_t)sh->num_cow * 2 * sizeof(int32_t));
}

bool step_output(const pa_step_host* h, const pa_step_device* d, const pa_step_shape* sh, cudaStream_t s) {
    const size_t qbytes = (size_t)sh->num_seqs * sh->num_heads * sh->head_dim * elem_bytes(sh->dtype);
    if (qbytes == 0) return true;
    return h->out && d->out && cudaMemcpyAsync(h->out, d->out, qbytes, cudaMemcpyDeviceToHost, s) == cudaSuccess;
}

bool step_shape_ok(const pa_step_shape* sh) {
    return sh->num_seqs >= 0 && sh->num_tokens >= 0 && sh->num_cow >= 0 && valid_dtype(sh->dtype);
}

}  // namespace

extern "C" {

const char* pa_status_string(pa_status s) {
    switch (s) {
        case PA_OK: return "ok";
        case PA_ERR_INVALID_ARG: return "invalid argument";
        case PA_ERR_UNSUPPORTED: return "unsupported shape or dtype";
        case PA_ERR_NO_BLOCKS: return "no free blocks";
        case PA_ERR_CUDA: return "CUDA error";
        case PA_ERR_DEVICE: return "device-side error flagged";
    }
    return "unknown status";
}

int64_t pa_launch_count(void) { return g_launches.load(); }

pa_status pa_set_decode_math(int mode) {
    if (mode != PA_MATH_AUTO && mode != PA_MATH_SIMT && mode != PA_MATH_TENSOR) return PA_ERR_INVALID_ARG;
    g_decode_math.store(mode);
    return PA_OK;
}

int pa_get_decode_math(void) { return g_decode_math.load(); }

pa_status pa_set_split_merge(int mode) {
    if (mode != PA_MERGE_FUSED && mode != PA_MERGE_KERNEL) return PA_ERR_INVALID_ARG;
    g_split_merge.store(mode);
    return PA_OK;
}

int pa_get_split_merge(void) { return g_split_merge.load(); }

pa_status pa_set_verify_kernel(int kind) {
    if (kind != PA_VERIFY_MMA_SYNC && kind != PA_VERIFY_TCGEN05 && kind != PA_VERIFY_AUTO) return PA_ERR_INVALID_ARG;
    g_verify_kernel.store(kind);
    return PA_OK;
}

int pa_get_verify_kernel(void) { return g_verify_kernel.load(); }

pa_status pa_profile_begin(void) { return pa_profile_begin_mask(0xffffffffu); }

pa_status pa_profile_begin_mask(uint32_t kernel_mask) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_mask = kernel_mask;
    for (auto& r : g_prof_records) {
        g_event_pool.push_back(r.start);
        g_event_pool.push_back(r.stop);
    }
    g_prof_records.clear();
    g_prof_on = true;
    return PA_OK;
}

pa_status pa_profile_end(double* total_ms, int64_t* launches) {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof_on = false;
    for (int k = 0; k < PA_KERNEL_COUNT; ++k) {
        if (total_ms) total_ms[k] = 0.0;
        if (launches) launches[k] = 0;
    }
    pa_status st = PA_OK;
    for (auto& r : g_prof_records) {
        float ms = 0.f;
        if (cudaEventSynchronize(r.stop) != cudaSuccess || cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) {
            st = PA_ERR_CUDA;
        } else if (r.kernel >= 0 && r.kernel < PA_KERNEL_COUNT) {
            if (total_ms) total_ms[r.kernel] += ms;
            if (launches) launches[r.kernel] += 1;
        }
        g_event_pool.push_back(r.start);
        g_event_pool.push_back(r.stop);
    }
    g_prof_records.clear();
    return st;
}

pa_status pa_cache_write(const void* k, const void* v, void* k_cache, void* v_cache, const int64_t* slot_mapping,
                         int num_tokens, const pa_cache_desc* cache, void* stream) {
    pa_dev::WriteArgs w{};
    const pa_status st = write_args(k, v, k_cache, v_cache, slot_mapping, num_tokens, cache, &w);
    if (st != PA_OK || num_tokens == 0) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    LaunchScope scope(PA_KERNEL_CACHE_WRITE, s);
    pa_dev::cache_write_kernel<<<write_grid(w), 256, 0, s>>>(w);
    return launch_status();
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* pairs, int num_pairs, const pa_cache_desc* cache,
                         void* stream) {
    pa_status st = check_cache_desc(cache);
    if (st != PA_OK) return st;
    if (num_pairs < 0) return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!k_cache || !v_cache || !pairs || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    const int64_t block_vecs =
        (int64_t)cache->block_size * cache->num_kv_heads * cache->head_dim * elem_bytes(cache->dtype) / 16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    LaunchScope scope(PA_KERNEL_COPY_BLOCKS, s);
    pa_dev::copy_blocks_kernel<<<dim3((unsigned)num_pairs, 2), 256, 0, s>>>(
        static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), pairs, block_vecs, cache->num_blocks);
    return launch_status();
}

pa_status pa_swap_blocks(void* dst_k, void* dst_v, int dst_blocks, const void* src_k, const void* src_v,
                         int src_blocks, const int32_t* pairs, int num_pairs, const pa_cache_desc* cache,
                         void* stream) {
    if (!cache || cache->num_kv_heads <= 0 || !valid_dtype(cache->dtype)) return PA_ERR_INVALID_ARG;
    if (!supported_block_size(cache->block_size) || !supported_head_dim(cache->head_dim)) return PA_ERR_UNSUPPORTED;
    if (num_pairs < 0 || dst_blocks <= 0 || src_blocks <= 0) return PA_ERR_INVALID_ARG;
    if (num_pairs == 0) return PA_OK;
    if (!dst_k || !dst_v || !src_k || !src_v || !pairs) return PA_ERR_INVALID_ARG;
    if (!aligned16(dst_k) || !aligned16(dst_v) || !aligned16(src_k) || !aligned16(src_v)) return PA_ERR_INVALID_ARG;
    // every pointer must be reachable from the device: device memory or pinned host memory
    const void* ptrs[5] = {dst_k, dst_v, src_k, src_v, pairs};
    void* dptr[5];
    for (int i = 0; i < 5; ++i) {
        cudaPointerAttributes at;
        if (cudaPointerGetAttributes(&at, ptrs[i]) != cudaSuccess) {
            cudaGetLastError();
            return PA_ERR_INVALID_ARG;
        }
        if (at.type == cudaMemoryTypeUnregistered || !at.devicePointer) return PA_ERR_INVALID_ARG;
        dptr[i] = at.devicePointer;      // the address through which kernels reach ptrs[i]
    }
    const int64_t block_vecs =
        (int64_t)cache->block_size * cache->num_kv_heads * cache->head_dim * elem_bytes(cache->dtype) / 16;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    LaunchScope scope(PA_KERNEL_SWAP, s);
    pa_dev::swap_blocks_kernel<<<dim3((unsigned)num_pairs, 2), 256, 0, s>>>(
        static_cast<uint4*>(dptr[0]), static_cast<uint4*>(dptr[1]), dst_blocks, static_cast<const uint4*>(dptr[2]),
        static_cast<const uint4*>(dptr[3]), src_blocks, static_cast<const int32_t*>(dptr[4]), block_vecs);
    return launch_status();
}

size_t pa_decode_workspace_size(int num_seqs, int num_heads, int head_dim, int max_context_len, int partition_size) {
    const int P = resolve_partition(partition_size);
    if (num_seqs <= 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 || !valid_partition(P)) return 0;
    const int64_t maxP = partitions_for(max_context_len, P);
    if (maxP <= 1) return 0;
    return ws_layout(num_seqs, num_heads, head_dim, maxP).total;
}

pa_status pa_decode(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                    const int32_t* context_lens, float scale, int block_size, int num_kv_heads, int num_seqs,
                    int num_heads, int head_dim, int max_blocks_per_seq, int max_context_len, int num_blocks,
                    pa_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes, void* stream) {
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, block_size, num_kv_heads, num_seqs,
                       num_heads, head_dim, max_blocks_per_seq, max_context_len, num_blocks, dtype, partition_size,
                       workspace, workspace_bytes, stream, nullptr);
}

pa_status pa_write_decode(const void* k, const void* v, const int64_t* slot_mapping, int num_tokens, void* out,
                          const void* q, void* k_cache, void* v_cache, const int32_t* block_tables,
                          const int32_t* context_lens, float scale, int block_size, int num_kv_heads, int num_seqs,
                          int num_heads, int head_dim, int max_blocks_per_seq, int max_context_len, int num_blocks,
                          pa_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes, void* stream) {
    const pa_cache_desc cd{num_blocks, block_size, num_kv_heads, head_dim, dtype};
    pa_dev::WriteArgs w{};
    const pa_status st = write_args(k, v, k_cache, v_cache, slot_mapping, num_tokens, &cd, &w);
    if (st != PA_OK) return st;
    return decode_impl(out, q, k_cache, v_cache, block_tables, context_lens, scale, block_size, num_kv_heads, num_seqs,
                       num_heads, head_dim, max_blocks_per_seq, max_context_len, num_blocks, dtype, partition_size,
                       workspace, workspace_bytes, stream, num_tokens > 0 ? &w : nullptr);
}

int pa_verify_partition_size(int num_seqs, int num_queries, int num_heads, int num_kv_heads, int max_context_len,
                             int block_size, int partition_size) {
    if (partition_size != 0) return partition_size;
    if (num_seqs <= 0 || num_queries <= 0 || num_kv_heads <= 0 || num_heads <= 0 || block_size <= 0)
        return kDefaultPartition;
    const int64_t rows = (int64_t)num_heads / num_kv_heads * num_queries;
    const int64_t per_seq = (int64_t)num_kv_heads * ((rows + 63) / 64);
    const int64_t ctx = std::max<int64_t>(1, max_context_len);
    auto items = [&](int64_t P) { return (int64_t)num_seqs * ((ctx + P - 1) / P) * per_seq; };
    // A split partition writes rows x (head_dim + 2) fp32 partials per kv head, which
    // the reduce reads back: at 32 rows or more that is over a tenth of the K/V bytes
    // of a 512-token partition.  There, larger partitions write fewer partials and
    // cross fewer item boundaries, as long as the work still spreads over the grid:
    // about six items per CTA of its 2 x 148 (the bound counts every sequence at the
    // longest context), and, for 2048, enough (sequence, kv head) items without any
    // split.  Their workspace need is below the 512-token one that
    // pa_verify_workspace_size reports for partition_size 0.
    constexpr int64_t kItems = 6 * 2 * 148;
    if (rows < 32) return kDefaultPartition;
    if (block_size >= 16 && num_seqs * per_seq >= 4 * 148 && items(2048) >= kItems) return 2048;
    if (items(1024) >= kItems) return 1024;
    return kDefaultPartition;
}

size_t pa_verify_workspace_size(int num_seqs, int num_queries, int num_heads, int head_dim, int max_context_len,
                                int partition_size) {
    const int P = resolve_partition(partition_size);
    if (num_queries <= 0 || num_seqs <= 0 || num_heads <= 0 || head_dim <= 0 || max_context_len < 0 ||
        !valid_verify_partition_size(P))
        return 0;
    const int64_t maxP = partitions_for(max_context_len, P);
    if (maxP <= 1) return 0;
    return ws_layout(num_seqs, (int64_t)num_queries * num_heads, head_dim, maxP).total;
}

pa_status pa_verify(void* out, const void* q, const void* k_cache, const void* v_cache, const int32_t* block_tables,
                    const int32_t* context_lens, float scale, int block_size, int num_kv_heads, int num_seqs,
                    int num_queries, int num_heads, int head_dim, int max_blocks_per_seq, int max_context_len,
                    int num_blocks, pa_dtype dtype, int partition_size, void* workspace, size_t workspace_bytes,
                    void* stream) {
    if (num_seqs < 0 || num_heads <= 0 || num_kv_heads <= 0 || max_blocks_per_seq <= 0 || num_blocks <= 0 ||
        max_context_len < 0 || !valid_dtype(dtype) || !std::isfinite(scale) || num_queries <= 0)
        return PA_ERR_INVALID_ARG;
    if (num_heads % num_kv_heads != 0) return PA_ERR_INVALID_ARG;
    if (dtype == PA_F32 || num_queries > 64) return PA_ERR_UNSUPPORTED;
    if (!supported_head_dim(head_dim) || !supported_block_size(block_size)) return PA_ERR_UNSUPPORTED;
    const int group = num_heads / num_kv_heads;
    const int rows = group * num_queries;
    const int n_chunks = (rows + 63) / 64;
    const int64_t table_cap0 = (int64_t)max_blocks_per_seq * block_size;
    const int P = pa_verify_partition_size(num_seqs, num_queries, num_heads, num_kv_heads,
                                           (int)std::min<int64_t>(max_context_len, table_cap0), block_size,
                                           partition_size);
    if (!valid_verify_partition(P, block_size)) return PA_ERR_INVALID_ARG;
    if (num_seqs == 0) return PA_OK;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PA_ERR_INVALID_ARG;
    if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache)) return PA_ERR_INVALID_ARG;
    if ((int64_t)num_blocks * block_size > INT32_MAX) return PA_ERR_UNSUPPORTED;
    const int64_t table_cap = (int64_t)max_blocks_per_seq * block_size;
    const int64_t cap = std::min<int64_t>(max_context_len, table_cap);
    if (cap > INT32_MAX / 2) return PA_ERR_INVALID_ARG;
    const int64_t maxP = partitions_for(cap, P);
    if (maxP > kMaxPartitions) return PA_ERR_UNSUPPORTED;
    if ((int64_t)num_seqs * maxP * num_kv_heads * n_chunks > INT32_MAX) return PA_ERR_INVALID_ARG;
    if ((int64_t)num_seqs * num_queries * num_heads > INT32_MAX / 2) return PA_ERR_INVALID_ARG;

    pa_dev::DecodeArgs a{};
    a.out = out;
    a.q = q;
    a.k_cache = k_cache;
    a.v_cache = v_cache;
    a.block_tables = block_tables;
    a.context_lens = context_lens;
    a.scale_log2 = scale * 1.4426950408889634f;
    a.num_seqs = num_seqs;
    a.num_heads = num_heads;
    a.num_kv_heads = num_kv_heads;
    a.group = group;
    a.n_gchunks = n_chunks;
    a.log2_bs = block_size == 8 ? 3 : block_size == 16 ? 4 : 5;
    a.max_blocks_per_seq = max_blocks_per_seq;
    a.ctx_cap = (int)cap;
    a.num_blocks = num_blocks;
    a.partition_size = P;
    a.max_partitions = (int)maxP;
    a.num_queries = num_queries;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (maxP > 1) {
        // partial rows are [num_seqs][Q][num_heads]: the decode layout with Q x num_heads heads
        const WsLayout L = ws_layout(num_seqs, (int64_t)num_queries * num_heads, head_dim, maxP);
        if (!workspace || workspace_bytes < L.total || (reinterpret_cast<uintptr_t>(workspace) & 255u))
            return PA_ERR_INVALID_ARG;
        char* ws = static_cast<char*>(workspace);
        a.plan = reinterpret_cast<const int2*>(ws + L.plan);
        a.plan_count = reinterpret_cast<const int*>(ws + L.count);
        a.split_seqs = reinterpret_cast<const int*>(ws + L.split);
        a.part_m = reinterpret_cast<float*>(ws + L.m);
        a.part_l = reinterpret_cast<float*>(ws + L.l);
        a.part_o = reinterpret_cast<float*>(ws + L.o);
        a.merge_count = nullptr;
        a.work_counter = reinterpret_cast<int*>(ws + L.count) + 2;   // zeroed by the plan kernel
        LaunchScope scope(PA_KERNEL_PLAN, s);
        const int threads = std::min(1024, std::max(32, (num_seqs + 31) / 32 * 32));
        if (launch_dependent(pa_dev::plan_kernel, dim3(1), dim3(threads), 0, s, a,
                             reinterpret_cast<int2*>(ws + L.plan), reinterpret_cast<int*>(ws + L.count),
                             reinterpret_cast<int*>(ws + L.split), reinterpret_cast<int*>(ws + L.counters),
                             0) != PA_OK)
            return PA_ERR_CUDA;
    }
    CUtensorMap tk, tv, tq;
    if (!encode_pool_map(&tk, k_cache, dtype, head_dim, num_kv_heads, num_blocks, block_size, block_size) ||
        !encode_pool_map(&tv, v_cache, dtype, head_dim, num_kv_heads, num_blocks, block_size, block_size))
        return PA_ERR_CUDA;
    const int64_t pair_upper = (int64_t)num_seqs * maxP;
    const int vk = g_verify_kernel.load(std::memory_order_relaxed);
    const bool tc5 = vk != PA_VERIFY_MMA_SYNC;
    // The tcgen05 kernel loads an item's q tile by TMA when its rows are one tile
    // (group x queries <= 64): q as (head_dim, num_heads, num_seqs x num_queries),
    // a box of one 128-byte slice x group heads x num_queries rows.
    std::memset(&tq, 0, sizeof(tq));
    if (tc5 && PA_VERIFY_TC_QTMA && n_chunks == 1 &&
        !encode_q_map(&tq, q, dtype, head_dim, num_heads, num_seqs * num_queries, group, num_queries))
        return PA_ERR_CUDA;
    pa_status st;
    if (dtype == PA_F16) {
        if (tc5)
            st = head_dim == 64 ? launch_verify_tc<__half, 64>(a, tk, tv, tq, pair_upper, s)
                                : launch_verify_tc<__half, 128>(a, tk, tv, tq, pair_upper, s);
        else
            st = head_dim == 64 ? launch_verify<__half, 64>(a, tk, tv, pair_upper, s)
                                : launch_verify<__half, 128>(a, tk, tv, pair_upper, s);
    } else {
        if (tc5)
            st = head_dim == 64 ? launch_verify_tc<__nv_bfloat16, 64>(a, tk, tv, tq, pair_upper, s)
                                : launch_verify_tc<__nv_bfloat16, 128>(a, tk, tv, tq, pair_upper, s);
        else
            st = head_dim == 64 ? launch_verify<__nv_bfloat16, 64>(a, tk, tv, pair_upper, s)
                                : launch_verify<__nv_bfloat16, 128>(a, tk, tv, pair_upper, s);
    }
    if (st != PA_OK || maxP <= 1) return st;
    pa_dev::DecodeArgs r = a;               // the reduce sees rows [s][i][h] as num_queries * num_heads heads
    r.num_heads = num_queries * num_heads;
    return dtype == PA_F16 ? launch_reduce<__half>(r, head_dim, s) : launch_reduce<__nv_bfloat16>(r, head_dim, s);
}

pa_status pa_step(const pa_step_host* h, const pa_step_device* d, void* k_cache, void* v_cache,
                  const pa_step_shape* sh, void* stream) {
    if (!h || !d || !sh || !k_cache || !v_cache || !step_shape_ok(sh)) return PA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (!step_inputs(h, d, sh, s)) return PA_ERR_CUDA;
    pa_status st = step_compute(d, k_cache, v_cache, sh, stream);
    if (st != PA_OK) return st;
    return step_output(h, d, sh, s) ? PA_OK : PA_ERR_CUDA;
}

}  // extern "C"

struct pa_pipeline {
    int depth = 0;
    int device = 0;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    std::vector<cudaEvent_t> staged, computed, drained;   // per staging set
    cudaEvent_t mark = nullptr;
    ~pa_pipeline() {
        for (auto* v : {&staged, &computed, &drained})
            for (cudaEvent_t e : *v)
                if (e) cudaEventDestroy(e);
        if (mark) cudaEventDestroy(mark);
        if (h2d) cudaStreamDestroy(h2d);
        if (d2h) cudaStreamDestroy(d2h);
    }
};


extern "C" {

pa_status pa_pipeline_create(int depth, pa_pipeline** out) {
    if (!out || depth < 1 || depth > 16) return PA_ERR_INVALID_ARG;
    *out = nullptr;
    pa_pipeline* p = new (std::nothrow) pa_pipeline();
    if (!p) return PA_ERR_INVALID_ARG;
    p->depth = depth;
    bool ok = cudaGetDevice(&p->device) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p->h2d, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&p->d2h, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&p->mark, cudaEventDisableTiming) == cudaSuccess;
    for (auto* v : {&p->staged, &p->computed, &p->drained}) {
        v->assign(depth, nullptr);
        for (int i = 0; i < depth && ok; ++i) ok = cudaEventCreateWithFlags(&(*v)[i], cudaEventDisableTiming) == cudaSuccess;
    }
    if (!ok) {
        delete p;
        return PA_ERR_CUDA;
    }
    *out = p;
    return PA_OK;
}

void pa_pipeline_destroy(pa_pipeline* p) { delete p; }

pa_status pa_pipeline_begin(pa_pipeline* p, void* stream) {
    if (!p) return PA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaEventRecord(p->mark, s) != cudaSuccess || cudaStreamWaitEvent(p->h2d, p->mark, 0) != cudaSuccess ||
        cudaStreamWaitEvent(p->d2h, p->mark, 0) != cudaSuccess)
        return PA_ERR_CUDA;
    return PA_OK;
}

pa_status pa_pipeline_step(pa_pipeline* p, int set, const pa_step_host* h, const pa_step_device* d, void* k_cache,
                           void* v_cache, const pa_step_shape* sh, void* stream) {
    if (!p || set < 0 || set >= p->depth || !h || !d || !sh || !k_cache || !v_cache || !step_shape_ok(sh))
        return PA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // inputs: after the previous compute that read this set
    if (cudaStreamWaitEvent(p->h2d, p->computed[set], 0) != cudaSuccess) return PA_ERR_CUDA;
    if (!step_inputs(h, d, sh, p->h2d) || cudaEventRecord(p->staged[set], p->h2d) != cudaSuccess) return PA_ERR_CUDA;
    // compute: after the inputs, and after the previous output copy read this set's `out`
    if (cudaStreamWaitEvent(s, p->staged[set], 0) != cudaSuccess ||
        cudaStreamWaitEvent(s, p->drained[set], 0) != cudaSuccess)
        return PA_ERR_CUDA;
    pa_status st = step_compute(d, k_cache, v_cache, sh, stream);
    if (st != PA_OK) return st;
    if (cudaEventRecord(p->computed[set], s) != cudaSuccess) return PA_ERR_CUDA;
    // output: after the compute
    if (cudaStreamWaitEvent(p->d2h, p->computed[set], 0) != cudaSuccess || !step_output(h, d, sh, p->d2h) ||
        cudaEventRecord(p->drained[set], p->d2h) != cudaSuccess)
        return PA_ERR_CUDA;
    return PA_OK;
}

pa_status pa_pipeline_end(pa_pipeline* p, void* stream) {
    if (!p) return PA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (cudaEventRecord(p->mark, p->h2d) != cudaSuccess || cudaStreamWaitEvent(s, p->mark, 0) != cudaSuccess ||
        cudaEventRecord(p->mark, p->d2h) != cudaSuccess || cudaStreamWaitEvent(s, p->mark, 0) != cudaSuccess)
        return PA_ERR_CUDA;
    return PA_OK;
}

pa_status pa_check_wait_expiry(void* stream) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    pa_dev::wait_expiry_kernel<<<1, 32, 0, s>>>();
    return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

pa_status pa_get_device_error(uint32_t* flags, void* stream) {
    if (!flags) return PA_ERR_INVALID_ARG;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned int v = 0;
    const unsigned int zero = 0;
    if (cudaMemcpyFromSymbolAsync(&v, pa_dev::g_error, sizeof(v), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return PA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
    if (cudaMemcpyToSymbolAsync(pa_dev::g_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
        return PA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess) return PA_ERR_CUDA;
    *flags = v;
    return v ? PA_ERR_DEVICE : PA_OK;
}

}  // extern "C"
