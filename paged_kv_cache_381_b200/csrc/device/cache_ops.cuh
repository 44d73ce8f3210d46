// KV-cache scatter (append new-token rows through the slot mapping) and
// whole-block copy for copy-on-write.
//
// Slot addressing ("大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解"
// 3.2-3.3): a new token goes to the end of the sequence's current block, or to
// a fresh block when the current one is full; the host resolves that to
// slot = block * block_size + offset.  In the pool layout
// [num_blocks, block_size, num_kv_heads, head_dim] the row of one slot (all kv
// heads) is contiguous, and so is a token's row of the new K / V, so each
// token is one contiguous copy of num_kv_heads * head_dim elements.
// Copy-on-write ("vLLM推理加速框架：PagedAttention与连续批处理技术解析" 2.2) copies a
// whole block (block_size * num_kv_heads * head_dim elements) in both pools.
#pragma once

#include "common.cuh"

namespace pa_dev {

// One thread per 16-byte vector of a token row (K and V), strided over the
// threads given (`first` = this thread's first vector, `stride` = all the
// threads' count); many independent loads in flight keep this short work from
// being latency-bound.  row_vecs = 16-byte vectors per token row.
__device__ __forceinline__ void write_rows(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                           uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                                           const int64_t* __restrict__ slot_mapping, int num_tokens, int row_vecs,
                                           int64_t num_slots, int64_t first, int64_t stride) {
    const int64_t total = (int64_t)num_tokens * row_vecs;
    for (int64_t i = first; i < total; i += stride) {
        const int64_t t = i / row_vecs;
        const int64_t j = i - t * row_vecs;
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0) continue;                 // padding token
        if (slot >= num_slots) {
            if (j == 0) flag_error(PA_DEVERR_SLOT);
            continue;
        }
        const uint4 a = __ldg(k + i);
        const uint4 b = __ldg(v + i);
        k_cache[slot * row_vecs + j] = a;
        v_cache[slot * row_vecs + j] = b;
    }
}

// The arguments of one cache write (pa_cache_write; also the first part of
// pa_write_decode's first kernel).
struct WriteArgs {
    const uint4* k;
    const uint4* v;
    uint4* k_cache;
    uint4* v_cache;
    const int64_t* slot_mapping;
    int num_tokens;
    int row_vecs;
    int64_t num_slots;
};

__global__ void __launch_bounds__(256) cache_write_kernel(const WriteArgs w) {
    write_rows(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, w.num_tokens, w.row_vecs, w.num_slots,
               (int64_t)blockIdx.x * blockDim.x + threadIdx.x, (int64_t)gridDim.x * blockDim.x);
}

// grid (num_pairs, 2): blockIdx.y selects the K or V pool.
__global__ void __launch_bounds__(256) copy_blocks_kernel(uint4* __restrict__ k_cache,
                                                          uint4* __restrict__ v_cache,
                                                          const int32_t* __restrict__ pairs,
                                                          int64_t block_vecs, int num_blocks) {
    const int pair = blockIdx.x;
    const int32_t src = pairs[2 * pair];
    const int32_t dst = pairs[2 * pair + 1];
    if (src < 0 || src >= num_blocks || dst < 0 || dst >= num_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0) flag_error(PA_DEVERR_BLOCK_ID);
        return;
    }
    uint4* pool = blockIdx.y == 0 ? k_cache : v_cache;
    const uint4* s = pool + (int64_t)src * block_vecs;
    uint4* d = pool + (int64_t)dst * block_vecs;
    for (int64_t i = threadIdx.x; i < block_vecs; i += blockDim.x) d[i] = s[i];
}

// Swap copies between two pools of the same block shape, either of which may
// be pinned host memory reached over the host link (the kernel reads or writes
// it in place, so one launch moves every block of a swap; many 16-byte
// accesses in flight per thread keep the link busy).  grid (num_pairs, 2):
// blockIdx.y selects the K or V pool; pairs[i] = (source block, destination
// block); ids outside their pool are skipped and flagged.
__global__ void __launch_bounds__(256) swap_blocks_kernel(uint4* __restrict__ dst_k, uint4* __restrict__ dst_v,
                                                          int dst_blocks, const uint4* __restrict__ src_k,
                                                          const uint4* __restrict__ src_v, int src_blocks,
                                                          const int32_t* __restrict__ pairs, int64_t block_vecs) {
    const int pair = blockIdx.x;
    const int32_t src = pairs[2 * pair];
    const int32_t dst = pairs[2 * pair + 1];
    if (src < 0 || src >= src_blocks || dst < 0 || dst >= dst_blocks) {
        if (threadIdx.x == 0 && blockIdx.y == 0) flag_error(PA_DEVERR_BLOCK_ID);
        return;
    }
    const uint4* s = (blockIdx.y == 0 ? src_k : src_v) + (int64_t)src * block_vecs;
    uint4* d = (blockIdx.y == 0 ? dst_k : dst_v) + (int64_t)dst * block_vecs;
    int64_t i = threadIdx.x;
    for (; i + 3 * 256 < block_vecs; i += 4 * 256) {
        const uint4 a = s[i], b = s[i + 256], c = s[i + 512], e = s[i + 768];
        d[i] = a;
        d[i + 256] = b;
        d[i + 512] = c;
        d[i + 768] = e;
    }
    for (; i < block_vecs; i += 256) d[i] = s[i];
}

}  // namespace pa_dev
