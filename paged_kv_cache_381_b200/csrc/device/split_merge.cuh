// The split-K planning and merge kernels shared by decode and the
// verification pass: plan_kernel orders the (sequence, partition) pairs that
// the attention kernels walk, reduce_kernel merges the partitions of split
// sequences by log-sum-exp.
#pragma once

#include <type_traits>

#include "cache_ops.cuh"
#include "decode.cuh"

namespace pa_dev {

// Orders the (sequence, partition) pairs that the attention kernels walk by
// their token count, longest first, so that each round of the persistent
// grid's walk (walk_next) deals its CTAs items of nearly the same length.  Counts
// are bucketed by 16-token step: a whole partition is bucket P / 16, a
// sequence's last partition the bucket of what is left of it, an empty
// context bucket 0.  One CTA: a histogram of the buckets, a descending scan
// that places them, then one atomic slot reservation per sequence (its whole
// partitions together) and one per last partition.  The order inside a bucket
// does not matter: results never depend on which CTA takes an item.  The plan
// kernel also lists the sequences with more than one partition for the reduce
// and clears the fused-merge counters and the decode kernel's item counter for
// this call.
constexpr int kPlanBuckets = 2048 / 16 + 1;        // partitions of up to 2048 tokens
__device__ __forceinline__ void build_plan(const DecodeArgs& a, int2* plan, int* count, int* split_seqs,
                                           int* merge_count, int num_counters) {
    __shared__ int hist[kPlanBuckets];
    __shared__ int cur[kPlanBuckets];
    __shared__ int nsplit;
    const int tid = threadIdx.x;
    const int P = a.partition_size;
    const int full = P >> 4;                     // bucket of a whole partition
    for (int i = tid; i < kPlanBuckets; i += blockDim.x) hist[i] = 0;
    for (int i = tid; i < num_counters; i += blockDim.x) merge_count[i] = 0;
    if (tid == 0) {
        nsplit = 0;
        count[2] = 0;                            // the counter of dynamically dealt items (decode, verify)
    }
    __syncthreads();
    for (int s = tid; s < a.num_seqs; s += blockDim.x) {
        const int ctx = clamp_context(a, s, true);
        const int np = partitions_of(a, ctx);
        if (np > 1) atomicAdd(&hist[full], np - 1);
        atomicAdd(&hist[(ctx - (np - 1) * P + 15) >> 4], 1);
    }
    __syncthreads();
    // cur[b] = pairs in buckets above b (one warp, descending, carried over chunks of 32)
    if (tid < 32) {
        int carry = 0;
        for (int c0 = 0; c0 <= full; c0 += 32) {
            const int bkt = full - (c0 + tid);
            const int x = bkt >= 0 ? hist[bkt] : 0;
            int incl = x;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                if (tid >= o) incl += y;
            }
            if (bkt >= 0) cur[bkt] = carry + incl - x;
            carry += __shfl_sync(0xffffffffu, incl, 31);
        }
        if (tid == 0) count[0] = carry;
    }
    __syncthreads();
    for (int s = tid; s < a.num_seqs; s += blockDim.x) {
        const int ctx = clamp_context(a, s, false);
        const int np = partitions_of(a, ctx);
        if (np > 1) {
            const int at = atomicAdd(&cur[full], np - 1);
            for (int p = 0; p < np - 1; ++p) plan[at + p] = make_int2(s, p);
            split_seqs[atomicAdd(&nsplit, 1)] = s;
        }
        plan[atomicAdd(&cur[(ctx - (np - 1) * P + 15) >> 4], 1)] = make_int2(s, np - 1);
    }
    __syncthreads();
    if (tid == 0) count[1] = nsplit;
}

__global__ void __launch_bounds__(1024) plan_kernel(const DecodeArgs a, int2* plan, int* count, int* split_seqs,
                                                    int* merge_count, int num_counters) {
    grid_dependency_wait();        // earlier kernels done before the plan and counters are rewritten
    grid_launch_dependents();      // the attention kernel may start its prologue meanwhile
    build_plan(a, plan, count, split_seqs, merge_count, num_counters);
}

// The first kernel of pa_write_decode: blocks [0, write_blocks) append the new
// tokens' K/V (pa_cache_write), block write_blocks builds the plan -- one
// launch instead of two.  Launched after everything before it in the stream;
// the attention kernel launched after it may start early and waits for it to
// complete before reading the cache or the plan.
__global__ void __launch_bounds__(256) write_plan_kernel(const WriteArgs w, int write_blocks, const DecodeArgs a,
                                                         int2* plan, int* count, int* split_seqs, int* merge_count,
                                                         int num_counters) {
    grid_launch_dependents();
    if ((int)blockIdx.x < write_blocks) {
        write_rows(w.k, w.v, w.k_cache, w.v_cache, w.slot_mapping, w.num_tokens, w.row_vecs, w.num_slots,
                   (int64_t)blockIdx.x * blockDim.x + threadIdx.x, (int64_t)write_blocks * blockDim.x);
    } else {
        build_plan(a, plan, count, split_seqs, merge_count, num_counters);
    }
}

// Log-sum-exp merge of a sequence's partitions (base-2 units): with
// M = max_i m_i, w_i = 2^(m_i - M):  out = sum_i w_i o_i / sum_i w_i l_i.
// One warp per (split sequence, query head) -- for the verification pass, per
// (sequence, query row, head) with num_heads = rows x heads.  The split
// sequences are the plan kernel's list of sequences with more than one
// partition, walked by a persistent grid; sequences with one partition were
// finished by the attention kernel.  A row's statistics (lane i holds those of
// partitions i and i + 32) and its first RB partials are all requested before
// any of them is used, then RB partials per round trip to L2, where the
// attention kernel has just left them.  RB = 4 keeps the kernel near 50
// registers, so about five CTAs of eight warps fit an SM and every split row
// of the 70B-shaped batch (5,824) has its own warp: measured on B200, one step
// of that batch took 0.2146 ms with RB = 4, 0.2160 ms with 8 and 0.2181 ms
// with 16.  Partials merge in partition order (the bits do not depend on the
// grid or on RB).
// Partials of a row a lane holds in flight (a build-time knob: more partials per
// round trip against more registers, so fewer warps resident).
#ifndef PA_REDUCE_RB
#define PA_REDUCE_RB 4
#endif
constexpr int kReduceWarps = 8;                   // warps per reduce CTA
template <typename T, int D>
__global__ void __launch_bounds__(kReduceWarps * 32) reduce_kernel(const DecodeArgs a) {
    using Tr = ElemTraits<T>;
    constexpr int PER = D / 32;                   // floats of a partial row per lane
    constexpr int RB = PA_REDUCE_RB;              // partials in flight per lane
    using Vec = typename std::conditional<PER == 4, float4, float2>::type;
    grid_dependency_wait();                       // the plan and the partials must be complete
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t units = (int64_t)a.plan_count[1] * a.num_heads;
    for (int64_t u = (int64_t)blockIdx.x * kReduceWarps + warp; u < units; u += (int64_t)gridDim.x * kReduceWarps) {
        const int k = (int)(u / a.num_heads);
        const int h = (int)(u - (int64_t)k * a.num_heads);
        const int s = a.split_seqs[k];
        const int np = partitions_of(a, clamp_context(a, s, false));
        const int64_t row = (int64_t)s * a.num_heads + h;
        const float* pm = a.part_m + row * a.max_partitions;
        const float* pl = a.part_l + row * a.max_partitions;
        const float* po = a.part_o + row * a.max_partitions * D + lane * PER;
        const float m0 = lane < np ? pm[lane] : -INFINITY;
        const float l0 = lane < np ? pl[lane] : 0.f;
        const float m1 = lane + 32 < np ? pm[lane + 32] : -INFINITY;
        const float l1 = lane + 32 < np ? pl[lane + 32] : 0.f;
        Vec x[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j)
            if (j < np) x[j] = *reinterpret_cast<const Vec*>(po + (int64_t)j * D);
        float M = fmaxf(m0, m1);
        for (int i = lane + 64; i < np; i += 32) M = fmaxf(M, pm[i]);
        M = warp_max(M);
        float L = (lane < np ? exp2f(m0 - M) * l0 : 0.f) + (lane + 32 < np ? exp2f(m1 - M) * l1 : 0.f);
        for (int i = lane + 64; i < np; i += 32) L += exp2f(pm[i] - M) * pl[i];
        L = warp_sum(L);
        float o[PER];
#pragma unroll
        for (int q = 0; q < PER; ++q) o[q] = 0.f;
        // partitions in order; the weight of partition j comes from the lane holding its max
        for (int b = 0; b < np; b += RB) {
            if (b > 0) {
#pragma unroll
                for (int j = 0; j < RB; ++j)
                    if (b + j < np) x[j] = *reinterpret_cast<const Vec*>(po + (int64_t)(b + j) * D);
            }
#pragma unroll
            for (int j = 0; j < RB; ++j) {
                const int i = b + j;
                const float mi = i < 32 ? __shfl_sync(0xffffffffu, m0, i & 31)
                                        : (i < 64 ? __shfl_sync(0xffffffffu, m1, i & 31) : (i < np ? pm[i] : 0.f));
                if (i < np) {
                    const float wgt = exp2f(mi - M);
                    const float* xv = reinterpret_cast<const float*>(&x[j]);
#pragma unroll
                    for (int q = 0; q < PER; ++q) o[q] = fmaf(wgt, xv[q], o[q]);
                }
            }
        }
        T* out = static_cast<T*>(a.out) + row * D + lane * PER;
        // L == 0 only for a verification row that sees no token (context shorter
        // than the query rows): a zero row, as for an empty context
#pragma unroll
        for (int j = 0; j < PER; ++j) out[j] = Tr::from_float(L > 0.f ? o[j] / L : 0.f);
    }
}

}  // namespace pa_dev
