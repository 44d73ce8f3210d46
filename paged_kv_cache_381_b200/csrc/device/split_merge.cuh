// The split-K planning and merge kernels shared by decode and the
// verification pass: plan_kernel orders the (sequence, partition) pairs that
// the attention kernels walk, reduce_kernel merges the partitions of split
// sequences by log-sum-exp.
#pragma once

#include <type_traits>

#include "decode.cuh"

namespace pa_dev {

// Orders (sequence, partition) pairs longest-first: all pairs of the highest
// partition index come first, then the next level, so the full partitions of
// long sequences start early and the short tails fill in at the end.  The
// order inside a level does not matter (results never depend on which CTA
// takes an item).  One CTA: a histogram of partition counts, a suffix scan that
// places the levels, then one atomic slot reservation per pair.  It also clears
// the fused-merge counters for this call.
// Dynamic shared memory: 2 * (max_partitions + 1) ints.
__global__ void __launch_bounds__(1024) plan_kernel(const DecodeArgs a, int2* plan, int* count, int* merge_count,
                                                    int num_counters) {
    extern __shared__ int plan_smem[];
    grid_dependency_wait();        // earlier kernels done before the plan and counters are rewritten
    grid_launch_dependents();      // the decode kernel may start its prologue meanwhile
    const int L = a.max_partitions;
    int* hist = plan_smem;                       // hist[k]: sequences with k partitions, k = 1 .. L
    int* cur = plan_smem + L + 1;                // first plan slot of level p, then its cursor
    __shared__ int warp_tot[32];
    __shared__ int carry;
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int nw = blockDim.x >> 5;
    for (int i = tid; i <= L; i += blockDim.x) hist[i] = 0;
    for (int i = tid; i < num_counters; i += blockDim.x) merge_count[i] = 0;
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int s = tid; s < a.num_seqs; s += blockDim.x)
        atomicAdd(&hist[partitions_of(a, clamp_context(a, s, true))], 1);
    __syncthreads();
    // level p holds the sequences with more than p partitions: size(p) = sum_{k > p} hist[k];
    // cur[p] = sum of size(p') over p' > p.  Scan k = L .. 1 (a running suffix of hist)
    // and levels p = L-1 .. 0 in the same descending pass.
    for (int c0 = 0; c0 < L; c0 += blockDim.x) {
        const int p = L - 1 - (c0 + tid);
        // size(p) = number of sequences with partitions > p, from a suffix scan of hist
        int x = p >= 0 ? hist[p + 1] : 0;
        int incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            if (lane < nw) warp_tot[lane] = t;
        }
        __syncthreads();
        // running suffix count of sequences with > p partitions
        const int size_p = carry + (warp ? warp_tot[warp - 1] : 0) + incl;
        if (p >= 0) cur[p] = size_p;              // sizes first; turned into offsets below
        __syncthreads();
        if (tid == 0) carry += warp_tot[nw - 1];
        __syncthreads();
    }
    // offsets: cur[p] = sum_{p' > p} size(p'), a second descending scan over the sizes
    if (tid == 0) carry = 0;
    __syncthreads();
    for (int c0 = 0; c0 < L; c0 += blockDim.x) {
        const int p = L - 1 - (c0 + tid);
        const int x = p >= 0 ? cur[p] : 0;
        int incl = x;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) warp_tot[warp] = incl;
        __syncthreads();
        if (warp == 0) {
            int t = lane < nw ? warp_tot[lane] : 0;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, t, o);
                if (lane >= o) t += y;
            }
            if (lane < nw) warp_tot[lane] = t;
        }
        __syncthreads();
        if (p >= 0) cur[p] = carry + (warp ? warp_tot[warp - 1] : 0) + incl - x;
        __syncthreads();
        if (tid == 0) carry += warp_tot[nw - 1];
        __syncthreads();
    }
    // level 1 lists every split sequence once, as (s, 1): the reduce walks it
    if (tid == 0) {
        count[1] = L > 1 ? cur[1] : 0;           // its first plan slot
        count[2] = L > 1 ? cur[0] - cur[1] : 0;  // its size: sequences with more than one partition
    }
    __syncthreads();
    for (int s = tid; s < a.num_seqs; s += blockDim.x) {
        const int np = partitions_of(a, clamp_context(a, s, false));
        for (int p = 0; p < np; ++p) plan[atomicAdd(&cur[p], 1)] = make_int2(s, p);
    }
    __syncthreads();
    if (tid == 0) count[0] = carry;
}

// Log-sum-exp merge of a sequence's partitions (base-2 units): with
// M = max_i m_i, w_i = 2^(m_i - M):  out = sum_i w_i o_i / sum_i w_i l_i.
// One warp per (split sequence, query head) -- for the verification pass, per
// (sequence, query row, head) with num_heads = rows x heads.  The split
// sequences come from the plan (its level 1: one (s, 1) entry per sequence with
// more than one partition), walked by a persistent grid; sequences with one
// partition were finished by the attention kernel.  A row's m, l and its first
// RB partials are all requested before the max and sum are formed.
constexpr int kReduceWarps = 8;                   // warps per reduce CTA
template <typename T, int D>
__global__ void __launch_bounds__(kReduceWarps * 32) reduce_kernel(const DecodeArgs a) {
    using Tr = ElemTraits<T>;
    constexpr int PER = D / 32;                   // floats of a partial row per lane
    constexpr int RB = 8;                         // partials in flight per lane
    using Vec = typename std::conditional<PER == 4, float4, float2>::type;
    grid_dependency_wait();                       // the plan and the partials must be complete
    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int split_base = a.plan_count[1];
    const int64_t units = (int64_t)a.plan_count[2] * a.num_heads;
    for (int64_t u = (int64_t)blockIdx.x * kReduceWarps + warp; u < units; u += (int64_t)gridDim.x * kReduceWarps) {
        const int k = (int)(u / a.num_heads);
        const int h = (int)(u - (int64_t)k * a.num_heads);
        const int s = a.plan[split_base + k].x;
        const int np = partitions_of(a, clamp_context(a, s, false));
        const int64_t row = (int64_t)s * a.num_heads + h;
        const float* pm = a.part_m + row * a.max_partitions;
        const float* pl = a.part_l + row * a.max_partitions;
        const float* po = a.part_o + row * a.max_partitions * D + lane * PER;
        Vec x[RB];
        float mb[RB];
#pragma unroll
        for (int j = 0; j < RB; ++j)
            if (j < np) {
                x[j] = *reinterpret_cast<const Vec*>(po + (int64_t)j * D);
                mb[j] = pm[j];
            }
        float M = -INFINITY;
        for (int i = lane; i < np; i += 32) M = fmaxf(M, pm[i]);
        M = warp_max(M);
        float L = 0.f;
        for (int i = lane; i < np; i += 32) L += exp2f(pm[i] - M) * pl[i];
        L = warp_sum(L);
        float o[PER];
#pragma unroll
        for (int j = 0; j < PER; ++j) o[j] = 0.f;
        // partitions in order
        for (int b = 0; b < np; b += RB) {
            if (b > 0) {
#pragma unroll
                for (int j = 0; j < RB; ++j)
                    if (b + j < np) {
                        x[j] = *reinterpret_cast<const Vec*>(po + (int64_t)(b + j) * D);
                        mb[j] = pm[b + j];
                    }
            }
#pragma unroll
            for (int j = 0; j < RB; ++j)
                if (b + j < np) {
                    const float wgt = exp2f(mb[j] - M);
                    const float* xv = reinterpret_cast<const float*>(&x[j]);
#pragma unroll
                    for (int q = 0; q < PER; ++q) o[q] = fmaf(wgt, xv[q], o[q]);
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
