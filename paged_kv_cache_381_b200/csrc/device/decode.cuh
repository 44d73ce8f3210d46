// Paged decode attention for sm_100a: single pass, split-K partitions and the
// log-sum-exp merge.
//
// What is computed ("大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
// section "PagedAttention分页注意力机制原理": the kernel resolves every logical block
// through the block table and runs attention over the non-contiguous physical
// blocks; "vLLM推理加速框架：PagedAttention与连续批处理技术解析" 2.2: the kernel works
// block by block; 6.2: out, q, k, v, block_tables): for sequence s, query
// head h and kv head g = h / group,
//     out[s][h] = sum_t softmax_t(scale * q[s][h] . K_s[t][g]) V_s[t][g].
//
// Design (B200):
//  * Work item = (sequence, context partition, kv head, query-head chunk).  A
//    CTA handles all query heads of a kv-head group that share the K/V rows it
//    streams, so each K/V byte leaves HBM once.  Contexts longer than the
//    partition size are split.  A planning kernel sorts the items by length,
//    longest first, and a persistent grid (a multiple of the SM count) walks
//    them with a fixed stride (walk_first / walk_next): every round of the
//    grid then takes items of nearly the same length.  The last rounds (the
//    shortest items) are dealt one at a time from an atomic counter, so CTAs
//    that ran faster absorb the tail.
//  * One producer warp looks items up one ahead of their use, publishes each
//    item's descriptor and q rows (one bulk copy) to the consumers through a
//    double-buffered shared-memory slot (an end-of-items slot closes the
//    sequence), resolves block ids through the block
//    table and issues tiled TMA loads into a ring of shared-memory stages of 32
//    token rows, each stage completed on an mbarrier with transaction counts.
//    The pool is seen by the TMA unit as a 3-D tensor [num_blocks * block_size
//    rows][num_kv_heads][head_dim]; one box is the block_size rows of one kv
//    head and one 128-byte slice of head_dim, so a 16-token block of a
//    128-wide bf16 head arrives in two 2 KiB loads (per-row 256-byte bulk
//    copies were measured to cap a producer warp near 7 GB/s).  Boxes land
//    with the 128-byte swizzle (16-byte chunk index XOR row % 8), which keeps
//    8-row ldmatrix and 16-byte vector reads free of bank conflicts; consumers
//    apply the same XOR when they address a row.
//  * Four consumer warps.  Tensor path (fp16 / bf16): phase 1 splits the K
//    stages over the warps and writes the scaled scores of every token of the
//    partition to shared memory with a running max; phase 2 gives each warp a
//    quarter of head_dim over every V stage, so each warp finishes its own
//    output columns (and the whole softmax denominator) without a cross-warp
//    reduction.  CUDA-core path (fp32, or on request): phase 1 as above with
//    16-byte vector reads, fp32 FMAs and a transposing butterfly that reduces
//    G partial dot products over the lanes of a row; phase 2 takes the exact
//    max, exponentials and their sum; phase 3 accumulates p * V per warp over
//    its stages, and an epilogue merges the warps in a fixed order.  Either
//    path writes the normalised row (one partition) or the partition's
//    unnormalised output, max and sum.
//  * Every reduction order depends only on logical token positions, so the
//    result is bitwise independent of the physical placement of blocks.
//  * All waits are bounded: on expiry the CTA records PA_DEVERR_TIMEOUT and
//    runs through its remaining work without touching the stages.
#pragma once

#include "common.cuh"

namespace pa_dev {

struct DecodeArgs {
    void* out;
    const void* q;
    const void* k_cache;
    const void* v_cache;
    const int32_t* block_tables;
    const int32_t* context_lens;
    float scale_log2;          // softmax scale * log2(e)
    int num_seqs;
    int num_heads;
    int num_kv_heads;
    int group;                 // num_heads / num_kv_heads
    int n_gchunks;             // query-head chunks per kv head
    int log2_bs;
    int max_blocks_per_seq;
    int ctx_cap;               // min(max_context_len, max_blocks_per_seq * block_size)
    int num_blocks;
    int partition_size;        // tokens per partition (multiple of 32)
    int max_partitions;        // 1: single pass, no plan / partials
    const int2* plan;          // split mode: (seq, partition), longest first
    const int* plan_count;     // [0]: pairs in the plan, [1]: split sequences
    const int* split_seqs;     // split mode: the sequences with more than one partition
    float* part_m;             // [num_seqs * num_heads, max_partitions] (log2 units)
    float* part_l;             // [num_seqs * num_heads, max_partitions]
    float* part_o;             // [num_seqs * num_heads, max_partitions, head_dim]
    int* merge_count;          // split mode, fused merge: finished partitions per (seq, kv head, chunk);
                               // nullptr: partitions are merged by reduce_kernel instead
    int* work_counter;         // split mode (decode, tcgen05 verification): items of the plan's tail handed
                               // out so far (zeroed by the plan kernel); nullptr: every item by the stride
    int num_queries;           // query rows per sequence and head (1: decode; > 1: verification pass)
};

struct WorkItem {
    int s, p, h, gc, t0, n, np;
};

__device__ __forceinline__ int clamp_context(const DecodeArgs& a, int s, bool report) {
    int c = a.context_lens[s];
    if (c < 0 || c > a.ctx_cap) {
        if (report) flag_error(PA_DEVERR_CONTEXT_LEN);
        c = c < 0 ? 0 : a.ctx_cap;
    }
    return c;
}

__device__ __forceinline__ int partitions_of(const DecodeArgs& a, int ctx) {
    return ctx == 0 ? 1 : (ctx + a.partition_size - 1) / a.partition_size;
}

// (sequence, partition) of a pair index: the plan's entry in split mode, the
// sequence itself in single-pass mode.
__device__ __forceinline__ int2 pair_at(const DecodeArgs& a, int pair) {
    return a.max_partitions == 1 ? make_int2(pair, 0) : a.plan[pair];
}

__device__ __forceinline__ WorkItem decode_item(const DecodeArgs& a, int i, bool report) {
    const int per = a.num_kv_heads * a.n_gchunks;
    const int pair = i / per;
    const int rem = i - pair * per;
    WorkItem w;
    w.h = rem / a.n_gchunks;
    w.gc = rem - w.h * a.n_gchunks;
    const int2 e = pair_at(a, pair);
    w.s = e.x;
    w.p = e.y;
    const int ctx = clamp_context(a, w.s, report);
    w.np = partitions_of(a, ctx);
    w.t0 = w.p * a.partition_size;
    w.n = min(max(ctx - w.t0, 0), a.partition_size);
    return w;
}

// The items a CTA of the persistent grid takes.  Round r covers items
// [r * G, (r + 1) * G) with G = gridDim.x; CTA c takes item r * G + c (a fixed
// stride), or, in snake order, r * G + c in even rounds and r * G + G - 1 - c
// in odd rounds.  With the plan sorted longest first, every round holds items
// of nearly the same length.  The sequence of items is increasing, so a walk
// ends at the first index past the total.
// Measured on B200 (70B-shaped batch, one box, two rounds each): the fixed
// stride over the length-sorted plan gave 194.5 us per decode launch against
// 196.6 us in snake order, although a model of per-CTA item lengths favours the
// snake order; PA_DECODE_SNAKE=1 (a build-time knob) walks in snake order.
#ifndef PA_DECODE_SNAKE
#define PA_DECODE_SNAKE 0
#endif
__device__ __forceinline__ int walk_first() { return (int)blockIdx.x; }

__device__ __forceinline__ int walk_next(int i) {
    const int64_t G = gridDim.x;
#if PA_DECODE_SNAKE
    const int64_t r = i / G + 1;
    const int64_t n = r * G + ((r & 1) ? G - 1 - (int64_t)blockIdx.x : (int64_t)blockIdx.x);
#else
    const int64_t n = (int64_t)i + G;
#endif
    return n > 0x7fffffff ? 0x7fffffff : (int)n;
}

// The decode kernel deals the last PA_DECODE_DYN_ROUNDS rounds of the sorted
// plan (its shortest items) dynamically: a CTA that runs out of its own items
// takes the next one from an atomic counter, so CTAs that ran faster absorb the
// tail.  0: every item by the fixed stride.  Measured on B200 (70B / 7B /
// long-context batches, two runs each): 0 rounds 194.8 / 195.1 / - us, 3 rounds
// 189.0 / 190.2 / 186.5 us, 6 rounds 190.1 / 190.9 / 188.8 us, every item
// dynamic 192.2 / 192.5 / 189.1 us.
#ifndef PA_DECODE_DYN_ROUNDS
#define PA_DECODE_DYN_ROUNDS 3
#endif

// Named barrier `id` over `threads` threads (a multiple of 32) that also returns
// the AND of every participating thread's `pred`: one answer for all of them.
__device__ __forceinline__ bool barrier_and(int id, int threads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.cta.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(threads)
        : "memory");
    return r != 0;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Reduce GC partial dot products held by each of the LPT lanes of a row.  Each
// halving step trades half of the values with the partner lane, so after the
// loop lane c of the row holds the complete sum for query c / (LPT / GC).
template <int GC, int LPT>
__device__ __forceinline__ float reduce_row_dots(float (&v)[GC], int lane) {
    constexpr int STEPS = ilog2(LPT);
#pragma unroll
    for (int step = 0; step < STEPS; ++step) {
        const int o = LPT >> (step + 1);
        const int n = GC >> step;
        if (n >= 2) {
            const int h = n >> 1;
            const bool upper = (lane & o) != 0;
#pragma unroll
            for (int i = 0; i < GC / 2; ++i) {
                if (i < h) {
                    const float send = upper ? v[i] : v[i + h];
                    const float keep = upper ? v[i + h] : v[i];
                    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, o);
                }
            }
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], o);
        }
    }
    return v[0];
}

// Merge the partitions of one (sequence, kv head, query chunk) in partition
// order: M = max_i m_i, out = sum_i 2^(m_i - M) o_i / sum_i 2^(m_i - M) l_i.
// Called by the CTA that finished the last of them, after a fence; reads the
// partials from L2.  Uses `stat_m` / `stat_l` (>= gq floats of shared memory)
// and named barrier 1 over the ncw consumer warps.
template <typename T, int D>
__device__ __forceinline__ void merge_partitions(const DecodeArgs& a, int64_t row0, int gq, int np, float* stat_m,
                                                 float* stat_l, int warp, int lane, int ctid, int ncw) {
    using Tr = ElemTraits<T>;
    T* outg = static_cast<T*>(a.out);
    for (int g = warp; g < gq; g += ncw) {       // one warp per query, lanes over partitions
        const float* pm = a.part_m + (row0 + g) * a.max_partitions;
        const float* pl = a.part_l + (row0 + g) * a.max_partitions;
        float M = -INFINITY;
        for (int i = lane; i < np; i += 32) M = fmaxf(M, __ldcg(pm + i));
        M = warp_max(M);
        float L = 0.f;
        for (int i = lane; i < np; i += 32) L += exp2f(__ldcg(pm + i) - M) * __ldcg(pl + i);
        L = warp_sum(L);
        if (lane == 0) {
            stat_m[g] = M;
            stat_l[g] = L;
        }
    }
    named_barrier(1, ncw * 32);
    // four consecutive head-dim elements per thread and step
    for (int e = ctid * 4; e < gq * D; e += ncw * 32 * 4) {
        const int g = e / D;
        const int d = e - g * D;
        const int64_t base = (row0 + g) * a.max_partitions;
        const float Mg = stat_m[g];
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        int i = 0;
        for (; i + 8 <= np; i += 8) {
            float4 x[8];
            float wt[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                x[j] = __ldcg(reinterpret_cast<const float4*>(a.part_o + (base + i + j) * D + d));
                wt[j] = exp2f(__ldcg(a.part_m + base + i + j) - Mg);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                o.x = fmaf(wt[j], x[j].x, o.x);
                o.y = fmaf(wt[j], x[j].y, o.y);
                o.z = fmaf(wt[j], x[j].z, o.z);
                o.w = fmaf(wt[j], x[j].w, o.w);
            }
        }
        for (; i < np; ++i) {
            const float4 xv = __ldcg(reinterpret_cast<const float4*>(a.part_o + (base + i) * D + d));
            const float wt = exp2f(__ldcg(a.part_m + base + i) - Mg);
            o.x = fmaf(wt, xv.x, o.x);
            o.y = fmaf(wt, xv.y, o.y);
            o.z = fmaf(wt, xv.z, o.z);
            o.w = fmaf(wt, xv.w, o.w);
        }
        const float Lg = stat_l[g];
        T* dst = outg + (row0 + g) * D + d;
        dst[0] = Tr::from_float(o.x / Lg);
        dst[1] = Tr::from_float(o.y / Lg);
        dst[2] = Tr::from_float(o.z / Lg);
        dst[3] = Tr::from_float(o.w / Lg);
    }
}

// Ring depth (stages of 32 token rows) and the CTAs per SM the launch bounds
// aim for (tensor-core path; the CUDA-core path holds more registers and aims
// for 2); build-time tuning knobs.  Measured on B200 (70B-shaped batch): 4
// stages at 4 CTAs per SM beat 8 stages at 2 (more independent items per SM
// hide the per-item phase barriers of short sequences).
#ifndef PA_DECODE_STAGES
#define PA_DECODE_STAGES 4
#endif
#ifndef PA_DECODE_BOX_BLOCK
// 1: one TMA box brings a whole block of one kv head (every 128-byte head_dim
// slice, through a 4-D view of the pool); 0: one box per (block, slice).
// Measured on B200 (two runs each): 188.75 vs 189.3 us per 70B-shaped launch,
// 189.65 vs 190.4 us (7B), 185.4 vs 186.4 us (long contexts).
#define PA_DECODE_BOX_BLOCK 1
#endif
#ifndef PA_DECODE_MIN_CTAS
#define PA_DECODE_MIN_CTAS 4
#endif

template <typename T, int D, int GC, bool TENSOR>
struct DecodeCfg {
    using Tr = ElemTraits<T>;
    static constexpr int ELT = (int)sizeof(T);
    static constexpr int VEC = Tr::VEC;             // elements per 16-byte vector
    static constexpr int LPT = D / VEC;             // lanes per token row (SIMT path)
    static constexpr int RPI = 32 / LPT;            // rows per warp instruction (SIMT path)
    static constexpr int ROW_BYTES = D * ELT;
    static constexpr int NH = ROW_BYTES / 128;      // 128-byte slices of a row (one TMA box each)
    static constexpr int BOX_ELEMS = 128 / ELT;     // head_dim elements per slice
    static constexpr int STAGE_ROWS = 32;
    static constexpr int STAGE_BYTES = STAGE_ROWS * ROW_BYTES;
    static constexpr int NSTAGES = PA_DECODE_STAGES;
    static constexpr int NCW = 4;                   // consumer warps
    static constexpr int THREADS = (NCW + 1) * 32;
    static constexpr int MAX_PARTITION = 1024;
    static constexpr int MAX_TABLE = MAX_PARTITION / 8;
    static constexpr int TPL = MAX_TABLE / 32;      // block-table entries per producer lane
    // Tensor path: every consumer warp reads every stage (phase 1 work goes to
    // one warp per stage, phase 2 work to all four), and a stage is free once
    // all four have released it.  CUDA-core path: each stage belongs to one warp.
    static constexpr int EMPTY_ARRIVALS = TENSOR ? NCW : 1;
    // scores row stride (floats): the tensor path reads 8-query rows as pairs;
    // the SIMT path pads to GC + 1 so per-query column walks avoid bank conflicts
    static constexpr int LSTRIDE = TENSOR ? GC : (GC == 1 ? 1 : GC + 1);
    static constexpr int Q_BYTES = GC * ROW_BYTES;  // one item's q rows
    static constexpr int OFF_FULL = NSTAGES * STAGE_BYTES;   // ring at a 1024-byte aligned base
    static constexpr int OFF_EMPTY = OFF_FULL + NSTAGES * 8;
    static constexpr int OFF_IFULL = OFF_EMPTY + NSTAGES * 8;    // item slot filled (descriptor + q)
    static constexpr int OFF_IEMPTY = OFF_IFULL + 2 * 8;         // item slot read by every consumer warp
    static constexpr int OFF_INFO = OFF_IEMPTY + 2 * 8;          // two WorkItem descriptors, 8 ints each
    static constexpr int OFF_TABLE = OFF_INFO + 2 * 32;
    static constexpr int OFF_QBUF = (OFF_TABLE + MAX_TABLE * 4 + 127) / 128 * 128;   // two q tiles
    static constexpr int OFF_STATS = OFF_QBUF + 2 * Q_BYTES;    // wmax, wsum [NCW][GC], m, l [GC], flags
    static constexpr int STATS_FLOATS = 2 * NCW * GC + 2 * GC + 4;
    // The scores (phases 1-3) and, on the CUDA-core path, the warps' output
    // partials (epilogue) share one region: a barrier separates the last score
    // read from the first partial write.
    static constexpr int OFF_LOGITS = ((OFF_STATS + STATS_FLOATS * 4) + 127) / 128 * 128;
    static constexpr int OFF_RED = OFF_LOGITS;
    static constexpr int RED_BYTES = TENSOR ? 0 : NCW * GC * D * 4;
    static_assert(TENSOR ? (GC == 8 && ELT == 2 && (D / 16) % NCW == 0) : (GC <= LPT), "unsupported query chunk");
    static_assert(LPT >= 1 && LPT <= 32 && (32 % LPT) == 0, "row must span a divisor of the warp");
    static_assert(ROW_BYTES % 128 == 0 && STAGE_BYTES % 1024 == 0, "swizzled boxes need 1024-byte alignment");
    static_assert(Q_BYTES % 16 == 0 && OFF_QBUF % 16 == 0, "bulk copies need 16-byte sizes and addresses");
    // CUDA-core path: consumer warp w takes the stages st = w, w + NCW, ... of
    // a phase, and a ring slot is reused every NSTAGES stages.  Only when
    // NSTAGES is a multiple of NCW does one warp own every use of a slot within
    // a phase; otherwise a warp could test a slot's full barrier for its next
    // use while the previous use (another warp's) is still in flight, and the
    // parity test would answer "complete" for the wrong phase.  (On the tensor
    // path every warp waits on every stage in order, which is safe at any
    // depth; the same rule is kept for both.)
    static_assert(NSTAGES % NCW == 0, "ring depth must be a multiple of the consumer warps");
    // + 1024: the dynamic shared-memory base is rounded up to 1024 bytes in the kernel
    static size_t smem_bytes(int partition) {
        const size_t scores = (size_t)partition * LSTRIDE * 4;
        return 1024 + (size_t)OFF_LOGITS + (scores > (size_t)RED_BYTES ? scores : (size_t)RED_BYTES);
    }
};

// Tensor path (fp16 / bf16), per warp and per 16-token tile, with G <= 8
// queries of one kv head padded to the n = 8 of mma.m16n8k16:
//   scores   S^T[16 tok x 8 q]  = K[16 x D] . Q^T[D x 8]    (A = K via ldmatrix, B = q in registers)
//   output   O^T[D x 8 q]      += V^T[D x 16 tok] . P^T[16 tok x 8 q]
//                                                (A = V via ldmatrix.trans, B = p built in registers,
//                                                 p split into a 16-bit value and its remainder)
// Fragment layouts (PTX m16n8k16): A regs {rows 0-7 | 8-15} x {cols 0-7 | 8-15},
// B reg0 = (k = 2*tig, 2*tig+1; n = gid), reg1 = same k + 8, C = (gid | gid+8, 2*tig | 2*tig+1),
// where gid = lane / 4 and tig = lane % 4.
template <typename T, int D, int GC, bool TENSOR>
__global__ void __launch_bounds__(DecodeCfg<T, D, GC, TENSOR>::THREADS, TENSOR ? PA_DECODE_MIN_CTAS : 2)
    decode_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v) {
    using C = DecodeCfg<T, D, GC, TENSOR>;
    using Tr = ElemTraits<T>;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_FULL);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + C::OFF_EMPTY);
    uint64_t* item_full = reinterpret_cast<uint64_t*>(smem + C::OFF_IFULL);
    uint64_t* item_empty = reinterpret_cast<uint64_t*>(smem + C::OFF_IEMPTY);
    int* info = reinterpret_cast<int*>(smem + C::OFF_INFO);           // [2][8]
    int32_t* tbl = reinterpret_cast<int32_t*>(smem + C::OFF_TABLE);
    unsigned char* qbuf = smem + C::OFF_QBUF;                          // [2][GC][D] elements
    float* wmax = reinterpret_cast<float*>(smem + C::OFF_STATS);   // [NCW][GC]
    float* wsum = wmax + C::NCW * GC;                                // [NCW][GC]
    float* stat_m = wsum + C::NCW * GC;                              // [GC]
    float* stat_l = stat_m + GC;                                     // [GC]
    volatile int* abort_flag = reinterpret_cast<volatile int*>(stat_l + GC);
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    float* logits = reinterpret_cast<float*>(smem + C::OFF_LOGITS);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NSTAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], C::EMPTY_ARRIVALS);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&item_full[i], 1);
            mbar_init(&item_empty[i], C::NCW);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    // launched as a programmatic dependent of the plan kernel (or of whatever
    // precedes it): nothing written by earlier kernels is read before this
    grid_dependency_wait();
    const int pairs = a.max_partitions == 1 ? a.num_seqs : a.plan_count[0];
    const int total = pairs * a.num_kv_heads * a.n_gchunks;
    const int bs = 1 << a.log2_bs;
    const int box_bytes = bs * 128;
    // byte offset, within a stage, of 16-byte chunk c of stage row r
    auto row_base = [&](int r) -> int {
        return ((r >> a.log2_bs) * C::NH) * box_bytes + (r & (bs - 1)) * 128;
    };
    auto chunk_off = [&](int r, int c) -> int {
        return row_base(r) + (c >> 3) * box_bytes + (((c & 7) ^ (r & 7)) << 4);
    };

    if (warp == C::NCW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmap_k);
            prefetch_tmap(&tmap_v);
        }
        const uint64_t policy = l2_policy_evict_first();
        const T* qg = static_cast<const T*>(a.q);
        // Block ids of an item, requested into registers (lane j holds entries
        // j, j + 32, ...) one item before they are needed; rows of the table
        // past the item's blocks are not read.
        auto request_ids = [&](const WorkItem& w, int32_t (&ids)[C::TPL]) {
            const int nblk = (w.n + bs - 1) >> a.log2_bs;
            const int32_t* trow = a.block_tables + (int64_t)w.s * a.max_blocks_per_seq + (w.t0 >> a.log2_bs);
#pragma unroll
            for (int k = 0; k < C::TPL; ++k) {
                const int j = lane + 32 * k;
                ids[k] = j < nblk ? trow[j] : 0;
            }
        };
        // Items below dyn_start follow the fixed stride; the rest are handed out
        // one at a time by the atomic counter (lane 0 takes, the warp shares).
        const int dyn_start = a.work_counter ? max(0, total - PA_DECODE_DYN_ROUNDS * (int)gridDim.x) : total;
        auto take_dynamic = [&]() -> int {
            int d = 0;
            if (lane == 0) d = atomicAdd(a.work_counter, 1);
            d = __shfl_sync(0xffffffffu, d, 0);
            return d >= total - dyn_start ? total : dyn_start + d;
        };
        auto next_item = [&](int cur) -> int {
            const int nx = walk_next(cur);
            return nx < dyn_start ? nx : (dyn_start < total ? take_dynamic() : total);
        };
        uint32_t stage = 0;
        uint32_t k = 0;                                   // items published
        bool ok = true;
        int i = walk_first();
        if (i >= dyn_start) i = dyn_start < total ? take_dynamic() : total;
        WorkItem w{};
        int32_t ids[C::TPL];
        if (i < total) {
            w = decode_item(a, i, lane == 0);
            request_ids(w, ids);
        }
        for (; i < total && ok; ++k) {
            // publish the item: descriptor, then its q rows by one bulk copy
            const int b = k & 1;
            if (!mbar_wait_warp(&item_empty[b], ((k >> 1) & 1u) ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            if (lane == 0) {
                int* dst = info + b * 8;
                dst[7] = 1;                   // an item (0: no more items)
                dst[0] = w.s;
                dst[1] = w.p;
                dst[2] = w.h;
                dst[3] = w.gc;
                dst[4] = w.t0;
                dst[5] = w.n;
                dst[6] = w.np;
                if (w.n > 0) {
                    const int gq = min(GC, a.group - w.gc * GC);
                    const int64_t row0 = (int64_t)w.s * a.num_heads + w.h * a.group + w.gc * GC;
                    mbar_arrive_expect_tx(&item_full[b], (uint32_t)(gq * C::ROW_BYTES));
                    bulk_copy_g2s(qbuf + b * C::Q_BYTES, qg + row0 * D, (uint32_t)(gq * C::ROW_BYTES),
                                  &item_full[b]);
                } else {
                    mbar_arrive(&item_full[b]);
                }
            }
            // look the next item up while this item's stages wait for ring slots
            const int inext = next_item(i);
            WorkItem wn{};
            int32_t idn[C::TPL];
            if (inext < total) {
                wn = decode_item(a, inext, lane == 0);
                request_ids(wn, idn);
            }
            if (w.n > 0) {
                const int nst = (w.n + C::STAGE_ROWS - 1) / C::STAGE_ROWS;
                const int nblk = (w.n + bs - 1) >> a.log2_bs;
                __syncwarp();                 // the previous item's table reads are done
#pragma unroll
                for (int kk = 0; kk < C::TPL; ++kk) {
                    const int j = lane + 32 * kk;
                    if (j < nblk) {
                        int32_t id = ids[kk];
                        if (id < 0 || id >= a.num_blocks) {
                            flag_error(PA_DEVERR_BLOCK_ID);
                            id = 0;
                        }
                        tbl[j] = id;
                    }
                }
                __syncwarp();
                for (int pass = 0; pass < 2 && ok; ++pass) {
                    const void* tmap = pass ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k);
                    for (int st = 0; st < nst; ++st, ++stage) {
                        const int slot = stage % C::NSTAGES;
                        const uint32_t parity = ((stage / C::NSTAGES) & 1u) ^ 1u;
                        if (!mbar_wait_warp(&empty[slot], parity, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const int rows = min(C::STAGE_ROWS, w.n - st * C::STAGE_ROWS);
                        const int nblk_st = (rows + bs - 1) >> a.log2_bs;      // whole blocks are loaded
                        const int nbox = nblk_st * C::NH;
                        if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)(nbox * box_bytes));
                        __syncwarp();
#if PA_DECODE_BOX_BLOCK
                        if (lane < nblk_st) {
                            // the block's slices land one after another: [slice][bs rows]
                            const int phys = tbl[((st * C::STAGE_ROWS) >> a.log2_bs) + lane];
                            tma_load_4d(smem + slot * C::STAGE_BYTES + lane * C::NH * box_bytes, tmap, 0, phys * bs,
                                        0, w.h, &full[slot], policy);
                        }
#else
                        if (lane < nbox) {
                            const int bb = lane / C::NH;
                            const int half = lane - bb * C::NH;
                            const int phys = tbl[((st * C::STAGE_ROWS) >> a.log2_bs) + bb];
                            tma_load_3d(smem + slot * C::STAGE_BYTES + (bb * C::NH + half) * box_bytes, tmap,
                                        half * C::BOX_ELEMS, w.h, phys * bs, &full[slot], policy);
                        }
#endif
                    }
                }
            }
            i = inext;
            w = wn;
#pragma unroll
            for (int kk = 0; kk < C::TPL; ++kk) ids[kk] = idn[kk];
        }
        if (ok) {
            // no more items: the closing slot tells the consumers to stop
            const int b = k & 1;
            if (mbar_wait_warp(&item_empty[b], ((k >> 1) & 1u) ^ 1u, abort_flag)) {
                if (lane == 0) {
                    info[b * 8 + 7] = 0;
                    mbar_arrive(&item_full[b]);
                }
                ++k;
            } else {
                ok = false;
            }
        }
        if (!ok) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            // let copies already issued land before the CTA can retire: every
            // stage issued, and the q copy of every item published
            const volatile int never = 0;
            const uint32_t issued = stage;
            for (int slot = lane; slot < C::NSTAGES; slot += 32) {
                if ((uint32_t)slot < issued) {
                    const uint32_t last = issued - 1 - ((issued - 1 - slot) % C::NSTAGES);
                    mbar_wait(&full[slot], (last / C::NSTAGES) & 1u, &never);
                }
            }
            for (int b = lane; b < 2; b += 32) {
                if ((uint32_t)b < k) {
                    const uint32_t last = k - 1 - ((k - 1 - b) & 1u);
                    mbar_wait(&item_full[b], (last >> 1) & 1u, &never);
                }
            }
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    constexpr int NCT = C::NCW * 32;
    const int ctid = threadIdx.x;
    T* outg = static_cast<T*>(a.out);
    uint32_t stage = 0;

    // Wait for a stage; false once the CTA has given up.  The answer is the
    // same for every lane of the warp (the lanes poll on their own, and the
    // warp-wide matrix instructions that follow need all of them).
    auto acquire = [&](uint32_t c) -> bool {
        if (!mbar_wait_warp(&full[c % C::NSTAGES], (c / C::NSTAGES) & 1u, abort_flag)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };
    auto release = [&](uint32_t c) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[c % C::NSTAGES]);
    };

    // Items in the order the producer publishes them, until its closing slot.
    // Whether the slot arrived is agreed by all four warps in one barrier
    // reduction, so that a wait giving up in one warp only cannot leave the
    // others at a named barrier of an item it will not take.
    for (uint32_t k = 0;; ++k) {
        const int b = k & 1;
        const bool got = mbar_wait(&item_full[b], (k >> 1) & 1u, abort_flag);
        if (!barrier_and(2, NCT, got)) {
            *abort_flag = 1;
            break;
        }
        const int* src = info + b * 8;
        if (src[7] == 0) break;                       // no more items
        WorkItem w;
        w.s = src[0];
        w.p = src[1];
        w.h = src[2];
        w.gc = src[3];
        w.t0 = src[4];
        w.n = src[5];
        w.np = src[6];
        const bool have_q = true;
        const int gq = min(GC, a.group - w.gc * GC);
        const int hq0 = w.h * a.group + w.gc * GC;
        const int64_t row0 = (int64_t)w.s * a.num_heads + hq0;
        const unsigned char* qs = qbuf + b * C::Q_BYTES;
        if (w.n == 0) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&item_empty[b]);
            for (int e = ctid; e < gq * D; e += NCT) outg[row0 * D + e] = Tr::from_float(0.f);
            continue;
        }
        const int nst = (w.n + C::STAGE_ROWS - 1) / C::STAGE_ROWS;

        if constexpr (TENSOR) {
            using M = MmaOps<T>;
            constexpr int KS = D / 16;                 // k-steps over head_dim
            constexpr int DMW = KS / C::NCW;           // 16-wide head_dim tiles per warp in phase 2
            const int gid = lane >> 2;
            const int tig = lane & 3;
            // ---- q as B fragments, from the item's tile (rows past the chunk are zero)
            uint32_t qb[KS][2];
#pragma unroll
            for (int kk = 0; kk < KS; ++kk) {
                if (have_q && gid < gq) {
                    const unsigned char* qrow = qs + gid * C::ROW_BYTES + (kk * 16 + tig * 2) * C::ELT;
                    qb[kk][0] = *reinterpret_cast<const uint32_t*>(qrow);
                    qb[kk][1] = *reinterpret_cast<const uint32_t*>(qrow + 8 * C::ELT);
                } else {
                    qb[kk][0] = qb[kk][1] = 0u;
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&item_empty[b]);
            // ---- phase 1: S^T tiles of the warp's stages, scaled to base-2 units, with a running max
            float mlo = -INFINITY, mhi = -INFINITY;      // queries 2*tig, 2*tig+1
            for (int st = 0; st < nst; ++st) {
                const uint32_t c = stage + st;
                if (!acquire(c)) continue;
                if ((st & (C::NCW - 1)) == warp) {
                    const int rows = min(C::STAGE_ROWS, w.n - st * C::STAGE_ROWS);
                    const uint32_t sb = smem_addr(smem + (c % C::NSTAGES) * C::STAGE_BYTES);
                    // ldmatrix row address of this lane: matrix lane/8 -> (+8 rows if odd, +8 cols if >= 2);
                    // row % 8 == lane % 8, the swizzle key
                    const int lrow = (lane & 7) + ((lane >> 3) & 1) * 8;
                    const int hi = lane >> 4;
                    const int x = lane & 7;
#pragma unroll
                    for (int mt = 0; mt < 2; ++mt) {
                        if (mt * 16 >= rows) break;
                        float acc[4] = {0.f, 0.f, 0.f, 0.f};
                        const uint32_t base = sb + row_base(mt * 16 + lrow);
#pragma unroll
                        for (int kk = 0; kk < KS; ++kk) {
                            uint32_t af[4];
                            const int cc = ((kk * 2) & 7) + hi;         // 16-byte chunk within the slice
                            ldsm_x4(base + (kk >> 2) * box_bytes + ((cc ^ x) << 4), af[0], af[1], af[2], af[3]);
                            M::mma(acc, af, qb[kk][0], qb[kk][1]);
                        }
                        const int t_lo = mt * 16 + gid;            // stage-relative token of acc[0..1]
                        float* lrow_lo = logits + (st * C::STAGE_ROWS + t_lo) * GC + tig * 2;
                        if (t_lo < rows) {
                            const float z0 = acc[0] * a.scale_log2, z1 = acc[1] * a.scale_log2;
                            *reinterpret_cast<float2*>(lrow_lo) = make_float2(z0, z1);
                            mlo = fmaxf(mlo, z0);
                            mhi = fmaxf(mhi, z1);
                        }
                        if (t_lo + 8 < rows) {
                            const float z2 = acc[2] * a.scale_log2, z3 = acc[3] * a.scale_log2;
                            *reinterpret_cast<float2*>(lrow_lo + 8 * GC) = make_float2(z2, z3);
                            mlo = fmaxf(mlo, z2);
                            mhi = fmaxf(mhi, z3);
                        }
                    }
                }
                release(c);
            }
            stage += nst;
#pragma unroll
            for (int o = 4; o < 32; o <<= 1) {
                mlo = fmaxf(mlo, __shfl_xor_sync(0xffffffffu, mlo, o));
                mhi = fmaxf(mhi, __shfl_xor_sync(0xffffffffu, mhi, o));
            }
            if (gid == 0) {
                wmax[warp * GC + tig * 2] = mlo;
                wmax[warp * GC + tig * 2 + 1] = mhi;
            }
            named_barrier(1, NCT);

            // ---- phase 2: p = 2^(z - max) built straight into B fragments for every
            // token; O^T += V^T P^T over this warp's head_dim tiles
            float mg = wmax[gid];
#pragma unroll
            for (int ww = 1; ww < C::NCW; ++ww) mg = fmaxf(mg, wmax[ww * GC + gid]);
            float oacc[DMW][4];
#pragma unroll
            for (int j = 0; j < DMW; ++j) oacc[j][0] = oacc[j][1] = oacc[j][2] = oacc[j][3] = 0.f;
            float lsum = 0.f;
            // ldmatrix.trans row address: matrix lane/8 -> (+8 tokens if >= 2, +8 head-dim cols if odd)
            const int vrow = (lane & 7) + (lane >> 4) * 8;
            const int vhi = (lane >> 3) & 1;
            const int vx = lane & 7;
            for (int st = 0; st < nst; ++st) {
                const uint32_t c = stage + st;
                if (!acquire(c)) continue;
                const int rows = min(C::STAGE_ROWS, w.n - st * C::STAGE_ROWS);
                const uint32_t sb = smem_addr(smem + (c % C::NSTAGES) * C::STAGE_BYTES);
#pragma unroll
                for (int mt = 0; mt < 2; ++mt) {
                    if (mt * 16 >= rows) break;
                    const int k0 = mt * 16 + tig * 2;       // stage-relative tokens of b0; b1 is k0 + 8
                    const float* lz = logits + (st * C::STAGE_ROWS + k0) * GC + gid;
                    const float p00 = k0 < rows ? exp2f(lz[0] - mg) : 0.f;
                    const float p01 = k0 + 1 < rows ? exp2f(lz[GC] - mg) : 0.f;
                    const float p10 = k0 + 8 < rows ? exp2f(lz[8 * GC] - mg) : 0.f;
                    const float p11 = k0 + 9 < rows ? exp2f(lz[9 * GC] - mg) : 0.f;
                    lsum += (p00 + p01) + (p10 + p11);
                    // p as a 16-bit pair (hi) plus its rounding remainder (lo): two mma per
                    // tile keep ~16 mantissa bits of p instead of 8 (bf16) or 11 (fp16)
                    uint32_t b0, b1, b0l, b1l;
                    split_pack<M>(p00, p01, b0, b0l);
                    split_pack<M>(p10, p11, b1, b1l);
                    const bool whole = mt * 16 + 16 <= rows;
                    const int vlo = rows - k0;              // valid tokens from k0 on (for masking)
                    const uint32_t base = sb + row_base(mt * 16 + vrow);
#pragma unroll
                    for (int j = 0; j < DMW; ++j) {
                        const int dm = warp * DMW + j;
                        uint32_t af[4];
                        const int cc = ((dm * 2) & 7) + vhi;
                        ldsm_x4_trans(base + (dm >> 2) * box_bytes + ((cc ^ vx) << 4), af[0], af[1], af[2], af[3]);
                        if (!whole) {   // rows past the context may hold stale bits (even NaN)
                            af[0] = keep_pair(af[0], vlo);
                            af[1] = keep_pair(af[1], vlo);
                            af[2] = keep_pair(af[2], vlo - 8);
                            af[3] = keep_pair(af[3], vlo - 8);
                        }
                        M::mma(oacc[j], af, b0, b1);
                        M::mma(oacc[j], af, b0l, b1l);
                    }
                }
                release(c);
            }
            stage += nst;
            // sum of p for query gid over the lanes holding it (tig = 0..3): every
            // warp formed the same sums in the same order
            lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
            lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);

            // ---- epilogue: this warp's columns; O^T fragment (d = 16*dm + gid [+8], query 2*tig [+1])
            const int qa = tig * 2, qc = tig * 2 + 1;
            const float la = __shfl_sync(0xffffffffu, lsum, qa * 4);     // lane with gid == query
            const float lc = __shfl_sync(0xffffffffu, lsum, qc * 4);
            const float ma = __shfl_sync(0xffffffffu, mg, qa * 4);
            const float mc = __shfl_sync(0xffffffffu, mg, qc * 4);
            const bool single = (w.np == 1);
            if (single) {
#pragma unroll
                for (int j = 0; j < DMW; ++j) {
                    const int d0 = (warp * DMW + j) * 16 + gid;
                    if (qa < gq) {
                        T* dst = outg + (row0 + qa) * D + d0;
                        dst[0] = Tr::from_float(oacc[j][0] / la);
                        dst[8] = Tr::from_float(oacc[j][2] / la);
                    }
                    if (qc < gq) {
                        T* dst = outg + (row0 + qc) * D + d0;
                        dst[0] = Tr::from_float(oacc[j][1] / lc);
                        dst[8] = Tr::from_float(oacc[j][3] / lc);
                    }
                }
            } else {
                const int64_t pa_ = (row0 + qa) * a.max_partitions + w.p;
                const int64_t pc_ = (row0 + qc) * a.max_partitions + w.p;
#pragma unroll
                for (int j = 0; j < DMW; ++j) {
                    const int d0 = (warp * DMW + j) * 16 + gid;
                    if (qa < gq) {
                        a.part_o[pa_ * D + d0] = oacc[j][0];
                        a.part_o[pa_ * D + d0 + 8] = oacc[j][2];
                    }
                    if (qc < gq) {
                        a.part_o[pc_ * D + d0] = oacc[j][1];
                        a.part_o[pc_ * D + d0 + 8] = oacc[j][3];
                    }
                }
                if (warp == 0 && gid == 0) {
                    if (qa < gq) {
                        a.part_m[pa_] = ma;
                        a.part_l[pa_] = la;
                    }
                    if (qc < gq) {
                        a.part_m[pc_] = mc;
                        a.part_l[pc_] = lc;
                    }
                }
            }
        } else {
            constexpr int LS = C::LSTRIDE;
            const int row_in = lane / C::LPT;                 // row within a warp instruction
            const int chunk = lane % C::LPT;                  // 16-byte chunk within the row
            const int gsel = chunk / (C::LPT / GC);           // query owned after the row reduction
            const bool gwriter = (chunk % (C::LPT / GC)) == 0;
            // ---- phase 1: z' = (q . k) * scale * log2(e) for every token
            {
                float qf[GC][C::VEC];
#pragma unroll
                for (int g = 0; g < GC; ++g) {
                    if (have_q && g < gq) {
                        const uint4 u = *reinterpret_cast<const uint4*>(qs + g * C::ROW_BYTES + chunk * 16);
                        Tr::unpack(u, qf[g]);
                    } else {
#pragma unroll
                        for (int v = 0; v < C::VEC; ++v) qf[g][v] = 0.f;
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&item_empty[b]);
                for (int st = warp; st < nst; st += C::NCW) {
                    const uint32_t c = stage + st;
                    if (!acquire(c)) continue;
                    const int rows = min(C::STAGE_ROWS, w.n - st * C::STAGE_ROWS);
                    const unsigned char* sb = smem + (c % C::NSTAGES) * C::STAGE_BYTES;
#pragma unroll 2
                    for (int r0 = 0; r0 < rows; r0 += C::RPI) {
                        const int r = r0 + row_in;
                        const uint4 u = *reinterpret_cast<const uint4*>(sb + chunk_off(r, chunk));
                        float kf[C::VEC];
                        Tr::unpack(u, kf);
                        float part[GC];
#pragma unroll
                        for (int g = 0; g < GC; ++g) {
                            float acc = 0.f;
#pragma unroll
                            for (int v = 0; v < C::VEC; ++v) acc = fmaf(qf[g][v], kf[v], acc);
                            part[g] = acc;
                        }
                        const float z = reduce_row_dots<GC, C::LPT>(part, lane);
                        if (gwriter && r < rows) logits[(st * C::STAGE_ROWS + r) * LS + gsel] = z * a.scale_log2;
                    }
                    release(c);
                }
                stage += nst;
            }
            named_barrier(1, NCT);

            // ---- phase 2: exact max, exponentials and their sum per query
            for (int g = warp; g < GC; g += C::NCW) {
                float m = -INFINITY;
                for (int t = lane; t < w.n; t += 32) m = fmaxf(m, logits[t * LS + g]);
                m = warp_max(m);
                float l = 0.f;
                for (int t = lane; t < w.n; t += 32) {
                    const float p = exp2f(logits[t * LS + g] - m);
                    logits[t * LS + g] = p;
                    l += p;
                }
                l = warp_sum(l);
                if (lane == 0) {
                    stat_m[g] = m;
                    stat_l[g] = l;
                }
            }
            named_barrier(1, NCT);

            // ---- phase 3: o = sum_t p_t v_t
            float acc[GC][C::VEC];
#pragma unroll
            for (int g = 0; g < GC; ++g)
#pragma unroll
                for (int v = 0; v < C::VEC; ++v) acc[g][v] = 0.f;
            for (int st = warp; st < nst; st += C::NCW) {
                const uint32_t c = stage + st;
                if (!acquire(c)) continue;
                const int rows = min(C::STAGE_ROWS, w.n - st * C::STAGE_ROWS);
                const unsigned char* sb = smem + (c % C::NSTAGES) * C::STAGE_BYTES;
#pragma unroll 2
                for (int r0 = 0; r0 < rows; r0 += C::RPI) {
                    const int r = r0 + row_in;
                    if (r < rows) {
                        const uint4 u = *reinterpret_cast<const uint4*>(sb + chunk_off(r, chunk));
                        float vf[C::VEC];
                        Tr::unpack(u, vf);
                        const float* pr = logits + (st * C::STAGE_ROWS + r) * LS;
                        float p[GC];
#pragma unroll
                        for (int g = 0; g < GC; ++g) p[g] = pr[g];
#pragma unroll
                        for (int g = 0; g < GC; ++g)
#pragma unroll
                            for (int v = 0; v < C::VEC; ++v) acc[g][v] = fmaf(p[g], vf[v], acc[g][v]);
                    }
                }
                release(c);
            }
            stage += nst;

            // merge the rows of a warp, then hand the warp's partial to the epilogue
#pragma unroll
            for (int o = C::LPT; o < 32; o <<= 1)
#pragma unroll
                for (int g = 0; g < GC; ++g)
#pragma unroll
                    for (int v = 0; v < C::VEC; ++v) acc[g][v] += __shfl_xor_sync(0xffffffffu, acc[g][v], o);
            named_barrier(1, NCT);            // every warp is done with the scores: reuse them as `red`
            if (row_in == 0) {
#pragma unroll
                for (int g = 0; g < GC; ++g) {
                    float* dst = red + (warp * GC + g) * D + chunk * C::VEC;
#pragma unroll
                    for (int v = 0; v < C::VEC; v += 4)
                        *reinterpret_cast<float4*>(dst + v) =
                            make_float4(acc[g][v], acc[g][v + 1], acc[g][v + 2], acc[g][v + 3]);
                }
            }
            named_barrier(1, NCT);

            // ---- epilogue: warps merged in a fixed order; final row or partition partials
            const bool single = (w.np == 1);
            for (int e = ctid; e < gq * D; e += NCT) {
                const int g = e / D;
                const int d = e - g * D;
                float o = 0.f;
#pragma unroll
                for (int ww = 0; ww < C::NCW; ++ww) o += red[(ww * GC + g) * D + d];
                const int64_t row = row0 + g;
                if (single) {
                    outg[row * D + d] = Tr::from_float(o / stat_l[g]);
                } else {
                    const int64_t pidx = row * a.max_partitions + w.p;
                    a.part_o[pidx * D + d] = o;
                    if (d == 0) {
                        a.part_m[pidx] = stat_m[g];
                        a.part_l[pidx] = stat_l[g];
                    }
                }
            }
        }

        if (w.np != 1 && a.merge_count != nullptr) {
            // The CTA that finishes the last partition of this (sequence, kv head,
            // chunk) merges all of them: partials are published with a fence
            // before the counter increment; the last arriver fences and reads
            // them from L2.  Nothing waits; the merge order is fixed (partition 0
            // first), so the bits do not depend on which CTA ends up merging.
            volatile int* last_flag = abort_flag + 1;
            __threadfence();
            named_barrier(1, NCT);
            if (ctid == 0) {
                const int64_t cidx = ((int64_t)w.s * a.num_kv_heads + w.h) * a.n_gchunks + w.gc;
                const int prev = atomicAdd(a.merge_count + cidx, 1);
                *last_flag = (prev == w.np - 1) ? 1 : 0;
            }
            named_barrier(1, NCT);
            if (*last_flag) {
                __threadfence();
                merge_partitions<T, D>(a, row0, gq, w.np, stat_m, stat_l, warp, lane, ctid, C::NCW);
            }
        }
        // every warp is done with this item's scores (and statistics) before the
        // next item's phase 1 writes them
        named_barrier(1, NCT);
    }
    // this CTA's work is done: a dependent kernel (the reduce) may start launching;
    // it still waits for this grid's completion before reading anything
    grid_launch_dependents();
}

}  // namespace pa_dev
