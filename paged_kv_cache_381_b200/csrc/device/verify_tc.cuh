// Multi-query paged attention (the verification pass of speculative decoding)
// on the fifth-generation tensor cores: tcgen05.mma with operands in shared
// memory and accumulators in tensor memory (TMEM).
//
// Same contract as verify_kernel (verify.cuh): query i of sequence s sits at
// position p = ctx_s - Q + i and attends causally to positions 0..p; work
// items, partitions, partials and the reduce are shared with decode.
//
// Design (2 CTAs per SM, each holding 256 of the SM's 512 TMEM columns):
//  * Item = (sequence, partition of 512, 1024 or 2048 tokens, kv head, chunk of
//    <= 64 query rows).  The rows form one M = 64 tile; the partition is walked in
//    chunks of 64 tokens.  A CTA walks the length-sorted plan with a fixed
//    stride; the last rounds are dealt from an atomic counter by the producer,
//    which publishes each item's index to the other warps in item slots.
//  * Warp 0 streams K and V chunks through TMA tiled boxes into a ring of
//    five slots, and each item's q rows into one of two q tiles an item ahead
//    (slot = 64 token rows of one kv head; each 128-byte head_dim
//    slice of the 64 rows is one 128-byte-swizzled array), K running one
//    chunk ahead of V: K0 K1 V0 K2 V1 ... .  A slot is refilled once the
//    products that read its previous contents are done: the producer waits
//    on the commit barrier the softmax (S done) or the epilogue (P.V done)
//    waits on, so no separate release barrier is committed.
//  * One elected thread of warp 1 issues the S products, one of warp 6 the P.V
//    products:
//        S(c) [64 x 64]  = Q K^T   KS MMAs M=64 N=64 K=16, into one of two S buffers
//        O    [64 x D]  += P V     4 (x 2) MMAs M=64 N=D K=16, P read from tensor
//                                  memory, V MN-major from the slot as loaded
//    S(c+1) is computed while the softmax of chunk c runs; S(c) waits for P.V
//    of chunk c - 2, the last reader of its buffer.  TMEM columns: S buffers
//    [0, 64) and [64, 128), O [128, 128 + D).  A tcgen05.mma costs its issuing
//    thread about as much as a commit or a barrier test, whatever its N, so a
//    chunk is covered by as few instructions as the shapes allow, over two
//    issuers.
//  * Warps 2-5 (one TMEM lane quarter each; a quarter's first 16 lanes hold 16
//    rows of an M = 64 accumulator, read as two half-warps of 32 columns)
//    stage q when its rows are not one TMA box, take the exact max of the chunk (causal mask, only where a
//    thread's tokens need it; max over raw scores, scaled once), rescale O in TMEM
//    when the running max grows by more than 8 (base 2), write p over the
//    chunk's S columns (arriving on one of two p_full copies), and finally read
//    O, normalise and store (or store the partition's partials) and release O
//    to the next item's first P.V.  For bf16, p is split into a 16-bit value and its
//    remainder (two products, as in decode); an fp16 p keeps 11 significant
//    bits and goes in one product.
//  * All waits are bounded; TMEM is freed after a final commit has drained
//    the MMAs.
#pragma once

#include "decode.cuh"
#include "tcgen05.cuh"

#include <type_traits>

namespace pa_dev {

#ifndef PA_VERIFY_TC_PSPLIT
// 1: P.V as two products (16-bit p and its remainder); 0: the 16-bit p only;
// 2: split for bf16 only (an fp16 p already carries 11 significant bits)
#define PA_VERIFY_TC_PSPLIT 2
#endif
#ifndef PA_VERIFY_TC_QTMA
// 1: two q tiles; when an item's query rows are one tile (group x queries <= 64)
// the producer brings its tile by TMA an item ahead.  0: one q tile, staged by
// the softmax warps after the previous item's last chunk.  Measured on B200 (6
// candidate tokens, one box, three runs each): 239.8 vs 248.2 us on the
// 70B-shaped batch, 207.5 vs 210.3 us (7B), 206.2 vs 210.3 us (long contexts).
#define PA_VERIFY_TC_QTMA 1
#endif
#ifndef PA_VERIFY_TC_SLOTS
// Measured on B200 (6 candidate tokens, two runs each): 6 slots 247.2 us vs 5
// slots 252.8 us on the 70B-shaped batch, 213.4 vs 213.65 us (7B), 211.85 vs
// 211.05 us (long contexts).  With two q tiles, five slots fit.
#define PA_VERIFY_TC_SLOTS (PA_VERIFY_TC_QTMA ? 5 : 6)
#endif
#ifndef PA_VERIFY_TC_DYN_ROUNDS
// The last rounds of the length-sorted plan (its shortest items) are handed out
// one at a time from an atomic counter; 0: every item by the fixed stride.
// Measured on B200 (6 candidate tokens, one box, three runs each, each batch at
// the partition pa_verify picks): 2 / 4 / 6 rounds 235.2 / 230.6 / 233.2 us on
// the 70B-shaped batch (2048-token partitions), 207.3 / 207.9 / 208.8 us (7B,
// 512), 195.5 / 196.5 / 196.9 us (long contexts, 1024); with the earlier
// 512-token partitions on the 70B batch, 0 / 2 / 3 rounds 249.9 / 247.7 /
// 248.2 us.
#define PA_VERIFY_TC_DYN_ROUNDS 4
#endif
#ifndef PA_VERIFY_TC_PTMEM
#define PA_VERIFY_TC_PTMEM 1     // 1: p written to tensor memory over its S buffer, P.V reads A from there
#endif
#ifndef PA_VERIFY_TC_PWAR
#define PA_VERIFY_TC_PWAR 1      // with p in tensor memory: S of chunk g waits for P.V of chunk g - 2
#endif
#ifndef PA_VERIFY_TC_TWO_ISSUERS
#define PA_VERIFY_TC_TWO_ISSUERS 1   // 1: S and P.V products issued by two warps; 0: one thread issues both
#endif
#ifndef PA_VERIFY_TC_PBUF
#define PA_VERIFY_TC_PBUF 1      // P tiles in shared memory: 2 = double-buffered, 1 = single
#endif

// 2^x by the PTX ex2.approx instruction (relative error about 2^-22; -inf -> +0;
// results below the normal range flush to zero)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

template <typename T, int D>
struct VerifyTcCfg {
    static constexpr int ELT = 2;
    static constexpr int NH = D * ELT / 128;                 // 128-byte head_dim slices
    static constexpr int BOX_ELEMS = 128 / ELT;
    static constexpr int CHUNK = 64;                         // tokens per chunk = rows of a ring slot
    static constexpr int SLICE_BYTES = CHUNK * 128;          // one head_dim slice of a slot
    static constexpr int SLOT_BYTES = NH * SLICE_BYTES;
    // K(c+1) and V(c) are in use while the rest of the ring loads.  The commit
    // barriers of S and P.V come in four copies (chunk g uses copy g % 4), so a
    // refill that waits on the element NSLOTS back in the stream can never see
    // its barrier four phases on: the same copy's next use is at least seven
    // elements later.
    static constexpr int NSLOTS = PA_VERIFY_TC_SLOTS;
    static constexpr int NPH = 4;                            // copies of the S / P.V commit barriers
    static constexpr int M = 64;                             // query rows per item
    static constexpr int Q_SLICE = M * 128;                  // one 128-byte slice of the Q tile
    static constexpr int Q_BYTES = NH * Q_SLICE;
    static constexpr int QBUF = PA_VERIFY_TC_QTMA ? 2 : 1;   // q tiles (item k uses tile k % QBUF)
    static constexpr int P_TILE = M * 128;                   // 64 rows x 64 tokens, one 128-byte atom column
    static constexpr bool PTMEM = PA_VERIFY_TC_PTMEM != 0;
    static constexpr int PBUF = PTMEM ? 0 : PA_VERIFY_TC_PBUF;  // P tiles in shared memory
    static constexpr bool PSPLIT =
        PA_VERIFY_TC_PSPLIT == 2 ? !std::is_same<T, __half>::value : PA_VERIFY_TC_PSPLIT != 0;
    static constexpr int TMEM_COLS = 256;
    static constexpr int S_COL = 0;                          // S buffer b: [64 b, 64 b + 64)
    static constexpr int O_COL = 128;
    // shared memory: ring, Q, P (buffers x {value, remainder}), barriers, table
    static constexpr int OFF_Q = NSLOTS * SLOT_BYTES;
    static constexpr int OFF_P = OFF_Q + QBUF * Q_BYTES;     // tile (buffer b, part h) at (2 b + h) * P_TILE
    static constexpr int OFF_BAR = OFF_P + 2 * PBUF * P_TILE;
    // barriers: full[NSLOTS], s_full[NPH], p_full[2], o_full[NPH], o_empty, drain, q_full[QBUF],
    // q_empty[QBUF], dyn_full[NDYN], dyn_empty[NDYN]
    static constexpr int NDYN = 4;                           // item slots of the dynamic tail
    static constexpr int NBAR = NSLOTS + 2 * NPH + 4 + 2 * QBUF + 2 * NDYN;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;      // allocated TMEM address
    static constexpr int OFF_ABORT = OFF_TMEM + 4;
    static constexpr int OFF_DYN = OFF_ABORT + 4;            // item index per slot (-1: no more items)
    static constexpr int OFF_TABLE = (OFF_DYN + NDYN * 4 + 15) / 16 * 16;
    static constexpr int MAX_TABLE = 1024 / 8;
    // 1024 bytes of slack let the kernel round its base up to 1024 bytes.  When
    // two CTAs fit on an SM (228 KB, 1 KB reserved per CTA) only without the
    // slack, the kernel needs the base it is given to be 1024-byte aligned, and
    // checks it.
    static constexpr int ALIGN_SLACK = 2 * (OFF_TABLE + MAX_TABLE * 4 + 2048) <= 228 * 1024 ? 1024 : 0;
    static constexpr size_t SMEM = ALIGN_SLACK + (size_t)OFF_TABLE + MAX_TABLE * 4;
    // A tcgen05.mma costs its issuing thread about 57 cycles whatever its N; two
    // issuing warps (S in warp 1, P.V in warp 6) double the rate the chunks need.
    // The S warp's wait for P.V of chunk g - 2 orders the two streams where they
    // share tensor memory, so this needs p in tensor memory with that wait.
    static constexpr bool TWO_ISSUERS = PA_VERIFY_TC_TWO_ISSUERS != 0 && PTMEM && PA_VERIFY_TC_PWAR != 0;
    static constexpr int PV_WARP = TWO_ISSUERS ? 6 : 1;
    static constexpr int THREADS = (TWO_ISSUERS ? 7 : 6) * 32;
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(SLOT_BYTES % 1024 == 0 && Q_BYTES % 1024 == 0 && P_TILE % 1024 == 0, "1024-byte atoms");
    static_assert((M * D * 2 / 16) % 128 == 0, "q tile chunks per staging thread");
    static_assert(PTMEM || PBUF == 1 || PBUF == 2, "P buffers");
    static_assert(NSLOTS >= 3 && NSLOTS <= 7, "ring refill rule");
    static_assert(CHUNK / 8 * NH <= 32, "one producer lane per box of a slot (8-token blocks at least)");
};

template <typename T, int D>
__global__ void __launch_bounds__(VerifyTcCfg<T, D>::THREADS, 2)
    verify_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_q) {
    using C = VerifyTcCfg<T, D>;
    using Tr = ElemTraits<T>;
    using MO = MmaOps<T>;
    constexpr bool BF16 = !std::is_same<T, __half>::value;
    constexpr uint32_t IDESC_S = tc::idesc_f16(BF16, false, C::M, C::CHUNK);
    constexpr uint32_t IDESC_PV = tc::idesc_f16(BF16, true, C::M, D);
    constexpr int KS = D / 16;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    if constexpr (C::ALIGN_SLACK == 0) {
        if (smem != smem_raw) {                  // no room to align: give up before any barrier
            if (threadIdx.x == 0) flag_error(PA_DEVERR_SMEM_ALIGN);
            return;
        }
    }
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bar;                        // [NSLOTS] a slot's TMA bytes landed
    uint64_t* s_full = bar + C::NSLOTS;          // [NPH] S of chunk g done (commit), copy g % NPH
    // [2] chunk g's S read, O rescaled, p written (128 arrivals), copy g % 2.  Two
    // copies: the P.V warp waits for chunk g's phase in order, and one barrier
    // could complete the phases of g and g + 1 before that warp looks (it may be
    // reading the next item's descriptor while the softmax warps finish two
    // chunks), after which the parity test would wait for a phase that never
    // comes.  The arrivals for chunk g + 2 need S(g + 2), which waits for P.V of
    // g, so copy g % 2 cannot move past the phase of g unseen; and a warp that
    // arrives for chunk g has seen S(g) done, so the phase of g - 2 on the same
    // copy is complete and the arrival counts toward the phase of g.
    uint64_t* p_full = s_full + C::NPH;
    uint64_t* o_full = p_full + 2;               // [NPH] P.V of chunk g done (commit), copy g % NPH
    uint64_t* o_empty = o_full + C::NPH;         // O read by the epilogue (128 arrivals)
    uint64_t* drain = o_empty + 1;               // every MMA done, before TMEM is freed (one commit per issuer)
    uint64_t* q_full = drain + 1;                // [QBUF] q tile written (TMA bytes, or 128 arrivals)
    uint64_t* q_empty = q_full + C::QBUF;        // [QBUF] last S of the tile's item done (commit)
    uint64_t* dyn_full = q_empty + C::QBUF;      // [NDYN] item slot written by the producer
    uint64_t* dyn_empty = dyn_full + C::NDYN;    // [NDYN] item slot read by the S, P.V and softmax warps
    volatile int* dyn_item = reinterpret_cast<volatile int*>(smem + C::OFF_DYN);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
    int32_t* tbl = reinterpret_cast<int32_t*>(smem + C::OFF_TABLE);
    unsigned char* qs = smem + C::OFF_Q;
    unsigned char* ps = smem + C::OFF_P;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    // An item's query rows are one box of q viewed as (head_dim, head, sequence x
    // query) when they are all of one kv head's group x queries (one row tile):
    // then the producer loads the tile by TMA and rows past them stay zero.
    const bool q_by_tma = C::QBUF == 2 && a.n_gchunks == 1;
    if (q_by_tma) {
        const int R = a.group * a.num_queries;
        for (int e = threadIdx.x; e < C::QBUF * C::NH * C::M * 8; e += blockDim.x) {
            const int row = (e >> 3) % C::M;
            if (row >= R) reinterpret_cast<uint4*>(smem + C::OFF_Q)[e] = make_uint4(0u, 0u, 0u, 0u);
        }
        tc::fence_proxy_async_smem();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NSLOTS; ++i) mbar_init(&full[i], 1);
        for (int i = 0; i < C::NPH; ++i) {
            mbar_init(&s_full[i], 1);
            mbar_init(&o_full[i], 1);
        }
        for (int b = 0; b < C::QBUF; ++b) {
            mbar_init(&q_full[b], q_by_tma ? 1 : 128);
            mbar_init(&q_empty[b], 1);
        }
        mbar_init(&p_full[0], 128);
        mbar_init(&p_full[1], 128);
        mbar_init(o_empty, 128);
        mbar_init(drain, C::TWO_ISSUERS ? 2 : 1);
        for (int i = 0; i < C::NDYN; ++i) {
            mbar_init(&dyn_full[i], 1);
            mbar_init(&dyn_empty[i], C::TWO_ISSUERS ? 6 : 5);     // one per consumer warp
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) {
        tc::tmem_alloc(tmem_slot, C::TMEM_COLS);
        tc::tmem_relinquish();
    }
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    grid_dependency_wait();
    // Items are taken with a fixed stride over the length-sorted plan (item
    // blockIdx.x, then + gridDim.x, ...): on the 70B-shaped batch with 6
    // candidate tokens this kernel measured 254.5 us with the stride and
    // 263.2 us in snake order (round r reversed when r is odd; same B200, same
    // build otherwise, five ring slots, no dynamic tail).
    const int pairs = a.max_partitions == 1 ? a.num_seqs : *a.plan_count;
    const int total = pairs * a.num_kv_heads * a.n_gchunks;
    const int bs = 1 << a.log2_bs;
    const int box_bytes = bs * 128;
    // A CTA takes items blockIdx.x, + gridDim.x, ... of the sorted plan while they
    // lie below dyn_start; past it (the last rounds, the shortest items) the
    // producer takes the next item from the counter and publishes its index in
    // the next item slot for the other warps.  Each role walks the same sequence:
    // next_static gives the successor of `cur` in the fixed-stride part (cur < 0:
    // the first item), or -1 once the walk reaches the dynamic part.
    const bool dyn_tail = a.work_counter != nullptr && PA_VERIFY_TC_DYN_ROUNDS > 0;
    const int dyn_start = dyn_tail ? max(0, total - PA_VERIFY_TC_DYN_ROUNDS * (int)gridDim.x) : total;
    auto next_static = [&](int cur) -> int {
        if (cur >= dyn_start) return -1;
        const int s = cur < 0 ? (int)blockIdx.x : cur + (int)gridDim.x;
        return s < dyn_start ? s : -1;
    };
    // a consumer warp's next dynamic item (total when there is none); the whole
    // warp reads the slot before its lane 0 releases it
    auto read_dynamic = [&](uint32_t& dk, bool& ok) -> int {
        if (!dyn_tail) return total;
        const int slot = (int)(dk % C::NDYN);
        if (!mbar_wait(&dyn_full[slot], (dk / C::NDYN) & 1u, abort_flag)) {
            ok = false;
            return total;
        }
        const int it = dyn_item[slot];
        __syncwarp();
        if (lane == 0) mbar_arrive(&dyn_empty[slot]);
        ++dk;
        return it < 0 ? total : it;
    };

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmap_k);
            prefetch_tmap(&tmap_v);
        }
        const uint64_t policy = l2_policy_evict_first();
        uint32_t seq = 0;                                   // stream elements issued so far
        uint32_t gch = 0;                                   // chunks of earlier items
        // the last NSLOTS stream elements (oldest first): chunk index << 1 | is_v
        uint32_t hist[C::NSLOTS];
#pragma unroll
        for (int k = 0; k < C::NSLOTS; ++k) hist[k] = 0;
        bool ok = true;
        uint32_t kq = 0;                                    // q tiles loaded (items with tokens)
        uint32_t dk = 0;                                    // dynamic items taken so far
        // the item after `cur`: by the stride, else the next one of the counter,
        // published in the next item slot (-1 there: no more items)
        auto take = [&](int cur) -> int {
            if (!ok) return total;
            const int st = next_static(cur);
            if (st >= 0) return st;
            if (!dyn_tail) return total;
            const int slot = (int)(dk % C::NDYN);
            if (!mbar_wait(&dyn_empty[slot], ((dk / C::NDYN) & 1u) ^ 1u, abort_flag)) {
                ok = false;
                return total;
            }
            int it = 0;
            if (lane == 0) {
                it = dyn_start + atomicAdd(a.work_counter, 1);
                if (it >= total) it = -1;
                dyn_item[slot] = it;
                mbar_arrive(&dyn_full[slot]);
            }
            it = __shfl_sync(0xffffffffu, it, 0);
            ++dk;
            return it < 0 ? total : it;
        };
        for (int i = take(-1); i < total && ok; i = take(i)) {
            const WorkItem w = decode_item(a, i, lane == 0);
            if (w.n == 0) continue;
            const int nblk = (w.n + bs - 1) >> a.log2_bs;
            const int32_t* trow = a.block_tables + (int64_t)w.s * a.max_blocks_per_seq + (w.t0 >> a.log2_bs);
            __syncwarp();
            for (int j = lane; j < nblk; j += 32) {
                int32_t id = trow[j];
                if (id < 0 || id >= a.num_blocks) {
                    flag_error(PA_DEVERR_BLOCK_ID);
                    id = 0;
                }
                tbl[j] = id;
            }
            __syncwarp();
            const int nc = (w.n + C::CHUNK - 1) / C::CHUNK;
            if (q_by_tma) {
                // the item's q rows into tile kq % 2 once the item two back has no S
                // product left to read it: rows (query i, head h * group + g) for all i,
                // g, i.e. row i * group + g of the tile
                const uint32_t b = kq & 1u;
                if (!mbar_wait(&q_empty[b], ((kq >> 1) & 1u) ^ 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                if (lane == 0)
                    mbar_arrive_expect_tx(&q_full[b], (uint32_t)(C::NH * a.group * a.num_queries * 128));
                __syncwarp();
                if (lane < C::NH)
                    tma_load_3d(qs + b * C::Q_BYTES + lane * C::Q_SLICE, &tmap_q, lane * C::BOX_ELEMS,
                                w.h * a.group, w.s * a.num_queries, &q_full[b], policy);
                ++kq;
            }
            // K or V of chunk c into the next slot, once the products that read the
            // slot's previous contents (the element NSLOTS back) are done
            auto issue = [&](int c, bool is_v) -> bool {
                if (seq >= (uint32_t)C::NSLOTS) {
                    const uint32_t g = hist[0] >> 1;
                    uint64_t* done = (hist[0] & 1u) ? &o_full[g % C::NPH] : &s_full[g % C::NPH];
                    if (!mbar_wait(done, (g / C::NPH) & 1u, abort_flag)) return false;
                }
                const int slot = seq % C::NSLOTS;
                const int rows = min(C::CHUNK, w.n - c * C::CHUNK);
                const int nbk = (rows + bs - 1) >> a.log2_bs;          // whole blocks
                if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)(nbk * C::NH * box_bytes));
                __syncwarp();
                if (lane < nbk * C::NH) {
                    static_assert(C::NH <= 2, "one or two slices");
                    const int half = C::NH == 2 && lane >= nbk ? 1 : 0;  // slice
                    const int b = lane - half * nbk;                    // block within the chunk
                    const int phys = tbl[((c * C::CHUNK) >> a.log2_bs) + b];
                    tma_load_3d(smem + slot * C::SLOT_BYTES + half * C::SLICE_BYTES + b * box_bytes,
                                is_v ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k),
                                half * C::BOX_ELEMS, w.h, phys * bs, &full[slot], policy);
                }
#pragma unroll
                for (int k = 0; k + 1 < C::NSLOTS; ++k) hist[k] = hist[k + 1];
                hist[C::NSLOTS - 1] = ((gch + (uint32_t)c) << 1) | (is_v ? 1u : 0u);
                ++seq;
                return true;
            };
            if (!(ok = issue(0, false))) break;
            for (int c = 0; c < nc && ok; ++c) {
                if (c + 1 < nc && !(ok = issue(c + 1, false))) break;
                ok = issue(c, true);
            }
            gch += nc;
        }
        if (!ok) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            const uint32_t issued = seq;
            const volatile int never = 0;
            for (int slot = lane; slot < C::NSLOTS; slot += 32) {
                if ((uint32_t)slot < issued) {
                    const uint32_t last = issued - 1 - ((issued - 1 - slot) % C::NSLOTS);
                    mbar_wait(&full[slot], (last / C::NSLOTS) & 1u, &never);
                }
            }
            if (lane < 2 && (uint32_t)lane < kq) {            // the q tiles' last loads
                const uint32_t last = kq - 1 - ((kq - 1 - lane) & 1u);
                mbar_wait(&q_full[lane], (last >> 1) & 1u, &never);
            }
        }
    }
    if (warp == 1 || warp == C::PV_WARP) {
        // ------------------------------------------------------------ MMA issue
        const bool do_s = warp == 1;                     // issues S products (and commits q_empty)
        const bool do_pv = warp == C::PV_WARP;           // issues P.V products
        uint32_t seq = 0, kq = 0, oe_ph = 0, gch = 0;
        bool ok = true;
        // operand descriptors built once; every MMA adds a byte offset to one of them
        const uint64_t qdesc = tc::sw128_desc(smem_addr(qs), 16, 1024);                 // Q, K-major
        const uint64_t pdesc = tc::sw128_desc(smem_addr(ps), 16, 1024);                 // P, K-major
        const uint64_t kdesc = tc::sw128_desc(smem_addr(smem), 16, 1024);               // slot 0 as K, K-major
        const uint64_t vdesc = tc::sw128_desc(smem_addr(smem), C::SLICE_BYTES, 1024);   // slot 0 as V, MN-major
        // S of global chunk g = Q K^T over its 64 tokens (stream element pos), into S
        // buffer g & 1 (token columns past the partition read stale rows; the softmax
        // masks them)
        auto issue_s = [&](uint32_t pos, uint32_t g, uint32_t qb) -> bool {
            const uint32_t buf = g & 1u;
            const int slot = pos % C::NSLOTS;
            if (!mbar_wait(&full[slot], (pos / C::NSLOTS) & 1u, abort_flag)) return false;
            if constexpr (C::PTMEM && PA_VERIFY_TC_PWAR) {
                // the buffer holds p of chunk g - 2, read by P.V of that chunk: a later
                // product may not overwrite an operand the tensor core may still read
                // (nor, with two issuers, one not yet read), so that P.V completes first
                if (g >= 2 && !mbar_wait(&o_full[(g - 2) % C::NPH], ((g - 2) / C::NPH) & 1u, abort_flag)) return false;
            }
            tc::fence_after_sync();
            if (lane == 0) {
                const uint64_t kd = tc::desc_add(kdesc, slot * C::SLOT_BYTES);
                const uint32_t d = tmem + C::S_COL + buf * 64;
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    const uint32_t koff = (kk >> 2) * C::SLICE_BYTES + (kk & 3) * 32;
                    const uint32_t qoff = (kk >> 2) * C::Q_SLICE + (kk & 3) * 32;
                    tc::mma_ss(d, tc::desc_add(qdesc, qb * C::Q_BYTES + qoff), tc::desc_add(kd, koff), IDESC_S, kk > 0);
                }
                tc::commit(&s_full[g % C::NPH]);    // also frees the slot for the producer
            }
            __syncwarp();
            return true;
        };
        // O += P V over the tokens of chunk c (global chunk g, stream element pos), p from
        // P buffer g & 1 (buffer 0 when single)
        auto issue_pv = [&](uint32_t pos, int c, int n, uint32_t g, bool first) -> bool {
            const uint32_t pbuf = C::PBUF == 2 ? (g & 1u) : 0u;
            const int slot = pos % C::NSLOTS;
            if (!mbar_wait(&full[slot], (pos / C::NSLOTS) & 1u, abort_flag)) return false;
            const int rows = min(C::CHUNK, n - c * C::CHUNK);
            if (rows < C::CHUNK) {
                // rows past the partition (stale or unwritten rows, maybe NaN): zero them
                // so that p = 0 meets finite values
                uint4* vrow = reinterpret_cast<uint4*>(smem + slot * C::SLOT_BYTES);
                for (int e = lane; e < C::NH * C::CHUNK * 8; e += 32)
                    if (((e >> 3) % C::CHUNK) >= rows) vrow[e] = make_uint4(0u, 0u, 0u, 0u);
                tc::fence_proxy_async_smem();
            }
            __syncwarp();
            tc::fence_after_sync();
            if (lane == 0) {
                const uint64_t vd = tc::desc_add(vdesc, slot * C::SLOT_BYTES);
                const uint64_t pd = tc::desc_add(pdesc, 2 * pbuf * C::P_TILE);
                // p in tensor memory: value in S buffer columns [0, 32), remainder in [32, 64)
                const uint32_t pt = tmem + C::S_COL + (g & 1u) * 64;
#pragma unroll
                for (int ks = 0; ks < C::CHUNK / 16; ++ks) {             // 16 tokens per MMA
                    const uint64_t bd = tc::desc_add(vd, ks * 16 * 128);
                    if constexpr (C::PTMEM) {
                        tc::mma_ts(tmem + C::O_COL, pt + ks * 8, bd, IDESC_PV, ks > 0 || !first);
                        if constexpr (C::PSPLIT) tc::mma_ts(tmem + C::O_COL, pt + 32 + ks * 8, bd, IDESC_PV, true);
                    } else {
                        tc::mma_ss(tmem + C::O_COL, tc::desc_add(pd, ks * 32), bd, IDESC_PV, ks > 0 || !first);
                        if constexpr (C::PSPLIT)
                            tc::mma_ss(tmem + C::O_COL, tc::desc_add(pd, C::P_TILE + ks * 32), bd, IDESC_PV, true);
                    }
                }
                tc::commit(&o_full[g % C::NPH]);    // also frees the slot for the producer
            }
            __syncwarp();
            return true;
        };
        // P.V of chunk c, once its p is written (and, for the item's first chunk, the
        // previous item's O has been read out)
        auto pv_chunk = [&](uint32_t pos, int c, int n, uint32_t g) -> bool {
            if (!mbar_wait(&p_full[g & 1u], (g >> 1) & 1u, abort_flag)) return false;
            if (c == 0) {
                if (!mbar_wait(o_empty, oe_ph ^ 1u, abort_flag)) return false;
                oe_ph ^= 1u;
            }
            tc::fence_after_sync();
            return issue_pv(pos, c, n, g, c == 0);
        };
        uint32_t dk = 0;
        auto next_item = [&](int cur) -> int {
            if (!ok) return total;
            const int st = next_static(cur);
            return st >= 0 ? st : read_dynamic(dk, ok);
        };
        for (int i = next_item(-1); i < total && ok; i = next_item(i)) {
            const WorkItem w = decode_item(a, i, false);
            if (w.n == 0) continue;
            const int nc = (w.n + C::CHUNK - 1) / C::CHUNK;
            // stream positions of the item's elements: K0, then K(c+1), V(c) per chunk
            auto kpos = [&](int c) -> uint32_t { return seq + (c == 0 ? 0u : (uint32_t)(2 * c - 1)); };
            auto vpos = [&](int c) -> uint32_t {
                return seq + (c + 1 < nc ? (uint32_t)(2 * c + 2) : (uint32_t)(2 * nc - 1));
            };
            const uint32_t qb = kq % C::QBUF;                   // the item's q tile
            if (do_s) {
                if (!mbar_wait(&q_full[qb], (kq / C::QBUF) & 1u, abort_flag)) {
                    ok = false;
                    break;
                }
                tc::fence_after_sync();
            }
            if constexpr (C::TWO_ISSUERS) {
                if (do_s) {
                    for (int c = 0; c < nc && ok; ++c) {
                        ok = issue_s(kpos(c), gch + c, qb);
                        if (ok && c + 1 == nc && lane == 0) tc::commit(&q_empty[qb]);   // the tile may be replaced
                        __syncwarp();
                    }
                } else {
                    for (int c = 0; c < nc && ok; ++c) ok = pv_chunk(vpos(c), c, w.n, gch + c);
                }
            } else {
                // one thread: S(c+1) is issued before P.V(c), so it runs during softmax(c)
                if (!(ok = issue_s(kpos(0), gch, qb))) break;
                if (nc == 1 && lane == 0) tc::commit(&q_empty[qb]);   // last S of the item: the tile may be replaced
                __syncwarp();
                for (int c = 0; c < nc && ok; ++c) {
                    if (c + 1 < nc) {
                        if (!(ok = issue_s(kpos(c + 1), gch + c + 1, qb))) break;
                        if (c + 2 == nc && lane == 0) tc::commit(&q_empty[qb]);
                        __syncwarp();
                    }
                    ok = pv_chunk(vpos(c), c, w.n, gch + c);
                }
            }
            seq += 2 * nc;
            gch += nc;
            ++kq;
        }
        if (!ok) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
        }
        // drain: every MMA this warp issued has completed before TMEM is released
        if (lane == 0) tc::commit(drain);
        __syncwarp();
        const volatile int never = 0;
        mbar_wait(drain, 0, &never);
    }
    if (warp >= 2 && warp < 6) {
        // ------------------------------------------------- softmax and epilogue
        const int ctid = threadIdx.x - 64;               // 0..127
        const int quarter = warp & 3;                    // TMEM lanes 32*quarter .. +15 hold rows 16*quarter ..
        const int half = lane >> 4;                      // which 32 columns of a 64-column group
        const int m = quarter * 16 + (lane & 15);        // accumulator row of this thread
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const T* qg = static_cast<const T*>(a.q);
        T* outg = static_cast<T*>(a.out);
        const int Q = a.num_queries;
        const int R = a.group * Q;
        uint32_t gch = 0;
        // P.V of global chunk g done: barrier copy g % NPH, its (g / NPH)-th phase
        auto wait_pv = [&](uint32_t g) -> bool {
            return mbar_wait(&o_full[g % C::NPH], (g / C::NPH) & 1u, abort_flag);
        };
        // output row and query position of local row lr of item w (orow < 0: no row)
        auto row_in = [&](const WorkItem& w, int ctx, int lr, int64_t& orow, int& pos) {
            const int r0 = w.gc * C::M;
            if (lr >= min(C::M, R - r0)) {
                orow = -1;
                pos = -1;
                return;
            }
            const int r = r0 + lr;
            const int qi = r / a.group;
            const int g = r - qi * a.group;
            orow = ((int64_t)w.s * Q + qi) * a.num_heads + (int64_t)w.h * a.group + g;
            pos = ctx - Q + qi;
        };
        // item w (the k-th item with tokens) as the A tile k % QBUF (rows past the
        // chunk are zero), once the item that last used the tile has no S product
        // left to read it
        auto stage_q = [&](const WorkItem& w, int ctx, uint32_t k) -> bool {
            const uint32_t b = k % C::QBUF;
            if (!mbar_wait(&q_empty[b], ((k / C::QBUF) & 1u) ^ 1u, abort_flag)) return false;
            unsigned char* qt = qs + b * C::Q_BYTES;
            // all loads of this thread first, then the swizzled stores
            constexpr int VPR = D * 2 / 16;               // 16-byte chunks per row
            constexpr int PER = C::M * VPR / 128;         // chunks per thread
            uint4 v[PER];
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int e = ctid + u * 128;
                int64_t orow;
                int pos;
                row_in(w, ctx, e / VPR, orow, pos);
                v[u] = orow >= 0 ? __ldg(reinterpret_cast<const uint4*>(qg + orow * D) + (e % VPR))
                                 : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < PER; ++u) {
                const int e = ctid + u * 128;
                const int lr = e / VPR;
                const int cc = e % VPR;
                *reinterpret_cast<uint4*>(qt + (cc >> 3) * C::Q_SLICE + lr * 128 + (((cc & 7) ^ (lr & 7)) << 4)) = v[u];
            }
            tc::fence_proxy_async_smem();
            mbar_arrive(&q_full[b]);
            return true;
        };
        bool ok = true;
        int staged = -1;                                 // item whose Q tile is already written
        uint32_t dk = 0;
        auto next_item = [&](int cur) -> int {
            if (!ok) return total;
            const int st = next_static(cur);
            return st >= 0 ? st : read_dynamic(dk, ok);
        };
        uint32_t kq = 0;                                 // items with tokens so far
        // the next item's descriptor, looked up while the current item ends
        WorkItem wpre{};
        int cpre = 0, ipre = -1;
        int i = next_item(-1);
        while (i < total && ok) {
            WorkItem w;
            int ctx;
            if (ipre == i) {
                w = wpre;
                ctx = cpre;
            } else {
                w = decode_item(a, i, false);
                ctx = clamp_context(a, w.s, false);
            }
            if (w.n == 0) {                              // empty context: zero rows
                const int nr = min(C::M, R - w.gc * C::M);
                for (int e = ctid; e < nr * D; e += 128) {
                    int64_t orow;
                    int pos;
                    row_in(w, ctx, e / D, orow, pos);
                    outg[orow * D + (e % D)] = Tr::from_float(0.f);
                }
                i = next_item(i);
                continue;
            }
            if (!q_by_tma && staged != i && !(ok = stage_q(w, ctx, kq))) break;
            int64_t orow;
            int pos;
            row_in(w, ctx, m, orow, pos);
            float m_run = -INFINITY, l_run = 0.f;        // l: this thread's half of the row
            const int nc = (w.n + C::CHUNK - 1) / C::CHUNK;
            for (int c = 0; c < nc && ok; ++c) {
                const uint32_t buf = (gch + c) & 1u;
                if (!(ok = mbar_wait(&s_full[(gch + c) % C::NPH], ((gch + c) / C::NPH) & 1u, abort_flag))) break;
                tc::fence_after_sync();
                uint32_t r[32];
                tc::ld16x2(tmem + lane_addr + C::S_COL + buf * 64, r);
                tc::wait_ld();
                // exact max of the chunk's visible scores (base-2 units); this thread holds
                // tokens c*64 + half*32 + k of row m
                const int t0 = c * C::CHUNK + half * 32;
                // With a positive scale the max commutes with scaling: scores stay raw (masked
                // ones -inf), the max is scaled once and p = 2^(fma(s, scale, -base)).  A
                // thread whose 32 tokens are all visible (most chunks) skips the mask.
                const float sl2 = a.scale_log2;
                const bool raw = sl2 > 0.f;
                const bool all_visible = t0 + 31 < w.n && w.t0 + t0 + 31 <= pos;
                float cmax = -INFINITY;
                if (raw && all_visible) {
#pragma unroll
                    for (int k = 0; k < 32; ++k) cmax = fmaxf(cmax, __uint_as_float(r[k]));
                } else {
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int t = t0 + k;
                        const float x = __uint_as_float(r[k]);
                        const float z = (t < w.n && w.t0 + t <= pos) ? (raw ? x : x * sl2) : -INFINITY;
                        r[k] = __float_as_uint(z);
                        cmax = fmaxf(cmax, z);
                    }
                }
                if (raw) cmax *= sl2;                    // -inf stays -inf
                cmax = fmaxf(cmax, __shfl_xor_sync(0xffffffffu, cmax, 16));
                // Lazy reference max: p = 2^(z - m_run) stays <= 2^8, so the reference only
                // moves (and O is rescaled) when a score beats it by more than 8 in base-2
                // units; a row that has seen nothing yet takes the chunk max (its O is zero).
                const bool fresh = m_run == -INFINITY;
                const bool raise = fresh ? cmax != -INFINITY : cmax > m_run + 8.f;
                const float m_new = raise ? cmax : m_run;
                const float base = m_new == -INFINITY ? 0.f : m_new;       // a row that saw nothing yet
                const float corr = raise && !fresh ? exp2f(m_run - m_new) : 1.f;
                uint32_t hi[16], lo[16];
                float lsum = 0.f;
                const float sc = raw ? sl2 : 1.f;       // scores are raw, or already scaled
#pragma unroll
                for (int k = 0; k < 32; k += 2) {
                    const float p0 = ex2_approx(fmaf(__uint_as_float(r[k]), sc, -base));
                    const float p1 = ex2_approx(fmaf(__uint_as_float(r[k + 1]), sc, -base));
                    if constexpr (C::PSPLIT) {
                        lsum += p0 + p1;
                        split_pack<MO>(p0, p1, hi[k >> 1], lo[k >> 1]);
                    } else {
                        hi[k >> 1] = MO::pack(p0, p1);            // the sum takes p as the product sees it
                        const float2 h = MO::unpack(hi[k >> 1]);
                        lsum += h.x + h.y;
                    }
                }
                const uint32_t gc = gch + c;
                // O rescale: only when some row of this warp moved its reference, after the
                // previous chunk's P.V has landed
                if (c > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
                    if (!(ok = wait_pv(gc - 1))) break;
                    tc::fence_after_sync();
#pragma unroll 1
                    for (int g = 0; g < D / 64; ++g) {
                        uint32_t o[32];
                        tc::ld16x2(tmem + lane_addr + C::O_COL + g * 64, o);
                        tc::wait_ld();
#pragma unroll
                        for (int k = 0; k < 32; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * corr);
                        tc::st16x2(tmem + lane_addr + C::O_COL + g * 64, o);
                    }
                    tc::wait_st();
                }
                m_run = m_new;
                l_run = l_run * corr + lsum;
                if constexpr (C::PTMEM && PA_VERIFY_TC_PWAR == 0) {
                    // S(gc) did not wait for P.V(gc - 2) here, so the phase of gc - 2 on this
                    // copy is not known complete: wait for chunk gc - 1's phase, which follows it
                    if (gc >= 1 && !(ok = mbar_wait(&p_full[(gc - 1) & 1u], ((gc - 1) >> 1) & 1u, abort_flag))) break;
                }
                if constexpr (C::PTMEM) {
                    // p over this chunk's S columns (already read): tokens half*32 .. +31 of row m
                    // are value columns half*16 .. +15 and remainder columns 32 + half*16 .. +15.
                    // The buffer's previous p was read by P.V of chunk gc - 2, which the tensor
                    // core finished before it wrote S of this chunk there.
                    tc::st16x2_x16(tmem + lane_addr + C::S_COL + buf * 64, hi);
                    if constexpr (C::PSPLIT) tc::st16x2_x16(tmem + lane_addr + C::S_COL + buf * 64 + 32, lo);
                    tc::wait_st();
                } else {
                    // the P buffer this chunk writes was last read by the P.V of chunk gc - PBUF
                    if (gc >= (uint32_t)C::PBUF && !(ok = wait_pv(gc - C::PBUF))) break;
                    // p of row m, tokens half*32 .. +31 of the chunk: 16-byte chunks 4*half .. +3 of the row
                    unsigned char* pt = ps + (C::PBUF == 2 ? 2 * buf : 0u) * C::P_TILE + m * 128;
#pragma unroll
                    for (int q4 = 0; q4 < 4; ++q4) {
                        const int off = (((half * 4 + q4) ^ (m & 7)) << 4);
                        *reinterpret_cast<uint4*>(pt + off) =
                            make_uint4(hi[4 * q4], hi[4 * q4 + 1], hi[4 * q4 + 2], hi[4 * q4 + 3]);
                        if constexpr (C::PSPLIT)
                            *reinterpret_cast<uint4*>(pt + C::P_TILE + off) =
                                make_uint4(lo[4 * q4], lo[4 * q4 + 1], lo[4 * q4 + 2], lo[4 * q4 + 3]);
                    }
                    tc::fence_proxy_async_smem();
                }
                tc::fence_before_sync();
                mbar_arrive(&p_full[gc & 1u]);
            }
            gch += nc;
            if (!ok) break;
            // ---- the next item now: its descriptor, and its q tile when the softmax
            // warps stage it, so that its first S products run while this item's
            // epilogue does
            const int inext = next_item(i);
            if (!ok) break;
            if (inext < total) {
                wpre = decode_item(a, inext, false);
                cpre = clamp_context(a, wpre.s, false);
                ipre = inext;
                if (!q_by_tma && wpre.n > 0) {
                    if (!(ok = stage_q(wpre, cpre, kq + 1))) break;
                    staged = inext;
                }
            }
            // ---- epilogue: O after the last chunk, normalised row or partition partials
            if (!(ok = wait_pv(gch - 1))) break;
            tc::fence_after_sync();
            const float l_row = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
            const bool single = w.np == 1;
            for (int g = 0; g < D / 64; ++g) {
                uint32_t o[32];
                tc::ld16x2(tmem + lane_addr + C::O_COL + g * 64, o);
                tc::wait_ld();
                if (orow >= 0) {
                    const int col = g * 64 + half * 32;
                    if (single) {
                        uint32_t packed[16];
#pragma unroll
                        for (int k = 0; k < 32; k += 2) {
                            const float o0 = l_row > 0.f ? __uint_as_float(o[k]) / l_row : 0.f;
                            const float o1 = l_row > 0.f ? __uint_as_float(o[k + 1]) / l_row : 0.f;
                            packed[k >> 1] = MO::pack(o0, o1);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(outg + orow * D + col);
#pragma unroll
                        for (int q4 = 0; q4 < 4; ++q4)
                            dst[q4] = make_uint4(packed[4 * q4], packed[4 * q4 + 1], packed[4 * q4 + 2], packed[4 * q4 + 3]);
                    } else {
                        const int64_t pidx = orow * a.max_partitions + w.p;
                        float4* dst = reinterpret_cast<float4*>(a.part_o + pidx * D + col);
#pragma unroll
                        for (int q8 = 0; q8 < 8; ++q8)
                            dst[q8] = make_float4(__uint_as_float(o[4 * q8]), __uint_as_float(o[4 * q8 + 1]),
                                                  __uint_as_float(o[4 * q8 + 2]), __uint_as_float(o[4 * q8 + 3]));
                    }
                }
            }
            if (!single && orow >= 0 && half == 0) {
                const int64_t pidx = orow * a.max_partitions + w.p;
                a.part_m[pidx] = m_run;
                a.part_l[pidx] = l_row;
            }
            tc::fence_before_sync();
            mbar_arrive(o_empty);
            ++kq;
            i = inext;
        }
        if (!ok) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
        }
    }
    // ---------------------------------------------------------------- teardown
    __syncthreads();
    if (warp == 1) {
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, C::TMEM_COLS);
    }
    grid_launch_dependents();
}

}  // namespace pa_dev
