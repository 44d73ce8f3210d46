// Multi-query paged attention (the verification pass of speculative decoding)
// on the fifth-generation tensor cores: tcgen05.mma with operands in shared
// memory and accumulators in tensor memory (TMEM).
//
// Same contract as verify_kernel (verify.cuh): query i of sequence s sits at
// position p = ctx_s - Q + i and attends causally to positions 0..p; work
// items, partitions, partials and the reduce are shared with decode.
//
// Design (one CTA per item at a time, 2 CTAs per SM):
//  * Item = (sequence, 512-token partition, kv head, chunk of <= 64 query
//    rows).  The rows are one M = 64 tile; the partition is walked in chunks
//    of 128 tokens = 4 slots of 32.
//  * Warp 0 streams, through TMA tiled boxes, the K slots of a chunk and then
//    its V slots into one ring (slot = 32 token rows of one kv head, the two
//    128-byte head_dim slices stored one after the other, 128-byte swizzle).
//  * Warp 1 issues the MMAs from one thread:
//        S[64 x 128] = Q K^T     4 x 8 MMAs M=64 N=32 K=16   (Q, K K-major)
//        O[64 x D]  += P V       4 x 2 x 2 MMAs M=64 N=D K=16 (P K-major, V
//                                 MN-major: the slot as loaded)
//    S (columns 0..127) and O (columns 128..) live in 256 TMEM columns; each
//    ring slot is released by a tcgen05.commit once the MMAs reading it are
//    done.  P is split into a 16-bit value and its remainder (two products),
//    as in decode, so p keeps ~16 mantissa bits.
//  * Warps 2-5 (one TMEM lane quarter each; a quarter's first 16 lanes hold
//    16 rows of an M = 64 accumulator) stage Q, read S row by row, take the
//    exact max of the chunk (causal mask), rescale O in TMEM when the running
//    max grows, write p to shared memory, and finally read O, normalise and
//    store (or store the partition's partials).
//  * All waits are bounded; TMEM is freed after a final commit has drained
//    the MMAs.
#pragma once

#include "decode.cuh"
#include "tcgen05.cuh"

#include <type_traits>

namespace pa_dev {

#ifndef PA_VERIFY_TC_SLOTS
#define PA_VERIFY_TC_SLOTS 6
#endif

template <typename T, int D>
struct VerifyTcCfg {
    static constexpr int ELT = 2;
    static constexpr int NH = D * ELT / 128;                 // 128-byte head_dim slices
    static constexpr int BOX_ELEMS = 128 / ELT;
    static constexpr int SLOT_ROWS = 32;
    static constexpr int SLICE_BYTES = SLOT_ROWS * 128;      // one slice of a slot
    static constexpr int SLOT_BYTES = NH * SLICE_BYTES;
    static constexpr int NSLOTS = PA_VERIFY_TC_SLOTS;
    static constexpr int CHUNK = 128;                        // tokens per softmax chunk
    static constexpr int CPS = CHUNK / SLOT_ROWS;            // slots per chunk
    static constexpr int M = 64;                             // query rows per item
    static constexpr int Q_SLICE = M * 128;                  // one 128-byte slice of the Q tile
    static constexpr int Q_BYTES = NH * Q_SLICE;
    static constexpr int P_ATOM = M * 128;                   // 64 tokens x 64 rows of p (bf16/fp16)
    static constexpr int P_BYTES = 2 * P_ATOM;               // 128 tokens
    static constexpr int TMEM_COLS = 256;                    // S: [0, 128), O: [128, 128 + D)
    static constexpr int S_COL = 0;
    static constexpr int O_COL = 128;
    // shared memory: ring, Q, P hi, P lo (1024-byte aligned), then barriers and the table
    static constexpr int OFF_Q = NSLOTS * SLOT_BYTES;
    static constexpr int OFF_PH = OFF_Q + Q_BYTES;
    static constexpr int OFF_PL = OFF_PH + P_BYTES;
    static constexpr int OFF_BAR = OFF_PL + P_BYTES;
    // barriers: full[NSLOTS], empty[NSLOTS], q_full, q_empty, s_full, p_full, o_full, o_empty, drain
    static constexpr int NBAR = 2 * NSLOTS + 7;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;      // allocated TMEM address
    static constexpr int OFF_ABORT = OFF_TMEM + 4;
    static constexpr int OFF_TABLE = (OFF_ABORT + 4 + 15) / 16 * 16;
    static constexpr int MAX_TABLE = 1024 / 8;
    static constexpr size_t SMEM = 1024 + (size_t)OFF_TABLE + MAX_TABLE * 4;
    static constexpr int THREADS = 6 * 32;
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(SLOT_BYTES % 1024 == 0 && Q_BYTES % 1024 == 0 && P_BYTES % 1024 == 0, "1024-byte atoms");
};

template <typename T, int D>
__global__ void __launch_bounds__(VerifyTcCfg<T, D>::THREADS, 2)
    verify_tc_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                     const __grid_constant__ CUtensorMap tmap_v) {
    using C = VerifyTcCfg<T, D>;
    using Tr = ElemTraits<T>;
    using MO = MmaOps<T>;
    constexpr bool BF16 = sizeof(T) == 2 && !std::is_same<T, __half>::value;
    constexpr uint32_t IDESC_S = tc::idesc_f16(BF16, false, C::M, C::SLOT_ROWS);
    constexpr uint32_t IDESC_PV = tc::idesc_f16(BF16, true, C::M, D);
    constexpr int KS = D / 16;
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* bar = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
    uint64_t* full = bar;
    uint64_t* empty = bar + C::NSLOTS;
    uint64_t* q_full = bar + 2 * C::NSLOTS;      // Q tile written (128 arrivals)
    uint64_t* q_empty = q_full + 1;              // last S of the item done (commit)
    uint64_t* s_full = q_full + 2;               // S of a chunk done (commit)
    uint64_t* p_full = q_full + 3;               // S read and p written (128 arrivals)
    uint64_t* o_full = q_full + 4;               // P.V of a chunk done (commit)
    uint64_t* o_empty = q_full + 5;              // O read by the epilogue (128 arrivals)
    uint64_t* drain = q_full + 6;                // every MMA done, before TMEM is freed
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
    int32_t* tbl = reinterpret_cast<int32_t*>(smem + C::OFF_TABLE);
    unsigned char* qs = smem + C::OFF_Q;
    unsigned char* ph = smem + C::OFF_PH;
    unsigned char* pl = smem + C::OFF_PL;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NSLOTS; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 1);
        }
        mbar_init(q_full, 128);
        mbar_init(q_empty, 1);
        mbar_init(s_full, 1);
        mbar_init(p_full, 128);
        mbar_init(o_full, 1);
        mbar_init(o_empty, 128);
        mbar_init(drain, 1);
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
    const int pairs = a.max_partitions == 1 ? a.num_seqs : *a.plan_count;
    const int total = pairs * a.num_kv_heads * a.n_gchunks;
    const int bs = 1 << a.log2_bs;
    const int box_bytes = bs * 128;

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmap_k);
            prefetch_tmap(&tmap_v);
        }
        const uint64_t policy = l2_policy_evict_first();
        uint32_t slot_seq = 0;
        bool ok = true;
        for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
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
            const int nst = (w.n + C::SLOT_ROWS - 1) / C::SLOT_ROWS;
            for (int c0 = 0; c0 < nst && ok; c0 += C::CPS) {
                const int nsl = min(C::CPS, nst - c0);
                for (int pass = 0; pass < 2 && ok; ++pass) {          // K slots of the chunk, then V slots
                    const void* tmap = pass ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k);
                    for (int j = 0; j < nsl; ++j, ++slot_seq) {
                        const int st = c0 + j;
                        const int slot = slot_seq % C::NSLOTS;
                        if (!mbar_wait(&empty[slot], ((slot_seq / C::NSLOTS) & 1u) ^ 1u, abort_flag)) {
                            ok = false;
                            break;
                        }
                        const int rows = min(C::SLOT_ROWS, w.n - st * C::SLOT_ROWS);
                        const int nb = (rows + bs - 1) >> a.log2_bs;       // whole blocks
                        const int nbox = nb * C::NH;
                        if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)(nbox * box_bytes));
                        __syncwarp();
                        if (lane < nbox) {
                            const int half = lane / nb;                     // slice
                            const int b = lane - half * nb;                 // block within the slot
                            const int phys = tbl[((st * C::SLOT_ROWS) >> a.log2_bs) + b];
                            tma_load_3d(smem + slot * C::SLOT_BYTES + half * C::SLICE_BYTES + b * box_bytes, tmap,
                                        half * C::BOX_ELEMS, w.h, phys * bs, &full[slot], policy);
                        }
                    }
                }
            }
        }
        if (!ok) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            const uint32_t issued = slot_seq;
            for (int slot = lane; slot < C::NSLOTS; slot += 32) {
                if ((uint32_t)slot < issued) {
                    const uint32_t last = issued - 1 - ((issued - 1 - slot) % C::NSLOTS);
                    const volatile int never = 0;
                    mbar_wait(&full[slot], (last / C::NSLOTS) & 1u, &never);
                }
            }
        }
    }
    if (warp == 1) {
        // ------------------------------------------------------------ MMA issue
        uint32_t slot_seq = 0, q_ph = 0, p_ph = 0, oe_ph = 0;
        bool ok = true;
        const uint32_t qb = smem_addr(qs), phb = smem_addr(ph), plb = smem_addr(pl);
        for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
            const WorkItem w = decode_item(a, i, false);
            if (w.n == 0) continue;
            if (!mbar_wait(q_full, q_ph, abort_flag)) {
                ok = false;
                break;
            }
            q_ph ^= 1u;
            tc::fence_after_sync();
            const int nst = (w.n + C::SLOT_ROWS - 1) / C::SLOT_ROWS;
            for (int c0 = 0; c0 < nst && ok; c0 += C::CPS) {
                const int nsl = min(C::CPS, nst - c0);
                // S = Q K^T for the chunk's slots (S columns were released by the previous p_full)
                for (int j = 0; j < nsl; ++j, ++slot_seq) {
                    const int slot = slot_seq % C::NSLOTS;
                    if (!mbar_wait(&full[slot], (slot_seq / C::NSLOTS) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    tc::fence_after_sync();
                    if (lane == 0) {
                        const uint32_t kb = smem_addr(smem + slot * C::SLOT_BYTES);
#pragma unroll
                        for (int kk = 0; kk < KS; ++kk) {
                            const uint32_t koff = (kk >> 2) * C::SLICE_BYTES + (kk & 3) * 32;
                            const uint32_t qoff = (kk >> 2) * C::Q_SLICE + (kk & 3) * 32;
                            tc::mma_ss(tmem + C::S_COL + j * C::SLOT_ROWS, tc::sw128_desc(qb + qoff, 16, 1024),
                                       tc::sw128_desc(kb + koff, 16, 1024), IDESC_S, kk > 0);
                        }
                        tc::commit(&empty[slot]);             // the K slot is free once these are done
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) {
                    tc::commit(s_full);
                    if (c0 + C::CPS >= nst) tc::commit(q_empty);   // last S of the item: Q may be replaced
                }
                __syncwarp();
                // O += P V once p is written (and, for the item's first chunk, once the
                // previous item's O has been read out)
                if (!mbar_wait(p_full, p_ph, abort_flag)) {
                    ok = false;
                    break;
                }
                p_ph ^= 1u;
                if (c0 == 0) {
                    if (!mbar_wait(o_empty, oe_ph ^ 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    oe_ph ^= 1u;
                }
                tc::fence_after_sync();
                for (int j = 0; j < nsl; ++j, ++slot_seq) {
                    const int slot = slot_seq % C::NSLOTS;
                    if (!mbar_wait(&full[slot], (slot_seq / C::NSLOTS) & 1u, abort_flag)) {
                        ok = false;
                        break;
                    }
                    const int st = c0 + j;
                    const int rows = min(C::SLOT_ROWS, w.n - st * C::SLOT_ROWS);
                    if (rows < C::SLOT_ROWS) {
                        // rows past the partition (stale or unwritten pool rows, maybe NaN):
                        // zero them so p = 0 meets finite values
                        uint4* vrow = reinterpret_cast<uint4*>(smem + slot * C::SLOT_BYTES);
                        for (int e = lane; e < C::NH * C::SLOT_ROWS * 8; e += 32) {
                            const int r = (e >> 3) % C::SLOT_ROWS;
                            if (r >= rows) vrow[e] = make_uint4(0u, 0u, 0u, 0u);
                        }
                        tc::fence_proxy_async_smem();
                    }
                    __syncwarp();
                    tc::fence_after_sync();
                    if (lane == 0) {
                        const uint32_t vb = smem_addr(smem + slot * C::SLOT_BYTES);
#pragma unroll
                        for (int ks = 0; ks < 2; ++ks) {                  // 16 tokens per MMA
                            const int tk = j * C::SLOT_ROWS + ks * 16;        // token within the chunk
                            const uint32_t poff = (tk >> 6) * C::P_ATOM + (tk & 63) * 2;
                            const uint64_t bdesc = tc::sw128_desc(vb + ks * 16 * 128, C::SLICE_BYTES, 1024);
                            const bool acc = !(c0 == 0 && j == 0 && ks == 0);
                            tc::mma_ss(tmem + C::O_COL, tc::sw128_desc(phb + poff, 16, 1024), bdesc, IDESC_PV, acc);
                            tc::mma_ss(tmem + C::O_COL, tc::sw128_desc(plb + poff, 16, 1024), bdesc, IDESC_PV, true);
                        }
                        tc::commit(&empty[slot]);
                    }
                    __syncwarp();
                }
                if (!ok) break;
                if (lane == 0) tc::commit(o_full);
                __syncwarp();
            }
        }
        if (!ok) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
        }
        // drain: every MMA issued above has completed before TMEM is released
        if (lane == 0) tc::commit(drain);
        __syncwarp();
        const volatile int never = 0;
        mbar_wait(drain, 0, &never);
    }
    if (warp >= 2) {
        // ------------------------------------------------- softmax and epilogue
        const int ctid = threadIdx.x - 64;               // 0..127
        const int quarter = warp & 3;                    // TMEM lanes 32*quarter .. +31
        const int m = quarter * 16 + lane;               // accumulator row of this thread (lane < 16)
        const bool holds_row = lane < 16;
        const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
        const T* qg = static_cast<const T*>(a.q);
        T* outg = static_cast<T*>(a.out);
        const int Q = a.num_queries;
        const int R = a.group * Q;
        uint32_t qe_ph = 0, s_ph = 0, o_ph = 0;
        bool ok = true;
        for (int i = blockIdx.x; i < total && ok; i += gridDim.x) {
            const WorkItem w = decode_item(a, i, false);
            const int ctx = clamp_context(a, w.s, false);
            const int r0 = w.gc * C::M;
            const int nr = min(C::M, R - r0);
            auto row_of = [&](int lr, int64_t& orow, int& pos) {
                if (lr >= nr) {
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
            if (w.n == 0) {                              // empty context: zero rows
                for (int e = ctid; e < nr * D; e += 128) {
                    int64_t orow;
                    int pos;
                    row_of(e / D, orow, pos);
                    outg[orow * D + (e % D)] = Tr::from_float(0.f);
                }
                continue;
            }
            // ---- stage this item's query rows as the A tile (rows past the chunk are zero),
            // once the previous item's last S product no longer reads the tile
            if (!mbar_wait(q_empty, qe_ph ^ 1u, abort_flag)) {
                ok = false;
                break;
            }
            qe_ph ^= 1u;
            {
                constexpr int VPR = D * 2 / 16;           // 16-byte chunks per row
                for (int e = ctid; e < C::M * VPR; e += 128) {
                    const int lr = e / VPR;
                    const int cc = e - lr * VPR;
                    int64_t orow;
                    int pos;
                    row_of(lr, orow, pos);
                    uint4 v = make_uint4(0u, 0u, 0u, 0u);
                    if (orow >= 0) v = __ldg(reinterpret_cast<const uint4*>(qg + orow * D) + cc);
                    *reinterpret_cast<uint4*>(qs + (cc >> 3) * C::Q_SLICE + lr * 128 + (((cc & 7) ^ (lr & 7)) << 4)) = v;
                }
                tc::fence_proxy_async_smem();
                mbar_arrive(q_full);
            }
            int64_t orow;
            int pos;
            row_of(m, orow, pos);
            if (!holds_row) pos = -1;
            float m_run = -INFINITY, l_run = 0.f;
            const int nst = (w.n + C::SLOT_ROWS - 1) / C::SLOT_ROWS;
            for (int c0 = 0; c0 < nst && ok; c0 += C::CPS) {
                const int nsl = min(C::CPS, nst - c0);
                const int tok0 = c0 * C::SLOT_ROWS;          // chunk's first token within the partition
                if (!mbar_wait(s_full, s_ph, abort_flag)) {
                    ok = false;
                    break;
                }
                s_ph ^= 1u;
                tc::fence_after_sync();
                // pass 1: exact max of the chunk's visible scores (base-2 units)
                float cmax = -INFINITY;
                for (int g = 0; g < nsl; ++g) {
                    uint32_t r[32];
                    tc::ld32(tmem + lane_addr + C::S_COL + g * 32, r);
                    tc::wait_ld();
#pragma unroll
                    for (int k = 0; k < 32; ++k) {
                        const int t = tok0 + g * 32 + k;
                        if (t < w.n && w.t0 + t <= pos) cmax = fmaxf(cmax, __uint_as_float(r[k]) * a.scale_log2);
                    }
                }
                const float m_new = fmaxf(m_run, cmax);
                const float base = m_new == -INFINITY ? 0.f : m_new;       // a row that saw nothing yet
                const float corr = exp2f(m_run - base);
                // the previous chunk's P.V must be done before O is rescaled and p rewritten
                if (c0 > 0) {
                    if (!mbar_wait(o_full, o_ph, abort_flag)) {
                        ok = false;
                        break;
                    }
                    o_ph ^= 1u;
                    tc::fence_after_sync();
                    if (__any_sync(0xffffffffu, holds_row && corr != 1.f)) {
                        for (int g = 0; g < D / 32; ++g) {
                            uint32_t r[32];
                            tc::ld32(tmem + lane_addr + C::O_COL + g * 32, r);
                            tc::wait_ld();
#pragma unroll
                            for (int k = 0; k < 32; ++k) r[k] = __float_as_uint(__uint_as_float(r[k]) * corr);
                            tc::st32(tmem + lane_addr + C::O_COL + g * 32, r);
                        }
                        tc::wait_st();
                    }
                }
                m_run = m_new;
                l_run *= corr;
                // pass 2: p = 2^(z - base) as a 16-bit value and its remainder, row m of the P tiles
                for (int g = 0; g < C::CPS; ++g) {
                    uint32_t r[32];
                    if (g < nsl) {
                        tc::ld32(tmem + lane_addr + C::S_COL + g * 32, r);
                        tc::wait_ld();
                    }
                    uint32_t hi[16], lo[16];
#pragma unroll
                    for (int k = 0; k < 32; k += 2) {
                        float p0 = 0.f, p1 = 0.f;
                        if (g < nsl) {
                            const int t = tok0 + g * 32 + k;
                            if (t < w.n && w.t0 + t <= pos) p0 = exp2f(__uint_as_float(r[k]) * a.scale_log2 - base);
                            if (t + 1 < w.n && w.t0 + t + 1 <= pos)
                                p1 = exp2f(__uint_as_float(r[k + 1]) * a.scale_log2 - base);
                        }
                        l_run += p0 + p1;
                        split_pack<MO>(p0, p1, hi[k >> 1], lo[k >> 1]);
                    }
                    if (holds_row) {
                        // tokens g*32 .. g*32+31 of the chunk: 4 chunks of 16 bytes in atom (g / 2)
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int cc = (g & 1) * 4 + c;                  // 16-byte chunk within the atom row
                            const int off = (g >> 1) * C::P_ATOM + m * 128 + ((cc ^ (m & 7)) << 4);
                            *reinterpret_cast<uint4*>(ph + off) = make_uint4(hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
                            *reinterpret_cast<uint4*>(pl + off) = make_uint4(lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
                        }
                    }
                }
                tc::fence_proxy_async_smem();
                tc::fence_before_sync();
                mbar_arrive(p_full);
            }
            if (!ok) break;
            // ---- epilogue: O of the last chunk, normalised row or partition partials
            if (!mbar_wait(o_full, o_ph, abort_flag)) {
                ok = false;
                break;
            }
            o_ph ^= 1u;
            tc::fence_after_sync();
            const bool single = w.np == 1;
            for (int g = 0; g < D / 32; ++g) {
                uint32_t r[32];
                tc::ld32(tmem + lane_addr + C::O_COL + g * 32, r);
                tc::wait_ld();
                if (holds_row && orow >= 0) {
                    if (single) {
                        uint32_t packed[16];
#pragma unroll
                        for (int k = 0; k < 32; k += 2) {
                            const float o0 = l_run > 0.f ? __uint_as_float(r[k]) / l_run : 0.f;
                            const float o1 = l_run > 0.f ? __uint_as_float(r[k + 1]) / l_run : 0.f;
                            packed[k >> 1] = MO::pack(o0, o1);
                        }
                        uint4* dst = reinterpret_cast<uint4*>(outg + orow * D + g * 32);
#pragma unroll
                        for (int c = 0; c < 4; ++c)
                            dst[c] = make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
                    } else {
                        const int64_t pidx = orow * a.max_partitions + w.p;
                        float4* dst = reinterpret_cast<float4*>(a.part_o + pidx * D + g * 32);
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            dst[c] = make_float4(__uint_as_float(r[4 * c]), __uint_as_float(r[4 * c + 1]),
                                                 __uint_as_float(r[4 * c + 2]), __uint_as_float(r[4 * c + 3]));
                    }
                }
            }
            if (!single && holds_row && orow >= 0) {
                const int64_t pidx = orow * a.max_partitions + w.p;
                a.part_m[pidx] = m_run;
                a.part_l[pidx] = l_run;
            }
            tc::fence_before_sync();
            mbar_arrive(o_empty);
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
