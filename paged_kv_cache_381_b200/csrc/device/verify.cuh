// Multi-query paged attention for sm_100a: the target model's verification
// pass of speculative decoding.
//
// What is computed ("大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache
// 实战拆解", section 5: a draft model proposes a handful of candidate tokens and
// the target model checks them in one parallel pass): each sequence brings Q
// query rows per head whose K/V are already the last Q positions of its paged
// context.  Query i of sequence s sits at position p = ctx_s - Q + i and
// attends causally to positions 0..p:
//     out[s][i][h] = sum_{t <= p} softmax_t(scale * q[s][i][h] . K_s[t][g]) V_s[t][g],  g = h / G.
//
// Design (B200).  One kv head of one sequence carries R = G * Q query rows
// (48 for a 70B-shaped GQA-8 model verifying 6 tokens), so every K/V row read
// from HBM feeds R dot products: enough arithmetic that the tensor cores take
// both products.
//  * Work item = (sequence, context partition, kv head, chunk of <= 64 rows);
//    items are ordered and split exactly as in decode (plan kernel, partials,
//    log-sum-exp reduce kernel), with the partial rows indexed [s][i][h].
//  * One producer warp streams a partition's K and V rows together, 32 tokens
//    per ring slot, through tiled TMA boxes (the pool seen as a 3-D tensor,
//    128-byte swizzle), completion on mbarriers with transaction counts.
//  * Four consumer warps own the chunk's 16-row tiles.  When a chunk has fewer
//    than four tiles, the warps of a tile split the slots among themselves
//    (slot st goes to warp st mod warps_per_tile) and merge at the end.  Per
//    slot and tile, with mma.m16n8k16 (fp32 accumulate):
//        S[16 q x 32 tok] = Q[16 x D] . K^T         (A = q in registers, B = K via ldmatrix)
//        online softmax over the slot (running max, base 2, causal mask)
//        O[16 q x D]     += P[16 x 32] . V[32 x D]   (A = p from the S fragments, split into a
//                                                     16-bit value and its remainder; B = V via
//                                                     ldmatrix.trans)
//  * Every consumer warp waits on every slot and releases it (the empty
//    barrier counts all four), so a slot is refilled only after all warps
//    are past it; all waits are bounded.
#pragma once

#include "decode.cuh"

namespace pa_dev {

#ifndef PA_VERIFY_STAGES
#define PA_VERIFY_STAGES 4
#endif

template <typename T, int D>
struct VerifyCfg {
    static constexpr int ELT = (int)sizeof(T);
    static constexpr int ROW_BYTES = D * ELT;
    static constexpr int NH = ROW_BYTES / 128;              // 128-byte slices of a row
    static constexpr int BOX_ELEMS = 128 / ELT;
    static constexpr int STAGE_ROWS = 32;                   // tokens per slot
    static constexpr int HALF_BYTES = STAGE_ROWS * ROW_BYTES;   // K, then V
    static constexpr int SLOT_BYTES = 2 * HALF_BYTES;
    static constexpr int NSTAGES = PA_VERIFY_STAGES;
    static constexpr int NCW = 4;                           // consumer warps
    static constexpr int THREADS = (NCW + 1) * 32;
    static constexpr int ROWS = 16 * NCW;                   // query rows per item
    static constexpr int MAX_TABLE = DecodeCfg<T, D, 8, true>::MAX_TABLE;
    static constexpr int OFF_FULL = NSTAGES * SLOT_BYTES;
    static constexpr int OFF_EMPTY = OFF_FULL + NSTAGES * 8;
    static constexpr int OFF_TABLE = OFF_EMPTY + NSTAGES * 8;
    static constexpr int OFF_STATS = OFF_TABLE + MAX_TABLE * 4;   // m, l [NCW][16], abort
    static constexpr int OFF_RED = ((OFF_STATS + (2 * NCW * 16 + 4) * 4) + 127) / 128 * 128;
    static constexpr int RED_STRIDE = D + 8;                // floats per row (spreads banks)
    static constexpr int RED_BYTES = NCW * 16 * RED_STRIDE * 4;
    // The item's query rows wait in shared memory (not registers) while its
    // slots stream by, in the region the epilogue later uses for the warps'
    // partial outputs; rows padded by 16 bytes so ldmatrix rows spread over banks.
    static constexpr int Q_STRIDE = D * ELT + 16;
    static_assert(ROWS * Q_STRIDE <= RED_BYTES, "query tile must fit the merge buffer");
    static constexpr size_t SMEM = 1024 + (size_t)OFF_RED + RED_BYTES;
    static_assert(ELT == 2, "tensor path: fp16 / bf16");
    static_assert(ROW_BYTES % 128 == 0 && HALF_BYTES % 1024 == 0, "swizzled boxes need 1024-byte alignment");
    // Every consumer warp waits on every use of every slot in order and releases
    // it, so a warp never tests a slot's full barrier more than one phase ahead
    // of it: any ring depth is safe here.
    static_assert(NSTAGES >= 2, "ring depth");
};

// Fragment layouts (PTX m16n8k16, gid = lane / 4, tig = lane % 4):
//   A regs {row gid | gid+8} x {k 2tig..2tig+1 | +8};  B reg0 = (k 2tig..2tig+1, n gid), reg1 = k + 8;
//   C = (row gid | gid+8, n 2tig | 2tig+1).
template <typename T, int D>
__global__ void __launch_bounds__(VerifyCfg<T, D>::THREADS, 2)
    verify_kernel(const DecodeArgs a, const __grid_constant__ CUtensorMap tmap_k,
                  const __grid_constant__ CUtensorMap tmap_v) {
    using C = VerifyCfg<T, D>;
    using Tr = ElemTraits<T>;
    using M = MmaOps<T>;
    constexpr int KS = D / 16;          // k-steps of S over head_dim
    constexpr int DT = D / 8;           // n8 tiles of O over head_dim
    extern __shared__ __align__(1024) unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_FULL);
    uint64_t* empty = reinterpret_cast<uint64_t*>(smem + C::OFF_EMPTY);
    int32_t* tbl = reinterpret_cast<int32_t*>(smem + C::OFF_TABLE);
    float* wm = reinterpret_cast<float*>(smem + C::OFF_STATS);      // [NCW][16] row max
    float* wl = wm + C::NCW * 16;                                    // [NCW][16] row sum
    volatile int* abort_flag = reinterpret_cast<volatile int*>(wl + C::NCW * 16);
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);        // [NCW][16][RED_STRIDE]
    unsigned char* qs = smem + C::OFF_RED;                           // [ROWS][Q_STRIDE] bytes, same region

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < C::NSTAGES; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], C::NCW);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    grid_dependency_wait();
    const int pairs = a.max_partitions == 1 ? a.num_seqs : *a.plan_count;
    const int total = pairs * a.num_kv_heads * a.n_gchunks;
    const int bs = 1 << a.log2_bs;
    const int box_bytes = bs * 128;
    auto row_base = [&](int r) -> int {
        return ((r >> a.log2_bs) * C::NH) * box_bytes + (r & (bs - 1)) * 128;
    };

    if (warp == C::NCW) {
        // ------------------------------------------------------------ producer
        if (lane == 0) {
            prefetch_tmap(&tmap_k);
            prefetch_tmap(&tmap_v);
        }
        const uint64_t policy = l2_policy_evict_first();
        uint32_t stage = 0;
        bool ok = true;
        for (int i = walk_first(); i < total && ok; i = walk_next(i)) {
            const WorkItem w = decode_item(a, i, lane == 0);
            if (w.n == 0) continue;
            const int nst = (w.n + C::STAGE_ROWS - 1) / C::STAGE_ROWS;
            const int nblk = (w.n + bs - 1) >> a.log2_bs;
            const int32_t* trow = a.block_tables + (int64_t)w.s * a.max_blocks_per_seq + (w.t0 >> a.log2_bs);
            __syncwarp();               // the previous item's table reads are done
            for (int j = lane; j < nblk; j += 32) {
                int32_t id = trow[j];
                if (id < 0 || id >= a.num_blocks) {
                    flag_error(PA_DEVERR_BLOCK_ID);
                    id = 0;
                }
                tbl[j] = id;
            }
            __syncwarp();
            for (int st = 0; st < nst; ++st, ++stage) {
                const int slot = stage % C::NSTAGES;
                const uint32_t parity = ((stage / C::NSTAGES) & 1u) ^ 1u;
                if (!mbar_wait_warp(&empty[slot], parity, abort_flag)) {
                    ok = false;
                    break;
                }
                const int rows = min(C::STAGE_ROWS, w.n - st * C::STAGE_ROWS);
                const int nbox = ((rows + bs - 1) >> a.log2_bs) * C::NH;    // whole blocks, K and V each
                if (lane == 0) mbar_arrive_expect_tx(&full[slot], (uint32_t)(2 * nbox * box_bytes));
                __syncwarp();
                if (lane < 2 * nbox) {
                    const int kv = lane >= nbox;                 // 0: K box, 1: V box
                    const int idx = lane - kv * nbox;
                    const int b = idx / C::NH;
                    const int half = idx - b * C::NH;
                    const int phys = tbl[((st * C::STAGE_ROWS) >> a.log2_bs) + b];
                    tma_load_3d(smem + slot * C::SLOT_BYTES + kv * C::HALF_BYTES + idx * box_bytes,
                                kv ? static_cast<const void*>(&tmap_v) : static_cast<const void*>(&tmap_k),
                                half * C::BOX_ELEMS, w.h, phys * bs, &full[slot], policy);
                }
            }
        }
        if (!ok) {
            if (lane == 0) flag_error(PA_DEVERR_TIMEOUT);
            *abort_flag = 1;
            const uint32_t issued = stage;
            for (int slot = lane; slot < C::NSTAGES; slot += 32) {
                if ((uint32_t)slot < issued) {
                    const uint32_t last = issued - 1 - ((issued - 1 - slot) % C::NSTAGES);
                    const volatile int never = 0;
                    mbar_wait(&full[slot], (last / C::NSTAGES) & 1u, &never);
                }
            }
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    constexpr int NCT = C::NCW * 32;
    const int ctid = threadIdx.x;
    const int gid = lane >> 2;
    const int tig = lane & 3;
    const T* qg = static_cast<const T*>(a.q);
    T* outg = static_cast<T*>(a.out);
    const int Q = a.num_queries;
    const int R = a.group * Q;                  // query rows per kv head
    uint32_t stage = 0;
    auto acquire = [&](uint32_t c) -> bool {
        const int slot = c % C::NSTAGES;
        const bool got = !*abort_flag && mbar_wait(&full[slot], (c / C::NSTAGES) & 1u, abort_flag);
        if (!warp_uniform(got)) {
            *abort_flag = 1;
            return false;
        }
        return true;
    };
    auto release = [&](uint32_t c) {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[c % C::NSTAGES]);
    };

    for (int i = walk_first(); i < total; i = walk_next(i)) {
        const WorkItem w = decode_item(a, i, false);
        const int ctx = clamp_context(a, w.s, false);
        const int r0 = w.gc * C::ROWS;
        const int nr = min(C::ROWS, R - r0);          // rows of this chunk
        const int RT = (nr + 15) >> 4;                // 16-row tiles
        const int WPR = RT == 1 ? 4 : (RT == 2 ? 2 : 1);
        const int rt = warp / WPR;
        const int wj = warp - rt * WPR;
        const bool active = rt < RT;
        // output row and position of chunk-local row lr; -1 for rows past the chunk
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
        if (w.n == 0) {                               // empty context: zero rows
            for (int e = ctid; e < nr * D; e += NCT) {
                int64_t orow;
                int pos;
                row_of(e / D, orow, pos);
                outg[orow * D + (e % D)] = Tr::from_float(0.f);
            }
            continue;
        }
        int64_t orow_lo, orow_hi;
        int pos_lo, pos_hi;
        row_of(rt * 16 + gid, orow_lo, pos_lo);
        row_of(rt * 16 + gid + 8, orow_hi, pos_hi);
        // query rows of the chunk -> shared memory (rows past the chunk as zeros); the
        // previous item's epilogue ended with a barrier, so the region is free
        {
            constexpr int VPR = D * C::ELT / 16;                   // 16-byte vectors per row
            for (int e = ctid; e < C::ROWS * VPR; e += NCT) {
                const int lr = e / VPR;
                const int vcol = e - lr * VPR;
                int64_t orow;
                int pos;
                row_of(lr, orow, pos);
                uint4 v = make_uint4(0u, 0u, 0u, 0u);
                if (orow >= 0) v = __ldg(reinterpret_cast<const uint4*>(qg + orow * D) + vcol);
                *reinterpret_cast<uint4*>(qs + lr * C::Q_STRIDE + vcol * 16) = v;
            }
            named_barrier(1, NCT);
        }
        // ldmatrix address of this lane in the warp's 16-row query tile: matrix lane/8 ->
        // (+8 rows if odd, +8 columns if >= 2)
        const uint32_t qaddr = smem_addr(qs) + (rt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * C::Q_STRIDE +
                               (lane >> 4) * 16;
        float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
        float oacc[DT][4];
#pragma unroll
        for (int dt = 0; dt < DT; ++dt) oacc[dt][0] = oacc[dt][1] = oacc[dt][2] = oacc[dt][3] = 0.f;
        const int nst = (w.n + C::STAGE_ROWS - 1) / C::STAGE_ROWS;
        const int x = lane & 7;                                   // swizzle key of the lane's ldmatrix row
        const int krow = (lane & 7) + ((lane >> 4) & 1) * 8;      // K: tokens 0-7 | 8-15 for matrices 2, 3
        const int kch = (lane >> 3) & 1;                          // K: +1 chunk for matrices 1, 3
        const int vrow = (lane & 7) + ((lane >> 3) & 1) * 8;      // V: tokens 8-15 for matrices 1, 3
        const int vch = lane >> 4;                                // V: +1 chunk for matrices 2, 3
        for (int st = 0; st < nst; ++st) {
            const uint32_t c = stage + st;
            if (!acquire(c)) continue;
            if (active && (st % WPR) == wj) {
                const int rows = min(C::STAGE_ROWS, w.n - st * C::STAGE_ROWS);
                const int tb = w.t0 + st * C::STAGE_ROWS;             // position of slot row 0
                const uint32_t kb = smem_addr(smem + (c % C::NSTAGES) * C::SLOT_BYTES);
                const uint32_t vb = kb + C::HALF_BYTES;
                // ---- S = Q K^T over the slot's 32 tokens (4 n-tiles).  Even and odd
                // k-steps accumulate separately: 8 independent mma chains of depth
                // KS / 2 instead of 4 of depth KS.  Rows past the partition are
                // computed too and masked below.
                float sc[4][4], se[4][4];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
                    se[nt][0] = se[nt][1] = se[nt][2] = se[nt][3] = 0.f;
                }
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    const int cidx = 2 * kk + kch;
                    const uint32_t off = (cidx >> 3) * box_bytes + (((cidx & 7) ^ x) << 4);
                    uint32_t qf[4];
                    ldsm_x4(qaddr + kk * 32, qf[0], qf[1], qf[2], qf[3]);
#pragma unroll
                    for (int np = 0; np < 2; ++np) {
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(kb + row_base(np * 16 + krow) + off, b0, b1, b2, b3);
                        float (&c0)[4] = (kk & 1) ? se[2 * np] : sc[2 * np];
                        float (&c1)[4] = (kk & 1) ? se[2 * np + 1] : sc[2 * np + 1];
                        M::mma(c0, qf, b0, b1);
                        M::mma(c1, qf, b2, b3);
                    }
                }
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    sc[nt][0] += se[nt][0];
                    sc[nt][1] += se[nt][1];
                    sc[nt][2] += se[nt][2];
                    sc[nt][3] += se[nt][3];
                }
                // ---- causal mask, slot max, rescale of the running state
                float mx_lo = -INFINITY, mx_hi = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int tt = nt * 8 + 2 * tig + (e & 1);
                        const int pos = e < 2 ? pos_lo : pos_hi;
                        const float z = (tt < rows && tb + tt <= pos) ? sc[nt][e] * a.scale_log2 : -INFINITY;
                        sc[nt][e] = z;
                        if (e < 2)
                            mx_lo = fmaxf(mx_lo, z);
                        else
                            mx_hi = fmaxf(mx_hi, z);
                    }
                }
                mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
                mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
                mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
                const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
                const float base_lo = mn_lo == -INFINITY ? 0.f : mn_lo;   // a row that saw nothing yet
                const float base_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
                const float cl = exp2f(m_lo - base_lo), ch = exp2f(m_hi - base_hi);
                m_lo = mn_lo;
                m_hi = mn_hi;
                l_lo *= cl;
                l_hi *= ch;
#pragma unroll
                for (int dt = 0; dt < DT; ++dt) {
                    oacc[dt][0] *= cl;
                    oacc[dt][1] *= cl;
                    oacc[dt][2] *= ch;
                    oacc[dt][3] *= ch;
                }
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    sc[nt][0] = exp2f(sc[nt][0] - base_lo);
                    sc[nt][1] = exp2f(sc[nt][1] - base_lo);
                    sc[nt][2] = exp2f(sc[nt][2] - base_hi);
                    sc[nt][3] = exp2f(sc[nt][3] - base_hi);
                    l_lo += sc[nt][0] + sc[nt][1];
                    l_hi += sc[nt][2] + sc[nt][3];
                }
                // ---- O += P V (p as a 16-bit value plus its remainder: two mma per tile)
#pragma unroll
                for (int kc = 0; kc < 2; ++kc) {     // a k-chunk past the partition has p = 0 and masked V
                    uint32_t ah[4], al[4];
                    split_pack<M>(sc[2 * kc][0], sc[2 * kc][1], ah[0], al[0]);
                    split_pack<M>(sc[2 * kc][2], sc[2 * kc][3], ah[1], al[1]);
                    split_pack<M>(sc[2 * kc + 1][0], sc[2 * kc + 1][1], ah[2], al[2]);
                    split_pack<M>(sc[2 * kc + 1][2], sc[2 * kc + 1][3], ah[3], al[3]);
                    const bool whole = kc * 16 + 16 <= rows;
                    const int vlo = rows - (kc * 16 + 2 * tig);         // valid tokens from this lane's first
                    const uint32_t base = vb + row_base(kc * 16 + vrow);
#pragma unroll
                    for (int dp = 0; dp < D / 16; ++dp) {
                        const int cidx = 2 * dp + vch;
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4_trans(base + (cidx >> 3) * box_bytes + (((cidx & 7) ^ x) << 4), b0, b1, b2, b3);
                        if (!whole) {     // slot rows past the partition may hold stale bits (even NaN)
                            b0 = keep_pair(b0, vlo);
                            b1 = keep_pair(b1, vlo - 8);
                            b2 = keep_pair(b2, vlo);
                            b3 = keep_pair(b3, vlo - 8);
                        }
                        M::mma(oacc[2 * dp], ah, b0, b1);
                        M::mma(oacc[2 * dp], al, b0, b1);
                        M::mma(oacc[2 * dp + 1], ah, b2, b3);
                        M::mma(oacc[2 * dp + 1], al, b2, b3);
                    }
                }
            }
            release(c);
        }
        stage += nst;
        // ---- epilogue: complete the row sums, merge the warps of a tile, write
        l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
        l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
        l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
        l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
        if (WPR > 1) {
            if (active && tig == 0) {
                wm[warp * 16 + gid] = m_lo;
                wm[warp * 16 + gid + 8] = m_hi;
                wl[warp * 16 + gid] = l_lo;
                wl[warp * 16 + gid + 8] = l_hi;
            }
            named_barrier(1, NCT);
            if (active) {
                // tile max M, this warp's weight 2^(m - M), and the tile's sum
                float Mlo = -INFINITY, Mhi = -INFINITY;
                for (int j = 0; j < WPR; ++j) {
                    Mlo = fmaxf(Mlo, wm[(rt * WPR + j) * 16 + gid]);
                    Mhi = fmaxf(Mhi, wm[(rt * WPR + j) * 16 + gid + 8]);
                }
                const float blo = Mlo == -INFINITY ? 0.f : Mlo, bhi = Mhi == -INFINITY ? 0.f : Mhi;
                float Llo = 0.f, Lhi = 0.f;
                for (int j = 0; j < WPR; ++j) {     // fixed order: the same bits whichever warp sums
                    Llo += exp2f(wm[(rt * WPR + j) * 16 + gid] - blo) * wl[(rt * WPR + j) * 16 + gid];
                    Lhi += exp2f(wm[(rt * WPR + j) * 16 + gid + 8] - bhi) * wl[(rt * WPR + j) * 16 + gid + 8];
                }
                const float slo = exp2f(m_lo - blo), shi = exp2f(m_hi - bhi);
                float* rlo = red + (warp * 16 + gid) * C::RED_STRIDE + 2 * tig;
                float* rhi = rlo + 8 * C::RED_STRIDE;
#pragma unroll
                for (int dt = 0; dt < DT; ++dt) {
                    *reinterpret_cast<float2*>(rlo + dt * 8) = make_float2(oacc[dt][0] * slo, oacc[dt][1] * slo);
                    *reinterpret_cast<float2*>(rhi + dt * 8) = make_float2(oacc[dt][2] * shi, oacc[dt][3] * shi);
                }
                m_lo = Mlo;
                m_hi = Mhi;
                l_lo = Llo;
                l_hi = Lhi;
            }
            named_barrier(1, NCT);
            if (active && wj == 0) {
#pragma unroll
                for (int dt = 0; dt < DT; ++dt) {
                    float2 slo = make_float2(0.f, 0.f), shi = make_float2(0.f, 0.f);
                    for (int j = 0; j < WPR; ++j) {
                        const float* rl = red + ((rt * WPR + j) * 16 + gid) * C::RED_STRIDE + dt * 8 + 2 * tig;
                        const float2 u = *reinterpret_cast<const float2*>(rl);
                        const float2 v = *reinterpret_cast<const float2*>(rl + 8 * C::RED_STRIDE);
                        slo.x += u.x;
                        slo.y += u.y;
                        shi.x += v.x;
                        shi.y += v.y;
                    }
                    oacc[dt][0] = slo.x;
                    oacc[dt][1] = slo.y;
                    oacc[dt][2] = shi.x;
                    oacc[dt][3] = shi.y;
                }
            }
        }
        if (active && wj == 0) {
            const bool single = w.np == 1;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int64_t orow = half ? orow_hi : orow_lo;
                if (orow < 0) continue;
                const float m = half ? m_hi : m_lo;
                const float l = half ? l_hi : l_lo;
                if (single) {
                    T* dst = outg + orow * D + 2 * tig;
#pragma unroll
                    for (int dt = 0; dt < DT; ++dt) {
                        const float o0 = oacc[dt][2 * half], o1 = oacc[dt][2 * half + 1];
                        *reinterpret_cast<uint32_t*>(dst + dt * 8) =
                            M::pack(l > 0.f ? o0 / l : 0.f, l > 0.f ? o1 / l : 0.f);
                    }
                } else {
                    const int64_t pidx = orow * a.max_partitions + w.p;
                    float* dst = a.part_o + pidx * D + 2 * tig;
#pragma unroll
                    for (int dt = 0; dt < DT; ++dt)
                        *reinterpret_cast<float2*>(dst + dt * 8) = make_float2(oacc[dt][2 * half], oacc[dt][2 * half + 1]);
                    if (tig == 0) {
                        a.part_m[pidx] = m;
                        a.part_l[pidx] = l;
                    }
                }
            }
        }
        named_barrier(1, NCT);          // stats and partial buffers are free for the next item
    }
    grid_launch_dependents();
}

}  // namespace pa_dev
