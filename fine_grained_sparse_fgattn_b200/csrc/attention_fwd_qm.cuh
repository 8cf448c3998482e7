// Query-major tile-sparse attention forward for 128-row query blocks (sm_100a).
//
// Same operation and inputs as fgattn_fwd_kernel (kept-key lists per query
// block, "FG-Attn: Leveraging Fine-Grained Sparse Attention in Video Diffusion
// Models", Abstract: skipped M x N tiles count as -inf), for the case where a
// query block fills the tensor core's M = 128 rows by itself: M = 128 tiles,
// and dense runs (every key kept, any M: the result does not depend on M).
//
// Each work item is one block of 128 query rows; its kept keys are taken in
// chunks of 128:
//     S [128 q x 128 keys]  = Q_blk [128 x D] . K_chunk^T      (MMA1, A and B in shared memory)
//     O [128 q x D]        += P [128 x 128 keys] . V_chunk     (MMA2, A = P in TMEM, B = V in shared memory)
// Two softmax warpgroups each take half of a chunk's keys; a softmax thread
// owns one query row (one TMEM lane) and 64 scores of the chunk, so a row's
// maximum needs no cross-lane reduction: the two halves combine their maxima
// through shared memory with one barrier of the 256 softmax threads per chunk.  Probabilities are taken
// against a reference mref that is raised only when a row maximum exceeds it
// by more than TAU (log2 units); raising it rescales the row's partial sum and
// its O row in TMEM (warp-collective TMEM access, so a warp rescales when any
// of its rows needs it).  P goes back to TMEM as bf16 pairs (two buffers) and
// feeds MMA2 directly, so P never touches shared memory.
//
// Each softmax thread reads its 64 scores twice: all at once for the row
// maximum, then 32 at a time in a rolled loop for the probabilities.  With a
// single softmax warpgroup (128 scores per thread) the kernel measured about
// 7 % slower; the speed follows the size of the loop body: fully unrolled
// passes (scores kept in registers) and double-buffered loads measured 2-12 %
// slower, and 16-wide pieces or a rolled first pass 4-14 % slower.
//
// Warp roles (512 threads):
//   warps 0-7   softmax + epilogue: warpgroup g = keys [64 g, 64 g + 64) of every chunk,
//               thread t of a warpgroup = query row t = TMEM lane t
//   warp  8     TMEM allocation + single-thread tcgen05.mma issue (S of chunk c+2 before P.V of chunk c)
//   warps 9-11  K producer: query tile (TMA), K rows (TMA boxes for 16-key runs, gather4 otherwise);
//               two warps for lists of 16-key runs, three for row-by-row lists
//   warps 12-15 V producer: V rows (TMA boxes for 16-key runs, cp.async otherwise)
// TMEM columns: S slots [0, 128) and [128, 256), P buffers [256, 320) and [320, 384) (bf16 pairs),
// O [384, 384 + DP) (DP = D, or 128 at D = 96: zero-padded V columns).
// Every mbarrier wait is bounded; on timeout the block records an error bit,
// drains its copies and MMAs, frees TMEM and exits (as fgattn_fwd_kernel).
#pragma once

#include "attention_fwd.cuh"

namespace fgattn {

template <int D, bool GATHER>
struct QmCfg {
    using HD = HeadDim<D>;  // panels of Q/K, V and O padded to DP columns at D = 96
    static constexpr int DP = HD::DP;
    static constexpr int MQ = 128;              // query rows per block = MMA M
    static constexpr int KC = 128;              // keys per chunk = MMA1 N
    static constexpr int KWARPS = GATHER ? 3 : 2;
    static constexpr int KV_TILE = KC * DP * 2;  // bytes of a K or V chunk slot
    static constexpr int Q_TILE = MQ * DP * 2;   // query tile slot
    static constexpr int Q_TX = MQ * D * 2;      // bytes a query-tile load delivers
    static constexpr int NV = 2;  // V slot (c % 2) is free once P.V of chunk c-2 completed
    static constexpr int LIMIT = 227 * 1024 - 1024 - 256;
    static constexpr int XCH = 2 * 2 * 128 * 4 + 2 * 128 * 4;  // row maxima [2][2][128], row sums [2][128]
    static constexpr int MISC = 64 * 8 + 64 + XCH;
    static constexpr int NK = (4 * KV_TILE + NV * KV_TILE + Q_TILE + MISC <= LIMIT) ? 4
                              : (3 * KV_TILE + NV * KV_TILE + Q_TILE + MISC <= LIMIT) ? 3
                                                                                      : 2;
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + NK * KV_TILE;
    static constexpr int OFF_Q = OFF_V + NV * KV_TILE;
    static constexpr int OFF_XMAX = OFF_Q + Q_TILE;        // float [chunk parity][key half][row]
    static constexpr int OFF_XSUM = OFF_XMAX + 2 * 2 * 128 * 4;  // float [key half][row]
    static constexpr int OFF_BAR = OFF_XSUM + 2 * 128 * 4;
    // barriers: k_full[NK] k_empty[NK] v_full[NV] q_full q_empty s_full[2] s_free[2] p_full[2] o_done[2] o_empty drain
    static constexpr int B_KFULL = 0, B_KEMPTY = NK, B_VFULL = 2 * NK, B_QFULL = 2 * NK + NV, B_QEMPTY = B_QFULL + 1;
    static constexpr int B_SFULL = B_QFULL + 2, B_SFREE = B_SFULL + 2, B_PFULL = B_SFREE + 2;
    static constexpr int B_ODONE = B_PFULL + 2, B_OEMPTY = B_ODONE + 2, B_DRAIN = B_OEMPTY + 1, NBAR = B_DRAIN + 1;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 8;
    static constexpr int BYTES = OFF_ABORT + 8;
    static_assert(BYTES <= LIMIT, "shared memory layout");
    static constexpr int SMEM_REQUEST = BYTES + 1024;  // + alignment slack
    static constexpr uint32_t COL_S = 0, COL_P = 256, COL_O = 384, TMEM_COLS = 512;
    static constexpr int THREADS = 512;
    // Register split: 256 softmax threads x 160 + 256 others x 96 = 512 x 128 (the
    // launch's allocation at 512 threads per block, one block per SM).
    static constexpr uint32_t LAUNCH_REGS = 128, SOFT_REGS = 160, AUX_REGS = 96;
    static_assert(256 * SOFT_REGS + 256 * AUX_REGS <= THREADS * LAUNCH_REGS, "register split");
};

template <int D, bool GATHER, bool STRIDED, bool FUSED>
__global__ void __launch_bounds__(512, 1) fgattn_fwd_qm_kernel(const __grid_constant__ FwdParams p) {
    using C = QmCfg<D, GATHER>;
    constexpr int NK = C::NK, NV = C::NV, MQ = C::MQ;
    constexpr float TAU = 8.0f;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    auto KSLOT = [&](int i) { return sbase + C::OFF_K + (uint32_t)i * C::KV_TILE; };
    auto VSLOT = [&](int i) { return sbase + C::OFF_V + (uint32_t)i * C::KV_TILE; };
    const uint32_t QTILE = sbase + C::OFF_Q;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 8) {
        ptx::tmem_alloc(sbase + C::OFF_TMEM, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < NK; ++i) {
            ptx::mbar_init(BAR(C::B_KFULL + i), C::KWARPS);
            ptx::mbar_init(BAR(C::B_KEMPTY + i), 1);
        }
        for (int i = 0; i < NV; ++i) ptx::mbar_init(BAR(C::B_VFULL + i), 128);
        ptx::mbar_init(BAR(C::B_QFULL), 1);
        ptx::mbar_init(BAR(C::B_QEMPTY), 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(BAR(C::B_SFULL + i), 1);
            ptx::mbar_init(BAR(C::B_SFREE + i), 256);
            ptx::mbar_init(BAR(C::B_ODONE + i), 1);
        }
        ptx::mbar_init(BAR(C::B_PFULL), 256);
        ptx::mbar_init(BAR(C::B_PFULL + 1), 256);
        ptx::mbar_init(BAR(C::B_OEMPTY), 256);
        ptx::mbar_init(BAR(C::B_DRAIN), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::OFF_TMEM);
    const uint32_t tS = tmem + C::COL_S;
    const uint32_t tP = tmem + C::COL_P;
    const uint32_t tO = tmem + C::COL_O;
    const int64_t L = p.L;

    if (warp >= 9 && warp < 12) {
        // ===================================================== K producer (TMA)
        ptx::regs_dec<C::AUX_REGS>();
        const int kw = warp - 9;
        if (kw < C::KWARPS) {
            // segments of 16 keys per warp: 0-3 / 4-7 (two warps) or 0-2 / 3-5 / 6-7 (three);
            // four lanes (4-row groups) per segment
            const int seg0 = GATHER ? kw * 3 : kw * 4;
            const int nseg = GATHER ? (kw < 2 ? 3 : 2) : 4;
            const int g4 = seg0 * 4 + lane;  // this lane's 4-row group in the chunk
            const bool issuer = lane < nseg * 4;
            const int lseg = lane >> 2;
            int64_t g = 0, it = 0;
            int64_t issued = 0, q_issued = 0;
            bool ok = true;
            for (int64_t item = blockIdx.x; item < p.items && ok; item += gridDim.x, ++it) {
                const int64_t bh = item / p.QB;
                const int64_t qb = item - bh * p.QB;
                int32_t bi = 0, hi = 0;
                int64_t krow0 = bh * L;  // first gather-map row of this head's keys
                if constexpr (STRIDED) {
                    bi = (int32_t)(bh / p.H);
                    hi = (int32_t)(bh - (int64_t)bi * p.H);
                    krow0 = bi * p.k_ub + hi * p.k_uh;
                }
                MaskRow mr;
                const int64_t cnt = item_keys<FUSED, MQ>(p, item, kw == 0 && lane == 0, mr, lane);
                const int64_t nch = (cnt + 127) / 128;
                const int32_t* lst = p.kept_idx ? p.kept_idx + item * p.cap : nullptr;
                auto fetch4 = [&](int64_t c) -> int4 {  // this lane's four entries of chunk c (-1: none)
                    if constexpr (FUSED) {
                        const int4 e = fused_idx4(mr, c, g4, lane);  // every lane takes part
                        return issuer ? e : make_int4(-1, -1, -1, -1);
                    } else {
                        return issuer ? fetch_idx(lst, cnt, c, g4) : make_int4(-1, -1, -1, -1);
                    }
                };
                if (kw == 0) {  // the query tile (rows past L are padding; never stored)
                    const bool okq =
                        it == 0 || bounded_wait(BAR(C::B_QEMPTY), (uint32_t)((it - 1) & 1), abort_flag);
                    if (!__all_sync(0xffffffffu, okq)) {
                        ok = false;
                        break;
                    }
                    if (lane == 0) {
                        ptx::mbar_arrive_expect_tx(BAR(C::B_QFULL), (uint32_t)C::Q_TX);
#pragma unroll
                        for (int pn = 0; pn < C::HD::KP; ++pn) {
                            const CUtensorMap* qm = (C::HD::NARROW && pn == 1) ? &p.tmap_q_hi : &p.tmap_q;
                            if constexpr (STRIDED)
                                ptx::tma_load_4d(QTILE + (uint32_t)pn * (MQ * 128), qm, pn * 64, (int32_t)(qb * MQ),
                                                 hi, bi, BAR(C::B_QFULL));
                            else
                                ptx::tma_load_2d(QTILE + (uint32_t)pn * (MQ * 128), qm, pn * 64,
                                                 (int32_t)(bh * L + qb * MQ), BAR(C::B_QFULL));
                        }
                    }
                    ++q_issued;
                    __syncwarp();
                }
                constexpr int PF = 4;  // index prefetch distance in chunks (the lists live in HBM)
                int4 ring[PF];
                // fused kernels: no ring, the next chunk's entries are computed one chunk ahead (one
                // copy of the expansion code per producer keeps the instruction cache warm)
                int4 nxt = make_int4(-1, -1, -1, -1);
                if constexpr (FUSED) {
                    if (nch > 0) nxt = fetch4(0);
                } else {
#pragma unroll
                    for (int i = 0; i < PF; ++i) ring[i] = i < nch ? fetch4(i) : make_int4(-1, -1, -1, -1);
                }
                for (int64_t c = 0; c < nch; ++c) {
                    const int64_t gc = g + c;
                    const int st = (int)(gc % NK);
                    int4 cur;
                    if constexpr (FUSED) {
                        cur = nxt;
                        if (c + 1 < nch) nxt = fetch4(c + 1);
                    } else {
                        cur = ring[0];
#pragma unroll
                        for (int i = 0; i < PF - 1; ++i) ring[i] = ring[i + 1];
                        ring[PF - 1] = c + PF < nch ? fetch4(c + PF) : make_int4(-1, -1, -1, -1);
                    }
                    const bool okw =
                        gc < NK || bounded_wait(BAR(C::B_KEMPTY + st), (uint32_t)((gc / NK - 1) & 1), abort_flag);
                    if (!__all_sync(0xffffffffu, okw)) {
                        ok = false;
                        break;
                    }
                    // a segment is one TMA box when its 16 keys are real and consecutive
                    const int64_t j0 = c * 128 + 4 * g4;
                    const int32_t first = __shfl_sync(0xffffffffu, cur.x, lane & ~3);
                    const bool run = issuer && j0 + 3 < cnt && cur.x == first + 4 * (lane & 3) &&
                                     cur.y == cur.x + 1 && cur.z == cur.x + 2 && cur.w == cur.x + 3 && first >= 0 &&
                                     first + 15 < L;
                    const uint32_t runs = __ballot_sync(0xffffffffu, run);
                    const bool seg_run = ((runs >> (lseg * 4)) & 0xFu) == 0xFu;
                    if (lane == 0)
                        ptx::mbar_arrive_expect_tx(BAR(C::B_KFULL + st), (uint32_t)(nseg * 16 * D * 2));
                    __syncwarp();
                    if (issuer) {
                        // this lane's 4 rows in panel pn (rows of pitch(pn) bytes)
                        auto dst = [&](int pn) {
                            return KSLOT(st) + (uint32_t)pn * (128 * 128) + (uint32_t)g4 * 4u * C::HD::pitch(pn);
                        };
                        if (seg_run) {
                            if ((lane & 3) == 0) {
#pragma unroll
                                for (int pn = 0; pn < C::HD::KP; ++pn) {
                                    const CUtensorMap* km = (C::HD::NARROW && pn == 1) ? &p.tmap_k16_hi : &p.tmap_k16;
                                    if constexpr (STRIDED)
                                        ptx::tma_load_4d(dst(pn), km, pn * 64, first, hi, bi, BAR(C::B_KFULL + st));
                                    else
                                        ptx::tma_load_2d(dst(pn), km, pn * 64, (int32_t)(bh * L + first),
                                                         BAR(C::B_KFULL + st));
                                }
                            }
                        } else {
                            int32_t rows[4];
                            rows_of<STRIDED>(p, cur, krow0, true, rows);
#pragma unroll
                            for (int pn = 0; pn < C::HD::KP; ++pn)
                                ptx::tma_gather4(dst(pn), (C::HD::NARROW && pn == 1) ? &p.tmap_k_hi : &p.tmap_k,
                                                 pn * 64, rows[0], rows[1], rows[2], rows[3], BAR(C::B_KFULL + st));
                        }
                    }
                    ++issued;
                }
                g += nch;
            }
            // every load this warp issued has landed before the block exits
            for (int64_t i = issued > NK ? issued - NK : 0; i < issued; ++i)
                bounded_wait(BAR(C::B_KFULL + (int)(i % NK)), (uint32_t)((i / NK) & 1), abort_flag, false);
            if (q_issued > 0) bounded_wait(BAR(C::B_QFULL), (uint32_t)((q_issued - 1) & 1), abort_flag, false);
        }
    } else if (warp >= 12) {
        // ===================================================== V producer (TMA boxes / cp.async)
        ptx::regs_dec<C::AUX_REGS>();
        const int vw = warp - 12;       // rows [32*vw, 32*vw + 32) of each chunk = two segments
        constexpr int DP = C::DP;
        constexpr int PPR = DP / 8;     // 16-byte pieces per row of a V slot (padding pieces zero-filled)
        constexpr int RPI = 32 / PPR;   // rows per warp instruction
        int64_t g = 0, v_issued = 0;  // v_issued: chunks this warp has issued
        bool ok = true;
        for (int64_t item = blockIdx.x; item < p.items && ok; item += gridDim.x) {
            const int64_t bh = item / p.QB;
            MaskRow mr;
            const int64_t cnt = item_keys<FUSED, MQ>(p, item, false, mr, lane);
            const int64_t nch = (cnt + 127) / 128;
            const int32_t* lst = p.kept_idx ? p.kept_idx + item * p.cap : nullptr;
            const __nv_bfloat16* vb = p.v_base + (size_t)bh * L * D;
            int32_t bi = 0, hi = 0, vrow0 = 0;
            if constexpr (STRIDED) {
                bi = (int32_t)(bh / p.H);
                hi = (int32_t)(bh - (int64_t)bi * p.H);
                vrow0 = (int32_t)(bi * p.v_ub + hi * p.v_uh);
            }
            auto fetch1 = [&](int64_t c) -> int32_t {
                const int64_t j = c * 128 + vw * 32 + lane;
                if constexpr (FUSED) {
                    const int32_t k = mask_row_key(mr, j, lane);  // every lane takes part
                    return j >= cnt ? -1 : k;
                } else {
                    if (j >= cnt) return -1;  // past the list
                    return lst ? __ldg(lst + j) : (int32_t)j;
                }
            };
            constexpr int PF = 4;
            int32_t ring[PF];
            int32_t nxt = -1;  // fused kernels: one chunk ahead, no ring
            if constexpr (FUSED) {
                if (nch > 0) nxt = fetch1(0);
            } else {
#pragma unroll
                for (int i = 0; i < PF; ++i) ring[i] = i < nch ? fetch1(i) : -1;
            }
            for (int64_t c = 0; c < nch; ++c) {
                const int64_t gc = g + c;
                const int st = (int)(gc % NV);
                int32_t idx;
                if constexpr (FUSED) {
                    idx = nxt;
                    if (c + 1 < nch) nxt = fetch1(c + 1);
                } else {
                    idx = ring[0];
#pragma unroll
                    for (int i = 0; i < PF - 1; ++i) ring[i] = ring[i + 1];
                    ring[PF - 1] = c + PF < nch ? fetch1(c + PF) : -1;
                }
                const bool okw = gc < 2 || bounded_wait(BAR(C::B_ODONE + (int)(gc & 1)),
                                                        (uint32_t)(((gc - 2) >> 1) & 1), abort_flag);
                if (!__all_sync(0xffffffffu, okw)) {
                    ok = false;
                    break;
                }
                const int32_t first = __shfl_sync(0xffffffffu, idx, lane & 16);
                const bool run = idx >= 0 && idx == first + (lane & 15) && first + 15 < L;
                const uint32_t runs = __ballot_sync(0xffffffffu, run);
                if (idx >= L) atomicOr(&g_device_error, kErrBadIndex);
                if (idx < 0 || idx >= L) idx = 0;  // past the list, or corrupt: key 0 (its scores are masked)
                const uint32_t vdst = VSLOT(st);
#pragma unroll
                for (int sg = 0; sg < 2; ++sg) {
                    const int r0 = vw * 32 + sg * 16;
                    if (((runs >> (16 * sg)) & 0xFFFFu) == 0xFFFFu) {
                        const int32_t fs = __shfl_sync(0xffffffffu, first, 16 * sg);
                        if (lane == 0) {
                            // whole boxes, including the zero-filled columns past D
                            ptx::mbar_expect_tx(BAR(C::B_VFULL + st), (uint32_t)(16 * DP * 2));
#pragma unroll
                            for (int pn = 0; pn < DP / 64; ++pn) {
                                if constexpr (STRIDED)
                                    ptx::tma_load_4d(vdst + (uint32_t)pn * (128 * 128) + (uint32_t)r0 * 128u,
                                                     &p.tmap_v16, pn * 64, fs, hi, bi, BAR(C::B_VFULL + st));
                                else
                                    ptx::tma_load_2d(vdst + (uint32_t)pn * (128 * 128) + (uint32_t)r0 * 128u,
                                                     &p.tmap_v16, pn * 64, (int32_t)(bh * L + fs),
                                                     BAR(C::B_VFULL + st));
                            }
                        }
                    } else {
#pragma unroll
                        for (int i = 0; i < 16 / RPI; ++i) {
                            const int rl = sg * 16 + i * RPI + lane / PPR;
                            const int pc = lane % PPR;
                            const int32_t ridx = __shfl_sync(0xffffffffu, idx, rl);
                            const int r = vw * 32 + rl;
                            // pieces past D (D = 96) are zero-filled: no bytes read from the row start
                            const bool real = pc * 8 < D;
                            const int pe = real ? pc * 8 : 0;
                            const __nv_bfloat16* src;
                            if constexpr (STRIDED)
                                src = p.v_base + (size_t)(uint32_t)(vrow0 + ridx * p.v_ul) * D + pe;
                            else
                                src = vb + (size_t)ridx * D + pe;
                            ptx::cp_async_16(vdst + (uint32_t)(pc / 8) * (128 * 128) + swz(r, pc % 8, 128), src,
                                             real ? 16u : 0u);
                        }
                    }
                }
                ptx::cp_async_arrive_noinc(BAR(C::B_VFULL + st));
                ++v_issued;
            }
            g += nch;
        }
        ptx::cp_async_wait_all();
        // Every V box this warp issued has landed before the block exits: on the normal
        // path the P.V issuer has consumed them all, after an abort nobody else waits
        // for them (a block must not exit with bulk copies into its shared memory in flight).
        for (int64_t i = v_issued > NV ? v_issued - NV : 0; i < v_issued; ++i)
            bounded_wait(BAR(C::B_VFULL + (int)(i % NV)), (uint32_t)((i / NV) & 1), abort_flag, false);
    } else if (warp == 8) {
        // ===================================================== MMA issuer
        ptx::regs_dec<C::AUX_REGS>();
        {
            constexpr uint32_t IDESC1 = umma_idesc_bf16(128, 128, false, false);  // S = Q . K^T
            constexpr uint32_t IDESC2 = umma_idesc_bf16(128, C::DP, false, true);  // O += P . V, V N-major
            constexpr uint32_t HI_V = umma_desc_hi(1024u, 2u);   // V rows: N-major, 128B swizzle
            const uint32_t qlo = umma_desc_lo(QTILE, 16u);
            bool ok = true;
            auto issue_s = [&](int64_t gc, int64_t c, int64_t it) -> bool {
                const int ks = (int)(gc % NK);
                const int s = (int)(gc & 1);
                if (c == 0 && !bounded_wait(BAR(C::B_QFULL), (uint32_t)(it & 1), abort_flag)) return false;
                if (!bounded_wait(BAR(C::B_KFULL + ks), (uint32_t)((gc / NK) & 1), abort_flag)) return false;
                if (gc >= 2 && !bounded_wait(BAR(C::B_SFREE + s), (uint32_t)(((gc >> 1) - 1) & 1), abort_flag))
                    return false;
                ptx::tc_fence_after();
                const uint32_t klo = umma_desc_lo(KSLOT(ks), 16u);
                const uint32_t dS = tS + (uint32_t)s * 128u;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    // Q tile and K chunk share one layout: 64-column panels of 128 rows (K-major, the
                    // panel's swizzle)
                    const uint32_t off = (uint32_t)(kk / 4) * (128 * 128) + (uint32_t)(kk % 4) * 32u;
                    const uint64_t ad = umma_desc_join(qlo + (off >> 4), C::HD::desc_hi(kk / 4));
                    const uint64_t bd = umma_desc_join(klo + (off >> 4), C::HD::desc_hi(kk / 4));
                    ptx::mma_bf16_ss(dS, ad, bd, IDESC1, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(BAR(C::B_SFULL + s));
                return true;
            };
            auto issue_pv = [&](int64_t gc, int64_t c, int64_t it) -> bool {
                const int vs = (int)(gc % NV);
                // O is free for a new item once the epilogue has read the previous one
                if (c == 0 && it > 0 && !bounded_wait(BAR(C::B_OEMPTY), (uint32_t)((it - 1) & 1), abort_flag))
                    return false;
                if (!bounded_wait(BAR(C::B_VFULL + vs), (uint32_t)((gc / NV) & 1), abort_flag)) return false;
                if (!bounded_wait(BAR(C::B_PFULL + (int)(gc & 1)), (uint32_t)((gc >> 1) & 1), abort_flag)) return false;
                ptx::tc_fence_after();
                ptx::fence_proxy_async_smem();
                const uint32_t vlo = umma_desc_lo(VSLOT(vs), 128u * 128u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t bd = umma_desc_join(vlo + (uint32_t)(kk * 2048 >> 4), HI_V);
                    ptx::mma_bf16_ts(tO, tP + (uint32_t)(gc & 1) * 64u + (uint32_t)kk * 8u, bd, IDESC2, (c > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::mma_commit(BAR(C::B_ODONE + (int)(gc & 1)));
                return true;
            };
            // The whole warp walks the items (a fused kernel reads each item's mask row
            // with all lanes); lane 0 issues and commits.
            int64_t g = 0, it = 0;
            for (int64_t item = blockIdx.x; item < p.items && ok; item += gridDim.x, ++it) {
                MaskRow mr;
                const int64_t nch = (item_keys<FUSED, MQ>(p, item, false, mr, lane) + 127) / 128;
                if (lane == 0) {
                    // S of chunks 0 and 1, then for every chunk c the S of chunk c+2 (its slot
                    // frees as soon as the softmax has read chunk c) before the P.V of chunk c
                    for (int64_t c = 0; c < nch && c < 2 && ok; ++c) ok = issue_s(g + c, c, it);
                    for (int64_t c = 0; c < nch && ok; ++c) {
                        if (c + 2 < nch) ok = issue_s(g + c + 2, c + 2, it);
                        if (ok) ok = issue_pv(g + c, c, it);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                g += nch;
            }
            // drain: every MMA issued has completed before TMEM is freed
            if (lane == 0) {
                ptx::mma_commit(BAR(C::B_DRAIN));
                bounded_wait(BAR(C::B_DRAIN), 0u, abort_flag, /*honour_abort=*/false);
            }
        }
        __syncwarp();
    } else {
        // ===================================================== softmax + epilogue (warps 0-7)
        // Two warpgroups, one per half of every chunk's keys: warpgroup g takes keys
        // [64 g, 64 g + 64).  Both own all 128 query rows (thread t = row t = TMEM lane t),
        // so a row's maximum is combined from the two halves once per chunk through
        // shared memory and one barrier of the 256 threads; both halves then use the same
        // reference.  O's columns are split between the two warpgroups for rescaling and
        // for the epilogue; the row sum is the sum of the two halves' partial sums.
        ptx::regs_inc<C::SOFT_REGS>();
        const int wg = warp >> 2;          // key half
        const int t = threadIdx.x & 127;   // query row of the block = TMEM lane
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        float* xmax = reinterpret_cast<float*>(smem + C::OFF_XMAX);
        float* xsum = reinterpret_cast<float*>(smem + C::OFF_XSUM);
        const float cs = p.scale_log2;  // never 0 (the host substitutes a tiny scale)
        // a masked key's score: scaled by cs it becomes -inf, and it never wins the row max
        const float masked = cs > 0.f ? -INFINITY : INFINITY;
        constexpr int OH = C::DP / 2;  // O columns per warpgroup (padding columns included)
        int64_t g = 0;
        for (int64_t item = blockIdx.x; item < p.items; item += gridDim.x) {
            const int64_t bh = item / p.QB;
            const int64_t qb = item - bh * p.QB;
            int64_t cnt;
            {
                MaskRow mr;
                cnt = item_keys<FUSED, MQ>(p, item, false, mr, lane);
            }
            const int64_t nch = (cnt + 127) / 128;
            float mref = -INFINITY;  // reference of this row (log2 units of the scaled scores)
            float lsum = 0.f;        // this half's partial row sum
            bool failed = false;
            for (int64_t c = 0; c < nch; ++c) {
                const int64_t gc = g + c;
                const int s = (int)(gc & 1);
                if (!bounded_wait(BAR(C::B_SFULL + s), (uint32_t)((gc >> 1) & 1), abort_flag)) failed = true;
                ptx::tc_fence_after();
                if (threadIdx.x == 0) {
                    // MMA1 of this chunk has finished reading its K slot (and, for the
                    // item's last chunk, the query tile)
                    ptx::mbar_arrive(BAR(C::B_KEMPTY + (int)(gc % NK)));
                    if (c == nch - 1) ptx::mbar_arrive(BAR(C::B_QEMPTY));
                }
                const uint32_t srow = tS + (uint32_t)s * 128u + (uint32_t)wg * 64u + lane_base;
                const int64_t rem = cnt - c * 128 - wg * 64;  // valid keys of this half
                // ---- this half's row maximum of the scaled scores
                float mloc;
                {
                    float sc[2][32];
                    ptx::tmem_ld32(srow, sc[0]);
                    ptx::tmem_ld32(srow + 32, sc[1]);
                    ptx::tmem_wait_ld();
                    if (rem < 64) {
#pragma unroll
                        for (int j = 0; j < 64; ++j)
                            if (j >= rem) sc[j / 32][j % 32] = masked;
                    }
                    if (cs > 0.f) {
                        float a = sc[0][0], b = sc[1][0];
#pragma unroll
                        for (int j = 1; j < 32; j += 2) {
                            a = ptx::max3(a, sc[0][j], sc[0][j + 1 < 32 ? j + 1 : j]);
                            b = ptx::max3(b, sc[1][j], sc[1][j + 1 < 32 ? j + 1 : j]);
                        }
                        mloc = fmaxf(a, b) * cs;
                    } else {
                        float a = sc[0][0], b = sc[1][0];
#pragma unroll
                        for (int j = 1; j < 32; ++j) {
                            a = fminf(a, sc[0][j]);
                            b = fminf(b, sc[1][j]);
                        }
                        mloc = fminf(a, b) * cs;
                    }
                }
                // ---- combine with the other half (buffers alternate by chunk parity: a half
                // writes parity gc & 1 again only after both passed the barrier of chunk gc+1)
                xmax[(s * 2 + wg) * 128 + t] = mloc;
                ptx::named_sync(1, 256);
                const float mx = fmaxf(mloc, xmax[(s * 2 + (wg ^ 1)) * 128 + t]);  // -inf if the half is empty
                // ---- raise the reference when the row maximum exceeds it by more than TAU
                const bool need = mx > mref + TAU;
                if (__any_sync(0xffffffffu, need)) {
                    const float mnew = need ? mx : mref;
                    const float alpha = ptx::ex2(mref - mnew);  // 0 on the item's first chunk, 1 for rows not raised
                    lsum *= alpha;
                    if (c > 0) {
                        // O holds this item's chunks < c: wait for the last of them, rescale
                        // this warpgroup's half of the row
                        const int64_t gp = gc - 1;
                        if (!bounded_wait(BAR(C::B_ODONE + (int)(gp & 1)), (uint32_t)((gp >> 1) & 1), abort_flag))
                            failed = true;
                        ptx::tc_fence_after();
#pragma unroll
                        for (int pi = 0; pi < OH / 32; ++pi) {
                            float o[32];
                            const uint32_t oa = tO + (uint32_t)(wg * OH + pi * 32) + lane_base;
                            ptx::tmem_ld32(oa, o);
                            ptx::tmem_wait_ld();
                            uint32_t ob[32];
#pragma unroll
                            for (int j = 0; j < 32; ++j) ob[j] = __float_as_uint(o[j] * alpha);
                            ptx::tmem_st32(oa, ob);
                        }
                        ptx::tmem_wait_st();
                        // the rescaled accumulator must reach TMEM before the next P.V
                        ptx::tc_fence_before();
                    }
                    mref = mnew;
                }
                // ---- probabilities of this half, 32 keys at a time (scores read from TMEM again)
                const float nm = -mref;
                const int pbuf = (int)(gc & 1);
                // P buffer pbuf is free once the P.V that last read it (chunk gc-2) has completed
                if (gc >= 2) {
                    const int64_t gp = gc - 2;
                    if (!bounded_wait(BAR(C::B_ODONE + (int)(gp & 1)), (uint32_t)((gp >> 1) & 1), abort_flag))
                        failed = true;
                }
                float ls[8];
#pragma unroll
                for (int j = 0; j < 8; ++j) ls[j] = 0.f;
#pragma unroll 1
                for (int pi = 0; pi < 2; ++pi) {
                    float x[32];
                    ptx::tmem_ld32(srow + pi * 32, x);
                    ptx::tmem_wait_ld();
                    if (rem < 64) {
#pragma unroll
                        for (int j = 0; j < 32; ++j)
                            if (pi * 32 + j >= rem) x[j] = masked;
                    }
#pragma unroll
                    for (int j = 0; j < 32; ++j) x[j] = ptx::ex2(fmaf(x[j], cs, nm));
#pragma unroll
                    for (int j = 0; j < 32; ++j) ls[j & 7] += x[j];
                    float pkf[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 h = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
                        pkf[j] = __uint_as_float(*reinterpret_cast<uint32_t*>(&h));
                    }
                    // P columns: keys 2k, 2k+1 of the chunk in column k
                    ptx::tmem_st16(tP + (uint32_t)pbuf * 64u + (uint32_t)wg * 32u + pi * 16 + lane_base, pkf);
                }
                lsum += ((ls[0] + ls[1]) + (ls[2] + ls[3])) + ((ls[4] + ls[5]) + (ls[6] + ls[7]));
                ptx::tmem_wait_st();
                ptx::tc_fence_before();
                // S slot s has been read for the last time; P of this chunk is in TMEM
                ptx::mbar_arrive(BAR(C::B_SFREE + s));
                ptx::mbar_arrive(BAR(C::B_PFULL + pbuf));
            }
            // ===================== epilogue: O / l -> bf16 row, lse
            const int64_t e = g + nch - 1;
            if (!bounded_wait(BAR(C::B_ODONE + (int)(e & 1)), (uint32_t)((e >> 1) & 1), abort_flag)) failed = true;
            if (ptx::named_red_or(1, 256, failed)) break;
            ptx::tc_fence_after();
            xsum[wg * 128 + t] = lsum;
            ptx::named_sync(1, 256);
            const float l = xsum[t] + xsum[128 + t];  // the same order in both halves
            const float inv = 1.0f / l;
            const int64_t row = qb * MQ + t;
            if (wg == 0 && p.lse != nullptr && row < L) {
                float lg;
                asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(l));
                p.lse[bh * L + row] = (mref + lg) * 0.69314718055994530942f;
            }
            __nv_bfloat16* orow;
            if constexpr (STRIDED) {
                const int64_t bi = bh / p.H;
                orow = p.out + bi * p.o_sb + (bh - bi * p.H) * p.o_sh + row * p.o_sl;
            } else {
                orow = p.out + ((size_t)bh * L + row) * D;
            }
#pragma unroll
            for (int pi = 0; pi < OH / 32; ++pi) {
                const int col = wg * OH + pi * 32;
                if (col >= D) continue;  // zero padding of V (D = 96)
                float o[32];
                ptx::tmem_ld32(tO + (uint32_t)col + lane_base, o);
                ptx::tmem_wait_ld();
                if (row < L) {
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4) {
                        uint32_t w[4];
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            __nv_bfloat162 h = __floats2bfloat162_rn(o[v4 * 8 + 2 * j] * inv, o[v4 * 8 + 2 * j + 1] * inv);
                            w[j] = *reinterpret_cast<uint32_t*>(&h);
                        }
                        *reinterpret_cast<uint4*>(orow + col + v4 * 8) = make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
            }
            // O has been read: the next item's first P.V may overwrite it
            ptx::tc_fence_before();
            ptx::mbar_arrive(BAR(C::B_OEMPTY));
            g += nch;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 8) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fgattn
