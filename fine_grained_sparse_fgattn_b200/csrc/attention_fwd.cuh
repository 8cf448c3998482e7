// Tile-sparse softmax attention forward for sm_100a (tcgen05 + TMEM).
//
// The method ("FG-Attn: Leveraging Fine-Grained Sparse Attention in Video
// Diffusion Models", Abstract): score computations are skipped for whole
// M x N tiles; skipped scores count as -inf.  Here the kept tiles arrive as a
// per-query-block list of kept key indices (mask compaction), and this kernel
// gathers only those K/V rows, so the tensor cores always see dense tiles
// whatever N is.
//
// Key-major formulation.  Each work item is one query block (b, h, qb) of MQ
// rows.  Its kept keys are processed in chunks of 128:
//     S^T [128 keys x MQ]  = K_chunk [128 x D] . Q_blk^T          (MMA1, M=128)
//     O^T [D x MQ]        += V_chunk^T [D x 128] . P^T [128 x MQ]  (MMA2, M=D)
// Putting the gathered keys on the MMA's M dimension keeps every MMA at the
// full-rate M=128 shape for any query-block height MQ in {16, 32, 64, 128}.
// A softmax thread owns one key (one TMEM lane) across all MQ queries, so the
// per-query running maximum is a cross-lane quantity.  It is refreshed lazily:
// probabilities are taken against a per-query reference mref and only when a
// score exceeds mref by more than TAU (log2 units) is the reference raised,
// after which the partial sums and the O accumulator are rescaled.  The final
// normalisation uses the same reference, so the result is exact up to
// rounding whatever reference was used.
//
// Warp roles (256 threads, two warps per SM sub-partition):
//   warps 0-3  softmax / correction / epilogue (thread t <-> TMEM lane t)
//   warps 4-6  producer: cp.async gathers of Q, K, V rows into 128B-swizzled
//              shared memory; completion tracked by mbarriers
//   warp  7    TMEM allocation + single-thread tcgen05.mma issue
// Every mbarrier wait is bounded; on timeout the block records an error bit,
// drains its in-flight copies and MMAs, frees TMEM and exits.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "sm100_ptx.cuh"

namespace fgattn {

__device__ unsigned int g_device_error = 0u;

constexpr uint32_t kErrBadIndex = 0x1u;
constexpr uint32_t kErrBadCount = 0x2u;
constexpr uint32_t kErrTimeout = 0x4u;
constexpr unsigned long long kWaitTimeoutNs = 2000000000ull;  // 2 s per wait

struct FwdParams {
    const __nv_bfloat16* q;
    const __nv_bfloat16* k;
    const __nv_bfloat16* v;
    const int32_t* kept_idx;  // nullptr: dense (every key kept)
    const int32_t* kept_cnt;
    __nv_bfloat16* out;
    float* lse;  // may be nullptr
    int64_t cap;
    int64_t L;
    int64_t QB;
    int64_t items;  // B * H * QB
    float scale_log2;  // scale * log2(e)
};

template <int D, int MQ>
struct FwdCfg {
    static_assert(D == 64 || D == 128, "head dim");
    static_assert(MQ == 16 || MQ == 32 || MQ == 64 || MQ == 128, "query block");
    static constexpr int KC = 128;                      // keys per chunk = MMA1 M
    static constexpr int NST = (MQ == 128) ? 2 : 3;     // K/V pipeline stages
    static constexpr int PPR = D / 8;                   // 16-byte pieces per K/V/Q row
    static constexpr int KV_TILE = KC * D * 2;          // bytes of a K or V chunk
    static constexpr int P_ROW = (MQ * 2 < 128) ? MQ * 2 : 128;  // bytes per key row of a P panel
    static constexpr int P_CPR = P_ROW / 16;            // 16-byte chunks per P row
    static constexpr int P_PANEL = KC * P_ROW;          // bytes per P panel
    static constexpr int P_TILE = KC * MQ * 2;
    static constexpr int KSLOT = (KV_TILE > P_TILE) ? KV_TILE : P_TILE;  // K slot also holds P
    static constexpr int Q_TILE = MQ * D * 2;
    static constexpr int STAGE_ROWS = 16;               // epilogue staging rows
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + NST * KSLOT;
    static constexpr int OFF_Q = OFF_V + NST * KV_TILE;
    static constexpr int OFF_STAGE = OFF_Q + Q_TILE;
    static constexpr int OFF_MREF = OFF_STAGE + STAGE_ROWS * D * 2;
    static constexpr int OFF_ALPHA = OFF_MREF + MQ * 4;
    static constexpr int OFF_LFIN = OFF_ALPHA + MQ * 4;
    static constexpr int OFF_RED = OFF_LFIN + MQ * 4;
    static constexpr int OFF_IDX = OFF_RED + 4 * MQ * 4;   // NST x 128 gathered row indices
    static constexpr int OFF_BAR = OFF_IDX + NST * KC * 4;
    // barriers: kv_full[NST], kv_empty[NST], q_full, q_empty, s_full[2], s_free[2],
    //           p_full[2], o_done[2], drain
    static constexpr int NBAR = 2 * NST + 11;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 8;
    static constexpr int BYTES = OFF_ABORT + 8;
    static constexpr int SMEM_REQUEST = BYTES + 1024;    // + alignment slack
    static constexpr uint32_t TMEM_COLS = (3 * MQ <= 64) ? 64 : (3 * MQ <= 128) ? 128 : (3 * MQ <= 256) ? 256 : 512;
    static constexpr int THREADS = 256;
    static constexpr int NPROD = 96;                    // producer threads (warps 4-6)
    static constexpr bool KEEP = MQ <= 64;              // keep a chunk's scores in registers
};

// UMMA shared-memory descriptor (sm_100): start, leading/stride byte offsets,
// version 1, swizzle mode (2 = 128B, 4 = 64B, 6 = 32B).
__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)layout << 61;
    return d;
}

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Byte offset of 16-byte chunk `c` of row `r` in a swizzled panel with `row_bytes`
// per row (128, 64 or 32): the chunk index is XORed with the row's position in its
// 8-row swizzle atom, matching both the UMMA canonical layouts and the panel base
// alignment of 1024 bytes.
__device__ __forceinline__ uint32_t swz(uint32_t r, uint32_t c, uint32_t row_bytes) {
    uint32_t off = r * row_bytes + c * 16u;
    const uint32_t cmask = row_bytes / 16u - 1u;
    return off ^ (((off >> 7) & cmask) << 4);
}

// Wait for the phase of `bar` with parity `parity`.  Gives up (returns false)
// when another role of the block has aborted (honour_abort) or after
// kWaitTimeoutNs, in which case it raises the block's abort flag and the
// device error bit.
__device__ __forceinline__ bool bounded_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                             bool honour_abort = true) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (;;) {
#pragma unroll 1
        for (int i = 0; i < 64; ++i)
            if (ptx::mbar_try_wait(bar, parity)) return true;
        if (honour_abort && *abort_flag) return false;
        if (ptx::globaltimer_ns() - t0 > kWaitTimeoutNs) {
            *abort_flag = 1;
            atomicOr(&g_device_error, kErrTimeout);
            return false;
        }
    }
}

__device__ __forceinline__ int64_t item_count(const FwdParams& p, int64_t item, bool report) {
    if (p.kept_idx == nullptr) return p.L;
    int64_t c = p.kept_cnt[item];
    if (c < 1 || c > p.cap) {
        if (report) atomicOr(&g_device_error, kErrBadCount);
        c = c < 1 ? 1 : p.cap;
    }
    return c;
}

template <int D, int MQ>
__global__ void __launch_bounds__(256, 1) fgattn_fwd_kernel(const FwdParams p) {
    using C = FwdCfg<D, MQ>;
    constexpr int NST = C::NST;
    constexpr float TAU = 8.0f;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    float* mref = reinterpret_cast<float*>(smem + C::OFF_MREF);
    float* alpha = reinterpret_cast<float*>(smem + C::OFF_ALPHA);
    float* lfin = reinterpret_cast<float*>(smem + C::OFF_LFIN);
    float* red = reinterpret_cast<float*>(smem + C::OFF_RED);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto KV_FULL = [&](int i) { return bar0 + 8u * i; };
    auto KV_EMPTY = [&](int i) { return bar0 + 8u * (NST + i); };
    const uint32_t Q_FULL = bar0 + 8u * (2 * NST);
    const uint32_t Q_EMPTY = bar0 + 8u * (2 * NST + 1);
    auto S_FULL = [&](int i) { return bar0 + 8u * (2 * NST + 2 + i); };
    auto S_FREE = [&](int i) { return bar0 + 8u * (2 * NST + 4 + i); };
    auto P_FULL = [&](int i) { return bar0 + 8u * (2 * NST + 6 + i); };
    auto O_DONE = [&](int i) { return bar0 + 8u * (2 * NST + 8 + i); };
    const uint32_t DRAIN = bar0 + 8u * (2 * NST + 10);
    auto KSLOT = [&](int st) { return sbase + C::OFF_K + (uint32_t)st * C::KSLOT; };
    auto VSLOT = [&](int st) { return sbase + C::OFF_V + (uint32_t)st * C::KV_TILE; };
    const uint32_t QTILE = sbase + C::OFF_Q;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (warp == 7) {
        ptx::tmem_alloc(sbase + C::OFF_TMEM, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < NST; ++i) {
            ptx::mbar_init(KV_FULL(i), C::NPROD);
            ptx::mbar_init(KV_EMPTY(i), 1);
        }
        ptx::mbar_init(Q_FULL, C::NPROD);
        ptx::mbar_init(Q_EMPTY, 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(S_FULL(i), 1);
            ptx::mbar_init(S_FREE(i), 128);
            ptx::mbar_init(P_FULL(i), 128);
            ptx::mbar_init(O_DONE(i), 1);
        }
        ptx::mbar_init(DRAIN, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::OFF_TMEM);
    const uint32_t tS0 = tmem;                 // S^T slots: columns [0, MQ) and [MQ, 2MQ)
    const uint32_t tO = tmem + 2u * MQ;        // O^T accumulator: columns [2MQ, 3MQ)

    const int64_t L = p.L;

    if (warp >= 4 && warp < 7) {
        // ===================================================== producer (gathers)
        const int u = threadIdx.x - 128;
        int32_t* idx_smem = reinterpret_cast<int32_t*>(smem + C::OFF_IDX);
        int64_t g = 0;
        int64_t it = 0;
        for (int64_t item = blockIdx.x; item < p.items; item += gridDim.x, ++it) {
            const int64_t bh = item / p.QB;
            const int64_t qb = item - bh * p.QB;
            const int64_t cnt = item_count(p, item, u == 0);
            const int64_t nch = (cnt + 127) / 128;
            bool okq = it == 0 || bounded_wait(Q_EMPTY, (uint32_t)((it - 1) & 1), abort_flag);
            okq = ptx::named_red_and(2, C::NPROD, okq);  // uniform exit: named barriers follow
            if (!okq) break;
            {  // query tile: MQ rows, zero-filled past L
                const __nv_bfloat16* qsrc = p.q + (size_t)bh * L * D;
                for (int id = u; id < MQ * C::PPR; id += C::NPROD) {
                    const int row = id / C::PPR, pc = id % C::PPR;
                    const int64_t grow = qb * MQ + row;
                    const bool in = grow < L;
                    const __nv_bfloat16* src = qsrc + (size_t)(in ? grow : 0) * D + pc * 8;
                    const uint32_t dst = QTILE + (uint32_t)(pc / 8) * (MQ * 128) + swz(row, pc % 8, 128);
                    ptx::cp_async_16(dst, src, in ? 16u : 0u);
                }
                ptx::cp_async_arrive_noinc(Q_FULL);
            }
            const int32_t* lst = p.kept_idx ? p.kept_idx + item * p.cap : nullptr;
            const __nv_bfloat16* kb = p.k + (size_t)bh * L * D;
            const __nv_bfloat16* vb = p.v + (size_t)bh * L * D;
            bool ok = true;
            for (int64_t c = 0; c < nch; ++c) {
                const int64_t gc = g + c;
                const int st = (int)(gc % NST);
                if (gc >= NST && !bounded_wait(KV_EMPTY(st), (uint32_t)((gc / NST - 1) & 1), abort_flag)) {
                    ok = false;
                }
                // the three producer warps agree before touching the stage
                ok = ptx::named_red_and(2, C::NPROD, ok);
                if (!ok) break;
                int32_t* sidx = idx_smem + st * 128;
                for (int r = u; r < 128; r += C::NPROD) {
                    const int64_t j = c * 128 + r;
                    int64_t idx = 0;  // rows past the list: any valid key (scores are masked)
                    if (j < cnt) {
                        idx = lst ? (int64_t)lst[j] : j;
                        if (idx < 0 || idx >= L) {
                            atomicOr(&g_device_error, kErrBadIndex);
                            idx = 0;
                        }
                    }
                    sidx[r] = (int32_t)idx;
                }
                ptx::named_sync(2, C::NPROD);
                const uint32_t kdst = KSLOT(st), vdst = VSLOT(st);
#pragma unroll 2
                for (int pid = u; pid < 128 * C::PPR; pid += C::NPROD) {
                    const int r = pid / C::PPR, pc = pid % C::PPR;
                    const size_t src = (size_t)sidx[r] * D + pc * 8;
                    const uint32_t off = (uint32_t)(pc / 8) * (128 * 128) + swz(r, pc % 8, 128);
                    ptx::cp_async_16(kdst + off, kb + src, 16u);
                    ptx::cp_async_16(vdst + off, vb + src, 16u);
                }
                ptx::cp_async_arrive_noinc(KV_FULL(st));
            }
            if (!ok) break;
            g += nch;
        }
        ptx::cp_async_wait_all();
    } else if (warp == 7) {
        // ===================================================== MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC1 = umma_idesc_bf16(128, MQ, false, false);
            constexpr uint32_t IDESC2 = umma_idesc_bf16(D, MQ, true, true);
            constexpr uint32_t P_LAYOUT = (C::P_ROW == 128) ? 2u : (C::P_ROW == 64) ? 4u : 6u;
            bool ok = true;
            auto issue_pv = [&](int64_t gm, int64_t cm) -> bool {
                const int st = (int)(gm % NST);
                const int s = (int)(gm & 1);
                if (!bounded_wait(P_FULL(s), (uint32_t)((gm >> 1) & 1), abort_flag)) return false;
                ptx::tc_fence_after();
                ptx::fence_proxy_async_smem();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = umma_desc(VSLOT(st) + kk * 2048u, 128u * 128u, 1024u, 2u);
                    const uint64_t bd = umma_desc(KSLOT(st) + kk * 16u * C::P_ROW, (uint32_t)C::P_PANEL,
                                                  8u * C::P_ROW, P_LAYOUT);
                    ptx::mma_bf16_ss(tO, ad, bd, IDESC2, (cm > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::mma_commit(KV_EMPTY(st));
                ptx::mma_commit(O_DONE(s));
                return true;
            };
            int64_t g = 0;
            int64_t it = 0;
            for (int64_t item = blockIdx.x; item < p.items && ok; item += gridDim.x, ++it) {
                const int64_t nch = (item_count(p, item, false) + 127) / 128;
                for (int64_t c = 0; c < nch; ++c) {
                    const int64_t gc = g + c;
                    const int st = (int)(gc % NST);
                    const int s = (int)(gc & 1);
                    if (c == 0 && !bounded_wait(Q_FULL, (uint32_t)(it & 1), abort_flag)) { ok = false; break; }
                    if (!bounded_wait(KV_FULL(st), (uint32_t)((gc / NST) & 1), abort_flag)) { ok = false; break; }
                    if (gc >= 2 && !bounded_wait(S_FREE(s), (uint32_t)(((gc >> 1) - 1) & 1), abort_flag)) {
                        ok = false;
                        break;
                    }
                    ptx::tc_fence_after();
                    ptx::fence_proxy_async_smem();
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t koff = (uint32_t)(kk / 4) * (128 * 128) + (uint32_t)(kk % 4) * 32u;
                        const uint32_t qoff = (uint32_t)(kk / 4) * (MQ * 128) + (uint32_t)(kk % 4) * 32u;
                        const uint64_t ad = umma_desc(KSLOT(st) + koff, 16u, 1024u, 2u);
                        const uint64_t bd = umma_desc(QTILE + qoff, 16u, 1024u, 2u);
                        ptx::mma_bf16_ss(tS0 + (uint32_t)s * MQ, ad, bd, IDESC1, kk > 0 ? 1u : 0u);
                    }
                    ptx::mma_commit(S_FULL(s));
                    if (c == nch - 1) ptx::mma_commit(Q_EMPTY);
                    if (c >= 1 && !issue_pv(gc - 1, c - 1)) { ok = false; break; }
                }
                if (!ok) break;
                if (!issue_pv(g + nch - 1, nch - 1)) { ok = false; break; }
                g += nch;
            }
            // drain: every MMA this thread issued has completed before TMEM is freed
            ptx::mma_commit(DRAIN);
            bounded_wait(DRAIN, 0u, abort_flag, /*honour_abort=*/false);
        }
        __syncwarp();
    } else {
        // ===================================================== softmax / epilogue
        const int t = threadIdx.x;  // key lane within a chunk; TMEM lane t
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        // d index held by this thread in the O^T accumulator (M = D layout)
        const int dt = (D == 128) ? t : ((lane < 16) ? warp * 16 + lane : -1);
        const float cs = p.scale_log2;
        int64_t g = 0;
        for (int64_t item = blockIdx.x; item < p.items; item += gridDim.x) {
            const int64_t bh = item / p.QB;
            const int64_t qb = item - bh * p.QB;
            const int64_t cnt = item_count(p, item, false);
            const int64_t nch = (cnt + 127) / 128;
            if (t < MQ) mref[t] = -INFINITY;
            float lp[MQ];
#pragma unroll
            for (int q = 0; q < MQ; ++q) lp[q] = 0.f;
            ptx::named_sync(1, 128);
            bool ok = true;
            for (int64_t c = 0; c < nch; ++c) {
                const int64_t gc = g + c;
                const int s = (int)(gc & 1);
                const int st = (int)(gc % NST);
                ok = bounded_wait(S_FULL(s), (uint32_t)((gc >> 1) & 1), abort_flag);
                ok = ptx::named_red_and(1, 128, ok);
                if (!ok) break;
                ptx::tc_fence_after();
                const bool valid = c * 128 + t < cnt;
                const uint32_t tS = tS0 + (uint32_t)s * MQ + lane_base;
                float xs[C::KEEP ? MQ : 1];
                // ---- pass 1: scores (log2 units) and the largest excess over the reference
                float dmax = -INFINITY;
#pragma unroll
                for (int pi = 0; pi < MQ / 16; ++pi) {
                    float v[16];
                    ptx::tmem_ld16(tS + pi * 16, v);
                    ptx::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const float x = valid ? v[j] * cs : -INFINITY;
                        if constexpr (C::KEEP) xs[pi * 16 + j] = x;
                        dmax = fmaxf(dmax, x - mref[pi * 16 + j]);
                    }
                }
                if constexpr (C::KEEP) {
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(S_FREE(s));
                }
                const bool need = ptx::named_red_or(1, 128, valid && dmax > TAU);
                if (need) {
                    // ---- exact column maxima of this chunk -> new references
#pragma unroll
                    for (int pi = 0; pi < MQ / 16; ++pi) {
                        float v[16];
                        if constexpr (!C::KEEP) {
                            ptx::tmem_ld16(tS + pi * 16, v);
                            ptx::tmem_wait_ld();
                        }
#pragma unroll
                        for (int j = 0; j < 16; ++j) {
                            float x;
                            if constexpr (C::KEEP) x = xs[pi * 16 + j];
                            else x = valid ? v[j] * cs : -INFINITY;
#pragma unroll
                            for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
                            if (lane == ((pi * 16 + j) & 31)) red[warp * MQ + pi * 16 + j] = x;
                        }
                    }
                    ptx::named_sync(1, 128);
                    if (t < MQ) {
                        const float mo = mref[t];
                        const float mn = fmaxf(mo, fmaxf(fmaxf(red[t], red[MQ + t]), fmaxf(red[2 * MQ + t], red[3 * MQ + t])));
                        alpha[t] = ptx::ex2(mo - mn);
                        mref[t] = mn;
                    }
                    ptx::named_sync(1, 128);
#pragma unroll
                    for (int q = 0; q < MQ; ++q) lp[q] *= alpha[q];
                    if (c > 0) {
                        // O holds chunks < c: wait for the last of them, then rescale its columns
                        const int64_t gp = gc - 1;
                        ok = bounded_wait(O_DONE((int)(gp & 1)), (uint32_t)((gp >> 1) & 1), abort_flag);
                        ok = ptx::named_red_and(1, 128, ok);
                        if (!ok) break;
                        ptx::tc_fence_after();
#pragma unroll
                        for (int pi = 0; pi < MQ / 16; ++pi) {
                            float o[16];
                            ptx::tmem_ld16(tO + lane_base + pi * 16, o);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 16; ++j) o[j] *= alpha[pi * 16 + j];
                            ptx::tmem_st16(tO + lane_base + pi * 16, o);
                        }
                        ptx::tmem_wait_st();
                    }
                }
                // ---- pass 2: probabilities -> bf16 P^T rows (this thread's key) in the K slot
                const uint32_t prow = KSLOT(st);
#pragma unroll
                for (int pi = 0; pi < MQ / 16; ++pi) {
                    float v[16];
                    if constexpr (!C::KEEP) {
                        ptx::tmem_ld16(tS + pi * 16, v);
                        ptx::tmem_wait_ld();
                    }
                    uint32_t packed[8];
#pragma unroll
                    for (int j = 0; j < 16; j += 2) {
                        float x0, x1;
                        if constexpr (C::KEEP) {
                            x0 = xs[pi * 16 + j];
                            x1 = xs[pi * 16 + j + 1];
                        } else {
                            x0 = valid ? v[j] * cs : -INFINITY;
                            x1 = valid ? v[j + 1] * cs : -INFINITY;
                        }
                        const float p0 = ptx::ex2(x0 - mref[pi * 16 + j]);
                        const float p1 = ptx::ex2(x1 - mref[pi * 16 + j + 1]);
                        lp[pi * 16 + j] += p0;
                        lp[pi * 16 + j + 1] += p1;
                        __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                        packed[j / 2] = *reinterpret_cast<uint32_t*>(&h);
                    }
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const int chunk = pi * 2 + h;  // 16-byte chunk = 8 queries
                        const int panel = chunk / C::P_CPR;
                        const uint32_t addr = prow + (uint32_t)panel * C::P_PANEL + swz(t, chunk % C::P_CPR, C::P_ROW);
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(packed[4 * h]),
                                     "r"(packed[4 * h + 1]), "r"(packed[4 * h + 2]), "r"(packed[4 * h + 3])
                                     : "memory");
                    }
                }
                if constexpr (!C::KEEP) {
                    ptx::tc_fence_before();
                    ptx::mbar_arrive(S_FREE(s));
                }
                ptx::fence_proxy_async_smem();
                ptx::tc_fence_before();
                ptx::mbar_arrive(P_FULL(s));
            }
            if (!ok) break;
            // ===================== epilogue: O / l -> bf16 rows, lse
            const int64_t e = g + nch - 1;
            ok = bounded_wait(O_DONE((int)(e & 1)), (uint32_t)((e >> 1) & 1), abort_flag);
            ok = ptx::named_red_and(1, 128, ok);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int q = 0; q < MQ; ++q) {
                float x = lp[q];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (lane == (q & 31)) red[warp * MQ + q] = x;
            }
            ptx::named_sync(1, 128);
            if (t < MQ) {
                const float l = (red[t] + red[MQ + t]) + (red[2 * MQ + t] + red[3 * MQ + t]);
                lfin[t] = 1.0f / l;
                const int64_t row = qb * MQ + t;
                if (p.lse != nullptr && row < L) {
                    float lg;
                    asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(l));
                    p.lse[bh * L + row] = (mref[t] + lg) * 0.69314718055994530942f;
                }
            }
            ptx::named_sync(1, 128);
            __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem + C::OFF_STAGE);
            __nv_bfloat16* outb = p.out + (size_t)bh * L * D;
#pragma unroll 1
            for (int pi = 0; pi < MQ / 16; ++pi) {
                float o[16];
                ptx::tmem_ld16(tO + lane_base + pi * 16, o);
                ptx::tmem_wait_ld();
                if (dt >= 0) {
#pragma unroll
                    for (int j = 0; j < 16; ++j) stage[j * D + dt] = __float2bfloat16_rn(o[j] * lfin[pi * 16 + j]);
                }
                ptx::named_sync(1, 128);
                for (int vi = t; vi < 16 * C::PPR; vi += 128) {
                    const int r = vi / C::PPR, pc = vi % C::PPR;
                    const int64_t row = qb * MQ + pi * 16 + r;
                    if (row < L) {
                        const uint4 val = *reinterpret_cast<const uint4*>(stage + r * D + pc * 8);
                        *reinterpret_cast<uint4*>(outb + row * D + pc * 8) = val;
                    }
                }
                ptx::named_sync(1, 128);
            }
            ptx::tc_fence_before();
            g += nch;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 7) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fgattn
