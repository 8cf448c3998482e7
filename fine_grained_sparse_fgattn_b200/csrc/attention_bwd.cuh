// Backward pass of tile-sparse softmax attention for sm_100a (tcgen05 + TMEM).
//
// The gradients of the forward ("FG-Attn: Leveraging Fine-Grained Sparse
// Attention in Video Diffusion Models", Abstract: a skipped M x N tile counts as
// -inf, so its scores have p = 0 and carry no gradient), over the same kept-key
// lists the forward reads.  With P recomputed from the forward's log-sum-exp,
//     P^T  = exp(scale * K Q^T - lse)           dP^T = V dO^T
//     dS^T = P^T o (dP^T - Delta),  Delta_i = dO_i . O_i
//     dV  += P^T dO      dK += scale * dS^T Q    dQ^T += scale * K^T dS^T
// per work item -- MQ <= 64 query rows of block (b, h, qb); a 128-row block is
// two items over the same list -- and each 128-key chunk of the list.
//
// Key-major, like the forward's kernel for short query blocks: a thread owns one
// key of the chunk (TMEM lane), so P^T and dS^T go to TMEM as the A operands of
// the dV and dK products (M = 128 keys, K = MQ queries), and dS^T also goes to
// shared memory as the B operand of dQ^T += K^T dS^T (the shape of the
// forward's O^T += V^T P^T).  dQ^T accumulates in TMEM over the block's chunks
// and is stored once per block.  A key is kept by many query blocks, so the
// chunk's dK and dV rows are ADDED to fp32 outputs, by the TMA unit: each warp
// stages its 32 rows in shared memory, 32 columns at a time, and a run of 16
// consecutive keys (what a list of 16-key groups is made of) goes out as one
// 16 x 32 box reduction; any other row goes out as one 128-byte bulk reduction.
// The adds happen in L2, with no per-thread atomics.
//
// One block of eight warps per SM (persistent, round-robin over query blocks).
// A warp can only read the TMEM lane quarter (w % 4), so the two warps of a
// quarter share its 32 keys and split the columns: the softmax's query halves,
// dV (warps 0-3) and dK (warps 4-7), K rows and V rows; thread 0 also issues
// the MMAs.  Per chunk c: softmax(c); the second half of chunk c-1's dK/dV drain
// (its TMEM columns are intact until the gradient products of c); then the
// dV/dK/dQ products of c and, behind them, the score products of c+1; then the
// first half of chunk c's drain while the tensor core computes S(c+1).  The TMA
// pushes (128 KB per chunk) thus overlap the softmax and the score products.  K
// rows of chunk c+2 are loaded with 16-byte cp.async copies into the stage of
// chunk c once its products are done (two K stages); V rows of chunk c+1 into
// the single V stage once the score products of c are done.  Every wait is
// bounded; on a timeout the block sets the device error bit and stops.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "attention_fwd.cuh"

namespace fgattn {

namespace ptx {

// 32 lanes x 4 / 8 / 16 consecutive 32-bit TMEM columns from raw words (packed bf16 pairs).
__device__ __forceinline__ void tmem_st4u(uint32_t taddr, const uint32_t (&r)[4]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%2,%3,%4};" ::"r"(taddr), "r"(r[0]), "r"(r[1]),
                 "r"(r[2]), "r"(r[3])
                 : "memory");
}

__device__ __forceinline__ void tmem_st8u(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}

__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}

// Close this thread's outstanding cp.async copies as one group; wait until at most N
// groups are still in flight.
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// TMA reduction: add the fp32 box at shared address src into the tensor at
// coordinates {x, y, z} (the tensor map fixes the box and the swizzle).
__device__ __forceinline__ void tma_reduce_add_3d(const void* tmap, uint32_t src, int32_t x, int32_t y, int32_t z) {
    asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(
                     reinterpret_cast<uint64_t>(tmap)),
                 "r"(x), "r"(y), "r"(z), "r"(src)
                 : "memory");
}

// Add `bytes` (a multiple of 16) contiguous fp32 values at shared address src to dst.
__device__ __forceinline__ void bulk_reduce_add_f32(float* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(dst), "r"(src),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// every bulk group of this thread has finished reading its shared-memory source
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// all but this thread's most recent bulk group have finished reading their sources
__device__ __forceinline__ void bulk_wait_read_but1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// every bulk group of this thread has completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

}  // namespace ptx

struct alignas(64) BwdParams {
    CUtensorMap tmap_dk, tmap_dv;            // fp32 {D, L, B*H}, box {32, 16, 1}, 128B swizzle
    const __nv_bfloat16 *q, *k, *v, *dout;  // [B][H][L][D], contiguous
    const float* lse;                        // [B][H][L], natural log (the forward's)
    const float* delta;                      // [B][H][L], dO_i . O_i
    const int32_t* kept_idx;                 // [B*H*QB][cap], or null: every key kept
    const int32_t* kept_cnt;                 // [B*H*QB]
    float *dq, *dk, *dv;                     // fp32 [B][H][L][D]; dk and dv accumulate (zeroed first)
    int64_t cap, L;
    int64_t QB;      // query blocks of the lists (M rows each) per (b, h)
    int64_t msplit;  // M / MQ: a 128-row block runs as two 64-row halves over one list
    int64_t items;   // B * H * QB * msplit
    float scale;       // softmax scale
    float scale_log2;  // scale * log2(e)
};

template <int D, int MQ>
struct BwdCfg {
    static_assert(D == 64 || D == 96 || D == 128, "head dim");
    static_assert(MQ == 16 || MQ == 32 || MQ == 64, "query block");
    // At D = 96 the tiles are 128 columns wide with columns 96..127 zero: the dV/dK
    // products run with N = 128 and the dQ^T product with M = 128 (the shapes
    // tcgen05 offers), and the padded columns are never stored.
    static constexpr int DP = D == 96 ? 128 : D;
    static constexpr int KC = 128;                // keys per chunk
    static constexpr int THREADS = 256;           // two warps per TMEM lane quarter
    static constexpr int ROW = DP * 2;            // bytes per bf16 row of a tile
    static constexpr int KV_TILE = KC * ROW;      // one chunk of K or V rows
    static constexpr int Q_TILE = MQ * ROW;       // the block's Q or dO rows
    static constexpr int P_ROW = (MQ * 2 < 128) ? MQ * 2 : 128;  // bytes per key row of a dS^T panel
    static constexpr int P_CPR = P_ROW / 16;
    static constexpr int P_PANEL = KC * P_ROW;
    static constexpr int P_TILE = KC * MQ * 2;
    static constexpr int STG = KC * 128;          // one staged 32-column slice of dV or dK (fp32)
    static constexpr int OFF_K = 0;                       // K stages [2]
    static constexpr int OFF_V = OFF_K + 2 * KV_TILE;     // V stage (one: only the score products read it)
    static constexpr int OFF_Q = OFF_V + KV_TILE;
    static constexpr int OFF_DO = OFF_Q + Q_TILE;
    static constexpr int OFF_DS = OFF_DO + Q_TILE;        // dS^T, MN-major panels
    static constexpr int OFF_STG = OFF_DS + P_TILE;       // 2 slots x {dV slice, dK slice}: [8 runs][16 rows][128 B]
    static constexpr int OFF_LSE = OFF_STG + 4 * STG;     // float [MQ]: lse * log2(e) (+inf past L)
    static constexpr int OFF_DELTA = OFF_LSE + MQ * 4;    // float [MQ]
    static constexpr int OFF_BAR = (OFF_DELTA + MQ * 4 + 7) / 8 * 8;  // s_done, g_done, drain
    static constexpr int OFF_TMEM = OFF_BAR + 3 * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 8;
    static constexpr int BYTES = OFF_ABORT + 8;
    static constexpr int SMEM_REQUEST = BYTES + 1024;     // + alignment slack
    static_assert(SMEM_REQUEST <= 227 * 1024, "shared memory");
    static_assert(OFF_STG % 1024 == 0, "staged boxes need 1024-byte aligned 128B-swizzle atoms");
    // TMEM columns: S^T, dP^T (MQ fp32 each), P^T and dS^T (MQ / 2 packed bf16 pairs
    // each), dV and dK (DP each, M = 128), dQ^T (MQ columns, M = DP)
    static constexpr uint32_t COL_S = 0, COL_DP = MQ, COL_P = 2 * MQ, COL_DS = COL_P + MQ / 2;
    static constexpr uint32_t COL_DV = COL_DS + MQ / 2, COL_DK = COL_DV + DP, COL_DQ = COL_DK + DP;
    static constexpr uint32_t COLS_USED = COL_DQ + MQ;
    static constexpr uint32_t TMEM_COLS = COLS_USED <= 128 ? 128 : COLS_USED <= 256 ? 256 : 512;
    static_assert(COLS_USED <= 512, "TMEM columns");
};

template <int D, int MQ>
__global__ void __launch_bounds__(BwdCfg<D, MQ>::THREADS, 1) fgattn_bwd_kernel(const __grid_constant__ BwdParams p) {
    using C = BwdCfg<D, MQ>;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
    const uint32_t bar_s = sbase + C::OFF_BAR, bar_g = bar_s + 8, bar_drain = bar_s + 16;
    float* s_lse = reinterpret_cast<float*>(smem + C::OFF_LSE);
    float* s_delta = reinterpret_cast<float*>(smem + C::OFF_DELTA);
    // Eight warps: warp w reads TMEM lanes 32 (w % 4) .. +31 (its quarter), so the two
    // warps of a quarter share one chunk's 32 keys and split the columns: softmax
    // query halves, dV (half 0) / dK (half 1), K rows (half 0) / V rows (half 1).
    const int t = threadIdx.x, warp = t >> 5, lane = t & 31;
    const int quarter = warp & 3, half = warp >> 2;
    const int kt = quarter * 32 + lane;  // this thread's key row of a chunk = its TMEM lane
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    const int64_t L = p.L;

    if (warp == 0) {
        ptx::tmem_alloc(sbase + C::OFF_TMEM, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (t == 0) {
        ptx::mbar_init(bar_s, 1);
        ptx::mbar_init(bar_g, 1);
        ptx::mbar_init(bar_drain, 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::OFF_TMEM);

    // Rows r0 .. r0+nrows of a K-major 128B-swizzled tile (64-column panels of prow
    // rows) from base[key_of(r)] (zero-filled where key_of returns -1): one 16-byte
    // piece per lane, PPR lanes per row.
    constexpr int PPR = C::DP / 8;
    constexpr int RPI = 32 / PPR;  // rows per warp instruction
    auto load_rows = [&](uint32_t dst, int prow, const __nv_bfloat16* base, int r0, int nrows, auto key_of) {
        for (int i = 0; i < nrows / RPI; ++i) {
            const int r = r0 + i * RPI + lane / PPR;
            const int pc = lane % PPR;
            const int64_t key = key_of(r);
            const bool in = key >= 0 && pc * 8 < D;  // padded columns read as zeros
            const __nv_bfloat16* src = base + (in ? key * D + pc * 8 : 0);
            ptx::cp_async_16(dst + (uint32_t)(pc / 8) * (uint32_t)(prow * 128) + swz((uint32_t)r, (uint32_t)(pc % 8), 128u),
                             src, in ? 16u : 0u);
        }
    };

    // S^T = K Q^T and dP^T = V dO^T of the chunk whose K rows are in stage st (K-major
    // operands, M = 128 keys, N = MQ), committed to bar_s.  Thread 0 only.
    auto issue_scores = [&](uint32_t st) {
        constexpr uint32_t IDESC = umma_idesc_bf16(128, MQ, false, false);
        constexpr uint32_t HI = umma_desc_hi(1024u, 2u);
        const uint32_t klo = umma_desc_lo(sbase + C::OFF_K + st * C::KV_TILE, 16u);
        const uint32_t vlo = umma_desc_lo(sbase + C::OFF_V, 16u);
        const uint32_t qlo = umma_desc_lo(sbase + C::OFF_Q, 16u);
        const uint32_t olo = umma_desc_lo(sbase + C::OFF_DO, 16u);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t aoff = (uint32_t)(kk / 4) * (128 * 128) + (uint32_t)(kk % 4) * 32u;
            const uint32_t boff = (uint32_t)(kk / 4) * (MQ * 128) + (uint32_t)(kk % 4) * 32u;
            ptx::mma_bf16_ss(tmem + C::COL_S, umma_desc_join(klo + (aoff >> 4), HI),
                             umma_desc_join(qlo + (boff >> 4), HI), IDESC, kk > 0 ? 1u : 0u);
            ptx::mma_bf16_ss(tmem + C::COL_DP, umma_desc_join(vlo + (aoff >> 4), HI),
                             umma_desc_join(olo + (boff >> 4), HI), IDESC, kk > 0 ? 1u : 0u);
        }
        ptx::mma_commit(bar_s);
    };
    // dV = P^T dO and dK = dS^T Q (A in TMEM; B = the Q / dO tiles read MN-major) and
    // dQ^T (+)= K^T dS^T (A = the K stage read MN-major; B = dS^T), committed to bar_g.
    auto issue_grads = [&](uint32_t st, bool first_chunk) {
        constexpr uint32_t IDESC_KV = umma_idesc_bf16(128, C::DP, false, true);
        constexpr uint32_t IDESC_Q = umma_idesc_bf16(C::DP, MQ, true, true);
        constexpr uint32_t HI_T = umma_desc_hi(1024u, 2u);
        constexpr uint32_t P_LAYOUT = (C::P_ROW == 128) ? 2u : (C::P_ROW == 64) ? 4u : 6u;
        constexpr uint32_t HI_DS = umma_desc_hi(8u * C::P_ROW, P_LAYOUT);
        const uint32_t olo = umma_desc_lo(sbase + C::OFF_DO, (uint32_t)(MQ * 128));
        const uint32_t qlo = umma_desc_lo(sbase + C::OFF_Q, (uint32_t)(MQ * 128));
        const uint32_t klo = umma_desc_lo(sbase + C::OFF_K + st * C::KV_TILE, 128u * 128u);
        const uint32_t dlo = umma_desc_lo(sbase + C::OFF_DS, (uint32_t)C::P_PANEL);
#pragma unroll
        for (int kk = 0; kk < MQ / 16; ++kk) {  // over the block's queries
            ptx::mma_bf16_ts(tmem + C::COL_DV, tmem + C::COL_P + (uint32_t)kk * 8u,
                             umma_desc_join(olo + (uint32_t)(kk * 2048 >> 4), HI_T), IDESC_KV, kk > 0 ? 1u : 0u);
            ptx::mma_bf16_ts(tmem + C::COL_DK, tmem + C::COL_DS + (uint32_t)kk * 8u,
                             umma_desc_join(qlo + (uint32_t)(kk * 2048 >> 4), HI_T), IDESC_KV, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)  // over the chunk's keys
            ptx::mma_bf16_ss(tmem + C::COL_DQ, umma_desc_join(klo + (uint32_t)(kk * 2048 >> 4), HI_T),
                             umma_desc_join(dlo + (uint32_t)(kk * 16 * C::P_ROW >> 4), HI_DS), IDESC_Q,
                             (!first_chunk || kk > 0) ? 1u : 0u);
        ptx::mma_commit(bar_g);
    };

    uint32_t ph_s = 0, ph_g = 0;  // phases of the two MMA barriers
    bool failed = false;
    int64_t gcount = 0;  // chunks this block has processed (K stage parity)
    const uint32_t stg_row = (uint32_t)(kt >> 4) * 2048u + (half ? (uint32_t)C::STG : 0u);  // 16-row box, dV | dK
    const int srow = kt & 15;  // this thread's row in the box
    uint32_t nsl = 0;          // slices this thread has staged
    const CUtensorMap* tmap_g = half ? &p.tmap_dk : &p.tmap_dv;
    float* const grad = half ? p.dk : p.dv;
    const float gscale = half ? p.scale : 1.f;
    const uint32_t col_g = half ? C::COL_DK : C::COL_DV;
    for (int64_t item = blockIdx.x; item < p.items && !failed; item += gridDim.x) {
        const int64_t blk = item / p.msplit;  // (b, h, qb) of the list
        const int64_t bh = blk / p.QB, qb = blk - bh * p.QB;
        int64_t cnt = L;
        const int32_t* lst = nullptr;
        if (p.kept_idx != nullptr) {
            cnt = p.kept_cnt[blk];
            if (cnt < 1 || cnt > p.cap) {
                if (t == 0) atomicOr(&g_device_error, kErrBadCount);
                cnt = cnt < 1 ? 1 : p.cap;
            }
            lst = p.kept_idx + blk * p.cap;
        }
        const int64_t nch = (cnt + 127) / 128;
        const __nv_bfloat16* kb = p.k + bh * L * D;
        const __nv_bfloat16* vb = p.v + bh * L * D;
        const int64_t row0 = (qb * p.msplit + (item - blk * p.msplit)) * MQ;  // this item's first query row
        // key at list position j; -1 past the list or for an entry outside [0, L)
        // (reported; such a row is loaded as zeros and gets no gradient)
        auto key_at = [&](int64_t j) -> int64_t {
            if (j >= cnt) return -1;
            if (lst == nullptr) return j;
            const int32_t x = __ldg(lst + j);
            if (x < 0 || (int64_t)x >= L) {
                atomicOr(&g_device_error, kErrBadIndex);
                return -1;
            }
            return x;
        };
        // K rows (half 0) of chunk c into stage (gcount + c) & 1, or V rows (half 1)
        // into the V stage, one cp.async group.  mykey = this thread's list entry of
        // chunk c (-1: none); the warp loads the rows of its quarter's 32 entries, PPR
        // lanes per row, reading the keys by shuffle.
        auto issue_rows = [&](uint32_t dst, const __nv_bfloat16* src_base, int32_t mykey) {
            const int pc = lane % PPR;
            const uint32_t panel = (uint32_t)(pc / 8) * (128u * 128u);
#pragma unroll
            for (int i = 0; i < 32 / RPI; ++i) {
                const int rl = i * RPI + lane / PPR;  // row within the quarter's 32
                const int32_t key = __shfl_sync(0xffffffffu, mykey, rl);
                const bool in = key >= 0 && pc * 8 < D;  // padded columns read as zeros
                const uint32_t off = panel + swz((uint32_t)(quarter * 32 + rl), (uint32_t)(pc % 8), 128u);
                ptx::cp_async_16(dst + off, src_base + (in ? (int64_t)key * D + pc * 8 : 0), in ? 16u : 0u);
            }
            ptx::cp_async_commit();
        };
        auto issue_k = [&](int64_t c, int32_t mykey) {
            issue_rows(sbase + C::OFF_K + (uint32_t)((gcount + c) & 1) * C::KV_TILE, kb, mykey);
        };
        auto issue_v = [&](int32_t mykey) { issue_rows(sbase + C::OFF_V, vb, mykey); };
        // ---- the block's Q (half 0) or dO (half 1) rows, zero past L; lse in log2 units
        //      and Delta; K (half 0) / V (half 1) of chunk 0, and K of chunk 1
        {
            auto qrow = [&](int r) -> int64_t { return row0 + r < L ? row0 + r : -1; };
            load_rows(sbase + (half ? C::OFF_DO : C::OFF_Q), MQ, (half ? p.dout : p.q) + bh * L * D, quarter * (MQ / 4),
                      MQ / 4, qrow);
            ptx::cp_async_commit();
            if (t < MQ) {
                const bool in = row0 + t < L;
                s_lse[t] = in ? p.lse[bh * L + row0 + t] * 1.4426950408889634f : INFINITY;
                s_delta[t] = in ? p.delta[bh * L + row0 + t] : 0.f;
            }
        }
        // this thread's list entries of chunks c (key0) and c+1 (key1)
        int32_t key0 = (int32_t)key_at(kt);
        int32_t key1 = nch > 1 ? (int32_t)key_at(128 + kt) : -1;
        if (half == 0) {
            issue_k(0, key0);
            if (nch > 1) {
                issue_k(1, key1);
                ptx::cp_async_wait_group<1>();  // Q and K of chunk 0 have landed
            } else {
                ptx::cp_async_wait_group<0>();
            }
        } else {
            issue_v(key0);
            ptx::cp_async_wait_group<0>();  // dO and V of chunk 0 have landed
        }
        ptx::fence_proxy_async_smem();  // this thread's copies -> visible to the tensor core
        ptx::tc_fence_before();
        __syncthreads();
        ptx::tc_fence_after();
        if (t == 0) issue_scores((uint32_t)(gcount & 1));
        // P^T and dS^T of this thread's key in chunk c for this half's QW query columns:
        // TMEM (A operands, two queries per column) and, for dS^T, shared memory (B
        // operand of dQ^T: MN-major, queries contiguous).
        constexpr int QW = MQ / 2;
        auto softmax_half = [&](int64_t c) {
            const bool valid = c * 128 + kt < cnt;
            const int q0 = half * QW;
            float sv[QW], dp[QW];
            if constexpr (QW == 32) {
                ptx::tmem_ld32(tmem + C::COL_S + (uint32_t)q0 + lane_base, sv);
                ptx::tmem_ld32(tmem + C::COL_DP + (uint32_t)q0 + lane_base, dp);
            } else if constexpr (QW == 16) {
                ptx::tmem_ld16(tmem + C::COL_S + (uint32_t)q0 + lane_base, sv);
                ptx::tmem_ld16(tmem + C::COL_DP + (uint32_t)q0 + lane_base, dp);
            } else {
                ptx::tmem_ld8(tmem + C::COL_S + (uint32_t)q0 + lane_base, sv);
                ptx::tmem_ld8(tmem + C::COL_DP + (uint32_t)q0 + lane_base, dp);
            }
            ptx::tmem_wait_ld();
            uint32_t pp[QW / 2], dd[QW / 2];
#pragma unroll
            for (int j = 0; j < QW; j += 2) {
                float pr[2], ds[2];
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int q = q0 + j + e;
                    pr[e] = valid ? ptx::ex2(fmaf(sv[j + e], p.scale_log2, -s_lse[q])) : 0.f;
                    ds[e] = pr[e] * (dp[j + e] - s_delta[q]);
                }
                __nv_bfloat162 hp = __floats2bfloat162_rn(pr[0], pr[1]);
                __nv_bfloat162 hd = __floats2bfloat162_rn(ds[0], ds[1]);
                pp[j / 2] = *reinterpret_cast<uint32_t*>(&hp);
                dd[j / 2] = *reinterpret_cast<uint32_t*>(&hd);
            }
            if constexpr (QW == 32) {
                ptx::tmem_st16u(tmem + C::COL_P + (uint32_t)(q0 / 2) + lane_base, pp);
                ptx::tmem_st16u(tmem + C::COL_DS + (uint32_t)(q0 / 2) + lane_base, dd);
            } else if constexpr (QW == 16) {
                ptx::tmem_st8u(tmem + C::COL_P + (uint32_t)(q0 / 2) + lane_base, pp);
                ptx::tmem_st8u(tmem + C::COL_DS + (uint32_t)(q0 / 2) + lane_base, dd);
            } else {
                ptx::tmem_st4u(tmem + C::COL_P + (uint32_t)(q0 / 2) + lane_base, pp);
                ptx::tmem_st4u(tmem + C::COL_DS + (uint32_t)(q0 / 2) + lane_base, dd);
            }
#pragma unroll
            for (int j = 0; j < QW; j += 8) {
                const int chunk = (q0 + j) / 8;  // 16-byte chunk = 8 queries
                const int panel = chunk / C::P_CPR;
                const uint32_t addr = sbase + C::OFF_DS + (uint32_t)panel * C::P_PANEL +
                                      swz((uint32_t)kt, (uint32_t)(chunk % C::P_CPR), (uint32_t)C::P_ROW);
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(dd[j / 2]), "r"(dd[j / 2 + 1]),
                             "r"(dd[j / 2 + 2]), "r"(dd[j / 2 + 3])
                             : "memory");
            }
        };
        // 32-column slices [sa, se) of this half's gradient (dV or dK) rows of the
        // chunk (this thread's key; -1: none) added to the output by the TMA unit,
        // through two staging slots.  run: the 16 keys of this half-warp are
        // consecutive (first = the half-warp's first key): one box per half-warp,
        // else one 128-byte row each.
        auto drain = [&](int sa, int se, int32_t key, int32_t first, bool run) {
#pragma unroll 1
            for (int sl = sa; sl < se; ++sl) {
                const int c0 = sl * 32;
                float a[32];
                ptx::tmem_ld32(tmem + col_g + (uint32_t)c0 + lane_base, a);
                ptx::tmem_wait_ld();
                // slot (nsl & 1) was last filled two slices ago: every lane committed one
                // bulk group per slice since, so "all but the newest group read" frees it
                ptx::bulk_wait_read_but1();
                __syncwarp();
                const uint32_t box = sbase + C::OFF_STG + (nsl & 1u) * (2u * C::STG) + stg_row;
                ++nsl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    // runs: the box's 128B-swizzled layout; single rows: plain 128-byte rows
                    const uint32_t off = run ? swz((uint32_t)srow, (uint32_t)j, 128u) : (uint32_t)(srow * 128 + j * 16);
                    asm volatile("st.shared.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(box + off), "f"(gscale * a[4 * j]),
                                 "f"(gscale * a[4 * j + 1]), "f"(gscale * a[4 * j + 2]), "f"(gscale * a[4 * j + 3])
                                 : "memory");
                }
                ptx::fence_proxy_async_smem();
                __syncwarp();
                if (run) {
                    if ((lane & 15) == 0) ptx::tma_reduce_add_3d(tmap_g, box, c0, first, (int32_t)bh);
                } else if (key >= 0) {
                    ptx::bulk_reduce_add_f32(grad + (bh * L + key) * D + c0, box + (uint32_t)srow * 128u, 128u);
                }
                ptx::bulk_commit();  // one group per lane and slice, empty or not
            }
        };
        // Per chunk c: softmax(c), then the second half of chunk c-1's drain (its TMEM
        // columns stay intact until the gradient products of c), then the products,
        // then the first half of chunk c's drain while the tensor core computes S(c+1).
        constexpr int NS = D / 32;  // 32-column slices of dV / dK
        int32_t key_prev = -1, first_prev = 0;
        bool run_prev = false;
        for (int64_t c = 0; c < nch; ++c) {
            const uint32_t st = (uint32_t)((gcount + c) & 1);
            // entry of chunk c+2, fetched now so that its latency hides behind the softmax
            const int32_t key2 = c + 2 < nch ? (int32_t)key_at((c + 2) * 128 + kt) : -1;
            if (!bounded_wait(bar_s, ph_s, abort_flag)) failed = true;
            ph_s ^= 1u;
            ptx::tc_fence_after();
            // the score products of c are done with the V stage: V rows of chunk c+1
            if (half == 1 && c + 1 < nch) issue_v(key1);
            softmax_half(c);
            if (c > 0) drain(NS / 2, NS, key_prev, first_prev, run_prev);
            ptx::tmem_wait_st();
            if (c + 1 < nch) ptx::cp_async_wait_group<0>();  // K or V of chunk c+1 (the newest group) has landed
            ptx::fence_proxy_async_smem();
            ptx::tc_fence_before();
            __syncthreads();
            ptx::tc_fence_after();
            // ---- gradient products of c, then the score products of c+1 behind them
            if (t == 0) {
                issue_grads(st, c == 0);
                if (c + 1 < nch) issue_scores(st ^ 1u);
            }
            if (!bounded_wait(bar_g, ph_g, abort_flag)) failed = true;
            ph_g ^= 1u;
            ptx::tc_fence_after();
            // K stage st is free (both products of c are done): K rows of chunk c+2 go there
            if (half == 0 && c + 2 < nch) issue_k(c + 2, key2);
            // ---- first half of this chunk's dV / dK drain
            {
                const int32_t first = __shfl_sync(0xffffffffu, key0, lane & 16);
                const bool in_run = key0 >= 0 && key0 == first + (lane & 15) && (int64_t)first + 15 < L;
                const uint32_t runs = __ballot_sync(0xffffffffu, in_run);
                const bool run = ((runs >> (lane & 16)) & 0xFFFFu) == 0xFFFFu;
                drain(0, NS / 2, key0, first, run);
                key_prev = key0;
                first_prev = first;
                run_prev = run;
            }
            key0 = key1;
            key1 = key2;
        }
        drain(NS / 2, NS, key_prev, first_prev, run_prev);  // second half of the last chunk
        gcount += nch;
        // ---- dQ rows of the block: dQ^T has D lanes x MQ columns (at D = 64 the M = 64
        //      accumulator holds row 16 * quarter + lane in lanes 0..15 of each quarter;
        //      at D = 96 lanes 96..127 hold the zero padding);
        //      each half reads its MQ / 2 columns
        const int dt = (C::DP == 128) ? (kt < D ? kt : -1) : ((lane < 16) ? quarter * 16 + lane : -1);
#pragma unroll 1
        for (int q0 = half * (MQ / 2); q0 < (half + 1) * (MQ / 2); q0 += 8) {
            float o[8];
            ptx::tmem_ld8(tmem + C::COL_DQ + (uint32_t)q0 + lane_base, o);
            ptx::tmem_wait_ld();
            if (dt >= 0) {
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    const int64_t row = row0 + q0 + j;
                    if (row < L) p.dq[(bh * L + row) * D + dt] = p.scale * o[j];
                }
            }
        }
        ptx::tc_fence_before();
        // TMEM (dQ^T, dV, dK) read before the next block's products overwrite it; leave together
        failed = __syncthreads_or(failed);
        ptx::tc_fence_after();
    }
    // drain: every MMA issued has completed before TMEM is freed, every copy and
    // reduction before the block exits
    if (t == 0) {
        ptx::mma_commit(bar_drain);
        bounded_wait(bar_drain, 0u, abort_flag, /*honour_abort=*/false);
    }
    ptx::cp_async_wait_all();
    ptx::bulk_wait_all();
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 0) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

// Delta_i = dO_i . O_i in fp32, one warp per row.
template <int D>
__global__ void __launch_bounds__(256) fgattn_bwd_delta_kernel(const __nv_bfloat16* __restrict__ out,
                                                               const __nv_bfloat16* __restrict__ dout,
                                                               float* __restrict__ delta, int64_t rows) {
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= rows) return;
    float acc = 0.f;
#pragma unroll
    for (int e = lane * 2; e < D; e += 64) {
        const __nv_bfloat162 a = *reinterpret_cast<const __nv_bfloat162*>(out + row * D + e);
        const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162*>(dout + row * D + e);
        acc = fmaf(__bfloat162float(a.x), __bfloat162float(b.x), acc);
        acc = fmaf(__bfloat162float(a.y), __bfloat162float(b.y), acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) delta[row] = acc;
}

}  // namespace fgattn
