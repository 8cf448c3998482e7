// Tile-sparse softmax attention forward for sm_100a (TMA gather + tcgen05 + TMEM).
//
// The method ("FG-Attn: Leveraging Fine-Grained Sparse Attention in Video
// Diffusion Models", Abstract): score computations are skipped for whole
// M x N tiles; skipped scores count as -inf.  The kept tiles arrive as a
// per-query-block list of kept key indices (mask compaction); this kernel
// gathers only those K/V rows with TMA row gathers, so the tensor cores always
// see dense 128-key tiles whatever N is.
//
// Key-major formulation.  Each work item is one query block (b, h, qb) of MQ
// rows.  Its kept keys are processed in chunks of 128:
//     S^T [128 keys x MQ]  = K_chunk [128 x D] . Q_blk^T          (MMA1, M=128)
//     O^T [D x MQ]        += V_chunk^T [D x 128] . P^T [128 x MQ]  (MMA2, M=D)
// Putting the gathered keys on the MMA's M dimension keeps every MMA at the
// full-rate M=128 shape for any query-block height MQ in {16, 32, 64, 128}.
// A softmax thread owns one key (TMEM lane) of the chunk; the softmax
// warpgroups split the chunk's MQ query columns between them (more groups =
// shorter per-thread dependency chains per chunk).  The per-query
// running maximum is a cross-lane quantity, so it is refreshed lazily:
// probabilities are taken against a per-query reference mref, and only when a
// score exceeds mref by more than TAU (log2 units) is the reference raised and
// the partial sums and the O accumulator rescaled.  The final normalisation
// uses the same reference, so the result is exact up to rounding whatever
// reference was used.
//
// Two warp layouts (template parameter GATHER), each the faster one for its kind
// of key list.  Tile layout (lists made of 16-key runs: N a multiple of 16, or a
// dense run): NSW softmax warpgroups (4, i.e. 768 threads, for MQ in {32, 64}; 2
// otherwise) + two auxiliary warpgroups:
//   warps 0 .. 4*NSW-1  softmax warpgroup g: query columns [g*CW, (g+1)*CW), CW = MQ/NSW
//   warps A, A+1        K producer (A = 4*NSW): TMA tile load of the query block; K rows by TMA
//   warp  A+2           single-thread tcgen05.mma issue of the P.V products (MMA2)
//   warp  A+3           TMEM allocation + single-thread tcgen05.mma issue of the scores (MMA1)
//   warps A+4 .. A+7    V producer: V rows by TMA or cp.async
// Gather layout (other lists: rows fetched one by one, where issuing the K row
// gathers dominates): two softmax warpgroups (512 threads), three K producer warps
// (A .. A+2) and one warp (A+3) issuing both MMA kinds, scores two chunks ahead.
// Each chunk is loaded as eight 16-row segments.  A segment whose 16 kept keys
// are consecutive (always the case for key groups of N >= 16 keys, N a multiple
// of 16) is one tiled TMA box; any other segment is gathered row by row (K with
// TMA gather4, V with cp.async).
// Gathering K and V through the two different copy paths (TMA and the LSU)
// keeps more row requests in flight per SM than either path alone; the
// producer warpgroups hand most of their registers to the softmax groups.
// Every mbarrier wait is bounded; on timeout the block records an error bit,
// drains its in-flight copies and MMAs, frees TMEM and exits.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>

#include "mask_row.cuh"
#include "sm100_ptx.cuh"

namespace fgattn {

__device__ unsigned int g_device_error = 0u;

constexpr uint32_t kErrBadIndex = 0x1u;
constexpr uint32_t kErrBadCount = 0x2u;
constexpr uint32_t kErrTimeout = 0x4u;
#ifndef FGATTN_WAIT_TIMEOUT_NS
#define FGATTN_WAIT_TIMEOUT_NS 2000000000ull  // 2 s per wait
#endif
constexpr unsigned long long kWaitTimeoutNs = FGATTN_WAIT_TIMEOUT_NS;

// Layouts (template parameter STRIDED).  Contiguous: q, k, v, out are
// [B][H][L][D]; the tile maps (q, k16, v16) and the gather map (k) are 2-D over
// the B*H*L rows.  Strided: q, k, v, out are [B][H][L][D] views with D
// contiguous and element strides (sb, sh, sl) in any order in memory
// ([B][L][H][D], a packed [B][L][3][H][D] projection ...); the tile maps are
// 4-D {D, L, H, B} with coordinates (x, l, h, b), and the gather map over k and
// the cp.async row copies of v count in rows of D elements (every stride is a
// whole number of rows).  The contiguous kernel is kept separate because its
// copy loops are sensitive to their code size: the general addressing measured
// 4-8 % slower on the sparse forward.
struct alignas(64) FwdParams {
    CUtensorMap tmap_q;    // q tiles: box {64, MQ} (contiguous) or {64, MQ, 1, 1} (strided), 128B swizzle
    CUtensorMap tmap_k;    // k rows of D elements, box {64, 1} (row gathers)
    CUtensorMap tmap_k16;  // k tiles: box {64, 16} or {64, 16, 1, 1} (16 consecutive keys)
    CUtensorMap tmap_v16;  // same for V (at D = 96 the box at column 64 is half outside: zero fill)
    // D = 96 only: columns 64..95 of q and k, 32-column boxes with 64B swizzle
    CUtensorMap tmap_q_hi, tmap_k_hi, tmap_k16_hi;
    const __nv_bfloat16* v_base;  // V rows, gathered with cp.async where not consecutive
    // strided layout only
    int64_t k_ub, k_uh;  // k batch / head strides in rows of D elements
    int64_t v_ub, v_uh;  // v batch / head strides in rows of D elements
    int32_t k_ul, v_ul;  // k / v token strides in rows of D elements
    int64_t o_sb, o_sh, o_sl;  // out element strides
    int64_t H;
    const int32_t* kept_idx;  // nullptr: dense (every key kept), or the mask below
    const int32_t* kept_cnt;
    // fused kernels only: the packed tile mask, read instead of kept lists
    const uint32_t* mask;
    int64_t mask_w, mask_g, mask_n;  // words per row, key groups, keys per group
    __nv_bfloat16* out;
    float* lse;  // may be nullptr
    int64_t cap;
    int64_t L;
    int64_t QB;
    int64_t items;     // B * H * QB
    float scale_log2;  // scale * log2(e)
};

// UMMA shared-memory descriptor (sm_100): start address >> 4 (bits 0-13), leading
// byte offset >> 4 (16-29), stride byte offset >> 4 (32-45), version 1 (bit 46),
// swizzle mode (bits 61-63: 2 = 128B, 4 = 64B, 6 = 32B), built as two halves.  The
// high half is a compile-time constant per operand; the low half moves by adding
// (byte offset >> 4), which never carries out of the 14-bit address field for
// shared-memory offsets below 256 KB.
__host__ __device__ constexpr uint32_t umma_desc_hi(uint32_t sbo, uint32_t layout) {
    return ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (layout << 29);
}
__device__ __forceinline__ uint32_t umma_desc_lo(uint32_t saddr, uint32_t lbo) {
    return ((saddr & 0x3FFFFu) >> 4) | (((lbo >> 4) & 0x3FFFu) << 16);
}
__device__ __forceinline__ uint64_t umma_desc_join(uint32_t lo, uint32_t hi) { return ((uint64_t)hi << 32) | lo; }

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Head dimensions D in {64, 96, 128}.  Q and K rows sit in shared memory as
// 64-column panels with 128-byte rows (128B swizzle); at D = 96 the second panel
// holds the last 32 columns in 64-byte rows (64B swizzle), so every load stays
// inside the rows and the score product runs D / 16 k-steps.  V rows always sit
// in 64-column 128B-swizzled panels; at D = 96 columns 96..127 of the second
// panel are zero, so the P.V product runs on V padded to DP = 128 columns (the
// only shape tcgen05 offers for that operand: M = D must be 64 or 128 in the
// key-major product), and the padded output columns are never stored.
template <int D>
struct HeadDim {
    static_assert(D == 64 || D == 96 || D == 128, "head dim");
    static constexpr int DP = D == 96 ? 128 : D;  // padded width of V, O and the shared-memory slots
    static constexpr int KP = (D + 63) / 64;      // panels of Q and K
    static constexpr bool NARROW = D == 96;       // second Q/K panel: 32 columns, 64B swizzle
    __host__ __device__ static constexpr uint32_t pitch(int pn) { return (NARROW && pn == 1) ? 64u : 128u; }
    // high word of the UMMA descriptor of Q/K panel pn (K-major; SBO = 8 rows)
    __host__ __device__ static constexpr uint32_t desc_hi(int pn) {
        return (NARROW && pn == 1) ? umma_desc_hi(8u * 64u, 4u) : umma_desc_hi(8u * 128u, 2u);
    }
};

template <int D, int MQ, bool GATHER>
struct FwdCfg {
    using HD = HeadDim<D>;
    static constexpr int DP = HD::DP;
    static_assert(MQ == 16 || MQ == 32 || MQ == 64 || MQ == 128, "query block");
    static constexpr int KC = 128;              // keys per chunk = MMA1 M
    static constexpr int NSW = (!GATHER && (MQ == 32 || MQ == 64)) ? 4 : 2;  // softmax warpgroups
    static constexpr int KWARPS = GATHER ? 3 : 2;                            // K producer warps
    static constexpr int CW = MQ / NSW;         // query columns per softmax warpgroup
    static constexpr int KV_TILE = KC * DP * 2;  // bytes of a K or V chunk slot
    static constexpr int P_ROW = (MQ * 2 < 128) ? MQ * 2 : 128;  // bytes per key row of a P panel
    static constexpr int P_CPR = P_ROW / 16;    // 16-byte chunks per P row
    static constexpr int P_PANEL = KC * P_ROW;  // bytes per P panel
    static constexpr int P_TILE = KC * MQ * 2;
    static constexpr int Q_TILE = MQ * DP * 2;  // query tile slot
    static constexpr int Q_TX = MQ * D * 2;     // bytes a query-tile load delivers
    static constexpr int SROWS = (CW < 8) ? CW : (NSW == 4 ? 8 : (CW < 16 ? CW : 16));  // staging rows per group
    static constexpr int STAGE = SROWS * D * 2;
    static constexpr int MISC = NSW * (3 * CW + 4 * CW) * 4 + 64 * 8 + 64;  // mref/alpha/lfin/red, barriers
    static constexpr int LIMIT = 227 * 1024 - 1024 - 256;
    static constexpr int fixed_bytes(int nk, int nv, int np) {
        return nk * KV_TILE + nv * KV_TILE + np * P_TILE + Q_TILE + NSW * STAGE + MISC;
    }
    // pipeline depths: K ring, V ring, P buffers (deepest that fits)
    // The V ring has two stages so that "V slot free" is exactly "MMA2 of the chunk
    // two back done" (o_done, no extra tensor-core commit); spare room deepens the K ring.
    static constexpr int NV = 2;
    static constexpr int NK = fixed_bytes(4, NV, 2) <= LIMIT ? 4 : fixed_bytes(3, NV, 1) <= LIMIT ? 3 : 2;
    static constexpr int NP = fixed_bytes(NK, NV, 2) <= LIMIT ? 2 : 1;
    static_assert(fixed_bytes(NK, NV, NP) <= LIMIT, "shared memory");
    static constexpr int OFF_K = 0;
    static constexpr int OFF_V = OFF_K + NK * KV_TILE;
    static constexpr int OFF_P = OFF_V + NV * KV_TILE;
    static constexpr int OFF_Q = OFF_P + NP * P_TILE;
    static constexpr int OFF_STAGE = OFF_Q + Q_TILE;           // NSW x STAGE
    static constexpr int OFF_MREF = OFF_STAGE + NSW * STAGE;   // [NSW][CW]
    static constexpr int OFF_ALPHA = OFF_MREF + NSW * CW * 4;  // [NSW][CW]
    static constexpr int OFF_LFIN = OFF_ALPHA + NSW * CW * 4;  // [NSW][CW]
    static constexpr int OFF_RED = OFF_LFIN + NSW * CW * 4;    // [NSW][4][CW]
    static constexpr int OFF_BAR = (OFF_RED + NSW * 4 * CW * 4 + 7) / 8 * 8;
    // barriers: k_full[NK] k_empty[NK] v_full[NV] v_empty[NV] (unused: o_done serves) q_full q_empty
    //           s_full[2] s_free[2] p_full[NP] o_done[2] drain
    // Only s_full and o_done are tensor-core commits (each commit costs tensor-pipe
    // time); k_empty and q_empty are arrived by a softmax thread once s_full shows
    // that the MMA reading them has finished.
    static constexpr int B_KFULL = 0, B_KEMPTY = NK, B_VFULL = 2 * NK, B_VEMPTY = 2 * NK + NV;
    static constexpr int B_QFULL = 2 * NK + 2 * NV, B_QEMPTY = B_QFULL + 1, B_SFULL = B_QFULL + 2;
    static constexpr int B_SFREE = B_SFULL + 2, B_PFULL = B_SFREE + 2, B_ODONE = B_PFULL + NP;
    static constexpr int B_DRAIN = B_ODONE + 2, B_DRAIN2 = B_DRAIN + 1, NBAR = B_DRAIN2 + 1;
    static constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
    static constexpr int OFF_ABORT = OFF_TMEM + 8;
    static constexpr int BYTES = OFF_ABORT + 8;
    static_assert(BYTES <= LIMIT, "shared memory layout");
    static constexpr int SMEM_REQUEST = BYTES + 1024;  // + alignment slack
    static constexpr uint32_t TMEM_COLS = (3 * MQ <= 64) ? 64 : (3 * MQ <= 128) ? 128 : (3 * MQ <= 256) ? 256 : 512;
    static constexpr int SOFT_THREADS = 128 * NSW;
    static constexpr int THREADS = SOFT_THREADS + 256;
    static constexpr int AUX_WARP = 4 * NSW;  // first auxiliary warp
    // Register split between the softmax warpgroups and the two producer/MMA
    // warpgroups; it must add up to the launch's allocation (THREADS x the per-thread
    // count the launch bounds give: 128 at 512 threads, 80 at 768):
    //   NSW = 2: 2*128*SOFT + 2*128*AUX = 512*128;  NSW = 4: 4*128*88 + 2*128*64 = 768*80.
    // (The producer and issuer warps fit in 64 registers at NSW = 4; at MQ = 128 they
    // keep 80, which measured faster than a 192/64 split.)
    // MQ = 128 keeps 64 columns of scores and sums per softmax thread.
    static constexpr uint32_t LAUNCH_REGS = NSW == 4 ? 80 : 128;
    static constexpr uint32_t SOFT_REGS = NSW == 4 ? 88 : (MQ == 128 ? 176 : 128);
    static constexpr uint32_t AUX_REGS = NSW == 4 ? 64 : (MQ == 128 ? 80 : 128);
    static_assert(NSW * 128 * SOFT_REGS + 256 * AUX_REGS <= THREADS * LAUNCH_REGS, "register split");
};

// Byte offset of 16-byte chunk `c` of row `r` in a swizzled panel with `row_bytes`
// per row (128, 64 or 32): the chunk index is XORed with the row's position in
// its 8-row swizzle atom (panel bases are 1024-byte aligned), the layout both
// the UMMA descriptors and the TMA 128B swizzle use.
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

// Kept-list entries 4*lane .. 4*lane+3 of chunk c (raw, unchecked).  Entries past
// the list read as 0.  Issued several chunks ahead of use: the lists live in HBM.
__device__ __forceinline__ int4 fetch_idx(const int32_t* lst, int64_t cnt, int64_t c, int lane) {
    const int64_t j0 = c * 128 + 4 * lane;
    if (lst == nullptr) {
        return make_int4(j0 < cnt ? (int)j0 : 0, j0 + 1 < cnt ? (int)(j0 + 1) : 0, j0 + 2 < cnt ? (int)(j0 + 2) : 0,
                         j0 + 3 < cnt ? (int)(j0 + 3) : 0);
    }
    if (j0 + 3 < cnt) return __ldg(reinterpret_cast<const int4*>(lst + j0));
    return make_int4(j0 < cnt ? __ldg(lst + j0) : 0, j0 + 1 < cnt ? __ldg(lst + j0 + 1) : 0,
                     j0 + 2 < cnt ? __ldg(lst + j0 + 2) : 0, j0 + 3 < cnt ? __ldg(lst + j0 + 3) : 0);
}

// Fused kernels: list entries 4*lane .. 4*lane+3 of chunk c from the mask row
// (warp-collective; every lane of the warp calls it).
__device__ __forceinline__ int4 fused_idx4(const MaskRow& mr, int64_t c, int lane4, int lane) {
    const int64_t j0 = c * 128 + 4 * lane4;
    if ((mr.n & 3) == 0) {  // four consecutive keys of one group
        const int32_t k = mask_row_key(mr, j0, lane);
        return make_int4(j0 < mr.keys ? k : 0, j0 + 1 < mr.keys ? k + 1 : 0, j0 + 2 < mr.keys ? k + 2 : 0,
                         j0 + 3 < mr.keys ? k + 3 : 0);
    }
    // four separate searches, one copy of the search code (kept small for the instruction cache)
    int4 e = make_int4(0, 0, 0, 0);
#pragma unroll 1
    for (int x = 0; x < 4; ++x) {
        const int32_t k = mask_row_key(mr, j0 + x, lane);
        e.x = x == 0 ? k : e.x;
        e.y = x == 1 ? k : e.y;
        e.z = x == 2 ? k : e.z;
        e.w = x == 3 ? k : e.w;
    }
    return e;
}

// Kept keys of work item `item`: from kept_cnt, L for a dense run, or the mask
// row (fused kernels; warp-collective, and `mr` keeps the row for the caller).
template <bool FUSED, int MQ>
__device__ __forceinline__ int64_t item_keys(const FwdParams& p, int64_t item, bool report, MaskRow& mr, int lane) {
    if constexpr (FUSED) {
        mask_row_load(mr, p.mask, item, p.QB, MQ, p.mask_n, p.mask_g, p.mask_w, p.L, lane);
        return mr.keys;
    } else {
        return item_count(p, item, report);
    }
}

// Gather-map row coordinates of four fetched entries: row0 + key * stride.
// Entries outside [0, L) are reported and replaced by key 0 of the head (as are
// entries past the list, whose scores the softmax masks).
template <bool STRIDED>
__device__ __forceinline__ void rows_of(const FwdParams& p, int4 raw, int64_t row0, bool report, int32_t (&rows)[4]) {
    const int32_t idx[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int32_t x = idx[i];
        if (x < 0 || (int64_t)x >= p.L) {
            if (report) atomicOr(&g_device_error, kErrBadIndex);
            x = 0;
        }
        if constexpr (STRIDED)
            rows[i] = (int32_t)row0 + x * p.k_ul;
        else
            rows[i] = (int32_t)(row0 + x);
    }
}

template <int D, int MQ, bool GATHER, bool STRIDED, bool FUSED>
__global__ void __launch_bounds__(FwdCfg<D, MQ, GATHER>::THREADS, 1)
    fgattn_fwd_kernel(const __grid_constant__ FwdParams p) {
    using C = FwdCfg<D, MQ, GATHER>;
    constexpr int NK = C::NK, NV = C::NV, NP = C::NP, CW = C::CW;
    // A reference is raised when a score exceeds it by more than TAU (log2 units):
    // probabilities stay below 2^16, far inside the range of bf16 and fp32 and at
    // the same relative precision.  8 raised the references (two extra warpgroup
    // barriers and an O rescale that waits for the previous P.V) often enough on
    // strongly peaked scores to cost 6 % on a low-rank-correlated layer.
    constexpr float TAU = 16.0f;

    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_ABORT);
    const uint32_t bar0 = sbase + C::OFF_BAR;
    auto BAR = [&](int i) { return bar0 + 8u * (uint32_t)i; };
    auto KSLOT = [&](int i) { return sbase + C::OFF_K + (uint32_t)i * C::KV_TILE; };
    auto VSLOT = [&](int i) { return sbase + C::OFF_V + (uint32_t)i * C::KV_TILE; };
    auto PBUF = [&](int i) { return sbase + C::OFF_P + (uint32_t)i * C::P_TILE; };
    const uint32_t QTILE = sbase + C::OFF_Q;

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    constexpr int AW = C::AUX_WARP;

    if (warp == AW + 3) {
        ptx::tmem_alloc(sbase + C::OFF_TMEM, C::TMEM_COLS);
        ptx::tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < NK; ++i) {
            ptx::mbar_init(BAR(C::B_KFULL + i), C::KWARPS);
            ptx::mbar_init(BAR(C::B_KEMPTY + i), 1);
        }
        for (int i = 0; i < NV; ++i) {
            ptx::mbar_init(BAR(C::B_VFULL + i), 128);
            ptx::mbar_init(BAR(C::B_VEMPTY + i), 1);
        }
        ptx::mbar_init(BAR(C::B_QFULL), 1);
        ptx::mbar_init(BAR(C::B_QEMPTY), 1);
        for (int i = 0; i < 2; ++i) {
            ptx::mbar_init(BAR(C::B_SFULL + i), 1);
            ptx::mbar_init(BAR(C::B_SFREE + i), C::SOFT_THREADS);
            ptx::mbar_init(BAR(C::B_ODONE + i), 1);
        }
        for (int i = 0; i < NP; ++i) ptx::mbar_init(BAR(C::B_PFULL + i), C::SOFT_THREADS);
        ptx::mbar_init(BAR(C::B_DRAIN), 1);
        ptx::mbar_init(BAR(C::B_DRAIN2), 1);
        *abort_flag = 0;
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + C::OFF_TMEM);
    const uint32_t tS0 = tmem;           // S^T slots: columns [0, MQ) and [MQ, 2MQ)
    const uint32_t tO = tmem + 2u * MQ;  // O^T accumulator: columns [2MQ, 3MQ)
    const int64_t L = p.L;

    if (warp >= AW && warp < AW + C::KWARPS) {
        // ===================================================== K producer (TMA)
        if constexpr (C::AUX_REGS != C::LAUNCH_REGS) ptx::regs_dec<C::AUX_REGS>();
        const int kw = warp - AW;
        // tile layout: segments 0-3 -> first warp, 4-7 -> second; gather layout: 0-2, 3-5, 6-7;
        // four lanes (4-row groups) per segment
        const int seg0 = GATHER ? kw * 3 : kw * 4;
        const int nseg = GATHER ? (kw < 2 ? 3 : 2) : 4;
        const int g4 = seg0 * 4 + lane;            // this lane's 4-row group in the chunk
        const bool issuer = lane < nseg * 4;
        const int lseg = lane >> 2;                // segment within the warp
        int64_t g = 0, it = 0;
        int64_t issued = 0;    // chunks whose loads this warp has issued
        int64_t q_issued = 0;  // query tiles issued (first K warp)
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
            if (kw == 0) {  // the query tile (rows past L are padding; their results are never stored)
                const bool okq = it == 0 || bounded_wait(BAR(C::B_QEMPTY), (uint32_t)((it - 1) & 1), abort_flag);
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
                            ptx::tma_load_4d(QTILE + (uint32_t)pn * (MQ * 128), qm, pn * 64, (int32_t)(qb * MQ), hi,
                                             bi, BAR(C::B_QFULL));
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
                const bool run = issuer && j0 + 3 < cnt && cur.x == first + 4 * (lane & 3) && cur.y == cur.x + 1 &&
                                 cur.z == cur.x + 2 && cur.w == cur.x + 3 && first >= 0 && first + 15 < L;
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
                            ptx::tma_gather4(dst(pn), (C::HD::NARROW && pn == 1) ? &p.tmap_k_hi : &p.tmap_k, pn * 64,
                                             rows[0], rows[1], rows[2], rows[3], BAR(C::B_KFULL + st));
                    }
                }
                ++issued;
            }
            g += nch;
        }
        // Before the block exits, every load this warp issued has landed (on the normal
        // path they all have already been consumed, so these waits return at once).
        for (int64_t i = issued > NK ? issued - NK : 0; i < issued; ++i)
            bounded_wait(BAR(C::B_KFULL + (int)(i % NK)), (uint32_t)((i / NK) & 1), abort_flag, false);
        if (q_issued > 0) bounded_wait(BAR(C::B_QFULL), (uint32_t)((q_issued - 1) & 1), abort_flag, false);
    } else if (warp >= AW + 4) {
        // ===================================================== V producer (TMA boxes / cp.async)
        if constexpr (C::AUX_REGS != C::LAUNCH_REGS) ptx::regs_dec<C::AUX_REGS>();
        const int vw = warp - (AW + 4);  // rows [32*vw, 32*vw + 32) of each chunk = two segments
        constexpr int DP = C::DP;
        constexpr int PPR = DP / 8;    // 16-byte pieces per row of a V slot (padding pieces zero-filled)
        constexpr int RPI = 32 / PPR;  // rows per warp instruction
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
                vrow0 = (int32_t)(bi * p.v_ub + hi * p.v_uh);  // first row (of D elements) of this head
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
                // slot (gc % 2) is free once MMA2 of chunk gc-2 has completed
                const bool okw =
                    gc < 2 || bounded_wait(BAR(C::B_ODONE + (int)(gc & 1)), (uint32_t)(((gc - 2) >> 1) & 1), abort_flag);
                if (!__all_sync(0xffffffffu, okw)) {
                    ok = false;
                    break;
                }
                const int32_t first = __shfl_sync(0xffffffffu, idx, lane & 16);
                const bool run = idx >= 0 && idx == first + (lane & 15) && first + 15 < L;
                const uint32_t runs = __ballot_sync(0xffffffffu, run);
                if (idx >= L) atomicOr(&g_device_error, kErrBadIndex);
                if (idx < 0 || idx >= L) idx = 0;  // past the list, or corrupt: key 0 (scores are masked)
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
                                                     &p.tmap_v16, pn * 64, (int32_t)(bh * L + fs), BAR(C::B_VFULL + st));
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
    } else if (warp == AW + 3 || (!GATHER && warp == AW + 2)) {
        // ===================================================== MMA issuers
        // Two issuing threads, one per MMA kind, so that neither waits behind the
        // other's inputs: warp A+3 issues the scores of a chunk as soon as its K rows
        // have landed and its TMEM slot is free; warp A+2 issues the P.V of a chunk as
        // soon as its V rows and probabilities are ready.  The tensor pipe takes the
        // two streams in arrival order; each thread's commits track its own MMAs.
        if constexpr (C::AUX_REGS != C::LAUNCH_REGS) ptx::regs_dec<C::AUX_REGS>();
        {
            constexpr uint32_t IDESC1 = umma_idesc_bf16(128, MQ, false, false);
            constexpr uint32_t IDESC2 = umma_idesc_bf16(C::DP, MQ, true, true);
            constexpr uint32_t P_LAYOUT = (C::P_ROW == 128) ? 2u : (C::P_ROW == 64) ? 4u : 6u;
            constexpr uint32_t HI_V = umma_desc_hi(1024u, 2u);   // V^T: MN-major, 128B swizzle
            constexpr uint32_t HI_P = umma_desc_hi(8u * C::P_ROW, P_LAYOUT);
            const uint32_t qlo = umma_desc_lo(QTILE, 16u);
            bool ok = true;
            auto issue_pv = [&](int64_t gm, int64_t cm) -> bool {
                const int vs = (int)(gm % NV);
                const int pb = (int)(gm % NP);
                if (!bounded_wait(BAR(C::B_VFULL + vs), (uint32_t)((gm / NV) & 1), abort_flag)) return false;
                if (!bounded_wait(BAR(C::B_PFULL + pb), (uint32_t)((gm / NP) & 1), abort_flag)) return false;
                ptx::tc_fence_after();
                ptx::fence_proxy_async_smem();
                // The descriptors are formed before the MMAs so that the eight issues run
                // back to back (descriptor arithmetic between issues stalls the single
                // issuing thread, and with it the tensor pipe).
                const uint32_t alo = umma_desc_lo(VSLOT(vs), 128u * 128u);
                const uint32_t blo = umma_desc_lo(PBUF(pb), (uint32_t)C::P_PANEL);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t ad = umma_desc_join(alo + (uint32_t)(kk * 2048 >> 4), HI_V);
                    const uint64_t bd = umma_desc_join(blo + (uint32_t)(kk * 16 * C::P_ROW >> 4), HI_P);
                    ptx::mma_bf16_ss(tO, ad, bd, IDESC2, (cm > 0 || kk > 0) ? 1u : 0u);
                }
                ptx::mma_commit(BAR(C::B_ODONE + (int)(gm & 1)));
                return true;
            };
            // S^T of chunk gc into its slot (MMA1), once its K rows have landed and the
            // softmax has copied the slot's previous contents (chunk gc-2) to registers.
            auto issue_s = [&](int64_t gc, int64_t c, int64_t it) -> bool {
                const int ks = (int)(gc % NK);
                const int s = (int)(gc & 1);
                if (c == 0 && !bounded_wait(BAR(C::B_QFULL), (uint32_t)(it & 1), abort_flag)) return false;
                if (!bounded_wait(BAR(C::B_KFULL + ks), (uint32_t)((gc / NK) & 1), abort_flag)) return false;
                if (gc >= 2 && !bounded_wait(BAR(C::B_SFREE + s), (uint32_t)(((gc >> 1) - 1) & 1), abort_flag))
                    return false;
                ptx::tc_fence_after();
                const uint32_t alo = umma_desc_lo(KSLOT(ks), 16u);
                const uint32_t dS = tS0 + (uint32_t)s * MQ;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (uint32_t)(kk / 4) * (128 * 128) + (uint32_t)(kk % 4) * 32u;
                    const uint32_t qoff = (uint32_t)(kk / 4) * (MQ * 128) + (uint32_t)(kk % 4) * 32u;
                    // K rows and Q rows: K-major, the panel's swizzle
                    const uint64_t ad = umma_desc_join(alo + (koff >> 4), C::HD::desc_hi(kk / 4));
                    const uint64_t bd = umma_desc_join(qlo + (qoff >> 4), C::HD::desc_hi(kk / 4));
                    ptx::mma_bf16_ss(dS, ad, bd, IDESC1, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(BAR(C::B_SFULL + s));
                return true;
            };
            // The whole warp walks the items (a fused kernel reads each item's mask row
            // with all lanes); lane 0 issues and commits.
            int64_t g = 0, it = 0;
            for (int64_t item = blockIdx.x; item < p.items && ok; item += gridDim.x, ++it) {
                MaskRow mr;
                const int64_t nch = (item_keys<FUSED, MQ>(p, item, false, mr, lane) + 127) / 128;
                if (lane == 0) {
                    if constexpr (GATHER) {
                        // one issuing thread: S of chunks 0 and 1, then for every chunk c the
                        // S of chunk c+2 (its slot frees early in softmax(c)) before the P.V of c
                        for (int64_t c = 0; c < nch && c < 2 && ok; ++c) ok = issue_s(g + c, c, it);
                        for (int64_t c = 0; c < nch && ok; ++c) {
                            if (c + 2 < nch) ok = issue_s(g + c + 2, c + 2, it);
                            if (ok) ok = issue_pv(g + c, c);
                        }
                    } else {
                        for (int64_t c = 0; c < nch && ok; ++c)
                            ok = (warp == AW + 3) ? issue_s(g + c, c, it) : issue_pv(g + c, c);
                    }
                }
                ok = __shfl_sync(0xffffffffu, ok, 0);
                g += nch;
            }
            // drain: every MMA this thread issued has completed before TMEM is freed
            if (lane == 0) {
                const int drain = (warp == AW + 3) ? C::B_DRAIN : C::B_DRAIN2;
                ptx::mma_commit(BAR(drain));
                bounded_wait(BAR(drain), 0u, abort_flag, /*honour_abort=*/false);
            }
        }
        __syncwarp();
    } else {
        // ===================================================== softmax / epilogue (NSW warpgroups)
        if constexpr (C::SOFT_REGS != C::LAUNCH_REGS) ptx::regs_inc<C::SOFT_REGS>();
        const int wg = warp >> 2;         // 0 .. NSW-1
        const int wq = warp & 3;          // warp within the group = TMEM lane quarter
        const int t = threadIdx.x & 127;  // key lane within a chunk; TMEM lane t
        const uint32_t nbar = 1u + (uint32_t)wg;
        const uint32_t lane_base = (uint32_t)(wq * 32) << 16;
        const uint32_t col0 = (uint32_t)(wg * CW);  // this group's first query column
        // d index held by this thread in the O^T accumulator (M = D layout)
        // (the O^T accumulator has DP lanes; at D = 96 lanes 96..127 hold the zero padding)
        const int dt = (C::DP == 128) ? (t < D ? t : -1) : ((lane < 16) ? wq * 16 + lane : -1);
        float* mref = reinterpret_cast<float*>(smem + C::OFF_MREF) + wg * CW;
        float* alpha = reinterpret_cast<float*>(smem + C::OFF_ALPHA) + wg * CW;
        float* lfin = reinterpret_cast<float*>(smem + C::OFF_LFIN) + wg * CW;
        float* red = reinterpret_cast<float*>(smem + C::OFF_RED) + wg * 4 * CW;
        __nv_bfloat16* stage = reinterpret_cast<__nv_bfloat16*>(smem + C::OFF_STAGE + wg * C::STAGE);
        const float cs = p.scale_log2;
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
            if (t < CW) mref[t] = -INFINITY;
            float lp[CW];
#pragma unroll
            for (int q = 0; q < CW; ++q) lp[q] = 0.f;
            ptx::named_sync(nbar, 128);
            // A wait that gives up (timeout or another role's abort) only sets `failed`:
            // the loop keeps its barrier sequence matched across the warpgroup and the
            // group leaves together after the item.
            bool failed = false;
            float v[CW];
            // Wait for the scores of item chunk cc, release what their MMA read, and load
            // them into dst.
            auto load_chunk = [&](int64_t cc, auto& dst) {
                const int64_t gx = g + cc;
                const int sx = (int)(gx & 1);
                if (!bounded_wait(BAR(C::B_SFULL + sx), (uint32_t)((gx >> 1) & 1), abort_flag)) failed = true;
                ptx::tc_fence_after();
                if (wg == 0 && t == 0) {
                    // MMA1 of this chunk has finished reading its K slot (and, for the
                    // item's last chunk, the query tile)
                    ptx::mbar_arrive(BAR(C::B_KEMPTY + (int)(gx % NK)));
                    if (cc == nch - 1) ptx::mbar_arrive(BAR(C::B_QEMPTY));
                }
                const uint32_t ta = tS0 + (uint32_t)sx * MQ + col0 + lane_base;
                if constexpr (CW >= 32) {
#pragma unroll
                    for (int pi = 0; pi < CW / 32; ++pi) {
                        float tmp[32];
                        ptx::tmem_ld32(ta + pi * 32, tmp);
#pragma unroll
                        for (int j = 0; j < 32; ++j) dst[pi * 32 + j] = tmp[j];
                    }
                } else if constexpr (CW == 16) {
                    ptx::tmem_ld16(ta, dst);
                } else {
                    ptx::tmem_ld8(ta, dst);
                }
            };
            load_chunk(0, v);
            for (int64_t c = 0; c < nch; ++c) {
                const int64_t gc = g + c;
                const int s = (int)(gc & 1);
                const int pb = (int)(gc % NP);
                if (c > 0) load_chunk(c, v);
                ptx::tmem_wait_ld();
                // the scores are in registers: the slot is free for the MMA of chunk gc+2
                ptx::tc_fence_before();
                ptx::mbar_arrive(BAR(C::B_SFREE + s));
                const bool valid = c * 128 + t < cnt;
                // ---- v <- score * scale * log2(e) - reference, and the largest excess over
                // the references (log2 units).  The first chunk of an item always takes the
                // exact path below (the references start at -inf).
                bool need = true;
                if (c > 0) {
                    float dmax = -INFINITY;
#pragma unroll
                    for (int q = 0; q < CW; q += 4) {
                        const float4 m4 = *reinterpret_cast<const float4*>(mref + q);
                        v[q] = fmaf(v[q], cs, -m4.x);
                        v[q + 1] = fmaf(v[q + 1], cs, -m4.y);
                        v[q + 2] = fmaf(v[q + 2], cs, -m4.z);
                        v[q + 3] = fmaf(v[q + 3], cs, -m4.w);
                        dmax = ptx::max3(dmax, v[q], v[q + 1]);
                        dmax = ptx::max3(dmax, v[q + 2], v[q + 3]);
                    }
                    need = ptx::named_red_or(nbar, 128, valid && dmax > TAU);
                }
                if (need) {
                    // ---- back to scaled scores, exact column maxima -> raised references
#pragma unroll
                    for (int q = 0; q < CW; ++q) v[q] = (c == 0) ? v[q] * cs : v[q] + mref[q];
#pragma unroll
                    for (int q = 0; q < CW; ++q) {
                        float x = valid ? v[q] : -INFINITY;
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
                        if (lane == (q & 31)) red[wq * CW + q] = x;
                    }
                    ptx::named_sync(nbar, 128);
                    if (t < CW) {
                        const float mo = mref[t];
                        const float mn =
                            fmaxf(mo, fmaxf(fmaxf(red[t], red[CW + t]), fmaxf(red[2 * CW + t], red[3 * CW + t])));
                        alpha[t] = ptx::ex2(mo - mn);
                        mref[t] = mn;
                    }
                    ptx::named_sync(nbar, 128);
#pragma unroll
                    for (int q = 0; q < CW; ++q) {
                        lp[q] *= alpha[q];
                        v[q] -= mref[q];
                    }
                    if (c > 0) {
                        // O holds this item's chunks < c: wait for the last of them, rescale our columns
                        const int64_t gp = gc - 1;
                        if (!bounded_wait(BAR(C::B_ODONE + (int)(gp & 1)), (uint32_t)((gp >> 1) & 1), abort_flag))
                            failed = true;
                        ptx::tc_fence_after();
#pragma unroll
                        for (int q0 = 0; q0 < CW; q0 += 8) {
                            float o[8];
                            ptx::tmem_ld8(tO + col0 + q0 + lane_base, o);
                            ptx::tmem_wait_ld();
#pragma unroll
                            for (int j = 0; j < 8; ++j) o[j] *= alpha[q0 + j];
                            ptx::tmem_st8(tO + col0 + q0 + lane_base, o);
                        }
                        ptx::tmem_wait_st();
                        // the rescaled accumulator must reach TMEM before the next P.V
                        ptx::tc_fence_before();
                    }
                }
                if (!valid) {
#pragma unroll
                    for (int q = 0; q < CW; ++q) v[q] = -INFINITY;
                }
                // ---- the P buffer is free once the MMA that last read it has completed
                if (gc >= NP) {
                    const int64_t gr = gc - NP;
                    if (!bounded_wait(BAR(C::B_ODONE + (int)(gr & 1)), (uint32_t)((gr >> 1) & 1), abort_flag))
                        failed = true;
                }
                // ---- probabilities -> bf16 P^T row of this key, our query columns
                const uint32_t prow = PBUF(pb);
#pragma unroll
                for (int q = 0; q < CW; q += 8) {
                    uint32_t packed[4];
#pragma unroll
                    for (int j = 0; j < 8; j += 2) {
                        const float p0 = ptx::ex2(v[q + j]);
                        const float p1 = ptx::ex2(v[q + j + 1]);
                        lp[q + j] += p0;
                        lp[q + j + 1] += p1;
                        __nv_bfloat162 h = __floats2bfloat162_rn(p0, p1);
                        packed[j / 2] = *reinterpret_cast<uint32_t*>(&h);
                    }
                    const int chunk = (int)(col0 + q) / 8;  // 16-byte chunk = 8 queries
                    const int panel = chunk / C::P_CPR;
                    const uint32_t addr = prow + (uint32_t)panel * C::P_PANEL + swz(t, chunk % C::P_CPR, C::P_ROW);
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(packed[0]),
                                 "r"(packed[1]), "r"(packed[2]), "r"(packed[3])
                                 : "memory");
                }
                // generic-proxy P writes -> visible to the tensor core's async proxy
                ptx::fence_proxy_async_smem();
                ptx::mbar_arrive(BAR(C::B_PFULL + pb));
            }
            // ===================== epilogue: O / l -> bf16 rows, lse (our query columns)
            const int64_t e = g + nch - 1;
            if (!bounded_wait(BAR(C::B_ODONE + (int)(e & 1)), (uint32_t)((e >> 1) & 1), abort_flag)) failed = true;
            if (ptx::named_red_or(nbar, 128, failed)) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int q = 0; q < CW; ++q) {
                float x = lp[q];
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
                if (lane == (q & 31)) red[wq * CW + q] = x;
            }
            ptx::named_sync(nbar, 128);
            if (t < CW) {
                const float l = (red[t] + red[CW + t]) + (red[2 * CW + t] + red[3 * CW + t]);
                lfin[t] = 1.0f / l;
                const int64_t row = qb * MQ + col0 + t;
                if (p.lse != nullptr && row < L) {
                    float lg;
                    asm("lg2.approx.f32 %0, %1;" : "=f"(lg) : "f"(l));
                    p.lse[bh * L + row] = (mref[t] + lg) * 0.69314718055994530942f;
                }
            }
            ptx::named_sync(nbar, 128);
            __nv_bfloat16* outb = p.out + (size_t)bh * L * D;
            int64_t ostride = D;  // elements between consecutive query rows of out
            if constexpr (STRIDED) {
                const int64_t bi = bh / p.H;
                outb = p.out + bi * p.o_sb + (bh - bi * p.H) * p.o_sh;
                ostride = p.o_sl;
            }
            constexpr int SR = C::SROWS;
#pragma unroll 1
            for (int q0 = 0; q0 < CW; q0 += SR) {
                float o[SR];
                if constexpr (SR == 16) {
                    ptx::tmem_ld16(tO + col0 + q0 + lane_base, o);
                } else {
                    ptx::tmem_ld8(tO + col0 + q0 + lane_base, o);
                }
                ptx::tmem_wait_ld();
                if (dt >= 0) {
#pragma unroll
                    for (int j = 0; j < SR; ++j) stage[j * D + dt] = __float2bfloat16_rn(o[j] * lfin[q0 + j]);
                }
                ptx::named_sync(nbar, 128);
                for (int vi = t; vi < SR * (D / 8); vi += 128) {
                    const int r = vi / (D / 8), pc = vi % (D / 8);
                    const int64_t row = qb * MQ + col0 + q0 + r;
                    if (row < L) {
                        const uint4 val = *reinterpret_cast<const uint4*>(stage + r * D + pc * 8);
                        *reinterpret_cast<uint4*>(outb + row * ostride + pc * 8) = val;
                    }
                }
                ptx::named_sync(nbar, 128);
            }
            ptx::tc_fence_before();
            g += nch;
        }
    }

    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == AW + 3) ptx::tmem_dealloc(tmem, C::TMEM_COLS);
}

}  // namespace fgattn
