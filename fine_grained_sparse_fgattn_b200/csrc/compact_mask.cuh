// Mask compaction: packed per-(b, h, query block) N-group bitmask -> ascending
// kept key indices and their count.  Which tiles are computed is the whole of
// the method's skipping rule ("FG-Attn: Leveraging Fine-Grained Sparse
// Attention in Video Diffusion Models", Abstract: skip M x N tiles); this
// kernel turns it into gather lists for the attention kernel.
//
// One warp per row.  The warp reads 32 mask words at a time (one per lane,
// coalesced), forces the row's diagonal groups, drops bits >= G, and takes
// warp-wide prefix sums (shuffles) of the set-group counts.  It then writes the
// batch's output cooperatively: lane l produces output vector l of every
// 32-vector round, locating the kept group that holds that position by a
// five-step binary search over the lanes' prefix counts and the n-th-set-bit
// instruction, so each warp store covers consecutive addresses.  Vectors are
// int4 when N is a multiple of 4 (every group starts 16-byte aligned), single
// ints otherwise.
#pragma once

#include <cstdint>

namespace fgattn {

template <int VW>  // keys written per lane per round: 4 (N % 4 == 0) or 1
__global__ void __launch_bounds__(256) compact_mask_kernel(const uint32_t* __restrict__ mask, int64_t rows,
                                                           int64_t QB, int64_t L, int64_t M, int64_t N,
                                                           int64_t G, int64_t W, int32_t* __restrict__ kept_idx,
                                                           int32_t* __restrict__ kept_cnt, int64_t cap) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int64_t qb = row % QB;
    const int64_t glo = (qb * M) / N;  // diagonal groups [glo, ghi]
    const int64_t ghi = ((qb * M + M < L ? qb * M + M : L) - 1) / N;
    const int64_t lastlen = L - (G - 1) * N;  // keys in group G-1
    const uint32_t* mrow = mask + row * W;
    int32_t* out = kept_idx + row * cap;
    int64_t base = 0;  // keys written so far for this row
    uint32_t next = (lane < W) ? __ldg(mrow + lane) : 0u;
    for (int64_t wb = 0; wb < W; wb += 32) {
        const int64_t wi = wb + lane;
        uint32_t word = next;
        next = (wb + 32 + lane < W) ? __ldg(mrow + wb + 32 + lane) : 0u;  // prefetch the next batch
        const int64_t g0 = wi * 32;
        const int64_t lo = glo - g0 > 0 ? glo - g0 : 0;
        const int64_t hi = ghi - g0 < 31 ? ghi - g0 : 31;
        if (lo <= hi) {
            const int nb = (int)(hi - lo + 1);
            word |= (nb == 32 ? 0xffffffffu : ((1u << nb) - 1u)) << lo;
        }
        const int64_t nvalid = G - g0;  // groups of this word that exist
        if (nvalid <= 0) word = 0u;
        else if (nvalid < 32) word &= (1u << nvalid) - 1u;
        // inclusive prefix sums of set groups over the 32 lanes
        const int cb = __popc(word);
        int inc = cb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        const int ngroups = __shfl_sync(0xffffffffu, inc, 31);
        if (ngroups == 0) continue;
        // keys in this batch: every group has N keys except group G-1
        const bool has_last = (G - 1 >= wb * 32) && (G - 1 < (wb + 32) * 32) &&
                              ((__shfl_sync(0xffffffffu, word, (int)(((G - 1) - wb * 32) / 32) & 31) >>
                                (((G - 1) - wb * 32) % 32)) & 1u);
        // (N <= L here, so every count and position below fits in 32 bits)
        const int n32 = (int)N;
        const int total = ngroups * n32 - (has_last ? (int)(N - lastlen) : 0);
        for (int pos0 = 0; pos0 < total; pos0 += 32 * VW) {
            const int n = pos0 + lane * VW;  // first key position of this lane's vector
            const int r = n / n32;           // rank of the kept group holding it
            const int off = n - r * n32;
            // first lane j whose inclusive count exceeds r
            int j = 0;
#pragma unroll
            for (int step = 16; step > 0; step >>= 1) {
                const int cand = __shfl_sync(0xffffffffu, inc, j + step - 1);
                if (cand <= r) j += step;
            }
            const uint32_t wj = __shfl_sync(0xffffffffu, word, j);
            const int exj = __shfl_sync(0xffffffffu, inc, j) - __popc(wj);
            if (n < total) {
                const int bit = __fns(wj, 0, r - exj + 1);
                const int32_t key = (int32_t)(((wb + j) * 32 + bit) * N + off);
                int32_t* dst = out + base + n;
                if constexpr (VW == 4) {
                    if (n + 4 <= total) {
                        *reinterpret_cast<int4*>(dst) = make_int4(key, key + 1, key + 2, key + 3);
                    } else {
                        for (int e = 0; e < 4 && n + e < total; ++e) dst[e] = key + e;
                    }
                } else {
                    *dst = key;
                }
            }
        }
        base += total;
    }
    if (lane == 0) kept_cnt[row] = (int32_t)base;
}

}  // namespace fgattn
