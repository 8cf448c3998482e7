// Mask compaction: packed per-(b, h, query block) N-group bitmask -> ascending
// kept key indices and their count.  Which tiles are computed is the whole of
// the method's skipping rule ("FG-Attn: Leveraging Fine-Grained Sparse
// Attention in Video Diffusion Models", Abstract: skip M x N tiles); this
// kernel turns it into gather lists for the attention kernel.
//
// One warp per row.  The warp reads 32 mask words at a time (one per lane,
// coalesced), forces the row's diagonal groups, drops bits >= G, counts the
// keys each word contributes (popc * N, minus the short last group), takes a
// warp-wide exclusive prefix sum with shuffles, and each lane then writes the
// key runs of its own set bits in ascending order (16-byte vector stores where
// the run is aligned).
#pragma once

#include <cstdint>

namespace fgattn {

__global__ void __launch_bounds__(256) compact_mask_kernel(const uint32_t* __restrict__ mask, int64_t rows,
                                                           int64_t QB, int64_t L, int64_t M, int64_t N,
                                                           int64_t G, int64_t W, int32_t* __restrict__ kept_idx,
                                                           int32_t* __restrict__ kept_cnt, int64_t cap) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int64_t qb = row % QB;
    const int64_t glo = (qb * M) / N;                                // diagonal groups [glo, ghi]
    const int64_t ghi = ((qb * M + M < L ? qb * M + M : L) - 1) / N;
    const int64_t lastlen = L - (G - 1) * N;                         // keys in group G-1
    const uint32_t* mrow = mask + row * W;
    int32_t* out = kept_idx + row * cap;
    int64_t base = 0;
    for (int64_t wb = 0; wb < W; wb += 32) {
        const int64_t wi = wb + lane;
        uint32_t word = (wi < W) ? __ldg(mrow + wi) : 0u;
        const int64_t g0 = wi * 32;
        const int64_t lo = glo - g0 > 0 ? glo - g0 : 0;
        const int64_t hi = ghi - g0 < 31 ? ghi - g0 : 31;
        if (lo <= hi) {
            const int nb = (int)(hi - lo + 1);
            word |= (nb == 32 ? 0xffffffffu : ((1u << nb) - 1u)) << lo;
        }
        const int64_t nvalid = G - g0;                               // groups of this word that exist
        if (nvalid <= 0) word = 0u;
        else if (nvalid < 32) word &= (1u << nvalid) - 1u;
        int64_t n = (int64_t)__popc(word) * N;
        if (nvalid >= 1 && nvalid <= 32 && ((word >> (nvalid - 1)) & 1u)) n -= N - lastlen;
        int64_t incl = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int64_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        const int64_t total = __shfl_sync(0xffffffffu, incl, 31);
        int64_t pos = base + incl - n;
        while (word) {
            const int b = __ffs(word) - 1;
            word &= word - 1u;
            const int64_t gidx = g0 + b;
            const int32_t start = (int32_t)(gidx * N);
            const int64_t len = (gidx == G - 1) ? lastlen : N;
            int64_t r = 0;
            for (; r < len && ((pos + r) & 3); ++r) out[pos + r] = start + (int32_t)r;
            for (; r + 4 <= len; r += 4) {
                const int32_t s = start + (int32_t)r;
                *reinterpret_cast<int4*>(out + pos + r) = make_int4(s, s + 1, s + 2, s + 3);
            }
            for (; r < len; ++r) out[pos + r] = start + (int32_t)r;
            pos += len;
        }
        base += total;
    }
    if (lane == 0) kept_cnt[row] = (int32_t)base;
}

}  // namespace fgattn
