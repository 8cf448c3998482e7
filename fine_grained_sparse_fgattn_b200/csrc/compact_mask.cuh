// Mask compaction: packed per-(b, h, query block) N-group bitmask -> ascending
// kept key indices and their count.  Which tiles are computed is the whole of
// the method's skipping rule ("FG-Attn: Leveraging Fine-Grained Sparse
// Attention in Video Diffusion Models", Abstract: skip M x N tiles); this
// kernel turns it into gather lists for the attention kernel.
//
// A warp takes 32 mask words at a time (one per lane, coalesced), forces the
// row's diagonal groups, drops bits >= G, and takes warp-wide prefix sums
// (shuffles) of the set-group counts.  It then writes the batch's output
// cooperatively: lane l produces output vector l of every 32-vector round,
// locating the kept group that holds that position by a five-step binary
// search over the lanes' prefix counts and the n-th-set-bit instruction, so
// each warp store covers consecutive addresses.  Vectors are int4 when N is a
// multiple of 4 (every group starts 16-byte aligned), single ints otherwise.
//
// Two launch shapes share that batch routine.  compact_mask_kernel: one warp
// per row, walking the row's batches in order (rows of up to 64 words, or
// enough rows to fill the GPU).  compact_mask_split_kernel: one block of eight
// warps per row, each warp owning a contiguous range of the row's batches; the
// warps first count their keys, take a block prefix sum through shared
// memory, then write at their offsets.  Long rows with few of them (the
// per-key layer: 1024 rows of 256 words) no longer wait on one warp walking
// eight batches in series (24 vs 39 us); with enough rows to fill the GPU the
// one-warp kernel stays faster, so the host picks by row count.
#pragma once

#include <cstdint>

namespace fgattn {

// Geometry of one row (b, h, qb).
struct CompactRow {
    int64_t glo, ghi;  // diagonal groups [glo, ghi]
    int64_t G, N, lastlen;
};

__device__ __forceinline__ CompactRow compact_row(int64_t row, int64_t QB, int64_t L, int64_t M, int64_t N,
                                                  int64_t G) {
    const int64_t qb = row % QB;
    CompactRow r;
    r.glo = (qb * M) / N;
    r.ghi = ((qb * M + M < L ? qb * M + M : L) - 1) / N;
    r.G = G;
    r.N = N;
    r.lastlen = L - (G - 1) * N;  // keys in group G-1
    return r;
}

// Word `wi` of the row with the diagonal groups forced and the bits of groups
// that do not exist cleared (`raw` = the stored word, 0 past the row).
__device__ __forceinline__ uint32_t forced_word(uint32_t raw, int64_t wi, const CompactRow& r) {
    const int64_t g0 = wi * 32;
    const int64_t lo = r.glo - g0 > 0 ? r.glo - g0 : 0;
    const int64_t hi = r.ghi - g0 < 31 ? r.ghi - g0 : 31;
    uint32_t word = raw;
    if (lo <= hi) {
        const int nb = (int)(hi - lo + 1);
        word |= (nb == 32 ? 0xffffffffu : ((1u << nb) - 1u)) << lo;
    }
    const int64_t nvalid = r.G - g0;  // groups of this word that exist
    if (nvalid <= 0)
        word = 0u;
    else if (nvalid < 32)
        word &= (1u << nvalid) - 1u;
    return word;
}

// Keys of one 32-word batch starting at word wb (every lane holds its word):
// returns the batch's key count; with WRITE, also writes the keys at out + base.
template <int VW, bool WRITE>
__device__ __forceinline__ int batch_keys(uint32_t word, int64_t wb, const CompactRow& r, int32_t* out, int64_t base,
                                          int lane) {
    // inclusive prefix sums of set groups over the 32 lanes
    const int cb = __popc(word);
    int inc = cb;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, inc, o);
        if (lane >= o) inc += y;
    }
    const int ngroups = __shfl_sync(0xffffffffu, inc, 31);
    if (ngroups == 0) return 0;
    const int64_t G = r.G, N = r.N;
    // keys in this batch: every group has N keys except group G-1
    const bool has_last = (G - 1 >= wb * 32) && (G - 1 < (wb + 32) * 32) &&
                          ((__shfl_sync(0xffffffffu, word, (int)(((G - 1) - wb * 32) / 32) & 31) >>
                            (((G - 1) - wb * 32) % 32)) & 1u);
    // (N <= L here, so every count and position below fits in 32 bits)
    const int n32 = (int)N;
    const int total = ngroups * n32 - (has_last ? (int)(N - r.lastlen) : 0);
    if constexpr (WRITE) {
        for (int pos0 = 0; pos0 < total; pos0 += 32 * VW) {
            const int n = pos0 + lane * VW;  // first key position of this lane's vector
            const int rk = n / n32;          // rank of the kept group holding it
            const int off = n - rk * n32;
            // first lane j whose inclusive count exceeds rk
            int j = 0;
#pragma unroll
            for (int step = 16; step > 0; step >>= 1) {
                const int cand = __shfl_sync(0xffffffffu, inc, j + step - 1);
                if (cand <= rk) j += step;
            }
            const uint32_t wj = __shfl_sync(0xffffffffu, word, j);
            const int exj = __shfl_sync(0xffffffffu, inc, j) - __popc(wj);
            if (n < total) {
                const int bit = __fns(wj, 0, rk - exj + 1);
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
    }
    return total;
}

template <int VW>  // keys written per lane per round: 4 (N % 4 == 0) or 1
__global__ void __launch_bounds__(256) compact_mask_kernel(const uint32_t* __restrict__ mask, int64_t rows,
                                                           int64_t QB, int64_t L, int64_t M, int64_t N,
                                                           int64_t G, int64_t W, int32_t* __restrict__ kept_idx,
                                                           int32_t* __restrict__ kept_cnt, int64_t cap) {
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (row >= rows) return;
    const CompactRow r = compact_row(row, QB, L, M, N, G);
    const uint32_t* mrow = mask + row * W;
    int32_t* out = kept_idx + row * cap;
    int64_t base = 0;  // keys written so far for this row
    uint32_t next = (lane < W) ? __ldg(mrow + lane) : 0u;
    for (int64_t wb = 0; wb < W; wb += 32) {
        const uint32_t word = forced_word(next, wb + lane, r);
        next = (wb + 32 + lane < W) ? __ldg(mrow + wb + 32 + lane) : 0u;  // prefetch the next batch
        base += batch_keys<VW, true>(word, wb, r, out, base, lane);
    }
    if (lane == 0) kept_cnt[row] = (int32_t)base;
}

// One block of eight warps per row; warp w owns batches [w * bpw, (w + 1) * bpw).
template <int VW>
__global__ void __launch_bounds__(256) compact_mask_split_kernel(const uint32_t* __restrict__ mask, int64_t QB,
                                                                 int64_t L, int64_t M, int64_t N, int64_t G,
                                                                 int64_t W, int32_t* __restrict__ kept_idx,
                                                                 int32_t* __restrict__ kept_cnt, int64_t cap) {
    __shared__ int64_t warp_keys[8];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int64_t row = blockIdx.x;
    const CompactRow r = compact_row(row, QB, L, M, N, G);
    const uint32_t* mrow = mask + row * W;
    int32_t* out = kept_idx + row * cap;
    const int64_t batches = (W + 31) / 32;
    const int64_t bpw = (batches + 7) / 8;
    const int64_t b0 = warp * bpw, b1 = (b0 + bpw < batches) ? b0 + bpw : batches;
    // pass 1: this warp's key count
    int64_t mine = 0;
    for (int64_t b = b0; b < b1; ++b) {
        const int64_t wi = b * 32 + lane;
        mine += batch_keys<VW, false>(forced_word(wi < W ? __ldg(mrow + wi) : 0u, wi, r), b * 32, r, out, 0, lane);
    }
    if (lane == 0) warp_keys[warp] = mine;
    __syncthreads();
    int64_t base = 0, total = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        base += i < warp ? warp_keys[i] : 0;
        total += warp_keys[i];
    }
    // pass 2: the keys, at this warp's offset
    for (int64_t b = b0; b < b1; ++b) {
        const int64_t wi = b * 32 + lane;
        base += batch_keys<VW, true>(forced_word(wi < W ? __ldg(mrow + wi) : 0u, wi, r), b * 32, r, out, base, lane);
    }
    if (threadIdx.x == 0) kept_cnt[row] = (int32_t)total;
}

}  // namespace fgattn
