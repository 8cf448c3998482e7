// Fused mask expansion: the kept keys of one query block read straight from the
// packed tile mask, by the warp that needs them, with no kept list in memory.
//
// The method skips M x N tiles ("FG-Attn: Leveraging Fine-Grained Sparse
// Attention in Video Diffusion Models", Abstract); the mask holds one bit per
// tile (row (b, h, qb) of W uint32 words, group g = bit g % 32 of word g / 32).
// A block's key list is its kept groups in ascending order, each expanded to
// its keys; the position of key j of the list is therefore fixed by the
// number of kept groups before it.  A warp loads the row once per work item
// (W <= 256 words: eight per lane), forces the block's diagonal groups and
// drops bits past the last group (the same rules as the compaction kernel),
// takes a prefix sum of the lanes' set-bit counts, and then finds the key at
// any list position by itself: a five-step search over the lanes' prefix
// counts, the lane's words by shuffle, and the n-th set bit of one word.  Every
// role of the forward kernel that reads list entries does this for its own
// entries, so the roles need no shared index structure.
#pragma once

#include <cstdint>

namespace fgattn {

constexpr int kFusedMaxWords = 256;  // mask words per row the fused expansion handles (G <= 8192)

struct MaskRow {
    static constexpr int WPL = kFusedMaxWords / 32;  // at most 8 words per lane
    uint32_t w[WPL];  // lane l holds words [l * wpl, l * wpl + wpl)
    int32_t wpl;      // words per lane: ceil(W / 32)
    int32_t incl;     // kept groups in lanes 0 .. lane (inclusive prefix over the warp)
    int32_t mine;     // kept groups in this lane's words
    int32_t keys;     // kept keys of the row = the list length (< 2^31)
    int32_t n;        // keys per group
};

// Warp-collective: row `item` (= (b * H + h) * QB + qb) of the mask.  mq = query
// rows per block, n = keys per group, g = groups per row, wds = words per row.
__device__ __forceinline__ void mask_row_load(MaskRow& r, const uint32_t* mask, int64_t item, int64_t qb_count,
                                              int64_t mq, int64_t n, int64_t g, int64_t wds, int64_t L, int lane) {
    const int64_t qb = item % qb_count;
    const uint32_t* row = mask + item * wds;
    const int32_t glo = (int32_t)((qb * mq) / n);  // diagonal groups [glo, ghi]
    const int32_t ghi = (int32_t)(((qb * mq + mq < L ? qb * mq + mq : L) - 1) / n);
    const int32_t wpl = (int32_t)((wds + 31) / 32);
    r.wpl = wpl;
    r.n = (int32_t)n;
    int mine = 0;
#pragma unroll
    for (int i = 0; i < MaskRow::WPL; ++i) {
        const int32_t wi = lane * wpl + i;
        uint32_t x = (i < wpl && wi < wds) ? __ldg(row + wi) : 0u;
        const int32_t g0 = wi * 32;
        const int32_t lo = glo - g0 > 0 ? glo - g0 : 0;
        const int32_t hi = ghi - g0 < 31 ? ghi - g0 : 31;
        if (lo <= hi) {
            const int nb = (int)(hi - lo + 1);
            x |= (nb == 32 ? 0xffffffffu : ((1u << nb) - 1u)) << lo;
        }
        const int64_t valid = (i < wpl) ? g - g0 : 0;  // groups of this word that exist
        if (valid <= 0)
            x = 0u;
        else if (valid < 32)
            x &= (1u << valid) - 1u;
        r.w[i] = x;
        mine += __popc(x);
    }
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
    }
    r.incl = incl;
    r.mine = mine;
    const int64_t total = __shfl_sync(0xffffffffu, incl, 31);
    // is the last group (which may hold fewer than n keys) kept?
    const int32_t wl = (int32_t)((g - 1) / 32);
    const int owner = wl / wpl, idx = wl % wpl;
    uint32_t mine_w = 0u;
#pragma unroll
    for (int i = 0; i < MaskRow::WPL; ++i)
        if (i == idx) mine_w = r.w[i];
    const uint32_t lw = __shfl_sync(0xffffffffu, mine_w, owner);
    const bool last_kept = (lw >> ((g - 1) % 32)) & 1u;
    const int64_t lastlen = L - (g - 1) * n;
    r.keys = (int32_t)(total * n - (last_kept ? n - lastlen : 0));
}

// Warp-collective: the key at list position pos (each lane its own pos); 0 for
// positions past the list (their scores are masked by the softmax).
__device__ __forceinline__ int32_t mask_row_key(const MaskRow& r, int64_t pos64, int lane) {
    const bool inside = pos64 >= 0 && pos64 < r.keys;
    const int32_t pos = inside ? (int32_t)pos64 : 0;
    const int32_t rank = pos / r.n;  // which kept group (32-bit division)
    const int32_t off = pos - rank * r.n;
    // first lane whose inclusive count exceeds rank
    int j = 0;
#pragma unroll
    for (int step = 16; step > 0; step >>= 1) {
        const int cand = __shfl_sync(0xffffffffu, r.incl, j + step - 1);
        if (cand <= rank) j += step;
    }
    int rr = rank - (__shfl_sync(0xffffffffu, r.incl, j) - __shfl_sync(0xffffffffu, r.mine, j));
    int32_t grp = 0;
    bool found = false;
#pragma unroll
    for (int i = 0; i < MaskRow::WPL; ++i) {
        if (i >= r.wpl) break;  // uniform across the warp
        const uint32_t wv = __shfl_sync(0xffffffffu, r.w[i], j);
        const int c = __popc(wv);
        if (!found && rr < c) {
            grp = (j * r.wpl + i) * 32 + (int)__fns(wv, 0u, rr + 1);
            found = true;
        }
        if (!found) rr -= c;
    }
    return inside ? grp * r.n + off : 0;
}

}  // namespace fgattn
