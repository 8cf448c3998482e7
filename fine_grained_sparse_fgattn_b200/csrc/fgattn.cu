// C ABI of the tile-sparse attention library (declared in include/fgattn.h).
// Host side only: argument validation, launch configuration, device error
// word, the host-to-host copy pipeline and the allocation-free entry point.
// The kernels are in compact_mask.cuh, attention_fwd.cuh (key-major),
// attention_fwd_qm.cuh (query-major) and attention_bwd.cuh (gradients).
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fgattn.h"
#include "attention_bwd.cuh"
#include "attention_fwd.cuh"
#include "attention_fwd_qm.cuh"
#include "compact_mask.cuh"

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int kMaxConfigDevices = 64;

// cuTensorMapEncodeTiled, fetched through the runtime so the library needs no -lcuda.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// Box shapes: 64 columns with 128B swizzle (128-byte shared-memory rows), or -- for
// columns 64..95 of a 96-element head -- 32 columns with 64B swizzle (64-byte rows).
struct BoxCols {
    uint32_t cols;
    CUtensorMapSwizzle swizzle;
};
constexpr BoxCols kWide = {64u, CU_TENSOR_MAP_SWIZZLE_128B};
constexpr BoxCols kNarrow = {32u, CU_TENSOR_MAP_SWIZZLE_64B};

// bf16 rows of d elements, `row_stride` elements apart, viewed in boxes of bc.cols
// columns x box_rows rows.
bool encode_rows(CUtensorMap* m, const void* base, int64_t rows, int64_t d, int64_t row_stride, uint32_t box_rows,
                 BoxCols bc = kWide) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)row_stride * 2};
    const cuuint32_t box[2] = {bc.cols, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, bc.swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// [B][H][L][d] view with element strides st = {sb, sh, sl} (d contiguous) as a 4-D
// map {d, L, H, B} in boxes of bc.cols columns x box_rows consecutive L positions.
bool encode_4d(CUtensorMap* m, const void* base, int64_t B, int64_t H, int64_t L, int64_t d, const int64_t* st,
               uint32_t box_rows, BoxCols bc = kWide) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)H, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)st[2] * 2, (cuuint64_t)st[1] * 2, (cuuint64_t)st[0] * 2};
    const cuuint32_t box[4] = {bc.cols, box_rows, 1u, 1u};
    const cuuint32_t estr[4] = {1u, 1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, bc.swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Strides of one tensor, in elements: {batch, head, token}.
struct Strides {
    int64_t s[3];
};

int current_sms() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    int sms = 0;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return sms;
}

// A tensor map is a pure function of a buffer's address, shape, strides and box, so
// the map set of a launch is cached under everything that determines it; repeated
// calls on the same buffers (the usual case for a layer called every denoising step)
// skip the host-side encodes.  Sixteen sets, replaced round-robin.
struct MapSetKey {
    const void* q;
    const void* k;
    const void* v;
    int64_t st[9];  // q, k, v strides
    int64_t B, H, L, d, k_rows;
    uint32_t mq;
    bool strided;
    bool operator==(const MapSetKey& o) const {
        if (q != o.q || k != o.k || v != o.v || B != o.B || H != o.H || L != o.L || d != o.d || k_rows != o.k_rows ||
            mq != o.mq || strided != o.strided)
            return false;
        for (int i = 0; i < 9; ++i)
            if (st[i] != o.st[i]) return false;
        return true;
    }
};
struct MapSet {
    CUtensorMap q, k, k16, v16, q_hi, k_hi, k16_hi;
};
constexpr int kMapCacheSize = 16;
std::mutex g_map_mutex;
MapSetKey g_map_keys[kMapCacheSize];
MapSet g_map_sets[kMapCacheSize];
bool g_map_valid[kMapCacheSize] = {};
int g_map_next = 0;

template <bool STRIDED>
bool encode_maps_uncached(fgattn::FwdParams& prm, const void* q, const Strides& qs, const void* k, const Strides& ks,
                          const void* v, const Strides& vs, int64_t B, int64_t H, int64_t d, int64_t k_rows,
                          uint32_t mq);

// The tensor maps of one launch: query tiles of mq rows, k row gathers, 16-key k and v
// boxes; at d = 96 also the 32-column maps of columns 64..95 of q and k.
template <bool STRIDED>
bool encode_maps(fgattn::FwdParams& prm, const void* q, const Strides& qs, const void* k, const Strides& ks,
                 const void* v, const Strides& vs, int64_t B, int64_t H, int64_t d, int64_t k_rows, uint32_t mq) {
    MapSetKey key = {q, k, v, {qs.s[0], qs.s[1], qs.s[2], ks.s[0], ks.s[1], ks.s[2], vs.s[0], vs.s[1], vs.s[2]},
                     B, H, prm.L, d, k_rows, mq, STRIDED};
    std::lock_guard<std::mutex> lock(g_map_mutex);
    for (int i = 0; i < kMapCacheSize; ++i)
        if (g_map_valid[i] && g_map_keys[i] == key) {
            const MapSet& m = g_map_sets[i];
            prm.tmap_q = m.q, prm.tmap_k = m.k, prm.tmap_k16 = m.k16, prm.tmap_v16 = m.v16;
            prm.tmap_q_hi = m.q_hi, prm.tmap_k_hi = m.k_hi, prm.tmap_k16_hi = m.k16_hi;
            return true;
        }
    if (!encode_maps_uncached<STRIDED>(prm, q, qs, k, ks, v, vs, B, H, d, k_rows, mq)) return false;
    const int i = g_map_next;
    g_map_next = (g_map_next + 1) % kMapCacheSize;
    g_map_keys[i] = key;
    g_map_sets[i] = {prm.tmap_q, prm.tmap_k, prm.tmap_k16, prm.tmap_v16, prm.tmap_q_hi, prm.tmap_k_hi, prm.tmap_k16_hi};
    g_map_valid[i] = true;
    return true;
}

template <bool STRIDED>
bool encode_maps_uncached(fgattn::FwdParams& prm, const void* q, const Strides& qs, const void* k, const Strides& ks,
                          const void* v, const Strides& vs, int64_t B, int64_t H, int64_t d, int64_t k_rows,
                          uint32_t mq) {
    const int64_t L = prm.L;
    const bool narrow = d == 96;
    if (STRIDED) {
        if (!encode_4d(&prm.tmap_q, q, B, H, L, d, qs.s, mq) || !encode_rows(&prm.tmap_k, k, k_rows, d, d, 1) ||
            !encode_4d(&prm.tmap_k16, k, B, H, L, d, ks.s, 16) || !encode_4d(&prm.tmap_v16, v, B, H, L, d, vs.s, 16))
            return false;
        if (narrow && (!encode_4d(&prm.tmap_q_hi, q, B, H, L, d, qs.s, mq, kNarrow) ||
                       !encode_rows(&prm.tmap_k_hi, k, k_rows, d, d, 1, kNarrow) ||
                       !encode_4d(&prm.tmap_k16_hi, k, B, H, L, d, ks.s, 16, kNarrow)))
            return false;
    } else {
        const int64_t rows = B * H * L;
        if (!encode_rows(&prm.tmap_q, q, rows, d, d, mq) || !encode_rows(&prm.tmap_k, k, rows, d, d, 1) ||
            !encode_rows(&prm.tmap_k16, k, rows, d, d, 16) || !encode_rows(&prm.tmap_v16, v, rows, d, d, 16))
            return false;
        if (narrow && (!encode_rows(&prm.tmap_q_hi, q, rows, d, d, mq, kNarrow) ||
                       !encode_rows(&prm.tmap_k_hi, k, rows, d, d, 1, kNarrow) ||
                       !encode_rows(&prm.tmap_k16_hi, k, rows, d, d, 16, kNarrow)))
            return false;
    }
    return true;
}

template <int D, int MQ, bool GATHER, bool STRIDED, bool FUSED>
fgattn_status launch_fwd(fgattn::FwdParams& prm, const void* q, const Strides& qs, const void* k, const Strides& ks,
                         const void* v, const Strides& vs, int64_t B, int64_t H, int64_t k_rows,
                         cudaStream_t stream) {
    using C = fgattn::FwdCfg<D, MQ, GATHER>;
    if (!encode_maps<STRIDED>(prm, q, qs, k, ks, v, vs, B, H, D, k_rows, MQ)) return FGATTN_ERR_CUDA;
    auto kernel = fgattn::fgattn_fwd_kernel<D, MQ, GATHER, STRIDED, FUSED>;
    // Request enough shared memory that exactly one block is resident per SM:
    // the grid is persistent (one block per SM, static round-robin over work).
    const int smem = C::SMEM_REQUEST > 120 * 1024 ? C::SMEM_REQUEST : 120 * 1024;
    // the attribute is per function and device: set and checked once per device
    static bool configured[kMaxConfigDevices] = {};
    int cdev = 0;
    if (cudaGetDevice(&cdev) != cudaSuccess || cdev < 0 || cdev >= kMaxConfigDevices) return FGATTN_ERR_CUDA;
    if (!configured[cdev]) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return FGATTN_ERR_CUDA;
        // The warp roles re-divide the block's registers with setmaxnreg, which only
        // completes if the launch allocates exactly the per-thread count the split
        // was sized for: refuse to launch otherwise (it would wait forever).
        cudaFuncAttributes attr;
        if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return FGATTN_ERR_CUDA;
        const bool split = C::SOFT_REGS != C::LAUNCH_REGS || C::AUX_REGS != C::LAUNCH_REGS;
        if (split && attr.numRegs != (int)C::LAUNCH_REGS) return FGATTN_ERR_UNSUPPORTED;
        configured[cdev] = true;
    }
    const int sms = current_sms();
    if (sms <= 0) return FGATTN_ERR_CUDA;
    const int64_t grid = prm.items < sms ? prm.items : sms;
    kernel<<<(unsigned)grid, C::THREADS, smem, stream>>>(prm);
    return cudaPeekAtLastError() == cudaSuccess ? FGATTN_OK : FGATTN_ERR_CUDA;
}

// Query-major kernel (128-row query blocks): M = 128 lists and dense runs.
template <int D, bool GATHER, bool STRIDED, bool FUSED>
fgattn_status launch_qm(fgattn::FwdParams& prm, const void* q, const Strides& qs, const void* k, const Strides& ks,
                        const void* v, const Strides& vs, int64_t B, int64_t H, int64_t k_rows, cudaStream_t stream) {
    using C = fgattn::QmCfg<D, GATHER>;
    if (!encode_maps<STRIDED>(prm, q, qs, k, ks, v, vs, B, H, D, k_rows, C::MQ)) return FGATTN_ERR_CUDA;
    auto kernel = fgattn::fgattn_fwd_qm_kernel<D, GATHER, STRIDED, FUSED>;
    const int smem = C::SMEM_REQUEST > 120 * 1024 ? C::SMEM_REQUEST : 120 * 1024;  // one block per SM
    // the attribute is per function and device: set and checked once per device
    static bool configured[kMaxConfigDevices] = {};
    int cdev = 0;
    if (cudaGetDevice(&cdev) != cudaSuccess || cdev < 0 || cdev >= kMaxConfigDevices) return FGATTN_ERR_CUDA;
    if (!configured[cdev]) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return FGATTN_ERR_CUDA;
        // setmaxnreg re-divides exactly the launch's registers: refuse any other count
        cudaFuncAttributes attr;
        if (cudaFuncGetAttributes(&attr, kernel) != cudaSuccess) return FGATTN_ERR_CUDA;
        if (attr.numRegs != (int)C::LAUNCH_REGS) return FGATTN_ERR_UNSUPPORTED;
        configured[cdev] = true;
    }
    const int sms = current_sms();
    if (sms <= 0) return FGATTN_ERR_CUDA;
    const int64_t grid = prm.items < sms ? prm.items : sms;
    kernel<<<(unsigned)grid, C::THREADS, smem, stream>>>(prm);
    return cudaPeekAtLastError() == cudaSuccess ? FGATTN_OK : FGATTN_ERR_CUDA;
}

template <int D, bool GATHER, bool STRIDED, bool FUSED>
fgattn_status dispatch_m(fgattn::FwdParams& prm, const void* q, const Strides& qs, const void* k, const Strides& ks,
                         const void* v, const Strides& vs, int64_t B, int64_t H, int64_t k_rows, int64_t M,
                         cudaStream_t s) {
    // 128-row query blocks (M = 128 lists or masks, or a dense run of any M: every key
    // is kept, so the result does not depend on M) go to the query-major kernel.
    if (M == 128 || (prm.kept_idx == nullptr && prm.mask == nullptr)) {
        prm.QB = (prm.L + 127) / 128;
        prm.items = B * H * prm.QB;
        // the query-major softmax needs a non-zero scale: a scale of magnitude below
        // 1e-30 (log2 units) gives the same probabilities (every score maps to 2^0)
        if (std::fabs(prm.scale_log2) < 1e-30f) prm.scale_log2 = prm.scale_log2 < 0.f ? -1e-30f : 1e-30f;
        return launch_qm<D, GATHER, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, s);
    }
    switch (M) {
        case 16: return launch_fwd<D, 16, GATHER, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, s);
        case 32: return launch_fwd<D, 32, GATHER, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, s);
        default: return launch_fwd<D, 64, GATHER, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, s);
    }
}

template <bool STRIDED, bool FUSED = false>
fgattn_status dispatch(fgattn::FwdParams& prm, const void* q, const Strides& qs, const void* k, const Strides& ks,
                       const void* v, const Strides& vs, int64_t B, int64_t H, int64_t k_rows, int64_t d, int64_t M,
                       bool gather, cudaStream_t s) {
    if (d == 128)
        return gather ? dispatch_m<128, true, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, M, s)
                      : dispatch_m<128, false, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, M, s);
    if (d == 96)
        return gather ? dispatch_m<96, true, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, M, s)
                      : dispatch_m<96, false, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, M, s);
    return gather ? dispatch_m<64, true, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, M, s)
                  : dispatch_m<64, false, STRIDED, FUSED>(prm, q, qs, k, ks, v, vs, B, H, k_rows, M, s);
}

// Shared by fgattn_forward (contiguous [B][H][L][d]) and fgattn_forward_strided.
fgattn_status forward_impl(const void* q, const Strides& qs, const void* k, const Strides& ks, const void* v,
                           const Strides& vs, const int32_t* kept_idx, const int32_t* kept_cnt, int64_t cap, int64_t B,
                           int64_t H, int64_t L, int64_t d, int64_t M, int64_t N, float scale, void* out,
                           const Strides& os, float* lse, fgattn_stream_t stream, const uint32_t* mask = nullptr) {
    if (!q || !k || !v || !out) return FGATTN_ERR_INVALID_ARG;
    if (kept_idx && !kept_cnt) return FGATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || L < 1 || M < 1 || N < 1 || d < 1) return FGATTN_ERR_INVALID_ARG;
    if (L > INT32_MAX || B > INT32_MAX || H > INT32_MAX) return FGATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return FGATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return FGATTN_ERR_INVALID_ARG;
    if (kept_idx && !aligned16(kept_idx)) return FGATTN_ERR_INVALID_ARG;  // rows are read as int4
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FGATTN_ERR_INVALID_ARG;
    if (kept_idx && (cap < L || (cap & 3))) return FGATTN_ERR_CAPACITY;
    if (d != 64 && d != 96 && d != 128) return FGATTN_ERR_UNSUPPORTED;
    if (M != 16 && M != 32 && M != 64 && M != 128) return FGATTN_ERR_UNSUPPORTED;
    // Strides: at least one row (d) and 16-byte multiples (TMA, vector stores); k and v
    // strides whole rows of d, so every key row is a row of the gather map over k.
    const Strides* all[4] = {&qs, &ks, &vs, &os};
    for (int t = 0; t < 4; ++t)
        for (int i = 0; i < 3; ++i) {
            const int64_t x = all[t]->s[i];
            if (x < d || (x & 7) || x >= (int64_t(1) << 38)) return FGATTN_ERR_INVALID_ARG;
            if (t >= 1 && t <= 2 && x % d) return FGATTN_ERR_INVALID_ARG;
        }
    const int64_t k_rows = ((B - 1) * ks.s[0] + (H - 1) * ks.s[1] + (L - 1) * ks.s[2]) / d + 1;
    const int64_t v_rows = ((B - 1) * vs.s[0] + (H - 1) * vs.s[1] + (L - 1) * vs.s[2]) / d + 1;
    // 32-bit TMA coordinates and row numbers in the kernels
    if (k_rows > INT32_MAX || v_rows > INT32_MAX || B * H * L > INT32_MAX) return FGATTN_ERR_UNSUPPORTED;

    fgattn::FwdParams prm;
    prm.kept_idx = kept_idx;
    prm.kept_cnt = kept_cnt;
    prm.mask = nullptr;
    prm.mask_w = prm.mask_g = prm.mask_n = 0;
    if (mask) {  // fused kernels: the mask is read in place of kept lists
        const int64_t Ng = N > L ? L : N;  // one key group either way when N > L
        prm.mask = mask;
        prm.mask_n = Ng;
        prm.mask_g = (L + Ng - 1) / Ng;
        prm.mask_w = (prm.mask_g + 31) / 32;
    }
    prm.out = static_cast<__nv_bfloat16*>(out);
    prm.lse = lse;
    prm.cap = kept_idx ? cap : L;
    prm.L = L;
    prm.H = H;
    prm.QB = (L + M - 1) / M;
    prm.items = B * H * prm.QB;
    prm.scale_log2 = scale * 1.4426950408889634f;
    prm.v_base = static_cast<const __nv_bfloat16*>(v);
    prm.k_ub = ks.s[0] / d, prm.k_uh = ks.s[1] / d, prm.k_ul = (int32_t)(ks.s[2] / d);
    prm.v_ub = vs.s[0] / d, prm.v_uh = vs.s[1] / d, prm.v_ul = (int32_t)(vs.s[2] / d);
    prm.o_sb = os.s[0], prm.o_sh = os.s[1], prm.o_sl = os.s[2];
    // Lists of whole 16-key runs (N a multiple of 16) load as TMA tiles: tile layout.
    // Anything else is gathered row by row: gather layout (more K producer warps).
    const bool gather = mask ? prm.mask_n % 16 != 0 : (kept_idx != nullptr && N % 16 != 0);
    // Contiguous [B][H][L][d] everywhere (strides of extent-1 dimensions aside): the
    // contiguous kernel.
    const Strides c = {{H * L * d, L * d, d}};
    const int64_t extent[3] = {B, H, L};
    bool contiguous = true;
    for (const Strides* t : {&qs, &ks, &vs, &os})
        for (int i = 0; i < 3; ++i) contiguous = contiguous && (extent[i] == 1 || t->s[i] == c.s[i]);
    cudaStream_t s = (cudaStream_t)stream;
    if (mask) {
        if (!contiguous) return FGATTN_ERR_UNSUPPORTED;
        return dispatch<false, true>(prm, q, qs, k, ks, v, vs, B, H, k_rows, d, M, gather, s);
    }
    if (contiguous) return dispatch<false>(prm, q, qs, k, ks, v, vs, B, H, k_rows, d, M, gather, s);
    return dispatch<true>(prm, q, qs, k, ks, v, vs, B, H, k_rows, d, M, gather, s);
}

}  // namespace

extern "C" {

int64_t fgattn_kept_capacity(int64_t L) {
    if (L < 1) return -1;
    return (L + 15) / 16 * 16;
}

fgattn_status fgattn_compact_mask(const uint32_t* mask, int64_t B, int64_t H, int64_t L, int64_t M, int64_t N,
                                  int32_t* kept_idx, int32_t* kept_cnt, int64_t cap, fgattn_stream_t stream) {
    if (!mask || !kept_idx || !kept_cnt) return FGATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || L < 1 || M < 1 || N < 1) return FGATTN_ERR_INVALID_ARG;
    if (L > INT32_MAX) return FGATTN_ERR_INVALID_ARG;
    if (!aligned16(kept_idx) || (reinterpret_cast<uintptr_t>(mask) & 3u)) return FGATTN_ERR_INVALID_ARG;
    if (cap < L || (cap & 3)) return FGATTN_ERR_CAPACITY;
    if (N > L) N = L;  // one key group either way (G = 1): same tiles, same keys
    const int64_t QB = (L + M - 1) / M;
    const int64_t G = (L + N - 1) / N;
    const int64_t W = (G + 31) / 32;
    const int64_t rows = B * H * QB;
    const int64_t blocks = (rows + 7) / 8;
    if (rows > INT32_MAX) return FGATTN_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    // Rows of more than two 32-word batches, and too few rows (one warp each) to fill
    // the GPU: eight warps per row.  (With enough rows the one-warp kernel is faster:
    // 0.55 vs 0.60 ms on 12288 rows of 1024 words.)
    const int sms = current_sms();
    if (W > 64 && rows < 32 * (int64_t)(sms > 0 ? sms : 148)) {
        if (N % 4 == 0)
            fgattn::compact_mask_split_kernel<4><<<(unsigned)rows, 256, 0, s>>>(mask, QB, L, M, N, G, W, kept_idx,
                                                                              kept_cnt, cap);
        else
            fgattn::compact_mask_split_kernel<1><<<(unsigned)rows, 256, 0, s>>>(mask, QB, L, M, N, G, W, kept_idx,
                                                                              kept_cnt, cap);
    } else if (N % 4 == 0) {
        fgattn::compact_mask_kernel<4><<<(unsigned)blocks, 256, 0, s>>>(mask, rows, QB, L, M, N, G, W, kept_idx,
                                                                       kept_cnt, cap);
    } else {
        fgattn::compact_mask_kernel<1><<<(unsigned)blocks, 256, 0, s>>>(mask, rows, QB, L, M, N, G, W, kept_idx,
                                                                       kept_cnt, cap);
    }
    return cudaPeekAtLastError() == cudaSuccess ? FGATTN_OK : FGATTN_ERR_CUDA;
}

fgattn_status fgattn_forward(const void* q, const void* k, const void* v, const int32_t* kept_idx,
                             const int32_t* kept_cnt, int64_t cap, int64_t B, int64_t H, int64_t L, int64_t d,
                             int64_t M, int64_t N, float scale, void* out, float* lse, fgattn_stream_t stream) {
    if (d < 1 || L < 1 || H < 1) return FGATTN_ERR_INVALID_ARG;
    const Strides c = {{H * L * d, L * d, d}};  // contiguous [B][H][L][d]
    return forward_impl(q, c, k, c, v, c, kept_idx, kept_cnt, cap, B, H, L, d, M, N, scale, out, c, lse, stream);
}

fgattn_status fgattn_forward_strided(const void* q, const int64_t* q_strides, const void* k, const int64_t* k_strides,
                                     const void* v, const int64_t* v_strides, const int32_t* kept_idx,
                                     const int32_t* kept_cnt, int64_t cap, int64_t B, int64_t H, int64_t L, int64_t d,
                                     int64_t M, int64_t N, float scale, void* out, const int64_t* out_strides,
                                     float* lse, fgattn_stream_t stream) {
    if (!q_strides || !k_strides || !v_strides || !out_strides) return FGATTN_ERR_INVALID_ARG;
    // The stride of a dimension of extent 1 is never applied: give it a valid value.
    auto norm = [&](const int64_t* st) {
        return Strides{{B == 1 ? d : st[0], H == 1 ? d : st[1], L == 1 ? d : st[2]}};
    };
    const Strides qs = norm(q_strides), ks = norm(k_strides), vs = norm(v_strides), os = norm(out_strides);
    return forward_impl(q, qs, k, ks, v, vs, kept_idx, kept_cnt, cap, B, H, L, d, M, N, scale, out, os, lse, stream);
}

fgattn_status fgattn_masked_forward(const void* q, const void* k, const void* v, const uint32_t* mask, int64_t B,
                                    int64_t H, int64_t L, int64_t d, int64_t M, int64_t N, float scale, void* out,
                                    float* lse, fgattn_stream_t stream) {
    if (!mask) return FGATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(mask) & 3u) return FGATTN_ERR_INVALID_ARG;
    if (d < 1 || L < 1 || H < 1 || N < 1) return FGATTN_ERR_INVALID_ARG;
    const int64_t Ng = N > L ? L : N;
    const int64_t W = ((L + Ng - 1) / Ng + 31) / 32;
    if (W > fgattn::kFusedMaxWords) return FGATTN_ERR_UNSUPPORTED;
    const Strides c = {{H * L * d, L * d, d}};  // contiguous [B][H][L][d]
    return forward_impl(q, c, k, c, v, c, nullptr, nullptr, L, B, H, L, d, M, N, scale, out, c, lse, stream, mask);
}

}  // extern "C"

namespace {

// fp32 gradient rows [B*H][L][d] as a 3-D map {d, L, B*H} in 32-column x 16-row boxes
// (128B swizzle): the target of the backward kernel's box reductions.  Boxes never
// reach past L, so a box never adds into another head's rows.
bool encode_grad_map(CUtensorMap* m, float* base, int64_t BH, int64_t L, int64_t d) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)L, (cuuint64_t)BH};
    const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)(L * d * 4)};
    const cuuint32_t box[3] = {32u, 16u, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int D, int MQ>
fgattn_status launch_bwd(const fgattn::BwdParams& prm, cudaStream_t s) {
    using C = fgattn::BwdCfg<D, MQ>;
    auto kernel = fgattn::fgattn_bwd_kernel<D, MQ>;
    // one block per SM: the block allocates up to all of the SM's TMEM columns
    const int smem = C::SMEM_REQUEST > 120 * 1024 ? C::SMEM_REQUEST : 120 * 1024;
    static bool configured[kMaxConfigDevices] = {};
    int cdev = 0;
    if (cudaGetDevice(&cdev) != cudaSuccess || cdev < 0 || cdev >= kMaxConfigDevices) return FGATTN_ERR_CUDA;
    if (!configured[cdev]) {
        if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
            return FGATTN_ERR_CUDA;
        configured[cdev] = true;
    }
    const int sms = current_sms();
    if (sms <= 0) return FGATTN_ERR_CUDA;
    const int64_t grid = prm.items < sms ? prm.items : sms;
    kernel<<<(unsigned)grid, C::THREADS, smem, s>>>(prm);
    return cudaPeekAtLastError() == cudaSuccess ? FGATTN_OK : FGATTN_ERR_CUDA;
}

template <int D>
fgattn_status launch_bwd_m(const fgattn::BwdParams& prm, int64_t M, cudaStream_t s) {
    switch (M) {
        case 16: return launch_bwd<D, 16>(prm, s);
        case 32: return launch_bwd<D, 32>(prm, s);
        default: return launch_bwd<D, 64>(prm, s);
    }
}

}  // namespace

extern "C" {

fgattn_status fgattn_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                              const float* lse, const int32_t* kept_idx, const int32_t* kept_cnt, int64_t cap,
                              int64_t B, int64_t H, int64_t L, int64_t d, int64_t M, int64_t N, float scale,
                              float* dq, float* dk, float* dv, float* delta, fgattn_stream_t stream) {
    if (!q || !k || !v || !out || !dout || !lse || !dq || !dk || !dv || !delta) return FGATTN_ERR_INVALID_ARG;
    if (kept_idx && !kept_cnt) return FGATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || L < 1 || M < 1 || N < 1 || d < 1) return FGATTN_ERR_INVALID_ARG;
    if (L > INT32_MAX || B > INT32_MAX || H > INT32_MAX) return FGATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return FGATTN_ERR_INVALID_ARG;
    for (const void* ptr : {q, k, v, out, dout, (const void*)dq, (const void*)dk, (const void*)dv})
        if (!aligned16(ptr)) return FGATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(lse) & 3u) || (reinterpret_cast<uintptr_t>(delta) & 3u) ||
        (kept_idx && (reinterpret_cast<uintptr_t>(kept_idx) & 3u)))
        return FGATTN_ERR_INVALID_ARG;
    if (kept_idx && (cap < L || (cap & 3))) return FGATTN_ERR_CAPACITY;
    if (d != 64 && d != 96 && d != 128) return FGATTN_ERR_UNSUPPORTED;
    if (M != 16 && M != 32 && M != 64 && M != 128) return FGATTN_ERR_UNSUPPORTED;
    if (B * H * L > INT32_MAX) return FGATTN_ERR_UNSUPPORTED;
    // tensor maps first: nothing is enqueued unless every host-side step succeeded
    fgattn::BwdParams prm;
    if (!encode_grad_map(&prm.tmap_dk, dk, B * H, L, d) || !encode_grad_map(&prm.tmap_dv, dv, B * H, L, d))
        return FGATTN_ERR_CUDA;
    const auto* gb = static_cast<const __nv_bfloat16*>(dout);
    prm.q = static_cast<const __nv_bfloat16*>(q);
    prm.k = static_cast<const __nv_bfloat16*>(k);
    prm.v = static_cast<const __nv_bfloat16*>(v);
    prm.dout = gb;
    prm.lse = lse;
    prm.delta = delta;
    prm.kept_idx = kept_idx;
    prm.kept_cnt = kept_cnt;
    prm.dq = dq;
    prm.dk = dk;
    prm.dv = dv;
    prm.cap = kept_idx ? cap : L;
    prm.L = L;
    // 128-row blocks run as two 64-row halves over the block's list (the kernel's
    // TMEM holds at most 64 query columns next to the dK/dV accumulators)
    const int64_t MQ = M > 64 ? 64 : M;
    prm.QB = (L + M - 1) / M;
    prm.msplit = M / MQ;
    prm.items = B * H * prm.QB * prm.msplit;
    prm.scale = scale;
    prm.scale_log2 = scale * 1.4426950408889634f;
    cudaStream_t s = (cudaStream_t)stream;
    const int64_t rows = B * H * L;
    const size_t grad_bytes = (size_t)rows * (size_t)d * sizeof(float);
    if (cudaMemsetAsync(dk, 0, grad_bytes, s) != cudaSuccess) return FGATTN_ERR_CUDA;
    if (cudaMemsetAsync(dv, 0, grad_bytes, s) != cudaSuccess) return FGATTN_ERR_CUDA;
    const auto* ob = static_cast<const __nv_bfloat16*>(out);
    const unsigned dblocks = (unsigned)((rows + 7) / 8);
    if (d == 128)
        fgattn::fgattn_bwd_delta_kernel<128><<<dblocks, 256, 0, s>>>(ob, gb, delta, rows);
    else if (d == 96)
        fgattn::fgattn_bwd_delta_kernel<96><<<dblocks, 256, 0, s>>>(ob, gb, delta, rows);
    else
        fgattn::fgattn_bwd_delta_kernel<64><<<dblocks, 256, 0, s>>>(ob, gb, delta, rows);
    if (cudaPeekAtLastError() != cudaSuccess) return FGATTN_ERR_CUDA;
    if (d == 96) return launch_bwd_m<96>(prm, MQ, s);
    return d == 128 ? launch_bwd_m<128>(prm, MQ, s) : launch_bwd_m<64>(prm, MQ, s);
}

fgattn_status fgattn_device_error(fgattn_stream_t stream, int clear, uint32_t* bits) {
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return FGATTN_ERR_CUDA;
    unsigned int word = 0;
    if (cudaMemcpyFromSymbol(&word, fgattn::g_device_error, sizeof(word)) != cudaSuccess) return FGATTN_ERR_CUDA;
    if (clear && word) {
        const unsigned int zero = 0;
        if (cudaMemcpyToSymbol(fgattn::g_device_error, &zero, sizeof(zero)) != cudaSuccess) return FGATTN_ERR_CUDA;
    }
    if (bits) *bits = word;
    return word ? FGATTN_ERR_DEVICE : FGATTN_OK;
}

int fgattn_num_sms(void) { return current_sms(); }


const char* fgattn_status_string(fgattn_status status) {
    switch (status) {
        case FGATTN_OK: return "ok";
        case FGATTN_ERR_INVALID_ARG: return "invalid argument";
        case FGATTN_ERR_UNSUPPORTED: return "unsupported head dimension or query-block height";
        case FGATTN_ERR_CAPACITY: return "kept-index capacity smaller than the sequence length";
        case FGATTN_ERR_CUDA: return "CUDA runtime or launch error";
        case FGATTN_ERR_DEVICE: return "a kernel reported a device-side error";
    }
    return "unknown status";
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Host-to-host attention with the transfers overlapped with the kernels.
//
// The (b, h) pairs are independent, so the call splits them into groups and
// pipelines, per group: host-to-device copies of q, k, v and the mask on one
// internal stream, compaction + forward on the caller's stream, device-to-host
// copies of out and lse on a second internal stream.  Events order the three;
// group i computes while group i+1 is copied in and group i-1 is copied out.
// ---------------------------------------------------------------------------


namespace {

constexpr int kMaxGroups = 64;

struct PipeState {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, end = nullptr;
    cudaEvent_t copied[kMaxGroups] = {}, computed[kMaxGroups] = {};
};
constexpr int kMaxPipeDevices = 64;
std::mutex g_pipe_mutex;
PipeState g_pipe[kMaxPipeDevices];

// Streams and events of the current device (created on first use).  The caller
// holds g_pipe_mutex: calls are enqueued one at a time, so every wait pairs
// with the record of its own call.
fgattn_status pipe_state(PipeState** st) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FGATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxPipeDevices) return FGATTN_ERR_UNSUPPORTED;
    PipeState& ps = g_pipe[dev];
    if (!ps.in) {
        const unsigned ef = cudaEventDisableTiming;
        if (cudaStreamCreateWithFlags(&ps.in, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&ps.out, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&ps.start, ef) != cudaSuccess || cudaEventCreateWithFlags(&ps.end, ef) != cudaSuccess)
            return FGATTN_ERR_CUDA;
        for (int i = 0; i < kMaxGroups; ++i)
            if (cudaEventCreateWithFlags(&ps.copied[i], ef) != cudaSuccess ||
                cudaEventCreateWithFlags(&ps.computed[i], ef) != cudaSuccess)
                return FGATTN_ERR_CUDA;
    }
    *st = &ps;
    return FGATTN_OK;
}

}  // namespace

extern "C" fgattn_status fgattn_attention_from_host(
    const void* q_host, const void* k_host, const void* v_host, const uint32_t* mask_host, void* q, void* k, void* v,
    uint32_t* mask, int32_t* kept_idx, int32_t* kept_cnt, int64_t cap, int64_t B, int64_t H, int64_t L, int64_t d,
    int64_t M, int64_t N, float scale, void* out, float* lse, void* out_host, float* lse_host, int64_t heads_per_group,
    fgattn_stream_t stream) {
    if (!q_host || !k_host || !v_host || !mask_host || !out_host) return FGATTN_ERR_INVALID_ARG;
    if (!q || !k || !v || !mask || !kept_idx || !kept_cnt || !out) return FGATTN_ERR_INVALID_ARG;
    if ((lse == nullptr) != (lse_host == nullptr)) return FGATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || L < 1 || M < 1 || N < 1 || d < 1 || heads_per_group < 1) return FGATTN_ERR_INVALID_ARG;
    if (L > INT32_MAX || !std::isfinite(scale)) return FGATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out) || !aligned16(kept_idx))
        return FGATTN_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(mask) & 3u) || (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)))
        return FGATTN_ERR_INVALID_ARG;
    if (cap < L || (cap & 3)) return FGATTN_ERR_CAPACITY;
    if (d != 64 && d != 96 && d != 128) return FGATTN_ERR_UNSUPPORTED;
    if (M != 16 && M != 32 && M != 64 && M != 128) return FGATTN_ERR_UNSUPPORTED;
    if (B * H * L > INT32_MAX) return FGATTN_ERR_UNSUPPORTED;
    const int64_t BH = B * H;
    int64_t hpg = heads_per_group;
    if ((BH + hpg - 1) / hpg > kMaxGroups) hpg = (BH + kMaxGroups - 1) / kMaxGroups;
    const int64_t groups = (BH + hpg - 1) / hpg;
    const int64_t QB = (L + M - 1) / M;
    const int64_t Ng = N > L ? L : N;
    const int64_t W = ((L + Ng - 1) / Ng + 31) / 32;
    const size_t row_bytes = (size_t)L * d * 2;  // one head of q, k, v or out

    std::lock_guard<std::mutex> lock(g_pipe_mutex);
    PipeState* ps = nullptr;
    fgattn_status st = pipe_state(&ps);
    if (st != FGATTN_OK) return st;
    cudaStream_t cs = (cudaStream_t)stream;
    // the copies start after everything already enqueued on the caller's stream
    if (cudaEventRecord(ps->start, cs) != cudaSuccess || cudaStreamWaitEvent(ps->in, ps->start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(ps->out, ps->start, 0) != cudaSuccess)
        return FGATTN_ERR_CUDA;
    auto at = [](const void* base, size_t off) { return static_cast<const char*>(base) + off; };
    auto atw = [](void* base, size_t off) { return static_cast<char*>(base) + off; };
    for (int64_t gi = 0; gi < groups; ++gi) {
        const int64_t h0 = gi * hpg;
        const int64_t hn = BH - h0 < hpg ? BH - h0 : hpg;
        const size_t off = (size_t)h0 * row_bytes, bytes = (size_t)hn * row_bytes;
        const size_t moff = (size_t)h0 * QB * W * 4, mbytes = (size_t)hn * QB * W * 4;
        if (cudaMemcpyAsync(atw(q, off), at(q_host, off), bytes, cudaMemcpyHostToDevice, ps->in) != cudaSuccess ||
            cudaMemcpyAsync(atw(k, off), at(k_host, off), bytes, cudaMemcpyHostToDevice, ps->in) != cudaSuccess ||
            cudaMemcpyAsync(atw(v, off), at(v_host, off), bytes, cudaMemcpyHostToDevice, ps->in) != cudaSuccess ||
            cudaMemcpyAsync(atw(mask, moff), at(mask_host, moff), mbytes, cudaMemcpyHostToDevice, ps->in) != cudaSuccess ||
            cudaEventRecord(ps->copied[gi], ps->in) != cudaSuccess || cudaStreamWaitEvent(cs, ps->copied[gi], 0) != cudaSuccess)
            return FGATTN_ERR_CUDA;
        st = fgattn_compact_mask(reinterpret_cast<const uint32_t*>(atw(mask, moff)), 1, hn, L, M, N,
                                 kept_idx + h0 * QB * cap, kept_cnt + h0 * QB, cap, stream);
        if (st != FGATTN_OK) return st;
        st = fgattn_forward(atw(q, off), atw(k, off), atw(v, off), kept_idx + h0 * QB * cap, kept_cnt + h0 * QB, cap, 1,
                            hn, L, d, M, N, scale, atw(out, off), lse ? lse + h0 * L : nullptr, stream);
        if (st != FGATTN_OK) return st;
        if (cudaEventRecord(ps->computed[gi], cs) != cudaSuccess ||
            cudaStreamWaitEvent(ps->out, ps->computed[gi], 0) != cudaSuccess ||
            cudaMemcpyAsync(atw(out_host, off), at(out, off), bytes, cudaMemcpyDeviceToHost, ps->out) != cudaSuccess)
            return FGATTN_ERR_CUDA;
        if (lse && cudaMemcpyAsync(lse_host + h0 * L, lse + h0 * L, (size_t)hn * L * 4, cudaMemcpyDeviceToHost,
                                   ps->out) != cudaSuccess)
            return FGATTN_ERR_CUDA;
    }
    // the caller's stream is complete (host results included) once it passes this point
    if (cudaEventRecord(ps->end, ps->out) != cudaSuccess || cudaStreamWaitEvent(cs, ps->end, 0) != cudaSuccess)
        return FGATTN_ERR_CUDA;
    return FGATTN_OK;
}

// ---------------------------------------------------------------------------
// Mask-driven forward for callers that cannot allocate device memory.
//
// Some callers are handed their input and output buffers and nothing else: a
// plug-in running inside another runtime that owns the device's memory, or a
// process whose memory is all reserved by a caching allocator, or code that
// must not allocate once set-up is over.  For them the kept lists that
// fgattn_compact_mask writes and fgattn_forward reads live in one fixed
// array that the library itself holds on every device that loads it.
// ---------------------------------------------------------------------------


namespace {

// Kept-list scratch: the counts first (rows rounded up to 64 entries, so the
// lists that follow start 256-byte aligned), then rows x cap kept indices.
// Nothing in it has to start at zero: the compaction writes every count and
// the first `count` entries of every list, and the forward reads no more.
static __device__ __align__(256) int32_t g_noalloc_scratch[FGATTN_NOALLOC_SCRATCH_BYTES / sizeof(int32_t)];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mutex;
int32_t* g_noalloc_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code
// g_noalloc_scratch names a host-side stand-in, never the device copy.
fgattn_status noalloc_scratch(int32_t** ptr) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FGATTN_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FGATTN_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_noalloc_mutex);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return FGATTN_ERR_CUDA;
        g_noalloc_ptr[dev] = static_cast<int32_t*>(p);
    }
    *ptr = g_noalloc_ptr[dev];
    return FGATTN_OK;
}

}  // namespace

extern "C" fgattn_status fgattn_masked_forward_noalloc(const void* q, const void* k, const void* v,
                                                       const uint32_t* mask, int64_t B, int64_t H, int64_t L,
                                                       int64_t d, int64_t M, int64_t N, float scale, void* out,
                                                       float* lse, fgattn_stream_t stream) {
    // Every check of both steps comes first, so an error status means nothing was enqueued.
    if (!q || !k || !v || !out || !mask) return FGATTN_ERR_INVALID_ARG;
    if (B < 1 || H < 1 || L < 1 || M < 1 || N < 1 || d < 1) return FGATTN_ERR_INVALID_ARG;
    if (L > INT32_MAX) return FGATTN_ERR_INVALID_ARG;
    if (!std::isfinite(scale)) return FGATTN_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return FGATTN_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(mask) & 3u) return FGATTN_ERR_INVALID_ARG;
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return FGATTN_ERR_INVALID_ARG;
    if (d != 64 && d != 96 && d != 128) return FGATTN_ERR_UNSUPPORTED;
    if (M != 16 && M != 32 && M != 64 && M != 128) return FGATTN_ERR_UNSUPPORTED;
    if (B * H * L > INT32_MAX) return FGATTN_ERR_UNSUPPORTED;
    const int64_t cap = fgattn_kept_capacity(L);
    const int64_t rows = B * H * ((L + M - 1) / M);
    const int64_t cnt_entries = (rows + 63) / 64 * 64;
    const int64_t limit = (int64_t)(FGATTN_NOALLOC_SCRATCH_BYTES / sizeof(int32_t));
    if (rows > limit || cap > limit || cnt_entries + rows * cap > limit) return FGATTN_ERR_CAPACITY;

    int32_t* scratch = nullptr;
    const fgattn_status st = noalloc_scratch(&scratch);
    if (st != FGATTN_OK) return st;
    int32_t* kept_cnt = scratch;
    int32_t* kept_idx = scratch + cnt_entries;
    const fgattn_status sc = fgattn_compact_mask(mask, B, H, L, M, N, kept_idx, kept_cnt, cap, stream);
    if (sc != FGATTN_OK) return sc;
    return fgattn_forward(q, k, v, kept_idx, kept_cnt, cap, B, H, L, d, M, N, scale, out, lse, stream);
}
