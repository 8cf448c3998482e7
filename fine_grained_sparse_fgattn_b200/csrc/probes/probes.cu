// Microbenchmarks that set the rooflines of the tile-sparse forward kernels on
// this GPU.  They are measurement tools, not part of the attention path: the
// library libfgattn_probes.so is built from this file alone and nothing in
// libfgattn.so calls it.
//
//  * Row loads from L2 into shared memory, no math: every block of a
//    persistent grid keeps NS chunks of 128 rows x 256 bytes (one 128-key
//    chunk of K or V at d = 128) in flight and re-issues a stage as soon as it
//    has landed.  Three ways of moving a row, the three the forward kernels use:
//      mode 0  tiled TMA boxes of 16 consecutive rows (16-key runs),
//      mode 1  TMA tile::gather4 of single rows (row-by-row gathers of K),
//      mode 2  16-byte cp.async copies per row (row-by-row gathers of V).
//    The rows come from a buffer the caller sizes (one head's K and V at the
//    Wan-480p-like shape is 16.8 MB, L2-resident); row numbers are a hash of
//    (block, chunk, row), uniform over the buffer.
//  * tcgen05.mma kind::f16 issue rate with the forward kernels' exact operand
//    layouts: the key-major score product (A = 128 keys x 128 d, K-major; B =
//    N query rows, K-major) and the key-major P.V product (A = V^T, MN-major;
//    B = P^T, MN-major), N in {64, 128, 256}, one commit per group of 8 MMAs
//    (one 128-key chunk), as in the kernels.
//  * MUFU ex2 throughput (8 independent chains per thread).
//
// Every mbarrier wait is bounded (2 s); a wait that gives up sets an error
// word that the host reads, and the block drains and exits.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "../attention_fwd.cuh"

namespace fgprobe {

using namespace fgattn;

__device__ unsigned int g_probe_error = 0u;

constexpr int KC = 128;            // rows per chunk
constexpr int ROWB = 256;          // bytes per row (d = 128 bf16)
constexpr int CHUNK = KC * ROWB;   // 32 KB
constexpr int NS = 6;              // chunks in flight per block (192 KB)

__device__ __forceinline__ uint32_t mix(uint32_t x) {
    x ^= x >> 16;
    x *= 0x7feb352du;
    x ^= x >> 15;
    x *= 0x846ca68bu;
    x ^= x >> 16;
    return x;
}

__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = ptx::globaltimer_ns();
    for (;;) {
        for (int i = 0; i < 64; ++i)
            if (ptx::mbar_try_wait(bar, parity)) return true;
        if (ptx::globaltimer_ns() - t0 > 2000000000ull) {
            atomicOr(&g_probe_error, 1u);
            return false;
        }
    }
}

struct RowParams {
    CUtensorMap tmap16;  // rows of 128 bf16, box {64, 16}, 128B swizzle
    CUtensorMap tmap1;   // rows of 128 bf16, box {64, 1}, 128B swizzle (gather4)
    const uint8_t* base;
    uint32_t rows;       // rows in the buffer (>= 16)
    uint32_t chunks;     // chunks per block
};

// 128 threads = 4 warps; warp w moves rows [32 w, 32 w + 32) of every chunk.
template <int MODE>
__global__ void __launch_bounds__(128, 1) probe_rows_kernel(const __grid_constant__ RowParams p) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const uint32_t bar0 = sbase + NS * CHUNK;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) ptx::mbar_init(bar0 + 8u * s, MODE == 2 ? 128u : 4u);
        ptx::fence_mbar_init();
    }
    __syncthreads();
    const uint32_t groups16 = p.rows / 16;
    auto issue = [&](uint32_t c, int s) {
        const uint32_t bar = bar0 + 8u * (uint32_t)s;
        const uint32_t dst = sbase + (uint32_t)s * CHUNK;
        const uint32_t seed = blockIdx.x * 0x9e3779b9u + c * 0x85ebca6bu;
        if (MODE == 0) {
            // two 16-row segments per warp, one box per 64-column panel
            if (lane == 0) ptx::mbar_arrive_expect_tx(bar, 32u * ROWB);
            __syncwarp();
            if (lane < 2) {
                const int seg = warp * 2 + lane;
                const int32_t r0 = (int32_t)(mix(seed + (uint32_t)seg) % groups16) * 16;
                for (int pn = 0; pn < 2; ++pn)
                    ptx::tma_load_2d(dst + pn * (KC * 128) + seg * 16 * 128, &p.tmap16, pn * 64, r0, bar);
            }
        } else if (MODE == 1) {
            // eight 4-row gathers per warp, per panel
            if (lane == 0) ptx::mbar_arrive_expect_tx(bar, 32u * ROWB);
            __syncwarp();
            if (lane < 8) {
                const int g4 = warp * 8 + lane;
                int32_t r[4];
                for (int i = 0; i < 4; ++i) r[i] = (int32_t)(mix(seed + (uint32_t)(4 * g4 + i)) % p.rows);
                for (int pn = 0; pn < 2; ++pn)
                    ptx::tma_gather4(dst + pn * (KC * 128) + g4 * 4 * 128, &p.tmap1, pn * 64, r[0], r[1], r[2], r[3],
                                     bar);
            }
        } else {
            // 16 pieces of 16 bytes per row; a warp instruction covers two rows
            const uint32_t myrow = mix(seed + (uint32_t)(warp * 32 + lane)) % p.rows;
            for (int i = 0; i < 16; ++i) {
                const int rl = 2 * i + (lane >> 4);
                const int pc = lane & 15;
                const uint32_t rr = __shfl_sync(0xffffffffu, myrow, rl);
                const int r = warp * 32 + rl;
                const uint8_t* src = p.base + (size_t)rr * ROWB + pc * 16;
                ptx::cp_async_16(dst + (uint32_t)(pc / 8) * (KC * 128) + swz(r, pc % 8, 128), src, 16u);
            }
            ptx::cp_async_arrive_noinc(bar);
        }
    };
    bool ok = true;
    for (uint32_t c = 0; c < p.chunks && c < NS; ++c) issue(c, (int)c);
    for (uint32_t c = 0; c < p.chunks; ++c) {
        const int s = (int)(c % NS);
        ok = wait_bounded(bar0 + 8u * s, (c / NS) & 1u);
        if (!__all_sync(0xffffffffu, ok)) break;
        if (c + NS < p.chunks) issue(c + NS, s);
    }
    // every copy this block issued has landed before it exits
    if (MODE == 2) ptx::cp_async_wait_all();
    if (!ok) {
        const uint32_t last = p.chunks;
        for (uint32_t c = last > NS ? last - NS : 0; c < last; ++c)
            wait_bounded(bar0 + 8u * (c % NS), (c / NS) & 1u);
    }
    __syncthreads();
}

// tcgen05.mma issue rate.  which = 1: score products only; 2: P.V products only;
// 3: both, one group of 8 after the other per chunk; 4: both, interleaved MMA by
// MMA (score k-step i, then P.V k-step i); 5: score products with the 8 k-steps
// alternating between two accumulators (two independent chains).  One thread
// issues `chunks` groups of 8 MMAs per kind, committing each group to a barrier,
// and waits for the commit of the group two back (the kernels' double buffering).
// Modes 4 and 5 separate the tensor pipe's throughput from the latency of a chain
// of dependent accumulations into one accumulator.
template <int N>
__global__ void __launch_bounds__(128, 1) probe_mma_kernel(int which, uint32_t chunks, unsigned long long* cycles) {
    constexpr int D = 128;
    constexpr int K_BYTES = KC * D * 2;          // K chunk: 2 panels of 128 rows x 128 B
    constexpr int Q_BYTES = N * D * 2;           // query tile: 2 panels of N rows x 128 B
    constexpr int V_BYTES = KC * D * 2;          // V chunk: same as K
    constexpr int P_ROW = 128;                   // bytes per key row of a P^T panel (64 queries)
    constexpr int P_PANEL = KC * P_ROW;          // 16 KB
    constexpr int P_BYTES = (N / 64) * P_PANEL;  // P^T: N / 64 panels
    constexpr int OFF_K = 0, OFF_Q = OFF_K + K_BYTES, OFF_V = OFF_Q + Q_BYTES, OFF_P = OFF_V + V_BYTES;
    constexpr int OFF_BAR = OFF_P + P_BYTES;
    constexpr uint32_t TCOLS = 2 * N <= 256 ? (2 * N <= 128 ? 128 : 256) : 512;
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    const uint32_t sbase = ptx::smem_u32(smem);
    const int warp = threadIdx.x >> 5;
    // finite operands: zeros
    for (int i = threadIdx.x; i < OFF_BAR / 16; i += blockDim.x)
        reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
    ptx::fence_proxy_async_smem();
    if (warp == 0) {
        ptx::tmem_alloc(sbase + OFF_BAR + 64, TCOLS);
        ptx::tmem_relinquish();
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < 5; ++i) ptx::mbar_init(sbase + OFF_BAR + 8u * i, 1u);
        ptx::fence_mbar_init();
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_BAR + 64);
    if (threadIdx.x == 0) {
        const uint32_t tS = tmem, tO = tmem + N;
        constexpr uint32_t IDESC1 = umma_idesc_bf16(128, N, false, false);
        constexpr uint32_t IDESC2 = umma_idesc_bf16(D, N, true, true);
        constexpr uint32_t HI_KQ = umma_desc_hi(1024u, 2u);
        constexpr uint32_t HI_V = umma_desc_hi(1024u, 2u);
        constexpr uint32_t HI_P = umma_desc_hi(8u * P_ROW, 2u);
        const uint32_t klo = umma_desc_lo(sbase + OFF_K, 16u);
        const uint32_t qlo = umma_desc_lo(sbase + OFF_Q, 16u);
        const uint32_t vlo = umma_desc_lo(sbase + OFF_V, 128u * 128u);
        const uint32_t plo = umma_desc_lo(sbase + OFF_P, (uint32_t)P_PANEL);
        const uint64_t t0 = clock64();
        bool ok = true;
        uint32_t n1 = 0, n2 = 0;  // commits per kind
        for (uint32_t c = 0; c < chunks && ok && which == 4; ++c) {
            if (n1 >= 2) ok = ok && wait_bounded(sbase + OFF_BAR + 8u * (n1 & 1), ((n1 - 2) >> 1) & 1u);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (uint32_t)(kk / 4) * (128 * 128) + (uint32_t)(kk % 4) * 32u;
                const uint32_t qoff = (uint32_t)(kk / 4) * (N * 128) + (uint32_t)(kk % 4) * 32u;
                ptx::mma_bf16_ss(tS, umma_desc_join(klo + (koff >> 4), HI_KQ), umma_desc_join(qlo + (qoff >> 4), HI_KQ),
                                 IDESC1, kk > 0 ? 1u : 0u);
                ptx::mma_bf16_ss(tO, umma_desc_join(vlo + (uint32_t)(kk * 2048 >> 4), HI_V),
                                 umma_desc_join(plo + (uint32_t)(kk * 16 * P_ROW >> 4), HI_P), IDESC2,
                                 (c > 0 || kk > 0) ? 1u : 0u);
            }
            ptx::mma_commit(sbase + OFF_BAR + 8u * (n1 & 1));
            ++n1;
        }
        for (uint32_t c = 0; c < chunks && ok && which == 5; ++c) {
            if (n1 >= 2) ok = ok && wait_bounded(sbase + OFF_BAR + 8u * (n1 & 1), ((n1 - 2) >> 1) & 1u);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t koff = (uint32_t)(kk / 4) * (128 * 128) + (uint32_t)(kk % 4) * 32u;
                const uint32_t qoff = (uint32_t)(kk / 4) * (N * 128) + (uint32_t)(kk % 4) * 32u;
                ptx::mma_bf16_ss(kk & 1 ? tO : tS, umma_desc_join(klo + (koff >> 4), HI_KQ),
                                 umma_desc_join(qlo + (qoff >> 4), HI_KQ), IDESC1, kk > 1 ? 1u : 0u);
            }
            ptx::mma_commit(sbase + OFF_BAR + 8u * (n1 & 1));
            ++n1;
        }
        for (uint32_t c = 0; c < chunks && ok && which <= 3; ++c) {
            if (which & 1) {
                if (n1 >= 2) ok = ok && wait_bounded(sbase + OFF_BAR + 8u * (n1 & 1), ((n1 - 2) >> 1) & 1u);
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (uint32_t)(kk / 4) * (128 * 128) + (uint32_t)(kk % 4) * 32u;
                    const uint32_t qoff = (uint32_t)(kk / 4) * (N * 128) + (uint32_t)(kk % 4) * 32u;
                    ptx::mma_bf16_ss(tS, umma_desc_join(klo + (koff >> 4), HI_KQ),
                                     umma_desc_join(qlo + (qoff >> 4), HI_KQ), IDESC1, kk > 0 ? 1u : 0u);
                }
                ptx::mma_commit(sbase + OFF_BAR + 8u * (n1 & 1));
                ++n1;
            }
            if (which & 2) {
                if (n2 >= 2) ok = ok && wait_bounded(sbase + OFF_BAR + 16u + 8u * (n2 & 1), ((n2 - 2) >> 1) & 1u);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    ptx::mma_bf16_ss(tO, umma_desc_join(vlo + (uint32_t)(kk * 2048 >> 4), HI_V),
                                     umma_desc_join(plo + (uint32_t)(kk * 16 * P_ROW >> 4), HI_P), IDESC2,
                                     (c > 0 || kk > 0) ? 1u : 0u);
                ptx::mma_commit(sbase + OFF_BAR + 16u + 8u * (n2 & 1));
                ++n2;
            }
        }
        // drain: everything issued has completed
        ptx::mma_commit(sbase + OFF_BAR + 32u);
        wait_bounded(sbase + OFF_BAR + 32u, 0u);
        const uint64_t t1 = clock64();
        if (blockIdx.x == 0) *cycles = t1 - t0;
    }
    ptx::tc_fence_before();
    __syncthreads();
    ptx::tc_fence_after();
    if (warp == 0) ptx::tmem_dealloc(tmem, TCOLS);
}

// MUFU ex2: 8 independent chains per thread; the result is kept live through `sink`.
__global__ void __launch_bounds__(256) probe_ex2_kernel(uint32_t iters, float* sink, unsigned long long* cyc,
                                                        unsigned long long* ns) {
    float x[8];
    for (int i = 0; i < 8; ++i) x[i] = -0.001f * (float)(threadIdx.x + i);
    const uint64_t c0 = clock64(), g0 = ptx::globaltimer_ns();
    for (uint32_t it = 0; it < iters; ++it) {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = ptx::ex2(x[i]) - 1.0f;
    }
    const uint64_t c1 = clock64(), g1 = ptx::globaltimer_ns();
    float s = 0.f;
    for (int i = 0; i < 8; ++i) s += x[i];
    if (s == 12345.f) sink[threadIdx.x] = s;  // never true in practice; keeps the chains live
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        *cyc = c1 - c0;
        *ns = g1 - g0;
    }
}

}  // namespace fgprobe

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
        return false;
    auto fn = reinterpret_cast<EncodeTiledFn>(ptr);
    const cuuint64_t dims[2] = {128u, rows};
    const cuuint64_t strides[1] = {256u};
    const cuuint32_t box[2] = {64u, box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sms() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return n;
}

template <typename F>
int timed(F launch, int reps, cudaStream_t s, float* ms) {
    cudaEvent_t a, b;
    if (cudaEventCreate(&a) != cudaSuccess || cudaEventCreate(&b) != cudaSuccess) return 4;
    launch();  // warm-up
    cudaEventRecord(a, s);
    for (int i = 0; i < reps; ++i) launch();
    cudaEventRecord(b, s);
    int st = cudaEventSynchronize(b) == cudaSuccess ? 0 : 4;
    float t = 0.f;
    if (st == 0 && cudaEventElapsedTime(&t, a, b) != cudaSuccess) st = 4;
    cudaEventDestroy(a);
    cudaEventDestroy(b);
    if (cudaPeekAtLastError() != cudaSuccess) st = 4;
    *ms = t / (float)reps;
    return st;
}

bool clear_error() {
    const unsigned int zero = 0;
    return cudaMemcpyToSymbol(fgprobe::g_probe_error, &zero, sizeof(zero)) == cudaSuccess;
}

int probe_error() {
    unsigned int w = 0;
    if (cudaMemcpyFromSymbol(&w, fgprobe::g_probe_error, sizeof(w)) != cudaSuccess) return 4;
    return w ? 5 : 0;
}

}  // namespace

extern "C" {

// Row loads from L2: src holds `rows` rows of 256 bytes (16-byte aligned,
// rows >= 16); one block per SM moves `chunks` chunks of 128 rows each, mode 0
// (16-row TMA boxes), 1 (TMA gather4) or 2 (cp.async).  *ms = mean time of one
// launch over `reps` launches; *bytes = bytes moved per launch.
// Returns 0, 1 (bad argument), 4 (CUDA error) or 5 (a wait gave up).
int fgprobe_rows(int mode, const void* src, int64_t rows, int chunks, int reps, void* stream, float* ms,
                 double* bytes) {
    if (!src || (reinterpret_cast<uintptr_t>(src) & 15u) || rows < 16 || rows > (1ll << 30) || chunks < 1 ||
        reps < 1 || mode < 0 || mode > 2 || !ms || !bytes)
        return 1;
    if (!clear_error()) return 4;
    fgprobe::RowParams p;
    if (!encode(&p.tmap16, src, (uint64_t)rows, 16) || !encode(&p.tmap1, src, (uint64_t)rows, 1)) return 4;
    p.base = static_cast<const uint8_t*>(src);
    p.rows = (uint32_t)rows;
    p.chunks = (uint32_t)chunks;
    const int smem = fgprobe::NS * fgprobe::CHUNK + 1024 + 64;
    const int grid = sms();
    if (grid <= 0) return 4;
    cudaStream_t s = (cudaStream_t)stream;
    auto k = mode == 0 ? fgprobe::probe_rows_kernel<0> : mode == 1 ? fgprobe::probe_rows_kernel<1>
                                                                   : fgprobe::probe_rows_kernel<2>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 4;
    const int st = timed([&] { k<<<grid, 128, smem, s>>>(p); }, reps, s, ms);
    *bytes = (double)grid * chunks * fgprobe::CHUNK;
    return st ? st : probe_error();
}

// tcgen05.mma issue rate (see probe_mma_kernel): n in {64, 128, 256}; which in
// {1, 2, 3}.  *ms = mean launch time; *flops = MMA FLOPs per launch; *cycles =
// SM clocks block 0 spent from the first issue to the last completion.
int fgprobe_mma(int which, int n, int chunks, int reps, void* stream, float* ms, double* flops,
                unsigned long long* cycles_dev, unsigned long long* cycles) {
    if (which < 1 || which > 5 || chunks < 1 || reps < 1 || !ms || !flops || !cycles_dev || !cycles) return 1;
    if (n != 64 && n != 128 && n != 256) return 1;
    if (!clear_error()) return 4;
    const int grid = sms();
    if (grid <= 0) return 4;
    cudaStream_t s = (cudaStream_t)stream;
    const int smem_of[3] = {32768 + 64 * 256 + 32768 + 16384, 32768 + 128 * 256 + 32768 + 32768,
                            32768 + 256 * 256 + 32768 + 65536};
    const int idx = n == 64 ? 0 : n == 128 ? 1 : 2;
    // at least 120 KB: exactly one block (one issuing thread) per SM
    const int smem = smem_of[idx] + 1024 + 128 > 120 * 1024 ? smem_of[idx] + 1024 + 128 : 120 * 1024;
    auto k = n == 64 ? fgprobe::probe_mma_kernel<64> : n == 128 ? fgprobe::probe_mma_kernel<128>
                                                                 : fgprobe::probe_mma_kernel<256>;
    if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) return 4;
    const int st = timed([&] { k<<<grid, 128, smem, s>>>(which, (uint32_t)chunks, cycles_dev); }, reps, s, ms);
    const double per_kind = 2.0 * 128.0 * n * 128.0;  // one chunk: M 128 x N x K 128
    const int kinds = which == 3 || which == 4 ? 2 : 1;
    *flops = (double)grid * chunks * per_kind * kinds;
    if (cudaMemcpy(cycles, cycles_dev, sizeof(unsigned long long), cudaMemcpyDeviceToHost) != cudaSuccess) return 4;
    return st ? st : probe_error();
}

// MUFU ex2: `blocks_per_sm` x SMs blocks of 256 threads, 8 chains x iters each.
// *ex2_per_clk_sm = ex2 results per SM clock per SM (block 0's clocks), *mhz = SM clock.
int fgprobe_ex2(int iters, int blocks_per_sm, void* stream, float* sink, unsigned long long* dev2, float* ms,
                double* ex2_per_clk_sm, double* mhz) {
    if (iters < 1 || blocks_per_sm < 1 || !sink || !dev2 || !ms || !ex2_per_clk_sm || !mhz) return 1;
    const int n = sms();
    if (n <= 0) return 4;
    cudaStream_t s = (cudaStream_t)stream;
    const int grid = n * blocks_per_sm;
    const int st = timed([&] { fgprobe::probe_ex2_kernel<<<grid, 256, 0, s>>>((uint32_t)iters, sink, dev2, dev2 + 1); },
                         3, s, ms);
    if (st) return st;
    unsigned long long h[2];
    if (cudaMemcpy(h, dev2, sizeof h, cudaMemcpyDeviceToHost) != cudaSuccess) return 4;
    *mhz = h[1] ? (double)h[0] / (double)h[1] * 1e3 : 0.0;
    const double total = (double)grid * 256.0 * 8.0 * iters;
    const double clocks = (double)(*ms) * 1e-3 * (*mhz) * 1e6;
    *ex2_per_clk_sm = clocks > 0 ? total / clocks / n : 0.0;
    return 0;
}

}  // extern "C"
