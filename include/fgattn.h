/*
 * fgattn.h -- C ABI of the B200 (sm_100a) tile-sparse attention library.
 *
 * The operation is the forward pass of softmax attention in which whole
 * M x N score tiles (M queries x N keys, M >= 16, N >= 1) are skipped; a
 * skipped score contributes exactly as if it were -inf.  Source: "FG-Attn:
 * Leveraging Fine-Grained Sparse Attention in Video Diffusion Models",
 * Abstract.  The page fixes neither the mask layout, the interface nor the
 * precision; this header states the readings the library implements.
 *
 * Conventions shared by every entry point
 *   - Tensor pointers are DEVICE pointers owned by the caller unless an entry
 *     point marks them HOST.  The library allocates no device memory per call
 *     and keeps no reference to any pointer after the call returns.
 *   - Work is enqueued on `stream` (0 = the legacy default stream) and runs
 *     asynchronously; argument validation happens synchronously on the host
 *     before anything is enqueued, and a call that returns an error status has
 *     enqueued nothing (fgattn_attention_from_host: unless the status is CUDA,
 *     which can leave the copies and kernels of earlier head groups enqueued;
 *     fgattn_backward: unless the status is CUDA, which can leave the zeroing of
 *     dk and dv and the delta pass enqueued).
 *   - Shapes: B batch, H heads, L tokens, d head dimension.
 *       QB = ceil(L / M) query blocks, G = ceil(L / N) key groups,
 *       W  = ceil(G / 32) mask words per query block.
 *   - Layouts (all contiguous, row-major, innermost last):
 *       q, k, v, out : bf16   [B][H][L][d]
 *       lse          : fp32   [B][H][L]         (natural logarithm)
 *       mask         : uint32 [B][H][QB][W]     tile (qb, g) kept <=> bit (g % 32)
 *                                               of word g / 32 is 1 (LSB first);
 *                                               bits >= G are ignored
 *       kept_idx     : int32  [B][H][QB][cap]   ascending kept key indices
 *       kept_cnt     : int32  [B][H][QB]        number of valid entries per row
 *   - Diagonal rule: whatever the mask says, query block qb keeps the key
 *     groups that hold its own rows' indices, floor(qb*M/N) ..
 *     floor((min(qb*M+M, L) - 1) / N), so every query row has at least one
 *     kept key and a finite log-sum-exp.
 *   - Ragged ends: keys >= L do not exist (the last group has L - (G-1)*N
 *     keys); query rows >= L are not computed and not written.
 *   - Pointer alignment: 16 bytes for q, k, v, out, kept_idx.
 *   - Errors never abort the process; every entry point returns a status.
 */
#ifndef FGATTN_H
#define FGATTN_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fgattn_stream_t; /* same type as cudaStream_t */

typedef enum {
    FGATTN_OK = 0,
    FGATTN_ERR_INVALID_ARG = 1, /* null pointer, non-positive size, misaligned pointer, bad scale */
    FGATTN_ERR_UNSUPPORTED = 2, /* a legal value this build has no kernel for (d, M) */
    FGATTN_ERR_CAPACITY = 3,    /* cap < L: a kept list might not fit */
    FGATTN_ERR_CUDA = 4,        /* a CUDA runtime call or a launch failed */
    FGATTN_ERR_DEVICE = 5       /* a kernel flagged an error (see fgattn_device_error) */
} fgattn_status;

/* Device error bits recorded by the kernels (fgattn_device_error). */
#define FGATTN_DEVERR_BAD_INDEX 0x1u   /* a kept_idx entry was outside [0, L); a safe row was used */
#define FGATTN_DEVERR_BAD_COUNT 0x2u   /* a kept_cnt entry was outside [0, cap]; it was clamped */
#define FGATTN_DEVERR_TIMEOUT 0x4u     /* a pipeline wait exceeded its bound; the block exited */

/*
 * Stride (in int32 elements) to use for one kept_idx row: L rounded up to a
 * multiple of 16 (keeps every row 64-byte aligned).  Returns -1 if L < 1.
 */
int64_t fgattn_kept_capacity(int64_t L);

/*
 * Mask compaction ("FG-Attn ...", Abstract: the M x N tiles to compute).
 * For every row (b, h, qb): kept_idx[row][0 .. kept_cnt[row]) = the key
 * indices of every kept group of the row, after the diagonal rule, ascending;
 * entries past kept_cnt[row] are left untouched.  Bit-exact integer work.
 *   mask      in   device uint32 [B][H][QB][W]
 *   kept_idx  out  device int32  [B][H][QB][cap], cap >= L, cap % 4 == 0
 *   kept_cnt  out  device int32  [B][H][QB]
 * Requires 1 <= M, 1 <= N (the method itself asks M >= 16; the compaction
 * accepts any M >= 1).  Errors: INVALID_ARG, CAPACITY, CUDA.
 */
fgattn_status fgattn_compact_mask(const uint32_t* mask, int64_t B, int64_t H, int64_t L, int64_t M,
                                  int64_t N, int32_t* kept_idx, int32_t* kept_cnt, int64_t cap,
                                  fgattn_stream_t stream);

/*
 * Tile-sparse attention forward ("FG-Attn ...", Abstract: scores of skipped
 * tiles are never computed and count as -inf).  For each query row i of
 * block qb, over the keys j listed in kept_idx for (b, h, qb):
 *   s_ij = scale * q_i . k_j,  p_ij = exp(s_ij - m_i),  l_i = sum_j p_ij,
 *   out_i = sum_j p_ij v_j / l_i  (stored as bf16),  lse_i = m_i + ln l_i.
 *   q, k, v   in   device bf16 [B][H][L][d]
 *   kept_idx  in   device int32 [B][H][QB][cap], cap >= L, cap % 4 == 0
 *                  (as written by fgattn_compact_mask,
 *                  or any ascending or unordered list of distinct keys < L),
 *                  or NULL for a dense run of the same kernel (every key kept)
 *   kept_cnt  in   device int32 [B][H][QB] (ignored when kept_idx is NULL);
 *                  every count must be >= 1 and <= cap
 *   out       out  device bf16 [B][H][L][d]
 *   lse       out  device fp32 [B][H][L], may be NULL
 * Supported: d in {64, 96, 128}, M in {16, 32, 64, 128}, any N >= 1, any L >= 1.
 * (At d = 96 the P.V product runs on V padded with zero columns to 128: the
 * tensor-core shape of that product needs 64 or 128; the padding is never
 * stored.)
 * Accumulation in fp32; P is rounded to bf16 for the P.V product; the sum l
 * is taken over the fp32 probabilities.
 * Errors: INVALID_ARG, UNSUPPORTED, CAPACITY, CUDA.  Kernel-side problems
 * (corrupt indices or counts, a wait that timed out) never fault: they set a
 * device error bit that fgattn_device_error reports.
 */
fgattn_status fgattn_forward(const void* q, const void* k, const void* v, const int32_t* kept_idx,
                             const int32_t* kept_cnt, int64_t cap, int64_t B, int64_t H, int64_t L,
                             int64_t d, int64_t M, int64_t N, float scale, void* out, float* lse,
                             fgattn_stream_t stream);

/*
 * fgattn_forward on tensors in any [B][H][L][d]-indexable layout with d
 * contiguous: [B][L][H][d] (the usual layout of a transformer's activations),
 * q, k, v as views of one packed [B][L][3][H][d] projection, and so on.  Same
 * operation, kept lists, lse layout ([B][H][L], contiguous) and errors as
 * fgattn_forward; the results are identical to fgattn_forward's on the same
 * values stored contiguously.
 *   x_strides  in  HOST int64[3]: element strides {batch, head, token} of x;
 *                  element (b, h, l, e) of x is x[b*s[0] + h*s[1] + l*s[2] + e].
 * Requirements (else INVALID_ARG): every stride >= d and a multiple of 8
 * elements (16 bytes); k and v strides multiples of d; the strides of a
 * dimension of extent 1 are ignored.  Views of out for different (b, h, l) must
 * not overlap.  UNSUPPORTED if the rows of k span 2^31 rows of d elements or
 * more.
 */
fgattn_status fgattn_forward_strided(const void* q, const int64_t* q_strides, const void* k, const int64_t* k_strides,
                                     const void* v, const int64_t* v_strides, const int32_t* kept_idx,
                                     const int32_t* kept_cnt, int64_t cap, int64_t B, int64_t H, int64_t L, int64_t d,
                                     int64_t M, int64_t N, float scale, void* out, const int64_t* out_strides,
                                     float* lse, fgattn_stream_t stream);

/*
 * Tile-sparse attention forward straight from the mask, in one kernel: the
 * mask compaction fused into the forward ("FG-Attn ...", Abstract: the M x N
 * tiles are skipped at that granularity; the mask is the tile list).  Every
 * warp of the kernel that needs kept keys reads its query block's mask row and
 * expands it itself (diagonal rule and ragged ends as fgattn_compact_mask), so
 * no kept list is written to or read from memory and nothing is allocated.
 *   q, k, v   in   device bf16 [B][H][L][d], contiguous
 *   mask      in   device uint32 [B][H][QB][W] (layout as above)
 *   out       out  device bf16 [B][H][L][d]
 *   lse       out  device fp32 [B][H][L], may be NULL
 * Results equal fgattn_compact_mask followed by fgattn_forward, bit for bit
 * (same kernels, same key order).  Supported: as fgattn_forward, and
 * W = ceil(ceil(L / N) / 32) <= 256 mask words per query block (for example
 * N = 16 up to L = 131072, N = 1 up to L = 8192); larger rows return
 * UNSUPPORTED (use fgattn_compact_mask + fgattn_forward).
 * Errors: INVALID_ARG (also a NULL or misaligned mask), UNSUPPORTED, CUDA;
 * device-side problems as for fgattn_forward.
 */
fgattn_status fgattn_masked_forward(const void* q, const void* k, const void* v, const uint32_t* mask, int64_t B,
                                    int64_t H, int64_t L, int64_t d, int64_t M, int64_t N, float scale, void* out,
                                    float* lse, fgattn_stream_t stream);

/*
 * Gradients of the tile-sparse forward ("FG-Attn ...", Abstract: a skipped
 * tile's scores are -inf, so p = 0 there and they carry no gradient; the page
 * gives only the forward, and this is its derivative).  Over the kept keys j
 * of each query row i, with p_ij = exp(scale * q_i . k_j - lse_i) recomputed
 * and g_i = dout_i:
 *   dp_ij = g_i . v_j,  delta_i = g_i . out_i,  ds_ij = p_ij (dp_ij - delta_i),
 *   dq_i = scale * sum_j ds_ij k_j,  dk_j = scale * sum_i ds_ij q_i,
 *   dv_j = sum_i p_ij g_i.
 *   q, k, v, out, dout  in   device bf16 [B][H][L][d] (out and lse as the
 *                            forward wrote them for the same lists and scale)
 *   lse                 in   device fp32 [B][H][L]
 *   kept_idx, kept_cnt  in   as for fgattn_forward (NULL kept_idx = dense)
 *   dq, dk, dv          out  device fp32 [B][H][L][d], 16-byte aligned; every
 *                            element is written (rows of keys that no query
 *                            block keeps get zeros)
 *   delta               out  device fp32 [B][H][L]: workspace owned by the
 *                            caller; holds delta_i on return
 * Supported: d in {64, 96, 128} (at d = 96 the products run on tiles padded
 * with zero columns to 128), M in {16, 32, 64, 128} (a 128-row block runs as
 * two 64-row halves over its list), any N >= 1, any L >= 1.
 * P and ds are rounded to bf16 for the tensor-core products; accumulation in
 * fp32.  dk and dv are accumulated with float atomics (many query blocks keep
 * one key), so their last bits depend on the order the blocks run in; dq is
 * deterministic.  Errors: INVALID_ARG, UNSUPPORTED, CAPACITY, CUDA; device-side
 * problems as for fgattn_forward, except that a kept_idx entry outside [0, L)
 * (flagged BAD_INDEX) is read as a zero row and receives no gradient.
 */
fgattn_status fgattn_backward(const void* q, const void* k, const void* v, const void* out, const void* dout,
                              const float* lse, const int32_t* kept_idx, const int32_t* kept_cnt, int64_t cap,
                              int64_t B, int64_t H, int64_t L, int64_t d, int64_t M, int64_t N, float scale,
                              float* dq, float* dk, float* dv, float* delta, fgattn_stream_t stream);

/*
 * Synchronise `stream`, then report (and, if clear != 0, reset) the device
 * error bits (FGATTN_DEVERR_*) recorded on the current device since the last
 * clear.  *bits may be NULL.  Returns DEVICE if any bit is set, CUDA if the
 * synchronisation failed, else OK.
 */
fgattn_status fgattn_device_error(fgattn_stream_t stream, int clear, uint32_t* bits);

/*
 * Host to host: the whole path (copy in, compaction, forward, copy out) for
 * inputs and results in host memory, with the transfers overlapped with the
 * kernels.  The (b, h) pairs are split into groups of heads_per_group (at
 * most 64 groups; more heads per group if needed); for each group the call
 * copies q, k, v and the mask to the device on an internal stream, runs
 * fgattn_compact_mask and fgattn_forward on `stream`, and copies out (and lse)
 * back on a second internal stream, so that one group computes while the next
 * is copied in and the previous one copied out.  Contiguous layouts only.
 *   q_host, k_host, v_host  in   HOST bf16 [B][H][L][d] (pinned memory for overlap)
 *   mask_host               in   HOST uint32 [B][H][QB][W]
 *   q, k, v, mask           out  DEVICE buffers of the same shapes (filled by the call)
 *   kept_idx, kept_cnt      out  DEVICE [B][H][QB][cap], [B][H][QB] (as fgattn_compact_mask)
 *   out, lse                out  DEVICE bf16 [B][H][L][d], fp32 [B][H][L] (lse may be NULL)
 *   out_host, lse_host      out  HOST, same shapes (lse_host NULL exactly when lse is NULL)
 * Asynchronous with respect to the host: the host results are complete once
 * `stream` has passed the point of the call (cudaStreamSynchronize(stream) or
 * an event).  The copies start after all work already enqueued on `stream`.
 * No device memory is allocated; the first call on a device creates two
 * streams and a set of events, kept until exit.  Calls from several host
 * threads are enqueued one at a time.
 * Errors: as fgattn_compact_mask and fgattn_forward; INVALID_ARG also for a
 * NULL host pointer or heads_per_group < 1.  The method of the paper has no
 * counterpart: this is transfer scheduling around its computation.
 */
fgattn_status fgattn_attention_from_host(const void* q_host, const void* k_host, const void* v_host,
                                         const uint32_t* mask_host, void* q, void* k, void* v, uint32_t* mask,
                                         int32_t* kept_idx, int32_t* kept_cnt, int64_t cap, int64_t B, int64_t H,
                                         int64_t L, int64_t d, int64_t M, int64_t N, float scale, void* out,
                                         float* lse, void* out_host, float* lse_host, int64_t heads_per_group,
                                         fgattn_stream_t stream);

/*
 * Size of the kept-list scratch array that fgattn_masked_forward_noalloc
 * uses: 64 MiB on every device the library is used on, held until exit.
 * The array belongs to the library's device code, so it is reserved when that
 * code is loaded onto a device: at the first call into the library on that
 * device, whichever entry point it is (with lazy module loading; at context
 * creation otherwise).  Every user of the library pays these 64 MiB per
 * device.  A caller that cannot allocate should make one call (any entry
 * point, e.g. fgattn_compact_mask on a tiny mask) before its allocator
 * reserves the device's memory; if the reservation fails, every entry point
 * returns FGATTN_ERR_CUDA.
 */
#define FGATTN_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * Mask to attention output without any device allocation: fgattn_compact_mask
 * followed by fgattn_forward, with the kept lists in a fixed scratch array
 * inside the library instead of caller memory.  The paper has no counterpart;
 * this entry point exists for callers that cannot allocate device memory
 * themselves (a plug-in handed only its input and output buffers by the
 * runtime that hosts it, a process whose device memory is all reserved by a
 * caching allocator, code that must not allocate once set-up is over).
 *   q, k, v   in   device bf16 [B][H][L][d]
 *   mask      in   device uint32 [B][H][QB][W]  (layout and diagonal rule as above)
 *   out       out  device bf16 [B][H][L][d]
 *   lse       out  device fp32 [B][H][L], may be NULL
 * Results equal fgattn_compact_mask + fgattn_forward on the same arguments.
 * Limit: the kept lists take 4 * (ceil(R / 64) * 64 + R * cap) bytes, with
 * R = B * H * QB rows and cap = fgattn_kept_capacity(L); a call that needs
 * more than FGATTN_NOALLOC_SCRATCH_BYTES returns CAPACITY and enqueues nothing
 * (for example B = 1, H = 8, L = 8192, M = 64 needs 32 MiB and fits).
 * No cudaMalloc, cudaFree or other allocating call is made.
 * Set-up: the first call on a device looks up that device's address of the
 * array (with the device current); make that first call before any stream
 * capture begins.  The address is kept for the life of the process, so the
 * library must not be used across a reset of that device (cudaDeviceReset or
 * any other teardown of its primary context): after one, the kept address
 * would no longer be the array's.
 * Sharing: every call on a device uses the same array, and it keeps the last
 * call's lists.  Calls in one stream are ordered and safe; calls that can run
 * at the same time on the GPU (different streams, no ordering between them)
 * race on the array and give wrong results.
 * Errors: INVALID_ARG, UNSUPPORTED, CAPACITY, CUDA; device-side problems as
 * for fgattn_forward.
 */
fgattn_status fgattn_masked_forward_noalloc(const void* q, const void* k, const void* v, const uint32_t* mask,
                                            int64_t B, int64_t H, int64_t L, int64_t d, int64_t M, int64_t N,
                                            float scale, void* out, float* lse, fgattn_stream_t stream);

/* Number of streaming multiprocessors the forward kernel's persistent grid uses
 * on the current device (0 on failure). */
int fgattn_num_sms(void);

/* Static, human-readable name of a status code. */
const char* fgattn_status_string(fgattn_status status);

#ifdef __cplusplus
}
#endif

#endif /* FGATTN_H */
