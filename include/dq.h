/*
 * dq.h -- C ABI of libdq: the int8 dynamic-quantization linear layer on
 * NVIDIA B200 (sm_100a), dense and block-sparse (BSR) weight, with its
 * dynamic FP8 sibling and the weight-only int4 (HQQ) linear.
 *
 * The layer (pytorch/ao PR 821, "int8 dynamic quant + bsr support",
 * description and review) is
 *
 *     q, s_row = per-token absmax int8 quantization of x        (bf16 -> int8)
 *     acc      = q . W_q^T                                        (int8 x int8 -> int32)
 *     out      = bf16( acc * s_row * s_col + bias )              (fused epilogue)
 *
 * with W_q an int8 weight quantized per output channel (absmax / 127, as the
 * Paddle "sparse_fc supported" PR 41770 computes its int8 weight scale, made
 * per channel as asked in its review).  The int32 accumulator never reaches
 * global memory in bf16 mode: the dequantization is fused into the GEMM,
 * which the PR 821 description names as the fix for its slowdown.
 *
 * Conventions for every entry point:
 *  - Tensor pointers are DEVICE pointers (unless stated), owned by the caller;
 *    libdq never frees or keeps them.  Calls are asynchronous on `stream`
 *    (a cudaStream_t; NULL = legacy default stream).
 *  - No entry point allocates device memory or synchronises, except where
 *    stated (dq_sync_status, dq_bsr_validate).  The first call on a device
 *    resolves the driver's tensor-map encoder and queries the device.
 *  - Arguments are validated on the host before any launch; a violation
 *    returns DQ_ERR_INVALID_ARG or DQ_ERR_UNSUPPORTED and launches nothing.
 *    Nothing aborts, throws or prints.
 *  - Matrices are row-major.  "ld" arguments are row strides in ELEMENTS.
 *  - Every wait inside a kernel is bounded (default 2 s, see
 *    dq_set_wait_timeout_ns).  A wait that runs out makes the kernel record
 *    DQ_ERR_TIMEOUT in a per-device error word and return; the error surfaces
 *    through dq_sync_status().
 *  - Only sm_100 devices (B200) are supported: anything else returns
 *    DQ_ERR_UNSUPPORTED.  There is no CPU or other fallback.
 */
#ifndef DQ_H_
#define DQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define DQ_API __attribute__((visibility("default")))
#else
#define DQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* A cudaStream_t (the runtime's stream handle) passed as a plain pointer. */
typedef struct CUstream_st* dq_stream_t;

typedef enum {
    DQ_OK = 0,
    DQ_ERR_INVALID_ARG = 1,   /* null pointer, negative size, bad stride, bad enum */
    DQ_ERR_UNSUPPORTED = 2,   /* shape / alignment / device outside what libdq handles */
    DQ_ERR_CUDA = 3,          /* a CUDA runtime or driver call failed: dq_last_cuda_error() */
    DQ_ERR_TIMEOUT = 4        /* a bounded device wait ran out (reported by dq_sync_status) */
} dq_status;

typedef enum {
    DQ_OUT_BF16 = 0,          /* out = bf16(acc * s_row * s_col + bias): the layer */
    DQ_OUT_S32 = 1,           /* out = acc as int32 (scales and bias ignored) */
    DQ_OUT_F32 = 2            /* FP8 path: out = acc as fp32 (scales and bias ignored) */
} dq_out_dtype;

/* Static description of a status code. Never NULL. */
DQ_API const char* dq_status_string(dq_status s);

/* The cudaError_t value behind the most recent DQ_ERR_CUDA on this host
 * thread (0 if none). */
DQ_API int dq_last_cuda_error(void);

/* Library version: major*10000 + minor*100 + patch. */
DQ_API int dq_version(void);

/* Synchronises `stream`, then reads and clears the current device's error
 * word.  Returns DQ_ERR_TIMEOUT if any kernel since the last call ran out a
 * bounded wait, DQ_ERR_CUDA if the synchronisation failed, DQ_OK otherwise.
 * Blocking. */
DQ_API dq_status dq_sync_status(dq_stream_t stream);

/* Limit, in nanoseconds of %globaltimer, for every bounded wait in kernels
 * launched after this call from any host thread (default 2e9).  0 restores
 * the default.  Host-side setting; takes effect at the next launch. */
DQ_API void dq_set_wait_timeout_ns(uint64_t ns);

/* Launches a one-CTA kernel that waits on an mbarrier nothing ever arrives
 * on, through the same bounded wait the GEMM kernels use, and so records
 * DQ_ERR_TIMEOUT after the configured limit.  For testing the failure path
 * without faulting the GPU.  Asynchronous. */
DQ_API dq_status dq_selftest_wait_timeout(dq_stream_t stream);

/* ------------------------------------------------------------------------
 * Quantization (first stage of the layer; pytorch/ao PR 821 "int8 dynamic
 * quant", Paddle PR 41770 absmax / 127 scale).
 *
 * For each row i:  a = max_k |x[i,k]|,  s[i] = fp32( max(a, 1e-8f) / 127 ),
 *                  q[i,k] = clamp( rint_half_even( fp32(x[i,k] / s[i]) ), -127, 127 ).
 * Guarantee: the scales are bit-equal to the IEEE fp32 quotient
 * max(a, 1e-8f) / 127, and every code is bit-equal to rint (half to even) of
 * the IEEE fp32 quotient x / s, clamped, i.e. to a scalar IEEE evaluation of
 * the formula with a true division.  (The kernels do not divide: for bf16
 * rows they form the correctly rounded quotient from a reciprocal by one
 * Markstein correction step, for fp32 rows they divide only near a tie.)
 * Non-finite inputs give unspecified (but in-bounds) results.
 *
 * x: bf16 [M, K] (as 16-bit patterns), row stride ldx >= K.
 * q: int8 [M, K], row stride ldq >= K.   scales: fp32 [M].
 * M >= 0, K >= 1 (M == 0 is a no-op).  Any alignment is accepted; rows
 * with K % 8 == 0, ldx % 8 == 0, ldq % 8 == 0 and 16-byte-aligned x and
 * 8-byte-aligned q take the vectorised single-pass kernel.
 * ------------------------------------------------------------------------ */
DQ_API dq_status dq_quantize_rows(const void* x_bf16, int64_t M, int64_t K, int64_t ldx,
                           int8_t* q, int64_t ldq, float* scales, dq_stream_t stream);

/* Weight preparation with the same formula per output channel: w fp32
 * [N, K] (nn.Linear layout: row n is output channel n), row stride ldw.
 * wq int8 [N, K] (row stride ldwq), s_col fp32 [N].  Offline step, not part
 * of the per-token hot path, but run on the GPU by the same kernel family. */
DQ_API dq_status dq_quantize_weight(const float* w, int64_t N, int64_t K, int64_t ldw,
                             int8_t* wq, int64_t ldwq, float* s_col, dq_stream_t stream);

/* ------------------------------------------------------------------------
 * Dense int8 linear (second and third stages fused).
 *
 *   acc[m,n] = sum_k A[m,k] * W[n,k]            exact int32 (|acc| <= K*127^2)
 *   DQ_OUT_BF16: out[m,n] = bf16_rne( ((float)acc * s_row[m]) * s_col[n] (+ bias[n]) )
 *                each step one fp32 op, round to nearest even, no FMA;
 *                bias == NULL means no addition at all.
 *   DQ_OUT_S32:  out[m,n] = acc (s_row, s_col, bias ignored, may be NULL).
 *
 * A: int8 [M, K], row-major, contiguous (K-major).   s_row: fp32 [M].
 * W: int8 [N, K], row-major, contiguous (K-major).   s_col: fp32 [N].
 * bias: bf16 [N] or NULL.   out: [M, N] row-major contiguous, bf16 or int32.
 * Requirements: M >= 0; 1 <= K <= 133144 (the int32 bound: 133144 * 127^2 <
 * 2^31) and K % 16 == 0; N >= 1 with N % 8 == 0; A, W, out 16-byte aligned.
 *
 * workspace / workspace_bytes: optional caller-owned device scratch for the
 * split-K (stream-K) schedules that keep all SMs busy when the output has
 * few tiles.  Pass NULL/0 to disable splitting (always correct, possibly
 * slower).  The size the library can use is dq_int8_linear_workspace_size();
 * a smaller buffer disables splitting.  The workspace must be ZERO-FILLED
 * before its first use; every call that completes leaves it zero-filled
 * again (after DQ_ERR_TIMEOUT, zero it again).  Two calls in flight at the
 * same time must not share a workspace.
 * ------------------------------------------------------------------------ */
DQ_API dq_status dq_int8_linear(const int8_t* A, const float* s_row, int64_t M, int64_t K,
                         const int8_t* W, const float* s_col, int64_t N,
                         const void* bias_bf16, void* out, dq_out_dtype out_dtype,
                         void* workspace, size_t workspace_bytes, dq_stream_t stream);

/* Bytes of workspace dq_int8_linear can use for this shape on the current
 * device (0 when the schedule never splits). */
DQ_API size_t dq_int8_linear_workspace_size(int64_t M, int64_t N, int64_t K);

/* ------------------------------------------------------------------------
 * Allocation-free variant of dq_int8_linear (the pages have no counterpart;
 * this is an interface convenience of libdq).
 *
 * Some callers cannot call cudaMalloc or own any device buffer to lend: a
 * plugin running inside an inference engine whose memory planner owns all
 * device memory, code that runs while another component is capturing a CUDA
 * graph (where an allocation would break the capture), or a latency-bound
 * caller that cannot afford the device-wide synchronisation cudaMalloc and
 * cudaFree can cause.  For them this entry point takes the same arguments as
 * dq_int8_linear minus the workspace: the stream-K scratch it needs lives in
 * a file-scope static device array of DQ_NOALLOC_SCRATCH_BYTES (32 MiB) that
 * every GPU which loads libdq holds until the process exits.  The caller still
 * passes inputs and outputs.  Nothing here calls cudaMalloc, cudaFree or any
 * allocating library routine.
 *
 *  - If the chosen schedule needs more scratch than DQ_NOALLOC_SCRATCH_BYTES
 *    (dq_int8_linear_workspace_size(M, N, K) > DQ_NOALLOC_SCRATCH_BYTES), the
 *    call launches nothing and returns DQ_ERR_UNSUPPORTED.
 *  - The first call on a device that needs the scratch looks up the array's
 *    device address for that device (cudaGetSymbolAddress, with that device
 *    current), zeroes the whole array on `stream` and waits for that (it
 *    synchronises `stream` once).  Make that first call before any stream
 *    capture.
 *  - The split-K kernel leaves every part of the array it used at zero when
 *    it completes, so later calls do not clear it.  After a bounded wait ran
 *    out (dq_sync_status returned DQ_ERR_TIMEOUT) partial sums may be left
 *    behind; the next call then zeroes the array again, on its `stream`,
 *    before its kernel.  All calls on a device share the one array: two
 *    calls whose work overlaps on the GPU (different streams, no ordering
 *    between them) race on it and may produce wrong results.  Serialise them.
 *  - The scratch size is dq_int8_linear_workspace_size(M, N, K) under the
 *    current measurement knobs (the same plan dq_int8_linear uses).
 *  - Everything else (requirements, results, errors) is as dq_int8_linear.
 * ------------------------------------------------------------------------ */
#define DQ_NOALLOC_SCRATCH_BYTES ((size_t)32 << 20)
DQ_API dq_status dq_int8_linear_noalloc(const int8_t* A, const float* s_row, int64_t M, int64_t K,
                                        const int8_t* W, const float* s_col, int64_t N,
                                        const void* bias_bf16, void* out, dq_out_dtype out_dtype,
                                        dq_stream_t stream);

/* ------------------------------------------------------------------------
 * Block-sparse (BSR) int8 linear, 64x64 blocks (pytorch/ao PR 821: the
 * kernel takes crow_indices / col_indices / values directly; vit_h_14
 * benchmark with --bsr 64).
 *
 * W [N, K] in BSR form: block row b (output channels 64b .. 64b+63) holds
 * blocks p = crow[b] .. crow[b+1]-1; block p covers input channels
 * 64*col[p] .. 64*col[p]+63 and values[p] is its 64x64 int8 tile, row j =
 * channel 64b+j, 64 contiguous k values.  Duplicate blocks add.
 *   acc[m, 64b+j] = sum_p sum_t A[m, 64 col[p] + t] * values[p][j][t]
 * then the same epilogue as dq_int8_linear.  Block rows with no block give
 * bias (or 0) in bf16 mode and 0 in int32 mode.
 *
 * crow: int32 [N/64 + 1], col: int32 [nnzb], values: int8 [nnzb, 64, 64].
 * Requirements: K % 64 == 0, N % 64 == 0, K <= 133120, nnzb >= 0, pointers
 * 16-byte aligned.  Indices must be canonical (crow[0] == 0, non-decreasing,
 * crow[N/64] == nnzb, 0 <= col < K/64; order inside a row is free).  The
 * kernel clamps block ranges to [0, nnzb] and a column outside [0, K/64)
 * reads zeros, so malformed indices give wrong numbers but never an
 * out-of-bounds access; dq_bsr_validate checks them on the host.
 * ------------------------------------------------------------------------ */
DQ_API dq_status dq_bsr_int8_linear(const int8_t* A, const float* s_row, int64_t M, int64_t K, int64_t N,
                             const int32_t* crow, const int32_t* col, const int8_t* values,
                             int64_t nnzb, const float* s_col, const void* bias_bf16,
                             void* out, dq_out_dtype out_dtype, dq_stream_t stream);

/* Gathers the 64x64 blocks named by (crow, col) out of a dense int8 weight
 * wq [N, K] (row stride K) into values [nnzb, 64, 64].  Offline weight
 * preparation (mask, quantize per channel, pack).  Same index requirements
 * as dq_bsr_int8_linear. */
DQ_API dq_status dq_bsr_pack(const int8_t* wq, int64_t N, int64_t K, const int32_t* crow,
                      const int32_t* col, int64_t nnzb, int8_t* values, dq_stream_t stream);

/* Host-side, synchronous: copies crow and col to the host and checks the
 * canonical form above.  DQ_OK or DQ_ERR_INVALID_ARG. */
DQ_API dq_status dq_bsr_validate(const int32_t* crow, const int32_t* col, int64_t N, int64_t K,
                          int64_t nnzb);

/* ------------------------------------------------------------------------
 * The same three calls for square blocks of 64, 32 or 16 (the BSR block
 * size is a parameter of the pages' benchmark, --sp-linear-tile-size in the
 * PR 821 review; PyTorch BSR tensors carry it as values' trailing shape).
 * `block` in {64, 32, 16}; every "64" above becomes `block`: crow int32
 * [N/block + 1], col int32 [nnzb] (0 <= col < K/block), values int8
 * [nnzb, block, block] (row j = channel block*b + j, `block` contiguous k
 * values).  Requirements: K % block == 0, N % block == 0, K % 16 == 0.
 * block == 64 is exactly dq_bsr_int8_linear / dq_bsr_pack / dq_bsr_validate.
 * Another block size returns DQ_ERR_UNSUPPORTED (DQ_ERR_INVALID_ARG from
 * the validator).  Smaller blocks cost more per useful MAC: a 16x16 block
 * still issues a K = 32 MMA (its other half multiplies zeros).
 * ------------------------------------------------------------------------ */
DQ_API dq_status dq_bsr_int8_linear_blocked(const int8_t* A, const float* s_row, int64_t M, int64_t K,
                                            int64_t N, int64_t block, const int32_t* crow,
                                            const int32_t* col, const int8_t* values, int64_t nnzb,
                                            const float* s_col, const void* bias_bf16, void* out,
                                            dq_out_dtype out_dtype, dq_stream_t stream);
DQ_API dq_status dq_bsr_pack_blocked(const int8_t* wq, int64_t N, int64_t K, int64_t block,
                                     const int32_t* crow, const int32_t* col, int64_t nnzb,
                                     int8_t* values, dq_stream_t stream);
DQ_API dq_status dq_bsr_validate_blocked(const int32_t* crow, const int32_t* col, int64_t N, int64_t K,
                                         int64_t block, int64_t nnzb);

/* ------------------------------------------------------------------------
 * Dynamic FP8 (e4m3) sibling of the int8 layer (the vLLM csrc/quantization
 * commits: dynamic activation scales, scaled values clamped to the e4m3
 * range so that no NaN appears; applied per token here like the int8 path).
 *
 * dq_quantize_rows_fp8 / dq_quantize_weight_fp8: per row
 *   s = fp32( max(absmax, 1e-8f) / 448 ),
 *   q = e4m3( clamp( fp32(x / s), -448, 448 ) )   round to nearest even,
 * codes are e4m3 bytes (1 sign, 4 exponent bits with bias 7, 3 mantissa
 * bits; 448 the largest value), layouts and requirements as
 * dq_quantize_rows / dq_quantize_weight.  Bit-identical to a scalar IEEE
 * evaluation.
 *
 * dq_fp8_linear: acc[m, n] = sum_k e4m3(A[m, k]) * e4m3(W[n, k]) on the
 * tensor cores (tcgen05.mma kind::f8f6f4, fp32 accumulator in TMEM), then
 *   DQ_OUT_BF16: out = bf16((acc * s_row[m]) * s_col[n] + bias[n]) as the
 *                int8 layer (each op rounded, left to right, no FMA);
 *   DQ_OUT_F32:  out = acc as fp32 (scales and bias ignored).
 * Every product of two e4m3 values is exact in fp32; the order and
 * precision of the tensor core's fp32 sum are the hardware's, so results are
 * not bit-reproducible by a scalar loop (the tests bound |acc - exact sum|).
 * A and W are uint8 e4m3 codes, K-major ([M,K] and [N,K] row-major).
 * Requirements: K % 16 == 0, N % 8 == 0 (bf16 out) or N % 4 == 0 (fp32 out),
 * pointers 16-byte aligned; M >= 0.  DQ_OUT_S32 is rejected here.
 * ------------------------------------------------------------------------ */
DQ_API dq_status dq_quantize_rows_fp8(const void* x_bf16, int64_t M, int64_t K, int64_t ldx, uint8_t* q,
                                      int64_t ldq, float* scales, dq_stream_t stream);
DQ_API dq_status dq_quantize_weight_fp8(const float* w, int64_t N, int64_t K, int64_t ldw, uint8_t* wq,
                                        int64_t ldwq, float* s_col, dq_stream_t stream);
DQ_API dq_status dq_fp8_linear(const uint8_t* A, const float* s_row, int64_t M, int64_t K, const uint8_t* W,
                               const float* s_col, int64_t N, const void* bias_bf16, void* out,
                               dq_out_dtype out_dtype, dq_stream_t stream);

/* ------------------------------------------------------------------------
 * Weight-only int4 linear with the groupwise asymmetric dequantization fused
 * into a bf16 GEMM ("Fused HQQ Quantization Gemm", pytorch/ao PR 153,
 * description and implementation details).
 *
 * Weight format (shared by every call below):
 *   codes   q[n, k], n < N output channels, k < K in-features; u4 (0..15) or,
 *           with DQ_HQQ_S4, s4 (-8..7);
 *   packed  uint8 [N, K/2] row-major: byte j of row n = q[n, 2j] in bits
 *           0..3 | q[n, 2j+1] in bits 4..7 (the page's "row interleave" of
 *           two codes per byte along K; s4 as two's-complement nibbles);
 *   scale, zero  bf16 [K/group, N] row-major, GROUP-MAJOR: element (g, n) is
 *           channel n's value for its group g of `group` consecutive k, so
 *           one contraction step's values for a run of channels are one
 *           contiguous slice (dq_hqq_group_major converts the per-channel
 *           [N, K/group] form);
 *   dequantized weight w[n, k] = bf16( bf16(q - zero[k/group, n]) *
 *           scale[k/group, n] ), each operation rounded once to nearest even.
 *
 * dq_hqq_pack: codes int8 [rows, cols] (cols even; values must lie in the
 *   u4 or s4 range, only the low 4 bits are kept) -> packed [rows, cols/2].
 * dq_hqq_group_major: src bf16 [N, G] -> dst bf16 [G, N] (the per-channel
 *   scale / zero-point layout to the group-major one; a weight-load step).
 * dq_hqq_dequantize: packed, scale, zero -> w bf16 [N, K] (the standalone
 *   dequantization; bit-exact).
 * dq_hqq_linear (forward):   out[m, n] = sum_k x[m, k] * w[n, k],
 *   x bf16 [M, K], out bf16 [M, N].
 * dq_hqq_linear_t (transposed, for the input gradient of the backward pass):
 *   out[m, k] = sum_n y[m, n] * w[n, k],  y bf16 [M, N], out bf16 [M, K].
 * Both run on the tensor cores (tcgen05.mma kind::f16, bf16 operands, fp32
 * accumulator in TMEM); the int4 weight is dequantized in shared memory by
 * the GEMM kernel itself and never exists as a bf16 matrix in global memory.
 * Every bf16 x bf16 product is exact in fp32; the order of the fp32 sum is
 * the hardware's (deterministic for a given shape and workspace), so results
 * are compared with the exact sum within a bound, not bit for bit.
 *
 * Requirements: group in {32, 64, 128, 256}; K % group == 0; N % 8 == 0;
 * M >= 0 (M == 0 launches nothing); all pointers 16-byte aligned.
 * workspace / workspace_bytes: accepted for interface stability and not
 * used; dq_hqq_workspace_size() returns 0.  Few-token calls split the
 * contraction over a thread-block cluster of up to 8 CTAs per output tile,
 * which add their partial sums through distributed shared memory in split
 * order (results do not depend on timing, and concurrent calls share no
 * state).
 * ------------------------------------------------------------------------ */
enum { DQ_HQQ_S4 = 1 };

DQ_API dq_status dq_hqq_pack(const int8_t* codes, int64_t rows, int64_t cols, uint8_t* packed,
                             dq_stream_t stream);
DQ_API dq_status dq_hqq_dequantize(const uint8_t* packed, const void* scale_bf16, const void* zero_bf16,
                                   int64_t N, int64_t K, int group, int flags, void* w_bf16,
                                   dq_stream_t stream);
DQ_API dq_status dq_hqq_group_major(const void* src_bf16, int64_t N, int64_t G, void* dst_bf16,
                                    dq_stream_t stream);
DQ_API size_t dq_hqq_workspace_size(int64_t M, int64_t N, int64_t K, int transposed);
DQ_API dq_status dq_hqq_linear(const void* x_bf16, int64_t M, const uint8_t* packed, const void* scale_bf16,
                               const void* zero_bf16, int64_t N, int64_t K, int group, int flags,
                               void* out_bf16, void* workspace, size_t workspace_bytes, dq_stream_t stream);
DQ_API dq_status dq_hqq_linear_t(const void* y_bf16, int64_t M, const uint8_t* packed, const void* scale_bf16,
                                 const void* zero_bf16, int64_t N, int64_t K, int group, int flags,
                                 void* out_bf16, void* workspace, size_t workspace_bytes, dq_stream_t stream);

/* ------------------------------------------------------------------------
 * 2:4 semi-structured sparse int8 weight ("sparse_fc supported",
 * PaddlePaddle PR 41770: FC weights with at most two nonzeros in every group
 * of four consecutive in-features, compressed on the device; its review asks
 * for the int8 product with only the dequantization fused and a 16-bit
 * output).
 *
 * dq_s24_compress: wq int8 [N, K] (K % 8 == 0, row-major) ->
 *   values int8 [N, K/2]: the two kept values of each group, in position order;
 *   meta uint8 [N, K/8]: per group the nibble p0 | p1 << 2 (kept positions
 *     p0 < p1), group 2b in the low nibble of byte b.
 *   A group with fewer than two nonzeros keeps them and fills up with its
 *   lowest free positions.  Groups with more than two nonzeros keep their two
 *   lowest nonzero positions and are counted into *violations (device int32,
 *   added to atomically; may be NULL).  wq 8-byte and values 4-byte aligned.
 * dq_s24_int8_linear: out = the int8 layer of dq_int8_linear with the weight
 *   given compressed: acc[m, n] = sum_k A[m, k] * W[n, k] (exact int32, W the
 *   decompressed weight), then DQ_OUT_BF16: bf16((acc * s_row[m]) * s_col[n]
 *   + bias[n]) or DQ_OUT_S32: acc.  A int8 [M, K] contiguous.  The product
 *   runs on the sparse tensor-core MMA (tcgen05.mma.sp kind::i8): the
 *   compressed values are its A operand as they are and the metadata, copied
 *   into tensor memory, its sparsity selectors, so only the kept half of the
 *   weight is multiplied; the weight crosses HBM compressed (5/8 of its dense
 *   int8 bytes).  meta nibbles must have p0 < p1 (as dq_s24_compress writes
 *   them); other nibbles give unspecified (but in-bounds) results.
 *   Requirements: K % 128 == 0, N % 8 == 0, M >= 0, pointers 16-byte
 *   aligned.  workspace: optional caller-owned device scratch that lets
 *   few-token calls split the contraction over more SMs; its usable size is
 *   dq_s24_workspace_size(), and NULL or a smaller buffer disables
 *   splitting.  Its first bytes are the split arrival counters, eight per
 *   tile, which must be zero when a call starts and which every completed
 *   call leaves zero; the rest holds int32 partial sums (exact, so results
 *   never depend on the split).  One zero-filled workspace serves any number
 *   of calls of one shape; re-zero it for another shape or after
 *   DQ_ERR_TIMEOUT, and do not share it between calls that may run at the
 *   same time.
 * ------------------------------------------------------------------------ */
DQ_API dq_status dq_s24_compress(const int8_t* wq, int64_t N, int64_t K, int8_t* values, uint8_t* meta,
                                 int32_t* violations, dq_stream_t stream);
DQ_API size_t dq_s24_workspace_size(int64_t M, int64_t N, int64_t K);
DQ_API dq_status dq_s24_int8_linear(const int8_t* A, const float* s_row, int64_t M, int64_t K, const int8_t* values,
                                    const uint8_t* meta, const float* s_col, int64_t N, const void* bias_bf16,
                                    void* out, dq_out_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                    dq_stream_t stream);

/* ------------------------------------------------------------------------
 * Measurement knobs.  Process-wide settings read by every later launch from
 * any host thread (relaxed atomics); they change which schedule or kernel a
 * call uses, never its result.  For benchmarks and tests of the alternative
 * schedules; the defaults (all 0 except where stated) are what the library
 * chooses by itself.  Not for concurrent use with different settings.
 *
 * dq_debug_set_schedule (dense int8 linear): 0 automatic; 1 the 1-SM kernel
 *   with whole tiles; 2 the 1-SM kernel with stream-K whenever a workspace
 *   is given; 3 the 2-SM pair kernel for every M; 4 the dense (tokens on
 *   MMA M) arrangement also for M <= 128; 5 as 4 with stream-K.  The FP8
 *   and 2:4 linears read it too: 1 keeps their 1-SM kernels, 3 takes their
 *   2-SM pair kernels (2:4: when its contraction is not split).
 * dq_debug_set_tile_n: force the dense tile width (128, 160, 192, 224, 256;
 *   pair kernel 160, 192, 256); 0 automatic.
 * dq_debug_set_two_widths: 1 (default) wave-balanced schedule of two tile
 *   widths where whole tiles leave a partial last wave; 0 uniform tiles.
 * dq_debug_set_bsr_panel: BSR activation-panel variant (K <= 1280):
 *   0 never, 1 (default) for blocks smaller than 64, 2 always.
 * dq_debug_set_quant_kernel: 0 automatic, 1 register-resident kernel,
 *   2 row-pipelined (shared-memory ring) kernel for int8 codes.
 * ------------------------------------------------------------------------ */
DQ_API void dq_debug_set_schedule(int mode);
DQ_API void dq_debug_set_tile_n(int n);
DQ_API void dq_debug_set_two_widths(int on);
DQ_API void dq_debug_set_bsr_panel(int mode);
DQ_API void dq_debug_set_quant_kernel(int mode);

/* ------------------------------------------------------------------------
 * Measurement helper: a kernel that only issues tcgen05.mma.kind::i8
 * (128x256x32, operands resident in shared memory, accumulator in TMEM) on
 * every SM, `iters` times per CTA, with no global-memory traffic.  Used to
 * state the measured dense INT8 tensor-pipe peak: ops = grid * iters *
 * 2*128*256*32.  grid <= 0 means one CTA per SM.
 * ------------------------------------------------------------------------ */
DQ_API dq_status dq_mma_peak_probe(int grid, int iters, dq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DQ_H_ */
