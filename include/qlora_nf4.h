/*
 * qlora_nf4.h -- C ABI of the NF4 + double-quantization codec and the QLoRA linear layer
 * for NVIDIA B200 (sm_100a).
 *
 * The operations follow the method described in:
 *   [T] "QLoRA Paper Breakdown: 4-Bit NormalFloat (NF4), Double Quantization, and Paged
 *       Optimizers" (fullstackaihub teardown): section 2 (code book), section 3 (blockwise
 *       quantization, double quantization), section 4 (forward pass, dequantization helper,
 *       backward through the frozen base).
 *   [E] "QLoRA, explained." (vibeengines): method steps 1-5 and the notation list.
 *
 * Conventions for every entry point:
 *  - Every pointer is a DEVICE pointer owned by the caller, except where stated.  The library
 *    allocates no device memory (except qnf4_paged_alloc, on request, for optimizer states) and
 *    keeps no state between calls other than the device error word (see qnf4_device_error) and
 *    the static scratch array of nf4_quantize_dq_noalloc.
 *  - bf16 tensors are passed as uint16_t bit patterns, row-major, densely packed.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Every call is
 *    stream-ordered and asynchronous: it returns after enqueueing its kernels.  Device-side
 *    faults surface at the caller's next synchronisation.
 *  - Every call returns an int status (QNF4_OK or a negative QNF4_ERR_*); on error nothing
 *    has been enqueued unless the status is QNF4_ERR_CUDA (a launch failed part-way), and
 *    qnf4_last_error() returns a human-readable reason (thread-local).
 *  - Sizes are int64_t element counts; a size <= 0 is QNF4_ERR_INVALID.
 *
 * Stored format of a quantized weight W with numel = N*K elements (row-major [N][K]):
 *  - blocks are flat runs of 64 consecutive elements of the row-major tensor (a block spans
 *    two rows when K is not a multiple of 64); nb = ceil(numel/64); the last block is
 *    zero-padded;
 *  - codes       : uint8[32*nb], two 4-bit NF4 indices per byte, element 2i in the low
 *                  nibble of byte i ([T] section 3 level 1, [E] step 2);
 *  - scale_codes : uint8[nb], the block absmax values centred by the tensor's mean, divided
 *                  by their group constant, as E4M3 8-bit floats ([T] section 3 level 2);
 *  - c2          : float[ceil(nb/256)], one fp32 constant per group of 256 scale codes;
 *  - mean        : float[1], the fp32 mean of all block absmax values.
 * Storage: 4 + 8/64 + 32/(64*256) = 4.126953125 bits per weight, plus 32 bits for the mean.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QNF4_OK 0
#define QNF4_ERR_INVALID (-1)     /* null pointer, size <= 0, size overflow */
#define QNF4_ERR_UNSUPPORTED (-2) /* unsupported shape or alignment (see each call) */
#define QNF4_ERR_ARCH (-3)        /* current device is not sm_100 */
#define QNF4_ERR_CUDA (-4)        /* a CUDA call or launch failed; see qnf4_last_error() */
#define QNF4_ERR_DEVICE (-5)      /* a kernel's bounded wait ran out (device error word set) */
#define QNF4_ERR_WORKSPACE (-6)   /* workspace too small */

/* Library version (major*10000 + minor*100 + patch). */
int qnf4_version(void);

/* Reason for the last non-OK status returned on this host thread ("" if none).  The
 * string is owned by the library and valid until the next call on this thread. */
const char* qnf4_last_error(void);

/* Synchronises `stream`, then reads and clears the device error word of the current device.
 * *word receives the bit flags (0 = no kernel gave up waiting).  Returns QNF4_ERR_DEVICE if
 * the word was non-zero, QNF4_ERR_CUDA if the synchronisation failed.  `word` is a HOST
 * pointer. */
int qnf4_device_error(void* stream, uint32_t* word);

/* Bounded-wait self-test (a diagnostic, no counterpart in the method): enqueues one kernel
 * whose single waiting thread waits on a barrier that nothing completes, through the same
 * bounded-wait code every pipeline wait of the library uses.  After `limit_ns` nanoseconds of
 * wall-clock time (1 ms .. 10 s, else QNF4_ERR_INVALID) the wait gives up, sets bit 5 (0x20)
 * of the device error word and the kernel returns; the CUDA context stays usable.  A following
 * qnf4_device_error() returns QNF4_ERR_DEVICE with that bit set (and clears the word). */
int qnf4_selftest_bounded_wait(uint64_t limit_ns, void* stream);

/* ---------------------------------------------------------------------------------------
 * NF4 blockwise quantization with double quantization.
 * [T] section 3 (both levels), [E] steps 2-3.
 *
 *   W           : bf16[numel], read only.
 *   codes       : uint8[32*nb], written.     16-byte aligned.
 *   scale_codes : uint8[nb], written.        8-byte aligned.
 *   c2          : float[ceil(nb/256)], written.
 *   mean        : float[1], written.
 *   workspace   : device scratch of at least nf4_quantize_workspace_bytes(numel) bytes,
 *                 256-byte aligned; its contents are undefined afterwards.
 * W must be 16-byte aligned.  numel <= 2^35.  Weights must be finite.  Bit-exact with the
 * method's definition: absmax per block, n = fp32(w / absmax) (correctly rounded), the
 * nearest code-book level (ties to the lower level; an all-zero block codes to level 7),
 * mean = fp32(float64 pairwise sum / nb), d = fp32(absmax - mean), c2 = max |d| per group,
 * scale code = E4M3 round-to-nearest-even of fp32(d / c2) (c2 == 0 gives code 0).
 * ------------------------------------------------------------------------------------- */
size_t nf4_quantize_workspace_bytes(int64_t numel);
int nf4_quantize_dq(const uint16_t* W, int64_t numel, uint8_t* codes, uint8_t* scale_codes, float* c2,
                    float* mean, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * NF4 blockwise quantization with double quantization, without a workspace argument.
 * The method has no counterpart to this entry point: it is a calling convention of this
 * library, and computes exactly what nf4_quantize_dq computes (bit-identical outputs).
 *
 * Meant for callers that cannot allocate device memory at the point of the call: a host
 * program or plug-in that is handed only the weight and the output buffers and has no device
 * allocator of its own, or a runtime that reserved device memory for its own pool up front
 * and has no way to lend a temporary buffer.  Such a caller cannot supply the workspace that
 * nf4_quantize_dq needs, so the library keeps that scratch itself: one static device array,
 * sized for numel <= QNF4_NOALLOC_MAX_NUMEL (2^28 weights: 16 MiB of per-block absmax plus
 * 128 KiB of per-group float64 sums), which the CUDA runtime reserves on each device when it
 * loads the library's kernels there.
 *
 *   W, codes, scale_codes, c2, mean : as for nf4_quantize_dq (same layouts and alignment).
 *
 *  - numel above QNF4_NOALLOC_MAX_NUMEL returns QNF4_ERR_UNSUPPORTED before any device work;
 *    quantize larger weights with nf4_quantize_dq and a workspace.
 *  - The first call on each device does a one-time set-up: with that device current it looks
 *    up the device address of the scratch array (and looks it up again if the device's
 *    context has been re-created since, e.g. after cudaDeviceReset).  Make that first call
 *    before any stream capture begins.
 *  - Nothing has to start at zero: every scratch element a call reads, the same call writes
 *    first.
 *  - There is one scratch array per device, shared by every call on that device.  Calls that
 *    overlap in time (on different streams, or from different host threads without ordering)
 *    race on it and produce wrong results: order them on one stream or synchronise between
 *    them.
 *  - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine is called.
 * ------------------------------------------------------------------------------------- */
#define QNF4_NOALLOC_MAX_NUMEL 268435456LL
int nf4_quantize_dq_noalloc(const uint16_t* W, int64_t numel, uint8_t* codes, uint8_t* scale_codes,
                            float* c2, float* mean, void* stream);

/* ---------------------------------------------------------------------------------------
 * NF4 + DQ -> bf16 dequantization (the standalone HBM stream).
 * [T] section 4, dequantization helper; [E] step 4.
 *
 *   W_out[e] = bf16_rn( fp32_rn( level[code_e] * s_b ) ),  s_b = fmaf(e4m3(scale_code_b), c2_g, mean)
 * codes must be 16-byte aligned and W_out 16-byte aligned.  Inputs are read only.
 * ------------------------------------------------------------------------------------- */
int nf4_dequant(const uint8_t* codes, const uint8_t* scale_codes, const float* c2, const float* mean,
                int64_t numel, uint16_t* W_out, void* stream);

/* ---------------------------------------------------------------------------------------
 * QLoRA linear layer, forward.  [T] section 4 (forward pass), [E] steps 4-5.
 *
 *   y = x W'^T + s (x A^T) B^T,   W' = dequant(codes, scale_codes, c2, mean)  ([N][K])
 *
 *   x       : bf16[M][K]          A : bf16[r][K]          B : bf16[N][r]
 *   y       : bf16[M][N], written
 *   t_saved : float[M][r], written: t = s x A^T (fp32), kept by the caller for the backward
 * W' is produced tile by tile on chip (in tensor memory for 256-token tiles, else in shared
 * memory) from the codes and is never written to HBM.
 * Requirements: K % 8 == 0, N % 8 == 0, r % 8 == 0, 8 <= r <= 256, bf16 and code pointers
 * 16-byte aligned.  Accuracy: fp32 accumulation of exact bf16 products; the adapter term uses
 * t split into bf16 hi + lo parts.  Workspace: qlora_linear_fwd_workspace_bytes(M, K, N, r)
 * bytes, 256-byte aligned.
 * ------------------------------------------------------------------------------------- */
size_t qlora_linear_fwd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r);
int qlora_linear_fwd(const uint16_t* x, int64_t M, int64_t K, int64_t N, const uint8_t* codes,
                     const uint8_t* scale_codes, const float* c2, const float* mean, const uint16_t* A,
                     const uint16_t* B, int r, float s, uint16_t* y, float* t_saved, void* workspace,
                     size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * QLoRA linear layer, backward.  [T] section 4 (gradients reach the input through the
 * dequantized frozen base; no gradient of W is formed), [E] step 5 (only the adapters train).
 *
 *   u  = s dY B              (fp32, split into bf16 hi + lo)
 *   dX = dY W' + u A         (W' produced on chip from the codes, transposed operand)
 *   dA = u^T x               (reduction over the M tokens)
 *   dB = dY^T t_saved        (t_saved from qlora_linear_fwd on the same x, A and s)
 *
 *   dY : bf16[M][N]   x : bf16[M][K]   t_saved : float[M][r]
 *   dX : bf16[M][K], written (may be NULL to skip)   dA : bf16[r][K]   dB : bf16[N][r]
 * Same shape / alignment requirements as the forward.  Workspace:
 * qlora_linear_bwd_workspace_bytes(M, K, N, r) bytes, 256-byte aligned.
 * ------------------------------------------------------------------------------------- */
size_t qlora_linear_bwd_workspace_bytes(int64_t M, int64_t K, int64_t N, int r);
int qlora_linear_bwd(const uint16_t* dY, const uint16_t* x, const float* t_saved, int64_t M, int64_t K, int64_t N,
                     const uint8_t* codes, const uint8_t* scale_codes, const float* c2, const float* mean,
                     const uint16_t* A, const uint16_t* B, int r, float s, uint16_t* dX, uint16_t* dA,
                     uint16_t* dB, void* workspace, size_t workspace_bytes, void* stream);

/* ---------------------------------------------------------------------------------------
 * Other 16-level code books and single-level (no double quantization) scales.
 * [T] section 1 (standard INT4: 16 equally spaced levels over [-c, +c]) and section 3
 * (single blockwise quantization: an fp32 absmax per block of 64, 4 + 32/64 = 4.5 bits per
 * weight); dmarx anthology sota-230 (the data types compared: Int4, Float4 (E2M1), NF4 + DQ).
 *
 * codebook:
 *   QNF4_CODEBOOK_NF4       the NF4 levels (the default of every other call);
 *   QNF4_CODEBOOK_FP4_E2M1  the 16 values of the 4-bit float E2M1 (0, 0.5, 1, 1.5, 2, 3, 4, 6,
 *                           both signs, both zeros) divided by 6, sorted; code j is the j-th
 *                           value in increasing order (-0 is code 7, +0 code 8), not the E2M1
 *                           bit pattern;
 *   QNF4_CODEBOOK_INT4      -1 + 2 j / 15 for j = 0 .. 15.
 * Each level is the nearest fp32 to its exact value.  A weight takes the code of the nearest
 * level (an exact tie goes to the lower code; for E2M1 a normalised value of exactly 0 codes
 * to -0 and any positive one below 1/24 to +0).
 *
 * double_quant = 1: the stored format of nf4_quantize_dq (scale_codes[nb] E4M3, scales =
 *   c2[ceil(nb/256)], mean[1]).
 * double_quant = 0: scales = one fp32 absmax per block, float[nb]; scale_codes and mean are
 *   unused (may be NULL); no workspace is needed (qnf4_quantize_workspace_bytes_ex returns a
 *   token size and the workspace pointer may be NULL).
 * Everything else (layouts, alignment, errors, bit-exactness) is as for the NF4 calls above;
 * the dequantized weight is bf16(fp32(level[code] * s_b)) with s_b the block's scale.  The
 * linear layer calls take the same workspace sizes as qlora_linear_fwd / _bwd.
 * ------------------------------------------------------------------------------------- */
#define QNF4_CODEBOOK_NF4 0
#define QNF4_CODEBOOK_FP4_E2M1 1
#define QNF4_CODEBOOK_INT4 2
size_t qnf4_quantize_workspace_bytes_ex(int64_t numel, int double_quant);
int qnf4_quantize_ex(const uint16_t* W, int64_t numel, int codebook, int double_quant, uint8_t* codes,
                     uint8_t* scale_codes, float* scales, float* mean, void* workspace, size_t workspace_bytes,
                     void* stream);
int qnf4_dequant_ex(const uint8_t* codes, int codebook, int double_quant, const uint8_t* scale_codes,
                    const float* scales, const float* mean, int64_t numel, uint16_t* W_out, void* stream);
int qlora_linear_fwd_ex(const uint16_t* x, int64_t M, int64_t K, int64_t N, int codebook, int double_quant,
                        const uint8_t* codes, const uint8_t* scale_codes, const float* scales, const float* mean,
                        const uint16_t* A, const uint16_t* B, int r, float s, uint16_t* y, float* t_saved,
                        void* workspace, size_t workspace_bytes, void* stream);
int qlora_linear_bwd_ex(const uint16_t* dY, const uint16_t* x, const float* t_saved, int64_t M, int64_t K, int64_t N,
                        int codebook, int double_quant, const uint8_t* codes, const uint8_t* scale_codes,
                        const float* scales, const float* mean, const uint16_t* A, const uint16_t* B, int r, float s,
                        uint16_t* dX, uint16_t* dA, uint16_t* dB, void* workspace, size_t workspace_bytes,
                        void* stream);

/* ---------------------------------------------------------------------------------------
 * Adapter merge and re-quantization.  [T] "Engineering Limitations" (full-rank updates need
 * the adapters dequantized and merged into 16-bit precision); [V] (merging / re-quantizing
 * adapters is a deployment step).
 *
 *   W''[n][k] = bf16( W'[n][k] + s * sum_j B[n][j] A[j][k] ),   then W'' is quantized again.
 *
 * The rank-r sum is formed in float64, term by term in index order j = 0 .. r-1; then
 * t = float64(s * sum), v = float64(W' + t), and W'' is v rounded once to the nearest bf16
 * (ties to even).  W' is the dequantized base (as nf4_dequant / qnf4_dequant_ex produce it).
 * The result is then coded exactly as qnf4_quantize_ex codes a bf16 weight, with the same
 * code book and format as the input (codebook, double_quant as in qnf4_quantize_ex).
 *
 *   codes, scale_codes, scales, mean          : the stored base W' [N][K], read only
 *   A : bf16[r][K]    B : bf16[N][r]    s : the LoRA scale alpha / r
 *   codes_out, scale_codes_out, scales_out, mean_out : the re-quantized W'' (may not alias the
 *                                               inputs), written
 *   merged_out : bf16[N][K] receiving W'' itself (16-byte aligned), or NULL to keep it in the
 *                workspace
 *   workspace  : qlora_merge_workspace_bytes(N, K, double_quant, merged_out != NULL) bytes,
 *                256-byte aligned
 * Requirements: K % 8 == 0, r <= 1024, N * K <= 2^35.
 * ------------------------------------------------------------------------------------- */
size_t qlora_merge_workspace_bytes(int64_t N, int64_t K, int double_quant, int merged_out_given);
int qlora_merge_requantize(const uint8_t* codes, const uint8_t* scale_codes, const float* scales, const float* mean,
                           int64_t N, int64_t K, int codebook, int double_quant, const uint16_t* A, const uint16_t* B,
                           int r, float s, uint8_t* codes_out, uint8_t* scale_codes_out, float* scales_out,
                           float* mean_out, uint16_t* merged_out, void* workspace, size_t workspace_bytes,
                           void* stream);

/* ---------------------------------------------------------------------------------------
 * Paged AdamW on the LoRA parameters.  [T] section 5 (the AdamW states of the adapters live in
 * CUDA unified memory, which the driver evicts to host RAM under memory pressure and pages back
 * for the optimizer step); [E] step 6.
 *
 * qlora_adamw_step: one AdamW step with decoupled weight decay on n parameters:
 *   m = b1 m + (1 - b1) g,  v = b2 v + (1 - b2) g^2,
 *   p = p - lr ( (m / (1 - b1^step)) / (sqrt(v / (1 - b2^step)) + eps) + weight_decay p ).
 *   param, m, v : float[n], updated in place (16-byte aligned);  grad : bf16[n] (8-byte aligned);
 *   param_bf16  : bf16[n] receiving the updated parameters rounded to bf16, or NULL.
 *   step is 1-based.  The hyper-parameters are doubles: the kernel uses lr, b1, 1 - b1, b2,
 *   1 - b2, eps, weight_decay and the two bias corrections each rounded once to fp32 from the
 *   value formed in double (so 1 - b2 = 0.001 is not lost to an fp32 b2).  fp32 arithmetic
 *   with IEEE division and square root.  Any of the pointers
 *   may be managed memory (qnf4_paged_alloc); such memory should be on the device
 *   (qnf4_paged_prefetch) when the step runs, or the driver migrates it page by page.
 *
 * qnf4_paged_alloc / qnf4_paged_free: CUDA managed memory for optimizer states (these two are
 *   the library's only allocating calls).  `ptr` is a HOST pointer receiving the address.
 * qnf4_paged_prefetch: stream-ordered migration of a managed range to the current device
 *   (to_device = 1) or to host memory (to_device = 0: eviction).
 * ------------------------------------------------------------------------------------- */
int qnf4_paged_alloc(size_t bytes, void** ptr);
int qnf4_paged_free(void* ptr);
int qnf4_paged_prefetch(const void* ptr, size_t bytes, int to_device, void* stream);
int qlora_adamw_step(float* param, const uint16_t* grad, float* m, float* v, uint16_t* param_bf16, int64_t n,
                     double lr, double beta1, double beta2, double eps, double weight_decay, int step,
                     void* stream);

/* ---------------------------------------------------------------------------------------
 * Launch plan of one forward / backward call of this shape (host-only, no device work):
 * the number of kernels each call enqueues, and the split factor of the K loop of the
 * fused dequant GEMMs (1 = no split).  Output pointers are HOST pointers and may be NULL.
 * ------------------------------------------------------------------------------------- */
int qlora_linear_plan(int64_t M, int64_t K, int64_t N, int r, int* fwd_launches, int* bwd_launches,
                      int* fwd_splits, int* dx_splits);

/* ---------------------------------------------------------------------------------------
 * Optional stage timing (a profiling aid, no counterpart in the method).  When `events`
 * is non-NULL, later calls made from this host thread record the caller's cudaEvent_t
 * handles on their stream at stage boundaries (events[i] for i < n only):
 *   qlora_linear_fwd: [0] start, [1] after the down-projection t = s x A^T, [2] end (after
 *                     the fused dequant GEMM and its split reduction, if any);
 *   qlora_linear_bwd: [0] start, [1] after the B transpose and t split, [2] after
 *                     u = s dY B, [3] after the fused dX GEMM, [4] after dA, [5] end (dB).
 * The handles stay owned by the caller; pass NULL (or n = 0) to stop recording.
 * ------------------------------------------------------------------------------------- */
int qnf4_set_timing_events(void* const* events, int n);

/* ---------------------------------------------------------------------------------------
 * E4M3 encoding of an fp32 array, as used for the scale codes (round to nearest even,
 * saturating at 448, sign kept).  mode 0 = hardware conversion (the one nf4_quantize_dq
 * uses), mode 1 = the library's software encoder.  A utility for checking the format.
 * ------------------------------------------------------------------------------------- */
int nf4_e4m3_encode(const float* v, int64_t n, uint8_t* out, int mode, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H */
