/*
 * fp4.h -- C ABI of libfp4: microscaling FP4 quantization (NVFP4, MXFP4 and
 * P1E8, one tensor or a batch), reconstruction to BF16, and the native W4A4
 * block-scaled GEMM (single, grouped, decode) on NVIDIA B200 (sm_100a).
 *
 * The operations come from these web pages (cited by title and section):
 *  [NVFP4-Arch] "NVFP4 Architecture: Microscaling & 4-Bit LLMs on Blackwell"
 *     "1. The E2M1 Floating-Point Format", "2. Micro-Block Exponent Scaling:
 *     E8M0 Format", "1. The Dual-Level Mathematical Formulation",
 *     "2. Hardware-Managed Tensor Core Dot-Products".
 *  [ia4pymes]   "NVIDIA NVFP4 quantization ..." - "The Physics of NVFP4:
 *     Block-Wise Microscaling Quantization" (16-element blocks, 8-bit scale).
 *  [MXFP4-BW]   "How Microscaling FP4 (MXFP4) Halves Memory Bandwidth in
 *     Frontier Models Without Training Divergence" - "The Microscaling
 *     Breakthrough: 32-Element Blocks", "Silicon Execution: Tensor Cores &
 *     Register Fusing".
 *  [MXFP4-kc]   "MXFP4" - "Core Facts" (E8M0 scale, block size 32).
 *
 * Conventions shared by every entry point
 *  - All data pointers are CUDA device pointers owned by the caller; the
 *    library never allocates or frees caller-visible memory.
 *  - Every call validates its arguments on the host first.  A call that
 *    returns anything but FP4_OK has launched nothing, except FP4_ERR_CUDA
 *    from a call that makes several launches (batches above 8 tensors or 16
 *    problems, the amax pass of a dynamic quantization), where launches
 *    before the failing one may have been queued.  A call that returns
 *    FP4_OK has queued its kernels on `stream` (asynchronous; the results are
 *    ready once the stream reaches that point).  Nothing is printed, nothing
 *    aborts the process.
 *  - BF16 inputs are row-major with a leading dimension `ld` in elements
 *    (ld >= the row length, ld % 8 == 0) and a 16-byte aligned base pointer.
 *    Outputs must be 16-byte aligned.
 *  - Inputs must be finite: NaN or infinity give unspecified output bytes
 *    (never a fault or a hang).
 *  - Packed FP4: two E2M1 codes per byte, the even index in the low nibble,
 *    K-major rows of K/2 bytes.  Code = sign bit (bit 3) | exponent (bits 2-1)
 *    | mantissa (bit 0); values {0, 0.5, 1, 1.5, 2, 3, 4, 6} with signed zero.
 *  - Scales: one byte per block (E4M3 for NVFP4, E8M0 for MXFP4 and P1E8) stored in
 *    512-byte tiles of 128 rows x 4 block-columns, tiles ordered with the
 *    block-column tile fastest; inside a tile the byte of (row r, block c) is
 *    at (r % 32) * 16 + ((r / 32) % 4) * 4 + (c % 4).  This is the layout the
 *    tensor core's block-scaled MMA reads.  Padding rows are written as 0.
 */
#ifndef FP4_H
#define FP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* fp4_stream_t;

typedef enum {
    /* 16-element blocks, unsigned E4M3 block scale, FP32 per-tensor scale
     * S_global ([NVFP4-Arch] dual-level formulation; [ia4pymes]). */
    FP4_NVFP4 = 0,
    /* 32-element blocks, E8M0 power-of-two block scale ([MXFP4-kc],
     * [MXFP4-BW] "32-Element Blocks"). */
    FP4_MXFP4 = 1,
    /* 16-element blocks with an E8M0 block scale under an FP32 S_global:
     * S_block = 2^ceil(log2(max(amax / (6 S_global), 1e-8))) (capped at
     * 2^127), the NVFP4 of [NVFP4-Arch] "1. The Dual-Level Mathematical
     * Formulation" read literally (its block scale is E8M0).  The GEMM runs
     * it as the 16-element block-scaled MMA with the UE8M0 scale type, with
     * alpha = S_global,A * S_global,B as for NVFP4. */
    FP4_P1E8 = 2
} fp4_format;

typedef enum {
    /* blocks run along each row (the row is the K dimension) */
    FP4_ROWWISE = 0,
    /* blocks run down each column; output row c is input column c, i.e. the
     * quantized result is the transpose (the K-major form of the other GEMM
     * operand) */
    FP4_COLWISE = 1
} fp4_axis;

typedef enum {
    FP4_OK = 0,
    FP4_ERR_INVALID_ARG = 1,       /* bad enum, NULL pointer, ld < length, small workspace */
    FP4_ERR_UNSUPPORTED_SHAPE = 2, /* a dimension breaks a divisibility rule */
    FP4_ERR_MISALIGNED = 3,        /* pointer or leading dimension not 16-byte aligned */
    FP4_ERR_CUDA = 4,              /* a CUDA runtime call or launch failed */
    FP4_ERR_TIMEOUT = 5,           /* a kernel gave up on a bounded wait (see fp4_get_device_status) */
    FP4_ERR_NO_DEVICE = 6,         /* no usable sm_100 device */
    FP4_ERR_WORKSPACE = 7          /* the decode workspace's counters were not zero (see fp4_gemm) */
} fp4_status;

typedef enum {
    FP4_GEMM_AUTO = 0,    /* decode kernel when M <= 16 and the workspace suffices, else prefill */
    FP4_GEMM_PREFILL = 1, /* persistent CTA-pair tensor-core kernel, 256x256 tiles */
    FP4_GEMM_DECODE = 2,  /* swap-AB, stream-K kernel for M <= 16 plus a split-K reduction */
    /* Flag, OR-ed into a kernel choice above: B and sB are not written by any
     * kernel that may still be running on the stream when the GEMM starts
     * (e.g. weights quantized ahead of time).  The decode kernel then requests
     * its first weight tiles before waiting for the previous kernel to
     * complete.  Without the flag no operand is read before that. */
    FP4_GEMM_B_STATIC = 0x100
} fp4_gemm_kernel;

/* Version of this ABI (incremented on any signature or contract change). */
int fp4_abi_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char* fp4_status_string(fp4_status s);

/* Detail of the most recent failing call on this host thread (which check or
 * CUDA call failed), or "" if none; valid until the thread's next failing
 * call. */
const char* fp4_last_error(void);

/* Bytes of packed FP4 data for `rows` rows of length k: rows * k / 2. */
size_t fp4_packed_bytes(int64_t rows, int64_t k);

/* Bytes of the tiled scale buffer for `rows` rows of length k in format
 * `fmt`: ceil(rows/128) * ceil(k/blk/4) * 512 (blk = 16 for NVFP4 and
 * P1E8, 32 for MXFP4).  0 for an invalid format. */
size_t fp4_scale_bytes(fp4_format fmt, int64_t rows, int64_t k);

/*
 * S_global of a BF16 matrix: amax over |x| divided by 6 * 448 = 2688 in FP32,
 * or 1.0 if the matrix is all zero.  With this value the block that holds the
 * tensor's largest magnitude gets the largest E4M3 block scale (448).
 * [NVFP4-Arch] "1. The Dual-Level Mathematical Formulation", item 1 (a
 * per-tensor scalar for the tensor's dynamic ceiling; FP32 is this library's
 * reading of its precision).
 *   in_bf16 : device, rows x cols, leading dimension ld (elements)
 *   gs_out  : device, one float, written asynchronously
 * Requires cols % 8 == 0.  One launch: the CTAs reduce their rows, the last
 * one to finish writes S_global.  Its partial maxima meet in one of 1024
 * reduction slots in the library's static device memory, taken in turn by
 * successive calls and left zeroed by each call, so up to 1024 calls may be
 * in flight at once (on any streams) without sharing a slot.  A call captured
 * in a CUDA graph keeps its slot in every replay of the graph.
 */
fp4_status fp4_compute_global_scale(const void* in_bf16, int64_t rows, int64_t cols,
                                    int64_t ld, float* gs_out, fp4_stream_t stream);

/*
 * fp4_compute_global_scale followed by alpha = S_global * (*other_gs) (the
 * product fp4_alpha_from_global_scales forms), both in the same single
 * launch: the two per-tensor factors of an NVFP4 GEMM whose other operand's
 * S_global is already known.  gs_out, other_gs and alpha_out are device
 * floats (other_gs written by earlier work on the stream, or constant).
 */
fp4_status fp4_compute_global_scale_alpha(const void* in_bf16, int64_t rows, int64_t cols,
                                          int64_t ld, float* gs_out, const float* other_gs,
                                          float* alpha_out, fp4_stream_t stream);

/*
 * S_global of both operands of an NVFP4 GEMM and alpha = gs_a * gs_b, in one
 * launch (the CTAs of that launch reduce the rows of either tensor; the last
 * to finish writes both scales and alpha): each value equal to what
 * fp4_compute_global_scale and fp4_alpha_from_global_scales give.  Same
 * reading of [NVFP4-Arch] "1. The Dual-Level Mathematical Formulation" as
 * above, for the two tensors whose product the GEMM forms.
 *   a_bf16, b_bf16 : device, rows x cols each, leading dimension ld_*
 *   gs_a_out, gs_b_out : device floats, written
 *   alpha_out : device float, or NULL
 * Requires cols_* % 8 == 0; an empty tensor gets S_global = 1.
 */
fp4_status fp4_compute_global_scales_pair(const void* a_bf16, int64_t rows_a, int64_t cols_a,
                                          int64_t ld_a, const void* b_bf16, int64_t rows_b,
                                          int64_t cols_b, int64_t ld_b, float* gs_a_out,
                                          float* gs_b_out, float* alpha_out, fp4_stream_t stream);

/*
 * Block quantization BF16 -> E2M1 codes + one scale per block.
 * [NVFP4-Arch] "1. The Dual-Level Mathematical Formulation" (S_block,j,
 * q_i = Quantize_E2M1(x_i / (S_global * S_block,j))) and the emulation script
 * in "End-to-End Implementation" (block amax, 1e-8 clamp, ceil(log2(amax/6))).
 *
 * Per block of k elements (k = 16 NVFP4 and P1E8, 32 MXFP4), amax = max |x_i|:
 *   MXFP4: e = ceil(log2(max(amax, 1e-8) / 6)); scale byte = e + 127;
 *          v_i = x_i * 2^-e.
 *   NVFP4: t = amax / (6 * gs) (FP32); scale byte = E4M3 round-to-nearest-
 *          even of t, saturating at 448; eff = E4M3(byte) * gs (FP32);
 *          v_i = x_i * RN(1/eff) (0 when eff == 0).
 *   P1E8:  a = max(amax / (6 * gs) (FP32), 1e-8); e = ceil(log2 a), at most
 *          127; scale byte = e + 127; eff = 2^e * gs (FP32); v_i as NVFP4.
 *   q_i  = E2M1 round-to-nearest-even of v_i, |v| >= 6 -> 6, sign of x_i kept.
 *
 *   axis = FP4_ROWWISE: blocks along each row of in[rows x cols];
 *          packed_out is [rows x cols/2] bytes, scales_out covers rows x
 *          cols/k scales.  Requires cols % (4k) == 0 (64 / 128).
 *   axis = FP4_COLWISE: blocks down each column; packed_out is
 *          [cols x rows/2] (the transpose), scales_out covers cols x rows/k.
 *          Requires rows % (4k) == 0 and cols % 8 == 0.
 *   global_scale: device pointer to S_global (NVFP4 and P1E8, required);
 *          ignored and may be NULL for MXFP4.
 *   Sizes of the outputs: fp4_packed_bytes / fp4_scale_bytes with the output
 *   row count and the blocked length.
 */
fp4_status fp4_quantize(fp4_format fmt, fp4_axis axis, const void* in_bf16, int64_t rows,
                        int64_t cols, int64_t ld, void* packed_out, void* scales_out,
                        const float* global_scale, fp4_stream_t stream);

/*
 * Reconstruction of a rowwise-quantized operand in BF16:
 *   out[r, i] = BF16_RNE(q[r, i] * S_block(r, i / k) * S_global)
 * ([NVFP4-Arch] "1. The Dual-Level Mathematical Formulation",
 * reconstruction x_hat), with S_global = 1 for MXFP4.  The product is exact
 * before the single rounding.  This is what a W4A16 path feeds a 16-bit GEMM;
 * the library's own GEMM never widens its operands.
 *   packed : device, [rows x k/2] (fp4_quantize's rowwise output)
 *   scales : device, its scale tiles
 *   global_scale : device S_global (NVFP4, P1E8: required; MXFP4: ignored)
 *   out_bf16 : device, [rows x k] BF16 with leading dimension ld (elements)
 * Requires k % (4 * block size) == 0, ld >= k, ld % 8 == 0, 16-byte aligned
 * packed and out_bf16.
 */
fp4_status fp4_dequantize(fp4_format fmt, const void* packed, const void* scales,
                          const float* global_scale, int64_t rows, int64_t k, void* out_bf16,
                          int64_t ld, fp4_stream_t stream);

/*
 * Rowwise quantization of several tensors in one launch (e.g. both GEMM
 * operands of a step), each exactly as fp4_quantize(fmt, FP4_ROWWISE, ...)
 * with its own sizes, buffers and S_global.  One launch covers the 128-row
 * tiles of up to 8 tensors (more are split into several launches), so small
 * tensors do not each pay a launch and a partial last wave.  Every
 * descriptor is validated before anything is launched; a failing one makes
 * the call return its status having launched nothing.
 *   n     : number of descriptors (>= 0)
 *   descs : host array of n descriptors
 */
typedef struct {
    const void* in_bf16;        /* device, rows x cols, leading dimension ld (elements) */
    int64_t rows, cols, ld;
    void* packed_out;           /* device, rows x cols/2 bytes */
    void* scales_out;           /* device, fp4_scale_bytes(fmt, rows, cols) bytes */
    const float* global_scale;  /* device S_global (NVFP4, P1E8: required); NULL for MXFP4 */
} fp4_quantize_desc;

fp4_status fp4_quantize_batch(fp4_format fmt, int n, const fp4_quantize_desc* descs,
                              fp4_stream_t stream);

/*
 * Dynamic NVFP4 quantization of a small tensor (e.g. the few rows of a decode
 * activation) in a single launch: S_global of the tensor (as
 * fp4_compute_global_scale), then the rowwise quantization with it (as
 * fp4_quantize), and optionally alpha = S_global * (*other_gs) (as
 * fp4_alpha_from_global_scales with the other operand's scale).  Results are
 * identical to those three calls.  One cluster of 16 CTAs (8 where the device
 * cannot place 16) holds the tensor in registers between the amax and the
 * quantization; a tensor above that capacity (32768 16-byte chunks, i.e.
 * 512 KiB of BF16, with 16 CTAs) is handled inside the same call by two
 * launches: S_global and alpha (as fp4_compute_global_scale_alpha), then the
 * rowwise quantizer, which visits the tensor's tiles last to first so that
 * the rows the first pass read last are still in L2.
 *   fmt      : FP4_NVFP4 only (MXFP4 needs no per-tensor scale: use
 *              fp4_quantize); else FP4_ERR_INVALID_ARG
 *   in_bf16  : device, rows x cols (ld), cols % 64 == 0, rows, cols > 0
 *   gs_out   : device float, S_global written here
 *   other_gs, alpha_out : device floats, both NULL or both set
 */
fp4_status fp4_quantize_dynamic(fp4_format fmt, const void* in_bf16, int64_t rows, int64_t cols,
                                int64_t ld, void* packed_out, void* scales_out, float* gs_out,
                                const float* other_gs, float* alpha_out, fp4_stream_t stream);

/* alpha = gsA * gsB (FP32), the factor that restores both per-tensor scales
 * after the block-scaled product (NVFP4).  All three are device pointers. */
fp4_status fp4_alpha_from_global_scales(const float* gsA, const float* gsB, float* alpha_out,
                                        fp4_stream_t stream);

/*
 * D = alpha * A_hat * B_hat^T with BF16 output, where A_hat[m,k] = q * S_block
 * of A's block and likewise for B.  The tensor core multiplies the E2M1 codes
 * of each block pair, scales the partial product by the two block scales and
 * accumulates in FP32 ([NVFP4-Arch] "2. Hardware-Managed Tensor Core
 * Dot-Products"; [MXFP4-BW] "Silicon Execution"); the operands are never
 * widened to 16 bits.  D = BF16_RNE(alpha * acc).
 *   A : packed [M x K/2], sA its scales (M rows, K/k blocks), from fp4_quantize
 *   B : packed [N x K/2], sB its scales (N rows)
 *   alpha : device pointer to one float, or NULL for 1.0
 *   D : BF16 [M x N], leading dimension ldd (elements, ldd >= N, ldd % 8 == 0)
 *   workspace / ws_bytes : scratch for the decode kernel's split-K partials
 *          (fp4_gemm_workspace_bytes); may be NULL / 0, then the prefill
 *          kernel runs for every M.  Its first 64 KB hold arrival counters
 *          that must be zero when a call starts: zero the whole workspace
 *          once after allocating it (cudaMemset); every call that completes
 *          leaves the counters zero again, for any later shape.  A call that
 *          finds a counter out of range records it and fp4_get_device_status
 *          returns FP4_ERR_WORKSPACE; after that, or after FP4_ERR_TIMEOUT,
 *          zero the workspace again.  Two calls that run at the same time
 *          need two workspaces.
 * Requires K % 64 == 0 (NVFP4, P1E8) or K % 128 == 0 (MXFP4) and N % 8 == 0.  M and
 * N tails are handled inside the kernels.  M == 0 or N == 0 is a no-op;
 * K == 0 writes zeros.
 *
 * The kernels are launched with programmatic stream serialization: one may
 * start its set-up while the previous kernel on the stream is still running,
 * and reads no operand, scale or alpha and writes no output before that
 * kernel has completed, so stream order is kept.
 */
fp4_status fp4_gemm(fp4_format fmt, const void* A, const void* sA, const void* B,
                    const void* sB, int64_t M, int64_t N, int64_t K, const float* alpha,
                    void* D, int64_t ldd, void* workspace, size_t ws_bytes,
                    fp4_stream_t stream);

/* Same as fp4_gemm with an explicit kernel choice (optionally OR-ed with
 * FP4_GEMM_B_STATIC; other bits: FP4_ERR_INVALID_ARG).  FP4_GEMM_DECODE needs
 * M <= 16, N <= 524288 and a workspace of fp4_gemm_workspace_bytes bytes
 * (else FP4_ERR_UNSUPPORTED_SHAPE / FP4_ERR_INVALID_ARG). */
fp4_status fp4_gemm_with_kernel(fp4_format fmt, const void* A, const void* sA, const void* B,
                                const void* sB, int64_t M, int64_t N, int64_t K,
                                const float* alpha, void* D, int64_t ldd, void* workspace,
                                size_t ws_bytes, fp4_gemm_kernel kernel, fp4_stream_t stream);

/*
 * Grouped GEMM: n independent problems D_i = alpha_i * A_i_hat * B_i_hat^T
 * (e.g. the experts of a mixture-of-experts layer, each with its own token
 * count M_i), each with the semantics and requirements of fp4_gemm, computed
 * by one persistent launch of the prefill kernel per 16 problems: the
 * 256 x 256 tiles of all problems form one list over the CTA pairs, so small
 * problems share the GPU instead of each paying a launch and a partial
 * wave.  Problems with M_i == 0 or N_i == 0 are skipped; K_i == 0 writes
 * zeros.  Every problem is validated before anything is launched.
 *   problems : host array of n descriptors (the pointers in them are device)
 */
typedef struct {
    const void* A;       /* packed [M x K/2] */
    const void* sA;      /* its scales */
    const void* B;       /* packed [N x K/2] */
    const void* sB;      /* its scales */
    int64_t M, N, K;
    const float* alpha;  /* device, or NULL for 1.0 */
    void* D;             /* BF16 [M x N], leading dimension ldd */
    int64_t ldd;
} fp4_gemm_problem;

fp4_status fp4_gemm_grouped(fp4_format fmt, int n, const fp4_gemm_problem* problems,
                            fp4_stream_t stream);

/* Workspace bytes the decode kernel needs for this shape on the current
 * device: 64 KB of counters plus the split-K partials (0 when the decode
 * kernel does not apply, i.e. M > 16 or N > 524288). */
size_t fp4_gemm_workspace_bytes(fp4_format fmt, int64_t M, int64_t N, int64_t K);

/*
 * Decode GEMM with the activation quantized inside the GEMM (NVFP4):
 *   S_global,A = amax|A| / 2688 (1 if zero)      -> *gsA_out
 *   alpha      = S_global,A * (*gsW)             -> *alpha_out
 *   D          = alpha * A_hat * W_hat^T (BF16)
 * where A_hat is the NVFP4 quantization of the BF16 activation A with
 * S_global,A (identical bytes to fp4_quantize_dynamic), formed block by
 * block in shared memory by the GEMM kernel itself as its K slices are
 * needed, never written to global memory.  Two launches: the one-launch
 * S_global/alpha kernel, then the decode GEMM, which streams its first
 * weight tiles while the first launch runs.  Every thread block quantizes
 * the activation slices its own K range needs, so for this path the BF16
 * activation (4x the bytes of its packed form) is read from L2 by every
 * block; fp4_quantize_dynamic followed by fp4_gemm is the faster decode
 * when the activation can go through global memory.  [NVFP4-Arch] "1. The
 * Dual-Level Mathematical Formulation" (per-tensor and block scales of an
 * activation quantized on the fly) and "2. Hardware-Managed Tensor Core
 * Dot-Products".
 *   act_bf16 : device, BF16 [M x K], leading dimension lda (elements)
 *   W, sW    : device, the packed NVFP4 weights [N x K/2] and their scales,
 *              quantized ahead of time with S_global *gsW; W, sW and gsW
 *              must not be written by a kernel still running on the stream
 *   D        : BF16 [M x N], leading dimension ldd
 *   gsA_out, alpha_out : device floats, written
 *   workspace / ws_bytes : as for fp4_gemm's decode kernel
 *              (fp4_gemm_workspace_bytes(FP4_NVFP4, M, N, K)), counters zero
 * Requires 1 <= M <= 16 (else FP4_ERR_UNSUPPORTED_SHAPE), K % 64 == 0,
 * N % 8 == 0, lda % 8 == 0; M == 0 or N == 0 is a no-op.
 */
fp4_status fp4_gemm_decode_dynamic(const void* act_bf16, int64_t lda, const void* W, const void* sW,
                                   const float* gsW, int64_t M, int64_t N, int64_t K, void* D,
                                   int64_t ldd, float* gsA_out, float* alpha_out, void* workspace,
                                   size_t ws_bytes, fp4_stream_t stream);

/*
 * Allocation-free form of the decode GEMM (no counterpart on the pages: it is
 * a service of this library, not part of the method).  Same operation,
 * arguments, result and kernels as fp4_gemm_with_kernel(..., FP4_GEMM_DECODE),
 * but the split-K partials live in a fixed 4 MiB array inside the library
 * instead of a caller-provided workspace, and the call makes no device
 * allocation of any kind.
 *
 * For callers that cannot call cudaMalloc on their hot path: plug-ins whose
 * host framework owns the device's memory through its own pool (an allocation
 * behind the pool's back escapes its accounting and fails once the pool has
 * reserved the memory), and latency-bound loops where cudaMalloc/cudaFree
 * would synchronize the device.
 *
 *  - Every GPU that loads the library holds the 4 MiB until the process exits.
 *  - The first call on a device looks up the array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.  The address is cached per device and
 *    context: after a cudaDeviceReset the next call looks it up again (and
 *    should, like the first, come before any capture).
 *  - All calls share the array.  It is zero when the library loads, and its
 *    counters (see fp4_gemm's workspace) are zero again after every call
 *    that completes; fp4_get_device_status zeroes them after reporting an
 *    error.  Calls that overlap on the GPU (e.g. on two streams at once) race
 *    on it: serialize them.
 *  - Shapes whose partials exceed 4 MiB (fp4_gemm_workspace_bytes) are
 *    rejected with FP4_ERR_UNSUPPORTED_SHAPE and an fp4_last_error() message;
 *    M > 16 is rejected the same way.  (N = 28672, K = 8192 needs 3.6 MB on
 *    148 SMs.)
 */
fp4_status fp4_gemm_decode_noalloc(fp4_format fmt, const void* A, const void* sA, const void* B,
                                   const void* sB, int64_t M, int64_t N, int64_t K,
                                   const float* alpha, void* D, int64_t ldd,
                                   fp4_stream_t stream);

/*
 * Synchronizes `stream`, then reports and clears the device error word of the
 * current device: FP4_ERR_TIMEOUT if a kernel of this library gave up on a
 * bounded wait since the last call (its outputs are then unspecified),
 * FP4_ERR_WORKSPACE if a decode call found its workspace counters not zero
 * (outputs unspecified), else FP4_OK; FP4_ERR_CUDA if the synchronization
 * itself failed.  After an error it also zeroes the counters of the static
 * scratch of fp4_gemm_decode_noalloc (a memset on `stream`, waited for):
 * every other stream that may hold an fp4_gemm_decode_noalloc call must be
 * idle when this is called, or that call's counters are cleared under it.
 */
fp4_status fp4_get_device_status(fp4_stream_t stream);

/*
 * Self-test of the failure path every kernel of this library uses: launches a
 * one-thread kernel that waits on a barrier nothing will ever complete.  The
 * bounded wait gives up after its time limit (2 s), records the timeout in
 * the device error word and returns, without trapping, so the context stays
 * usable.  After the stream reaches it, fp4_get_device_status reports
 * FP4_ERR_TIMEOUT (and clears the word).  Not part of the method on the
 * pages; a check of the library's fault handling.
 */
fp4_status fp4_selftest_bounded_wait(fp4_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FP4_H */
