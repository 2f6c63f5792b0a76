/*
 * qlora.h -- C ABI of libqlora: a frozen linear layer stored as blockwise NF4
 * with double quantization, dequantized on the fly to bf16 and contracted with
 * activations, plus the 16-bit LoRA branch, forward and backward, on one
 * sm_100a (B200) GPU.
 *
 * Method: QLoRA (Dettmers, Pagnoni, Holtzman, Zettlemoyer, arXiv:2305.14314),
 * as described on
 *   - automatone "QLoRA paper explained", section "How it works" (weights kept
 *     frozen in 4-bit, dequantized to bf16 on the fly for the forward and
 *     backward passes; gradients land only on the 16-bit LoRA adapters),
 *     paragraphs "4-bit NormalFloat (NF4)" (levels at standard-normal
 *     quantiles) and "Double Quantization (DQ)" (one scaling constant per
 *     block, the constants quantized again, about 0.37 bits per parameter
 *     saved);
 *   - creativeworksofknowledge "QLoRA: Fine-Tune 70B on One GPU", sections
 *     "1. NF4", "2. Double quantization" (constants FP32 -> FP8) and "Code"
 *     (quant type nf4, compute dtype bf16, double quant on, LoRA r / alpha,
 *     bias none);
 *   - aiwiki "QLoRA", section "Key Concepts and Technology" (one storage
 *     type NF4, one compute type bf16).
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, 16-byte
 *     aligned.  bf16 tensors are passed as uint16_t bit patterns, row-major.
 *   - The library never allocates device memory and never synchronizes the
 *     stream; every call is asynchronous on `stream` (NULL = legacy default
 *     stream).  Work buffers are supplied by the caller (sizes below).
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns an error status and launches nothing.  A CUDA
 *     launch failure returns QLORA_ERR_CUDA.
 *   - Inputs must be finite.  Non-finite weights give unspecified codes.
 *   - Thread safety: calls may be made concurrently on different streams;
 *     calls sharing a work buffer must be ordered by the caller.
 *   - Reproducibility: NF4 codes, E4M3 constants, c2, the mean and the
 *     dequantized weight are bit-exact and deterministic.  Y, X A^T, dA, dB
 *     and (with more than 16 tokens) dX are bit-reproducible from run to run
 *     on the same device: split contractions sum their partials in a fixed
 *     order.  The one exception is dX with 16 tokens or fewer, whose split-K
 *     partials are added with fp32 atomics and can differ in the last bits.
 */
#ifndef QLORA_H_
#define QLORA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define QLORA_EXPORT __attribute__((visibility("default")))
#else
#define QLORA_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* qlora_stream_t;   /* a cudaStream_t */

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_NULL = -1,         /* a required pointer is NULL */
  QLORA_ERR_SHAPE = -2,        /* a size is out of range or not a supported multiple */
  QLORA_ERR_ALIGN = -3,        /* a pointer is not 16-byte aligned */
  QLORA_ERR_UNSUPPORTED = -4,  /* block sizes, quant type, or no sm_100 device */
  QLORA_ERR_CUDA = -5,         /* a CUDA runtime / driver call failed */
  QLORA_ERR_WORKSPACE = -6     /* the work buffer is smaller than required */
} qlora_status;

/*
 * The 4-bit data type of a quantized weight (its 16 levels, ascending, in
 * [-1, 1]; qlora_get_levels returns them).  NF4 is the method's type
 * (automatone "QLoRA paper explained", paragraph "4-bit NormalFloat (NF4)");
 * INT4 and FP4 are the types that paragraph compares it with:
 *   QLORA_NF4   normal quantiles with an exact zero at index 7 (see
 *               qlora_get_codebook);
 *   QLORA_FP4   the E2M1 4-bit float values divided by 6: 15 distinct levels
 *               (+0 and -0 are one), index 7 is 0, the last entry repeats +1
 *               and is never chosen by the encoder;
 *   QLORA_INT4  16 evenly spaced levels (2i - 15) / 15 (no exact zero).
 */
typedef enum { QLORA_NF4 = 0, QLORA_FP4 = 1, QLORA_INT4 = 2 } qlora_quant_type;

/*
 * A quantized weight W [rows, cols] (rows = out features N, cols = in
 * features K).  Layout of the flattened row-major weight e = n*cols + k:
 *   codes      [ceil(rows*cols/2)] bytes; byte j holds element 2j in its high
 *              nibble and element 2j+1 in its low nibble; a ragged tail is
 *              padded with code 7; a block whose absmax is 0 is all code 7.
 * The block constants, one per 64 weights, are stored in one of two forms:
 *   with double quantization (blocksize2 = 256; creativeworksofknowledge
 *   "QLoRA: Fine-Tune 70B on One GPU", "2. Double quantization"):
 *     absmax_q   [ceil(rows*cols/64)] OCP E4M3 codes, one per 64-weight block.
 *     absmax_c2  [ceil(ceil(rows*cols/64)/256)] float, one per 256 blocks.
 *     absmax_mean[1] float, the mean of all block absmax values.
 *     Dequantized weight: c1' = fma(e4m3(q[b]), c2[b/256] / 448, mean);
 *                         w'  = bf16_RNE(L[code] * c1').
 *   without it (blocksize2 = 0, 0.5 bits of constants per weight):
 *     absmax     [ceil(rows*cols/64)] float, the block absmax c1 itself.
 *     Dequantized weight: w' = bf16_RNE(L[code] * c1).
 * Pointers of the form not in use are ignored (may be NULL).  All buffers are
 * caller-owned device memory.  A zero-initialised quant_type is NF4.
 */
typedef struct {
  uint8_t* codes;
  uint8_t* absmax_q;
  float* absmax_c2;
  float* absmax_mean;
  int64_t rows;
  int64_t cols;
  int32_t blocksize;    /* must be 64 */
  int32_t blocksize2;   /* 256: double quantization; 0: fp32 block constants */
  float* absmax;        /* blocksize2 == 0 only */
  int32_t quant_type;   /* a qlora_quant_type */
  int32_t reserved;     /* must be 0 */
} qlora_nf4_tensor;

/* Human-readable name of a status. Never NULL. */
QLORA_EXPORT const char* qlora_status_string(qlora_status s);

/*
 * The 16 NF4 levels (ascending; L[0] = -1, L[7] = 0, L[15] = 1): normal
 * quantiles, 8 positive at Phi^-1(1/2 + (d - 1/2) j / 8), j = 1..8, 7 negative
 * at -Phi^-1(1/2 + (d - 1/2) j / 7), j = 1..7, each divided by Phi^-1(d), with
 * d = 1 - (1/30 + 1/32) / 2 (automatone, "4-bit NormalFloat (NF4)").  Host only.
 */
QLORA_EXPORT void qlora_get_codebook(float out[16]);

/*
 * The 16 levels of a 4-bit type (see qlora_quant_type).  Host only.
 * Errors: QLORA_ERR_NULL, QLORA_ERR_UNSUPPORTED (unknown type).
 */
QLORA_EXPORT qlora_status qlora_get_levels(int32_t quant_type, float out[16]);

/*
 * Byte sizes of the buffers of a quantized [rows, cols] weight and of the
 * work buffer qlora_quantize_nf4_dq needs.  Any output pointer may be NULL.
 * With blocksize2 = 0 (no double quantization) absmax_q_bytes receives the
 * size of the fp32 `absmax` array and absmax_c2_bytes 0.
 * Errors: QLORA_ERR_SHAPE (rows or cols < 0), QLORA_ERR_UNSUPPORTED (block sizes).
 */
QLORA_EXPORT qlora_status qlora_nf4_sizes(int64_t rows, int64_t cols, int32_t blocksize, int32_t blocksize2,
                             size_t* codes_bytes, size_t* absmax_q_bytes, size_t* absmax_c2_bytes,
                             size_t* workspace_bytes);

/*
 * Blockwise absmax encode of a bf16 weight with the levels of
 * out->quant_type, then double quantization of the block constants
 * (automatone, "4-bit NormalFloat (NF4)" and "Double Quantization (DQ)";
 * creativeworksofknowledge, "2. Double quantization"):
 *   per 64 weights: c1 = max|x|, n = x / c1 (IEEE), code = nearest level
 *   (ties to the lower index); per tensor: mean = float(sum(c1) / count)
 *   with the sum in double; per 256 constants: c2 = max|c1 - mean|,
 *   q = E4M3_RNE(float((c1 - mean) / c2) * 448), q = 0 when c2 == 0.
 * With out->blocksize2 == 0 the constants c1 are written to out->absmax as
 * they are (no double quantization).
 * W: [out->rows * out->cols] bf16.  out: the destination buffers and shape.
 * workspace: >= workspace_bytes of qlora_nf4_sizes.
 * A zero-sized weight is a no-op.
 */
QLORA_EXPORT qlora_status qlora_quantize_nf4_dq(const uint16_t* W, const qlora_nf4_tensor* out, void* workspace,
                                   size_t workspace_bytes, qlora_stream_t stream);

/*
 * Dequantization to bf16 (automatone "How it works": dequantize to the
 * BFloat16 compute type): two-level with double quantization, one fp32
 * constant per block without it (see qlora_nf4_tensor).  W_out: [rows * cols] bf16.
 */
QLORA_EXPORT qlora_status qlora_dequantize(const qlora_nf4_tensor* W, uint16_t* W_out, qlora_stream_t stream);

/*
 * Work-buffer sizes of qlora_linear_fwd / qlora_linear_bwd for a weight of
 * shape [rows, cols], M token rows and LoRA rank r.  A work buffer is
 * caller-owned device scratch: it needs no initialisation (each call clears or
 * overwrites what it uses on its own stream), and two calls that may run at
 * the same time must not share one.
 */
QLORA_EXPORT qlora_status qlora_linear_workspace_size(int64_t rows, int64_t cols, int64_t M, int32_t r,
                                         size_t* fwd_bytes, size_t* bwd_bytes);

/*
 * Forward of the frozen NF4 linear layer with LoRA (automatone "How it works";
 * creativeworksofknowledge "Code": bias none, LoRA scale s = alpha / r):
 *   Y = X deq(W)^T + s (X A^T) B^T
 * X [M, cols] bf16, A [r, cols] bf16, B [rows, r] bf16, Y [M, rows] bf16 out.
 * XA_out [M, r] float receives X A^T (unscaled, fp32) when non-NULL; the
 * backward pass takes it back.
 * Requirements: cols % 64 == 0, rows % 8 == 0, r % 8 == 0, 8 <= r <= 256, M >= 1.
 * M <= 16 takes the decode-shaped path; larger M the prefill-shaped one.
 */
QLORA_EXPORT qlora_status qlora_linear_fwd(const qlora_nf4_tensor* W, const uint16_t* X, int64_t M,
                              const uint16_t* A, const uint16_t* B, int32_t r, float s, uint16_t* Y,
                              float* XA_out, void* workspace, size_t workspace_bytes,
                              qlora_stream_t stream);

/*
 * Decode-shaped forward with a LoRA adapter per token: several adapters served
 * over one frozen 4-bit weight in one pass over it (automatone "QLoRA paper
 * explained", "Results": the 4-bit base is also the deployed model).  Token t
 * uses adapter a = adapter_idx[t]:
 *   Y[t] = X[t] deq(W)^T + s (X[t] A_a^T) B_a^T,   XA_out[t] = X[t] A_a^T
 * A_stack [n_adapters][r, cols] bf16 and B_stack [n_adapters][rows, r] bf16,
 * each adapter contiguous; adapter_idx: device int32 [M], 4-byte aligned.  A
 * negative index means "no adapter" (the base weight alone, XA_out row 0).
 * An index >= n_adapters is treated the same way and sets bit 3 of the device
 * error flag (qlora_read_device_errors): it cannot be checked on the host.
 * The weight is read once whatever the number of adapters; every adapter in
 * use adds one rank-r up-projection per output tile.
 * Requirements as qlora_linear_fwd, and 1 <= M <= 16, n_adapters >= 1; the
 * work buffer is qlora_linear_workspace_size's fwd_bytes for the same M.
 */
QLORA_EXPORT qlora_status qlora_linear_fwd_multi(const qlora_nf4_tensor* W, const uint16_t* X, int64_t M,
                                    const uint16_t* A_stack, const uint16_t* B_stack, int32_t n_adapters,
                                    const int32_t* adapter_idx, int32_t r, float s, uint16_t* Y,
                                    float* XA_out, void* workspace, size_t workspace_bytes,
                                    qlora_stream_t stream);

/*
 * Backward of the same layer; W is frozen and gets no gradient (automatone
 * "How it works": gradients land only on the LoRA adapters; gptget Deep
 * Analysis: backward dequantizes to 16-bit for the matmul):
 *   G  = dY B                      [M, r]
 *   dX = dY deq(W) + s G A          [M, cols] bf16   (skipped when dX is NULL)
 *   dB = s dY^T (X A^T)             [rows, r] float
 *   dA = s G^T X                    [r, cols] float
 * The LoRA gradients are written in fp32 (the optimizer's input); X, dY, A, B
 * are bf16.  XA: X A^T (fp32 [M, r]) as returned by the forward, or NULL to
 * recompute it from X and A.
 * Same shape requirements as the forward.
 */
QLORA_EXPORT qlora_status qlora_linear_bwd(const qlora_nf4_tensor* W, const uint16_t* X, const uint16_t* dY,
                              int64_t M, const uint16_t* A, const uint16_t* B, int32_t r, float s,
                              const float* XA, uint16_t* dX, float* dA, float* dB,
                              void* workspace, size_t workspace_bytes, qlora_stream_t stream);

/*
 * Device error flag of the calling thread's current device: bit 0 is set when
 * a kernel's internal wait gave up after its time limit (a bug, reported
 * instead of hanging); bit 2 when a kernel's shared-memory window did not fit
 * its fixed map; bit 3 when a per-token adapter index was out of range
 * (qlora_linear_fwd_multi).  Reading synchronizes the device; clear = 1
 * resets it.
 */
QLORA_EXPORT qlora_status qlora_read_device_errors(uint32_t* flags, int clear);

/*
 * Largest weight (rows * cols) qlora_quantize_nf4_dq_noalloc accepts.
 */
#define QLORA_NOALLOC_MAX_ELEMENTS 134217728LL   /* 2^27, e.g. 8192 x 16384 */

/*
 * qlora_quantize_nf4_dq without a work buffer and without any allocation.
 * The pages have no counterpart to this entry point; it exists for callers
 * that cannot obtain device memory when they quantize: a server that reserves
 * all of its memory at start-up and forbids allocation afterwards, code that
 * runs inside another framework's allocator or out-of-memory path, or a loader
 * with no allocator handle.  Its scratch (one float per 64 weights plus 2048
 * partial sums, 8 MiB + 16 KiB) is a fixed array inside the library that
 * every GPU loading the library holds until the process exits.
 *   - Same arguments and results as qlora_quantize_nf4_dq, bit for bit.
 *   - Validation as for qlora_quantize_nf4_dq, in the same order; where that
 *     entry point checks its work buffer's size, this one checks rows * cols
 *     against QLORA_NOALLOC_MAX_ELEMENTS (QLORA_ERR_WORKSPACE above it, with
 *     nothing launched).
 *   - The first call on a device (with that device current) looks up the
 *     array's device address; make that first call before any stream capture.
 *   - All calls share the one array: calls that can overlap on the GPU (other
 *     streams, other host threads) race on it and must be ordered by the
 *     caller.  No part of the array needs clearing between calls.
 *   - Calls no cudaMalloc / cudaFree or other allocating routine.
 */
QLORA_EXPORT qlora_status qlora_quantize_nf4_dq_noalloc(const uint16_t* W, const qlora_nf4_tensor* out,
                                                     qlora_stream_t stream);

/*
 * Self-test of the failure path (no counterpart on the pages): launches one
 * CTA that waits on an mbarrier nothing arrives on, with the library's bounded
 * wait and a limit of `limit_cycles` SM cycles (0 .. 1e8) instead of the
 * pipelines' two seconds.  No copy or MMA is in flight, so the wait gives up:
 * the kernel sets bit 0 (wait timed out) of the device error flag that
 * qlora_read_device_errors reads, writes 1 to *outcome (2 if the wait had
 * completed; outcome may be NULL, else a 4-byte aligned device pointer) and
 * returns, leaving the context usable.
 * Errors: QLORA_ERR_SHAPE (limit out of range), QLORA_ERR_ALIGN.
 */
QLORA_EXPORT qlora_status qlora_selftest_bounded_wait(int64_t limit_cycles, uint32_t* outcome,
                                                     qlora_stream_t stream);

/*
 * Number of kernels this library has launched in the process so far (all
 * devices).  Host only; used to count launches inside a timed region.
 */
QLORA_EXPORT uint64_t qlora_kernel_launches(void);

/*
 * Measurement hook: when both are non-NULL cudaEvent_t handles, the next fused
 * dequant-GEMM launch made by the calling thread (inside qlora_linear_fwd or
 * qlora_linear_bwd) is bracketed by cudaEventRecord(start) / (stop) on its
 * stream; the hook then clears itself.  Pass NULL, NULL to cancel.
 */
QLORA_EXPORT qlora_status qlora_time_next_gemm(void* start_event, void* stop_event);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_H_ */
