/*
 * qlora_nf4.h -- C ABI of libqlora_nf4.so: blockwise NF4 quantisation, double
 * quantisation and the QLoRA linear layer (forward, input/adapter backward)
 * on NVIDIA B200 (sm_100a).
 *
 * Method sources (web pages, cited by title and section):
 *   [QE]  "QLoRA Explained: A 4-Bit Base, NF4, and What It Really Costs"
 *         (skillsuites.com)
 *   [LQ]  "LoRA vs QLoRA: Efficient Fine-Tuning Explained" (masterainow.com)
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller.  The
 *    library allocates nothing: scratch space is a caller-provided workspace
 *    whose size comes from qlora_workspace_bytes().
 *  - Work is enqueued asynchronously on `stream` (NULL = legacy default
 *    stream).  Returning QLORA_OK means "validated and enqueued".
 *  - Arguments are validated synchronously before anything is enqueued; on a
 *    validation error nothing is launched and the status is returned.
 *  - Errors detected on the device (a non-finite weight, a bounded wait that
 *    ran out) set a sticky per-device status word; qlora_check_status()
 *    synchronises the stream, returns that word and clears it.
 *  - Matrices are row-major with dense rows.  bf16 is IEEE bfloat16 passed
 *    as 16-bit storage (uint16_t / torch.bfloat16).
 *  - Every device pointer must be 16-byte aligned.
 *  - There is no CPU fallback: without a usable sm_100 device every compute
 *    entry point returns QLORA_ERR_CUDA or QLORA_ERR_UNSUPPORTED.
 *  - Per-device state (the status word's address, kernel attributes) is set
 *    up on first use of each device and kept for the life of the process:
 *    the library must not be used across cudaDeviceReset.
 */
#ifndef QLORA_NF4_H
#define QLORA_NF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream. */
typedef struct CUstream_st* qlora_stream_t;

typedef enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = 1,   /* null pointer, bad enum, bad rank/alpha      */
  QLORA_ERR_SHAPE = 2,         /* a dimension violates a stated constraint    */
  QLORA_ERR_ALIGN = 3,         /* a pointer is not 16-byte aligned            */
  QLORA_ERR_NONFINITE = 4,     /* device: NaN/Inf weight met while quantising */
  QLORA_ERR_TIMEOUT = 5,       /* device: a bounded pipeline wait gave up     */
  QLORA_ERR_CUDA = 6,          /* a CUDA runtime/driver call failed           */
  QLORA_ERR_UNSUPPORTED = 7,   /* no sm_100 device, or a mode not built       */
  QLORA_ERR_WORKSPACE = 8      /* workspace null or smaller than required     */
} qlora_status;

typedef enum { QLORA_F32 = 0, QLORA_BF16 = 1 } qlora_dtype;

/* 4-bit data types ([QE] config walk-through: bnb_4bit_quant_type picks the
 * table; "the library's other 4-bit option is a small floating-point layout
 * ... it costs exactly the same memory").
 *   QLORA_QUANT_NF4: the 16 normal quantiles of [QE] "That is NF4"; code =
 *     rank of the value (0 = -1, 7 = exact 0, 15 = +1).
 *   QLORA_QUANT_FP4: a 4-bit float, sign bit 3, 2 exponent bits, 1 mantissa
 *     bit, no infinities or NaNs: code c holds
 *     (-1)^(c>>3) * {0, 0.5, 1, 1.5, 2, 3, 4, 6}[c & 7] / 6, so that the
 *     largest magnitude meets the block absmax.  Code 8 (-0) decodes to -0
 *     and is never produced by quantisation. */
typedef enum { QLORA_QUANT_NF4 = 0, QLORA_QUANT_FP4 = 1 } qlora_quant_type;

/* Formats of the 8-bit block-scale codes (nf4_weight.double_quant):
 *   QLORA_DQ_INT8: symmetric int8, c = round-half-even(RN32(RN32(d / s_g) * 127))
 *   QLORA_DQ_FP8:  the E4M3 8-bit float (sign, 4 exponent bits with bias 7,
 *                  3 mantissa bits), c = E4M3(256 * RN32(d / s_g)) rounded to
 *                  nearest with ties to the even code (the sign of a zero
 *                  result is kept); decoded exactly as e4m3(c) / 256. */
typedef enum { QLORA_DQ_NONE = 0, QLORA_DQ_INT8 = 1, QLORA_DQ_FP8 = 2 } qlora_dq_type;

/* Bytes of the double-quantisation exponent histogram: 256 int64 bins; bin e
 * holds the sum of the 24-bit significands of the absmax values whose fp32
 * exponent field is e (bin 255 unused).  Histograms of disjoint parts of a
 * tensor add up (integer sum) to the whole tensor's histogram. */
#define QLORA_DQ_HIST_BYTES 2048

/* Operation ids for qlora_workspace_bytes(). */
typedef enum {
  QLORA_OP_DOUBLE_QUANT = 0,
  QLORA_OP_FWD = 1,
  QLORA_OP_BWD = 2,
  QLORA_OP_FWD_DROPOUT = 3,
  QLORA_OP_BWD_DROPOUT = 4
} qlora_op;

/* LoRA dropout on the adapter's input ([QE] config walk-through:
 * lora_dropout=0.05).  Element e = m * K + k of X is kept with probability
 * 1 - p: Philox4x64-10 (Salmon et al., "Parallel Random Numbers: As Easy as
 * 1, 2, 3", SC 2011) with key (seed, 0) and counter (e / 8, 0, 0, 0); word
 * (e % 8) / 2 of the block, bits 40..63 (e even) or 16..39 (e odd), as a
 * 24-bit uniform u; kept when u >= floor(p * 2^24 + 1/2).  Kept inputs are
 * RNbf16(RN32(x * c)) with c = RN32(1 / RN32(1 - p)); the same mask is
 * regenerated in the backward.  p in [0, 1); p = 0 is the plain layer. */
typedef struct {
  float p;
  uint32_t reserved;      /* 0 */
  uint64_t seed;
} qlora_dropout;

/*
 * A quantised frozen weight W[rows, cols] (rows = N output features,
 * cols = K input features).  [QE] "Why the groups are small": one scale per
 * block of 64 consecutive weights of the row-major flattening (cols % 64 == 0,
 * so blocks never straddle rows).  [QE] "Shrink the scale factors too": with
 * double quantisation the block scales are int8 in groups of 256 with one
 * fp32 scale per group, plus one fp32 mean offset per tensor.
 *
 *   packed   [rows*cols/2]  two codes per byte, element 2j in the HIGH nibble
 *   absmax   [rows*cols/64] fp32 block scales      (used when double_quant == 0)
 *   qabsmax  [rows*cols/64] int8 block-scale codes in [-127, 127], as
 *            nf4_double_quantize writes them (used when double_quant == 1;
 *            -128 is outside the format)
 *   dq_scale [ceil(rows*cols/64/256)] fp32 group scales (double_quant == 1)
 *   dq_mean  [1] fp32 per-tensor mean offset, device     (double_quant == 1)
 *
 * Dequantised value of element i in block b (code c, table q of quant_type):
 *   a^ = absmax[b]                                              (no DQ)
 *   a^ = RN32(RN32(v(qabsmax[b]) * dq_scale[b/256]) + dq_mean)  (DQ)
 *   v(c) = RN32(c / 127) for int8 codes (double_quant 1), e4m3(c) / 256 for
 *   8-bit float codes (double_quant 2; c is the E4M3 byte)
 *   w' = RNbf16(RN32(q[c] * a^))
 * quant_type is QLORA_QUANT_NF4 (0) or QLORA_QUANT_FP4 (1); a zero-filled
 * struct is NF4.
 */
typedef struct {
  const uint8_t* packed;
  int64_t rows;
  int64_t cols;
  int32_t blocksize;      /* must be 64  */
  int32_t double_quant;   /* 0: none, 1 (QLORA_DQ_INT8) or 2 (QLORA_DQ_FP8) */
  const float* absmax;
  const int8_t* qabsmax;
  const float* dq_scale;
  const float* dq_mean;
  int32_t dq_blocksize;   /* must be 256 */
  int32_t quant_type;     /* QLORA_QUANT_NF4 or QLORA_QUANT_FP4 */
} nf4_weight;

/* ---- host-only queries (no GPU needed) -------------------------------- */

/* The library's 16-entry NF4 table and its 15 decision thresholds, computed
 * on the host at load time ([QE] "Put the rows where the weights are",
 * "That is NF4": normal quantiles normalised to [-1, 1], exact zero; ties
 * between two rows go to the higher row, [QE] "The two failures ...").
 * Writes 16 (resp. 15) floats.  Returns QLORA_OK or QLORA_ERR_INVALID_ARG. */
int nf4_code_table(float* table16);
int nf4_code_thresholds(float* thresholds15);

/* The same for either 4-bit type: table16 receives the value of each code;
 * thresholds15 the decision thresholds between consecutive distinct values,
 * ascending (15 for NF4, 14 for FP4), and *count their number.  Returns
 * QLORA_OK or QLORA_ERR_INVALID_ARG. */
int qlora_code_table(int quant_type, float* table16);
int qlora_code_thresholds(int quant_type, float* thresholds15, int* count);

/* The double-quantisation mean from a complete exponent histogram over
 * n_total absmax values (QLORA_DQ_HIST_BYTES of int64, host memory): the
 * same exact rounding as the device, RN32(RN64(exact sum) / n_total), on
 * the host -- for a caller that gathers shard histograms on the host.
 * Returns QLORA_OK or QLORA_ERR_INVALID_ARG (null, n_total < 1, a negative
 * bin). */
int qlora_dq_mean_from_hist(const int64_t* hist, int64_t n_total, float* mean);

/* Bytes of caller workspace needed by an operation (0 if none).
 *   QLORA_OP_DOUBLE_QUANT: M, K, r ignored; N = number of absmax values.
 *   QLORA_OP_FWD / QLORA_OP_BWD: layer with M tokens, weight N x K, rank r. */
size_t qlora_workspace_bytes(int op, int64_t M, int64_t N, int64_t K, int r);

/* Human-readable name of a status code (static string). */
const char* qlora_status_string(int status);

/* ABI version of this header (major*100 + minor). */
int qlora_abi_version(void);

/* Number of kernels this library has launched in this process (all devices);
 * a measurement aid: the difference across a region counts its launches. */
uint64_t qlora_kernel_launches(void);

/* Measurement aid.  Registers two CUDA events (cudaEvent_t, created by the
 * caller).  The next tensor-core GEMM launch of qlora_linear_fwd or
 * qlora_linear_bwd records `start` on its stream immediately before the GEMM
 * kernel and `stop` immediately after it, then the registration is cleared.
 * Passing NULL for both clears a pending registration.  Host-only, per
 * process; returns QLORA_OK or QLORA_ERR_INVALID_ARG (exactly one NULL). */
int qlora_profile_gemm_events(void* start, void* stop);

/* ---- device entry points ---------------------------------------------- */

/*
 * Blockwise NF4 quantisation ([QE] "The table, and the number that stretches
 * it", steps 1-3; "Why the groups are small").
 *   W       device [rows, cols], fp32 or bf16 (dtype)
 *   packed  device out [rows*cols/2]
 *   absmax  device out [rows*cols/64] fp32
 * Per block: a = max|w| (exact); x = RN32(w / a) (IEEE division); code =
 * index of the nearest table row, ties to the higher row; a zero block gives
 * code 7 (the exact zero) everywhere.  Constraints: rows >= 1, cols >= 64,
 * cols % 64 == 0, blocksize == 64.  A NaN/Inf weight sets
 * QLORA_ERR_NONFINITE in the device status word (outputs then undefined).
 */
int nf4_quantize(const void* W, int dtype, int64_t rows, int64_t cols,
                 int blocksize, uint8_t* packed, float* absmax,
                 qlora_stream_t stream);

/*
 * Blockwise quantisation to either 4-bit type, optionally building the
 * double-quantisation histogram in the same pass ([QE] "The table, and the
 * number that stretches it"; "Shrink the scale factors too").  Same as
 * nf4_quantize with the table of quant_type; ties between two rows go to the
 * higher value.
 *   dq_hist  NULL, or device [256] int64 (QLORA_DQ_HIST_BYTES): zeroed by the
 *            call, then filled with the exponent histogram of this call's
 *            absmax values (input of nf4_double_quantize_hist).
 * A shard of a larger weight (a range of whole rows) is quantised the same
 * way; the shards' histograms summed (for instance by an all-reduce) give
 * the whole weight's histogram.
 */
int qlora_quantize_4bit(const void* W, int dtype, int64_t rows, int64_t cols, int blocksize,
                        int quant_type, uint8_t* packed, float* absmax, int64_t* dq_hist,
                        qlora_stream_t stream);

/*
 * Double quantisation of the block scales ([QE] "Shrink the scale factors
 * too").  mean = RN32(RN64(exact sum of absmax) / n) (one per tensor);
 * d = RN32(a - mean); s_g = max|d| over each group of 256 (the last group may
 * be partial); c = round-half-even(RN32(RN32(d / s_g) * 127)), 0 if s_g == 0.
 *   absmax   device [n_absmax] fp32, finite and >= 0
 *   qabsmax  device out [n_absmax] int8
 *   dq_scale device out [ceil(n_absmax/256)] fp32
 *   dq_mean  device out [1] fp32
 *   ws       device workspace of qlora_workspace_bytes(QLORA_OP_DOUBLE_QUANT, ..)
 * The mean is bit-identical for any launch order (exact integer sum: an
 * exponent histogram of the significands, written to ws, then the exact
 * total rounded once).  A negative, NaN or Inf absmax sets
 * QLORA_ERR_NONFINITE in the device status word.
 */
int nf4_double_quantize(const float* absmax, int64_t n_absmax, int dq_blocksize,
                        int8_t* qabsmax, float* dq_scale, float* dq_mean,
                        void* ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * The second pass of double quantisation on its own: the mean from a
 * complete exponent histogram over n_total absmax values (dq_hist from
 * qlora_quantize_4bit, summed over shards when the weight is sharded), then
 * the int8 codes and group scales of this array's n_absmax values.  When
 * sharding, every shard but the last must hold a multiple of 256 absmax
 * values so that the groups of 256 do not straddle shards; the results then
 * equal nf4_double_quantize of the whole absmax array bit for bit.
 *   dq_hist  device [256] int64, read only; n_total >= n_absmax >= 1.
 */
int nf4_double_quantize_hist(const float* absmax, int64_t n_absmax, const int64_t* dq_hist,
                             int64_t n_total, int dq_blocksize, int8_t* qabsmax,
                             float* dq_scale, float* dq_mean, qlora_stream_t stream);

/* The same with the code format chosen: dq_type QLORA_DQ_INT8 (as above) or
 * QLORA_DQ_FP8 (see qlora_dq_type); the weight's double_quant field must
 * then name the same format. */
int qlora_double_quantize_hist(const float* absmax, int64_t n_absmax, const int64_t* dq_hist,
                               int64_t n_total, int dq_blocksize, int dq_type, int8_t* qabsmax,
                               float* dq_scale, float* dq_mean, qlora_stream_t stream);

/*
 * Dequantise to bf16 ([QE] worked example step 4; "That is NF4": every
 * matmul runs on values expanded back to bf16).
 *   W_out device out [rows, cols] bf16,  w' = RNbf16(RN32(q[code] * a^)).
 */
int nf4_dequantize(const nf4_weight* w, void* W_out, qlora_stream_t stream);

/*
 * Merge the trained adapter into the base weight for export ([QE] "Why a
 * 16-bit adapter will not fold into a 4-bit base": expand the base to 16
 * bits first, then add; [LQ] "How LoRA Works": W' = W + (alpha/r) B A):
 *   W_out[n, k] = RNbf16(RN32(w'[n, k] + RN32(s * sum_j B[n, j] A[j, k])))
 *   w' = RNbf16(RN32(q[c] * a^)) (the nf4_dequantize values), s = alpha / r,
 *   the sum over j accumulated in fp32 on tensor cores.
 *   A device [r, K] bf16, B device [N, r] bf16, W_out device out [N, K] bf16.
 * Constraints: r in {8,16,32,64,128}, alpha finite; one pass over the codes
 * and one write of W_out.
 */
int qlora_merge(const nf4_weight* w, const void* A, const void* B, int r, float alpha,
                void* W_out, qlora_stream_t stream);

/*
 * QLoRA linear forward ([LQ] "How LoRA Works": W' = W + (alpha/r) B A;
 * [QE] "Why the expansion cannot be skipped": codes -> table -> scale ->
 * bf16 on chip -> tensor core):
 *   Y = X deq(W)^T + s (X A^T) B^T,   s = alpha / r,  fp32 accumulation.
 *   X  device [M, K] bf16      A device [r, K] bf16    B device [N, r] bf16
 *   Y  device out [M, N] bf16
 *   T_save device out [M, r] bf16 = RNbf16(X A^T), or NULL
 *   ws device workspace of qlora_workspace_bytes(QLORA_OP_FWD, M, N, K, r)
 * Constraints: M >= 1, N % 8 == 0, K % 64 == 0, r in {8,16,32,64,128},
 * alpha finite.  M <= 16 runs the decode (GEMV) kernel, larger M the fused
 * dequantise-in-mainloop tensor-core GEMM (on pairs of SMs when N > 128).  The decode kernel applies each
 * block's scale to that block's fp32 partial product (the table rounded to
 * bf16 rather than each scaled weight); the GEMM uses the bf16 weights of
 * nf4_dequantize exactly.  Both are within the layer's tolerance.
 */
int qlora_linear_fwd(const nf4_weight* w, const void* X, int64_t M,
                     const void* A, const void* B, int r, float alpha,
                     void* Y, void* T_save, void* ws, size_t ws_bytes,
                     qlora_stream_t stream);

/*
 * QLoRA linear backward ([LQ] "How QLoRA Works": the frozen base gets no
 * gradient; only the adapters do).  With U = dY B:
 *   dX = dY deq(W) + s U A      [M, K] bf16
 *   dA = s U^T X                [r, K] bf16
 *   dB = s dY^T (X A^T)         [N, r] bf16
 *   T  device [M, r] bf16 = X A^T saved by the forward, or NULL to recompute
 * Same constraints as the forward; reductions over M are fixed-order
 * (deterministic).
 */
int qlora_linear_bwd(const nf4_weight* w, const void* X, const void* dY,
                     int64_t M, const void* A, const void* B, int r,
                     float alpha, const void* T, void* dX, void* dA, void* dB,
                     void* ws, size_t ws_bytes, qlora_stream_t stream);

/*
 * The layer with LoRA dropout on the adapter's input (see qlora_dropout):
 *   Y  = X deq(W)^T + s (X' A^T) B^T,   X' = dropout(X)
 *   T_save = RNbf16(X' A^T)
 *   dX = dY deq(W) + D * c * (s U A),  dA = s U^T X',  dB = s dY^T T
 * with D the keep mask and c its scale.  Same arguments and constraints as
 * qlora_linear_fwd / qlora_linear_bwd plus `dropout` (not null; p outside
 * [0, 1) is QLORA_ERR_INVALID_ARG); workspaces from
 * qlora_workspace_bytes(QLORA_OP_FWD_DROPOUT / QLORA_OP_BWD_DROPOUT, ...).
 * Every token count runs the tensor-core GEMM (the decode kernel reads X once
 * for base and adapter alike).  The backward's dX is the GEMM of dY deq(W)
 * followed by a rank-r pass that adds the masked adapter term in place.
 */
int qlora_linear_fwd_dropout(const nf4_weight* w, const void* X, int64_t M,
                             const void* A, const void* B, int r, float alpha,
                             const qlora_dropout* dropout, void* Y, void* T_save,
                             void* ws, size_t ws_bytes, qlora_stream_t stream);
int qlora_linear_bwd_dropout(const nf4_weight* w, const void* X, const void* dY,
                             int64_t M, const void* A, const void* B, int r,
                             float alpha, const qlora_dropout* dropout, const void* T,
                             void* dX, void* dA, void* dB, void* ws, size_t ws_bytes,
                             qlora_stream_t stream);

/*
 * Forward without a workspace argument, for callers that cannot allocate
 * device memory: a plugin inside a host program that owns all device
 * allocations, code running during CUDA stream capture (where cudaMalloc is
 * not allowed), or a loop that forbids allocation after start-up.  The pages
 * have no counterpart to this entry point; it only changes where the scratch
 * lives.
 *
 * Same arguments, constraints, results and errors as qlora_linear_fwd, minus
 * ws / ws_bytes; the argument checks run first and in the same order.
 * Scratch is a fixed array of QLORA_FWD_NOALLOC_SCRATCH_BYTES compiled into
 * the library; every GPU that loads the library holds it until the process
 * exits.  A call whose qlora_workspace_bytes(QLORA_OP_FWD, M, N, K, r) exceeds
 * that size returns QLORA_ERR_WORKSPACE before anything is enqueued.  That
 * size depends on M, N, K and r together and is not monotonic in M (the
 * split-contraction partial sums of X A^T vanish once M alone fills the GPU;
 * the decode path's partials grow with N), so no single token limit exists:
 * check qlora_workspace_bytes(QLORA_OP_FWD, M, N, K, r) <=
 * QLORA_FWD_NOALLOC_SCRATCH_BYTES before relying on this entry point.  For
 * reference, 8192 tokens at K = 3584, r = 64 need about 11 MiB; with
 * N = K = 4096 and r = 128 the token counts 18,725-18,816 and 26,215-37,760
 * are refused while 18,817-26,214 and 37,761 and more are accepted.
 *   - The first call on each device resolves the array's device address
 *     (cudaGetSymbolAddress) with that device current and keeps it for the
 *     life of the process; make that first call before any stream capture,
 *     and do not use the library across cudaDeviceReset (the kept address,
 *     like the device status word's, belongs to the context it came from).
 *   - No call allocates or frees memory (no cudaMalloc, cudaFree or
 *     allocating library routine).
 *   - All calls share the array: calls whose work overlaps on the GPU (other
 *     streams, other host threads, the same device) race and corrupt each
 *     other's results; order them on one stream or synchronise between them.
 *   - Each call writes every scratch byte it reads, so nothing carries over
 *     from the previous call.
 */
#define QLORA_FWD_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int qlora_linear_fwd_noalloc(const nf4_weight* w, const void* X, int64_t M,
                             const void* A, const void* B, int r, float alpha,
                             void* Y, void* T_save, qlora_stream_t stream);

/*
 * Synchronise `stream`, return the sticky device status word (QLORA_OK if
 * no device-side error was recorded since the last call) and clear it.
 */
int qlora_check_status(qlora_stream_t stream);

/*
 * Failure detection.  Every pipeline wait in the library's kernels (on a
 * TMA stage, a tensor-core commit, the partner SM of a pair) gives up after
 * a wall-time limit: the kernel records QLORA_ERR_TIMEOUT in the status
 * word, lets the copies it issued land (bounded too), releases its tensor
 * memory and returns, so the context stays usable.
 *   qlora_set_wait_limit: the limit for the current device, in ns (0 = the
 *     default 1 s; otherwise 1 ms .. 60 s, else QLORA_ERR_INVALID_ARG).
 *     Synchronous; do not change it while the library's kernels run.
 *   qlora_test_withhold_first_fill: a test switch (default off).  While on,
 *     the decode kernel's first CTA leaves its first pipeline stage
 *     unfilled, so that its waits run out and the call reports
 *     QLORA_ERR_TIMEOUT -- a wait that nothing satisfies, with no fault.
 * Both return QLORA_OK or QLORA_ERR_CUDA / QLORA_ERR_UNSUPPORTED.
 */
int qlora_set_wait_limit(uint64_t ns);
int qlora_test_withhold_first_fill(int on);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif /* QLORA_NF4_H */
