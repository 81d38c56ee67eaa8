/*
 * qlora_nf4.h -- C ABI of the B200 (sm_100a) QLoRA NF4 library.
 *
 * The library implements the hot path of QLoRA for one linear layer:
 *
 *   * the blockwise NF4 quantizer with double quantization that turns a frozen
 *     fp32 weight W0 into 4-bit codes plus 8-bit second-level scale codes;
 *   * dequantization of that format to bf16;
 *   * the QLoRA linear forward  h = dequant(W0) x + (alpha/r) B A x
 *     ("QLoRA", llm-compass, section 方法与公式, the displayed formula);
 *   * its backward: dx through the frozen quantized base plus the LoRA branch,
 *     and dA, dB for the adapters (same section, the sentence after the
 *     formula: gradients only for B, A; W0 is never updated; "QLoRA",
 *     aigrafen.se, opening paragraph: gradients flow through the quantized
 *     base).
 *
 * Conventions shared by every call
 * --------------------------------
 *   Shapes use the PyTorch Linear convention: x [M, in], W0 [out, in],
 *   A [r, in], B [out, r], h [M, out], s = alpha / r.  All matrices are dense
 *   row-major with no padding between rows.
 *   bf16 tensors are passed as uint16_t bit patterns.
 *   Every pointer except the host arrays of qlora_nf4_codebook is a DEVICE
 *   pointer on the current CUDA device and must be 16-byte aligned.
 *   `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   All device work is enqueued on `stream` (the grouped calls fork it onto
 *   internal streams and join them back) and the calls return without
 *   synchronizing; outputs are valid once the stream reaches that point.
 *   The caller owns every buffer, including the workspace; the library never
 *   allocates device memory and keeps no per-call state (the grouped calls
 *   keep their internal streams and events for the process).
 *   Arguments are validated before anything is launched: a call that returns
 *   a negative status has enqueued no work and written no output.
 *
 * NF4 storage format (qlora_nf4_weight)
 * -------------------------------------
 *   blocks    64 consecutive weights of a row ("QLoRA", llm-compass,
 *             方法与公式 item 1: one scale per block of 64);
 *             n_blocks = rows*cols/64, block b = row*(cols/64) + col/64.
 *   codes     uint8 [rows, cols/2]; weight (row, 2i) in the low nibble of byte
 *             (row, i), weight (row, 2i+1) in the high nibble.  Code j means
 *             level j of qlora_nf4_codebook (ascending; level 7 is exactly 0).
 *   q8        int8 [n_blocks], second-level code of each block's absmax.
 *   step2     fp32 [ceil(n_blocks/256)], one step per group of 256 blocks.
 *   mean      fp32 [1], mean of all block absmaxes.
 *   The block scale is  c_hat = fp32(fp32(q8 * step2) + mean)  and a weight
 *   is  bf16_rne(fp32(level[code] * c_hat))  (double quantization of the
 *   block constants to 8 bit: llm-compass, 方法与公式 item 2; auryth glossary
 *   "Hoe het werkt", item 2).
 */
#ifndef QLORA_NF4_H_
#define QLORA_NF4_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every call. */
enum {
  QLORA_OK = 0,
  QLORA_ERR_INVALID_ARG = -1,      /* null or misaligned pointer, bad scalar      */
  QLORA_ERR_UNSUPPORTED_SHAPE = -2,/* a size rule below is violated               */
  QLORA_ERR_WORKSPACE = -3,        /* workspace missing or smaller than required  */
  QLORA_ERR_CUDA = -4,             /* a CUDA runtime/driver call failed           */
  QLORA_ERR_TIMEOUT = -5,          /* a device-side wait gave up (see below)      */
  QLORA_ERR_SCRATCH_LIMIT = -6     /* size beyond the built-in scratch of a
                                      no-allocation entry point               */
};

/* Operation selector of qlora_workspace_size. */
enum {
  QLORA_OP_QUANTIZE = 0,
  QLORA_OP_DEQUANTIZE = 1,
  QLORA_OP_LINEAR_FWD = 2,
  QLORA_OP_LINEAR_BWD = 3,
  QLORA_OP_LINEAR_FWD_DROPOUT = 4,
  QLORA_OP_LINEAR_BWD_DROPOUT = 5
};

/* A quantized weight: device pointers in the format described above. */
typedef struct qlora_nf4_weight {
  const uint8_t* codes;  /* [rows, cols/2]            */
  const int8_t* q8;      /* [rows*cols/64]            */
  const float* step2;    /* [ceil(rows*cols/64/256)]  */
  const float* mean;     /* [1]                       */
  int64_t rows;          /* out features              */
  int64_t cols;          /* in features, multiple of 64 */
} qlora_nf4_weight;

/*
 * qlora_nf4_codebook -- the 16 NF4 levels and 15 decision thresholds (host).
 *
 * NF4 places 16 levels at standard-normal quantiles with equal expected mass
 * per bin, normalised to [-1, 1] ("QLoRA", llm-compass, 方法与公式 item 1;
 * learn-interview-questions QLoRA page, section 2).  The exact construction
 * (an exact zero, 8 positive and 7 negative levels): with
 * delta = 1 - (1/32 + 1/30)/2, positive levels Phi^-1(delta - i(delta-1/2)/8),
 * i = 0..7, negative levels -Phi^-1(delta - i(delta-1/2)/7), i = 0..6, and 0,
 * all divided by Phi^-1(delta), rounded to fp32, ascending.
 * thresholds[j] is the exact midpoint of levels j and j+1 rounded toward
 * -infinity to fp32, so that for fp32 v: v > thresholds[j] <=> v lies above
 * the midpoint (nearest level, ties to the lower index).
 *
 * levels: host array of 16 floats (written).  thresholds: host array of 15
 * floats, or NULL.  Pure host computation, no CUDA call.
 * Returns QLORA_OK, or QLORA_ERR_INVALID_ARG if levels is NULL.
 */
int qlora_nf4_codebook(float levels[16], float thresholds[15]);

/*
 * qlora_workspace_size -- bytes of device workspace a call needs.
 *
 * op is one of QLORA_OP_*.  Sizes are those the call will receive (for
 * QLORA_OP_QUANTIZE and _DEQUANTIZE: rows = out_features, cols = in_features;
 * M and r are ignored).  Returns 0 when the call needs no workspace, and
 * (size_t)-1 for an unknown op or negative sizes.  The workspace must be
 * 256-byte aligned; its contents on entry do not matter.
 */
size_t qlora_workspace_size(int op, int64_t M, int64_t in_features,
                            int64_t out_features, int r);

/*
 * qlora_quantize_nf4 -- blockwise NF4 quantization with double quantization.
 *
 * Per block b of 64 weights: c_b = max|w| (exact); if c_b = 0 every code is 7;
 * otherwise v = fp32(w * fp32(1/c_b)), or v = fp32(w / c_b) for a block whose
 * fp32(1/c_b) overflows (a subnormal c_b below ~2.9e-39), and
 * code = #{j : v > thresholds[j]}, the nearest level with ties to the lower.
 * Second level: mean = fp32(T / n_blocks) where T is the fp64 sum of all c_b
 * in a fixed binary tree (zero-padded to a power of two, adjacent pairs added
 * level by level) and the division is done in fp64; d_b = fp32(c_b - mean);
 * per group g of 256 blocks step2_g = fp32(max|d_b| / 127);
 * q8_b = clamp(round_half_even(fp32(d_b * fp32(1/step2_g))), -127, 127), with
 * fp32(d_b / step2_g) in place of the product when fp32(1/step2_g) overflows,
 * or 0 when step2_g = 0.  All fp32 operations are correctly
 * rounded (no fused multiply-add), so the result is bit-reproducible.
 * ("QLoRA", llm-compass, 方法与公式 items 1-2.)
 *
 * W       device fp32 [rows, cols], finite values.
 * codes   device uint8 [rows, cols/2]      (written)
 * q8      device int8 [rows*cols/64]       (written)
 * step2   device fp32 [ceil(n_blocks/256)] (written)
 * mean    device fp32 [1]                  (written)
 * workspace / workspace_bytes: at least
 *         qlora_workspace_size(QLORA_OP_QUANTIZE, 0, cols, rows, 0) bytes.
 * Size rules: rows >= 1, cols >= 64, cols % 64 == 0.
 */
int qlora_quantize_nf4(const float* W, int64_t rows, int64_t cols,
                       uint8_t* codes, int8_t* q8, float* step2, float* mean,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Codebooks.  QLORA_CODEBOOK_NF4 is the NF4 code of qlora_nf4_codebook.
 * QLORA_CODEBOOK_INT4 is the uniform INT4 absmax code the pages compare NF4
 * with (learn-interview-questions QLoRA page, section 2, NF4 vs. Standard
 * INT4; llm-compass, 方法与公式 item 1): levels fp32(k/7) for k = -7..7 at
 * codes 0..14 (zero at code 7), code 15 a second +1.  Both run through the
 * same kernels; only the 16-entry level table and its thresholds differ.
 */
#define QLORA_CODEBOOK_NF4 0
#define QLORA_CODEBOOK_INT4 1

/*
 * qlora_codebook -- host only: the 16 levels and 15 thresholds (exact
 * midpoints of consecutive levels rounded toward -infinity) of a codebook
 * kind.  Returns QLORA_ERR_INVALID_ARG for an unknown kind.
 */
int qlora_codebook(int kind, float levels[16], float thresholds[15]);

/*
 * qlora_quantize_codebook / qlora_dequantize_codebook -- qlora_quantize_nf4
 * and qlora_dequantize_nf4 with the levels of codebook `kind` (same blocks,
 * normalisation, tie rule, packing, double quantization, dequantization and
 * workspace).  The stored weight does not record its codebook: dequantize it
 * with the kind it was quantized with.  The linear-layer calls use NF4.
 * Returns as qlora_quantize_nf4 / qlora_dequantize_nf4, and
 * QLORA_ERR_INVALID_ARG for an unknown kind.
 */
int qlora_quantize_codebook(int kind, const float* W, int64_t rows, int64_t cols,
                            uint8_t* codes, int8_t* q8, float* step2, float* mean,
                            void* workspace, size_t workspace_bytes, void* stream);
int qlora_dequantize_codebook(int kind, const qlora_nf4_weight* w, uint16_t* W_out, void* stream);

/*
 * qlora_quantize_nf4_bf16 -- qlora_quantize_nf4 for a weight loaded in bf16
 * (the 16-bit checkpoint form; "QLoRA: Fine-Tuning on One Consumer GPU",
 * skillbyai, Merging the adapter for serving, loads the base in bfloat16).
 * Every step is that of qlora_quantize_nf4 applied to the exact fp32 value of
 * each bf16 weight (bf16 -> fp32 widening is exact), so the outputs equal
 * those of qlora_quantize_nf4 on the widened tensor, bit for bit.
 *
 * W       device bf16 (uint16 bit patterns) [rows, cols], 16-byte aligned,
 *         finite values.  Other arguments, workspace, size rules and return
 *         values as qlora_quantize_nf4 (same workspace size).
 */
int qlora_quantize_nf4_bf16(const uint16_t* W, int64_t rows, int64_t cols,
                            uint8_t* codes, int8_t* q8, float* step2, float* mean,
                            void* workspace, size_t workspace_bytes, void* stream);

/*
 * qlora_merge_adapter -- the adapter merged into a bf16 copy of the
 * dequantized base for serving: W_out = dequant(W0) + (alpha/r) B A.
 * Merging needs the base dequantized first and goes into a higher-precision
 * copy, since merging straight back into 4 bit is lossy ("QLoRA",
 * llm-compass, 调参与实践经验; skillbyai, Merging the adapter for serving).
 * Per element: acc = fp32 sum over j = 0..r-1, in that order, of
 * B[o][j] * A[j][i] (each product exact in fp32);
 * W_out[o][i] = bf16_rne(fp32(w_hat[o][i] + fp32(s * acc))) with
 * s = fp32(alpha / r) and w_hat the bf16 weight of qlora_dequantize_nf4.
 * Re-quantizing W_out with qlora_quantize_nf4_bf16 is the lossy "merge back
 * into 4 bit".
 *
 * w       quantized base [out, in]
 * A       device bf16 [r, in], 16-byte aligned
 * B       device bf16 [out, r], 16-byte aligned
 * W_out   device bf16 [out, in], 16-byte aligned (written)
 * Size rules: in % 64 == 0, out % 64 == 0, 1 <= r <= 256; alpha finite.
 * Returns QLORA_OK, QLORA_ERR_INVALID_ARG, QLORA_ERR_UNSUPPORTED_SHAPE or
 * QLORA_ERR_CUDA; nothing is launched on an error.
 */
int qlora_merge_adapter(const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r, float alpha,
                        uint16_t* W_out, void* stream);

/*
 * qlora_dequantize_nf4 -- NF4 weight to bf16, bit-exact with the formula in
 * the format description above ("QLoRA", auryth glossary, "Hoe het werkt":
 * dequantize NF4 on the fly per layer).
 *
 * w      quantized weight (device pointers), cols % 64 == 0.
 * W_out  device bf16 [rows, cols] (written).
 */
int qlora_dequantize_nf4(const qlora_nf4_weight* w, uint16_t* W_out, void* stream);

/*
 * qlora_linear_fwd -- QLoRA linear forward
 *   h  = x dequant(W0)^T + us B^T,   us = bf16(s * x A^T),   s = alpha / r
 * ("QLoRA", llm-compass, 方法与公式, displayed formula).  The dequantized
 * weight is produced tile by tile inside the GEMM and never written to memory.
 * M > 16 runs the fused tensor-core GEMM; M <= 16 a split-K streaming GEMV.
 * The GEMM's token tile is 512 rows on a CTA pair for M > 384, else 256 or
 * 128 rows on one CTA; the environment variable QLORA_NF4_GEMM_TILE_M = 128,
 * 256 or 512 (read once per process) forces one of them for every M > 16, so
 * that each GEMM kernel can be exercised on any shape (results agree within
 * fp32 summation order).  The backward's dx GEMM follows the same rule.
 *
 * x       device bf16 [M, in]
 * w       quantized W0, rows = out, cols = in
 * A       device bf16 [r, in];  B  device bf16 [out, r]
 * h       device bf16 [M, out] (written)
 * us_out  device bf16 [M, r] (written): the scaled LoRA activation, kept for
 *         the backward.
 * workspace: qlora_workspace_size(QLORA_OP_LINEAR_FWD, M, in, out, r) bytes.
 * Size rules: M >= 1; in % 64 == 0; out % 64 == 0; 1 <= r <= 256 ("QLoRA",
 * llm-compass, 调参与实践经验: the rank is a free hyper-parameter, 16-64
 * typical).  The kernels work on rank multiples of 8 (16-byte rows of the
 * [tokens, r] and [out, r] tensors); for any other r the call runs at r
 * rounded up to 8 on zero-padded copies of A, B and us held in the
 * workspace (the padding adds exactly zero) and copies us back to [M, r].
 */
int qlora_linear_fwd(const uint16_t* x, int64_t M, const qlora_nf4_weight* w,
                     const uint16_t* A, const uint16_t* B, int r, float alpha,
                     uint16_t* h, uint16_t* us_out,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * qlora_linear_bwd -- QLoRA linear backward with W0 frozen.
 *   du = bf16(s * dh B)                 [M, r]
 *   dx = dh dequant(W0) + du A          [M, in]  (bf16 out)
 *   dB = dh^T us                        [out, r] (fp32 out)
 *   dA = du^T x                         [r, in]  (fp32 out)
 * us is the us_out of the matching forward (us = bf16(s x A^T)), so
 * dB = s dh^T x A^T and dA = s (dh B)^T x up to bf16 rounding of us and du.
 * No gradient is formed for W0 ("QLoRA", llm-compass, 方法与公式: gradients
 * only for B, A; aigrafen.se: gradients back-propagate through the quantized
 * base, only the adapters are updated).
 *
 * dh, x, us, A, B: device bf16 as in the forward; dh [M, out].
 * dx device bf16 [M, in]; dA device fp32 [r, in]; dB device fp32 [out, r]
 * (all written, not accumulated).
 * workspace: qlora_workspace_size(QLORA_OP_LINEAR_BWD, M, in, out, r) bytes.
 * Size rules as for qlora_linear_fwd; for r % 8 != 0 the padded copies of A,
 * B, us and of dA, dB (fp32) live in the workspace and dA, dB are copied back
 * to [r, in] and [out, r].
 */
int qlora_linear_bwd(const uint16_t* dh, const uint16_t* x, const uint16_t* us,
                     int64_t M, const qlora_nf4_weight* w,
                     const uint16_t* A, const uint16_t* B, int r, float alpha,
                     uint16_t* dx, float* dA, float* dB,
                     void* workspace, size_t workspace_bytes, void* stream);

/*
 * qlora_linear_fwd_dropout / qlora_linear_bwd_dropout -- the layer with LoRA
 * dropout on the adapter input (lora_dropout = 0.05 in every configuration on
 * the pages: "QLoRA", aigrafen.se; llm-compass, 实现要点; skillbyai;
 * learn-interview-questions, section 3).  With keep mask k (0/1 per element
 * of x) and drop probability p, inverted scaling:
 *   h  = x W0^T + s ((x * k) / (1 - p)) A^T B^T
 *   dx = dh W0 + s ((dh B) A) * k / (1 - p)
 *   dB = dh^T us,  dA = du^T (x * k) / (1 - p)
 * with us = bf16((s / (1 - p)) (x * k) A^T) (returned by the forward and
 * passed to the backward), du = bf16(s dh B); the backward must receive the
 * same k and p as the forward.  The base GEMMs are those of
 * qlora_linear_fwd / _bwd; dx adds the masked rank-r term to the bf16 result
 * of dh W0 in fp32 and rounds again to bf16.
 *
 * The masked input x * k is never stored: the rank-r kernels zero the
 * dropped elements of the activation tiles they stage.  The backward forks
 * `stream` onto the library's internal streams (the dx GEMM beside du, dB
 * and dA) and joins them back before returning, like the grouped calls.
 *
 * keep_bits  device uint8 [M, in/8], 4-byte aligned: bit (i % 8) of byte i/8
 *            of row m is the keep flag of x[m][i] (the caller draws the mask).
 * p          drop probability, 0 <= p < 1.
 * workspace: qlora_workspace_size(QLORA_OP_LINEAR_FWD_DROPOUT / _BWD_DROPOUT,
 *            M, in, out, r) bytes (the same as without dropout; none for the
 *            forward with M > 16).  Other arguments, rules and returns as
 *            qlora_linear_fwd / qlora_linear_bwd; QLORA_ERR_INVALID_ARG for a
 *            null or misaligned mask or p outside [0, 1).
 */
int qlora_linear_fwd_dropout(const uint16_t* x, int64_t M, const qlora_nf4_weight* w, const uint16_t* A,
                             const uint16_t* B, int r, float alpha, const uint8_t* keep_bits, float p, uint16_t* h,
                             uint16_t* us_out, void* workspace, size_t workspace_bytes, void* stream);
int qlora_linear_bwd_dropout(const uint16_t* dh, const uint16_t* x, const uint16_t* us, int64_t M,
                             const qlora_nf4_weight* w, const uint16_t* A, const uint16_t* B, int r, float alpha,
                             const uint8_t* keep_bits, float p, uint16_t* dx, float* dA, float* dB, void* workspace,
                             size_t workspace_bytes, void* stream);

/*
 * Grouped projections: n independent QLoRA linears issued together, e.g.
 * the seven projections of one decoder layer ("QLoRA", llm-compass, 实现要点:
 * target_modules q/k/v/o and gate/up/down).  One problem per projection:
 *
 *   x, w, A, B, M, r, alpha   as in qlora_linear_fwd
 *   h, us                     forward outputs (us is the backward's input)
 *   dh                        backward input [M, out]
 *   dx, dA, dB                backward outputs
 *
 * qlora_linear_fwd_group computes what n calls of qlora_linear_fwd would, in
 * order, on `stream`; qlora_linear_bwd_group what n calls of qlora_linear_bwd
 * would (the fields a direction does not use may be null).  Results are bit
 * for bit those of the single calls.  The difference is the issue order: the
 * rank-r products (us in the forward; du, dA and dB in the backward) run on
 * an internal low-priority stream and the fused GEMMs on an internal
 * high-priority stream of the current device, projection i + 1's rank-r work
 * beside projection i's GEMM, so that it fills the SMs the GEMM's last
 * partial wave of CTA pairs leaves idle.  Both internal streams first wait for
 * the work issued to `stream` before the call, and `stream` waits for both
 * before anything issued after it.  Projections with M <= 16 or r % 8 != 0
 * run as the single call would, on the high-priority stream.
 *
 * The projections must not overlap: no output of one may alias any input or
 * output of another.  workspace: qlora_linear_group_workspace_size(backward,
 * n, problems) bytes (each projection's single-call workspace, one after
 * another).  Returns the first failing projection's error before anything is
 * issued when an argument check fails; QLORA_ERR_INVALID_ARG for n < 0 or a
 * null `problems` with n > 0.  Calls from several host threads on one device
 * are serialized while they issue work.  Dropout is not offered grouped.
 */
typedef struct qlora_linear_problem {
  const uint16_t* x;
  const qlora_nf4_weight* w;
  const uint16_t* A;
  const uint16_t* B;
  int64_t M;
  int r;
  float alpha;
  uint16_t* h;
  uint16_t* us;
  const uint16_t* dh;
  uint16_t* dx;
  float* dA;
  float* dB;
} qlora_linear_problem;

/* (size_t)-1 for n < 0, a null `problems` with n > 0 or a projection whose
 * sizes qlora_workspace_size rejects. */
size_t qlora_linear_group_workspace_size(int backward, int n, const qlora_linear_problem* problems);
int qlora_linear_fwd_group(int n, const qlora_linear_problem* problems, void* workspace, size_t workspace_bytes,
                           void* stream);
int qlora_linear_bwd_group(int n, const qlora_linear_problem* problems, void* workspace, size_t workspace_bytes,
                           void* stream);

/*
 * qlora_last_device_status -- synchronizes `stream`, then reads and clears
 * the current device's error flag.  Kernels that wait on another part of the
 * device (pipeline barriers inside the GEMMs) give up after a bounded time
 * (qlora_set_wait_timeout_ns), set the flag and return.  Returns QLORA_OK,
 * QLORA_ERR_TIMEOUT when the flag was set, or QLORA_ERR_CUDA when the
 * synchronization itself reports an error.
 */
int qlora_last_device_status(void* stream);

/*
 * qlora_set_wait_timeout_ns -- bound, in nanoseconds of %globaltimer, of every
 * device-side wait launched after this call (process-wide; default 2e9 = 2 s).
 * Values below 1000 are raised to 1000.  Returns the previous bound.
 */
uint64_t qlora_set_wait_timeout_ns(uint64_t ns);

/*
 * qlora_selftest_wait_timeout -- diagnostic: launches one kernel that waits on
 * a pipeline barrier that nothing will ever complete, bounded by the current
 * wait timeout, so that the timeout path (error flag set, kernel returns,
 * context stays usable) can be exercised without faulting or hanging a GPU.
 * Returns the status of qlora_last_device_status after the kernel
 * (QLORA_ERR_TIMEOUT when the path works).
 */
int qlora_selftest_wait_timeout(void* stream);

/*
 * Per-kernel timing (diagnostics for benchmarks).  While enabled, every kernel
 * the library launches is bracketed by two CUDA events recorded on the
 * launching stream; qlora_timing_collect synchronizes on those events and
 * returns, for one kernel name, the summed device time in milliseconds and
 * the number of launches since the last reset.  Names: "quantize_blocks",
 * "scale_mean_tree", "dq_scales", "dequantize", "gemm_fwd", "gemm_dx",
 * "gemv", "gemv_finalize", "lora_rowwise" (us), "lora_rowwise_du" (du),
 * "lora_colwise" (dA and dB), "merge_adapter", "dropout_dx".  Events are created by the library on first use (host-side
 * CUDA objects, no device memory).  Not for use during stream capture.
 *
 * qlora_timing_enable: on != 0 enables, 0 disables; returns the previous state.
 * qlora_timing_reset: forgets all recorded launches.
 * qlora_timing_collect: kernel name (NUL-terminated), outputs may be NULL.
 *   Returns QLORA_OK, QLORA_ERR_INVALID_ARG for a NULL name, or
 *   QLORA_ERR_CUDA if an event query fails.
 */
int qlora_timing_enable(int on);
void qlora_timing_reset(void);
int qlora_timing_collect(const char* kernel, double* total_ms, int64_t* launches);

/*
 * qlora_quantize_nf4_noalloc -- qlora_quantize_nf4 without a caller workspace.
 *
 * The pages describe no such variant; it exists for callers that cannot
 * obtain device memory at the moment they quantize: a host that forbids
 * cudaMalloc after start-up (an allocation can synchronize the device and
 * break a memory budget planned in advance), or a plugin that has no access
 * to its host framework's allocator and so cannot size and pass the
 * workspace that qlora_quantize_nf4 needs.  It computes exactly what
 * qlora_quantize_nf4 computes (same kernels, bit-identical outputs); its
 * scratch (block absmaxes and the partial sums of the scale-mean tree) lives
 * in a fixed device array inside the library, QLORA_NOALLOC_MAX_BLOCKS blocks
 * of 64 weights large (16 MiB + 8.5 KiB), which every GPU that loads the
 * library holds until the process exits.  The call itself allocates nothing.
 *
 * The first call on a device looks up that array's device address (once per
 * device, with the device current), and so does the first call after the
 * device's context was destroyed and recreated (cudaDeviceReset), which
 * gives the array a new address; make the first call (and the first after
 * a reset) before any stream capture begins.  Every call shares the one array: calls that can overlap on
 * the GPU (different streams, or different host threads) race on it and must
 * be ordered by the caller.  The array keeps the previous call's contents;
 * each call overwrites every scratch value before reading it, so nothing has
 * to start at zero.
 *
 * Arguments and size rules as qlora_quantize_nf4, without the workspace.
 * Returns QLORA_ERR_SCRATCH_LIMIT (nothing launched) when
 * rows*cols/64 > QLORA_NOALLOC_MAX_BLOCKS, QLORA_ERR_CUDA if the address
 * lookup fails.
 */
#define QLORA_NOALLOC_MAX_BLOCKS (1LL << 22)
int qlora_quantize_nf4_noalloc(const float* W, int64_t rows, int64_t cols,
                               uint8_t* codes, int8_t* q8, float* step2, float* mean,
                               void* stream);

/*
 * Sharded quantization -- qlora_quantize_nf4 split over `world` ranks that
 * each hold a contiguous slice of the flattened weight (data parallelism over
 * blocks; the pages quantize on one device, the split is this library's).
 *
 * The blocks (64 consecutive weights of the row-major weight) are grouped in
 * chunks of 4096; rank k owns the chunks [k*cpr, (k+1)*cpr) with
 * cpr = ceil(chunks / world), i.e. the blocks [block_begin, block_end), so
 * every shard starts on a chunk boundary and hence on a 256-block boundary of
 * the second-level groups.  The only quantity that needs every block is the
 * scale mean.  Its tree (qlora_quantize_nf4: fp64, zero-padded to a power of
 * two, adjacent pairs added level by level) is cut at the chunk level: each
 * rank sums its own chunks (roots), the ranks all-gather the roots in rank
 * order (world * cpr doubles, zeros for chunks past the weight), and every
 * rank finishes the same tree over them.  Adding zero-padded power-of-two
 * subtrees is exact, so codes, q8, step2 and mean are bit-identical to one
 * qlora_quantize_nf4 call on the whole weight.
 *
 * qlora_quantize_shard_plan (host only): the block range of `rank` and cpr.
 *   n_blocks_total = rows * cols / 64 of the whole weight (1 .. 2^34);
 *   1 <= world, 0 <= rank < world.  A trailing rank may own no block.
 *
 * qlora_quantize_shard_workspace_size: bytes of the workspace one rank keeps
 *   from its local call to its finishing call (n_roots_total = world * cpr);
 *   (size_t)-1 for bad sizes.
 *
 * qlora_quantize_nf4_shard_local: the rank's codes and roots.
 *   W_shard      device fp32, n_blocks_shard * 64 weights (the shard's slice
 *                of the flattened weight), finite values.
 *   codes_shard  device uint8 [n_blocks_shard * 32]             (written)
 *   roots        device fp64 [roots_per_rank], 16-byte aligned  (written;
 *                chunk sums of the shard's block absmaxes, zero past it)
 *   The workspace must stay untouched until the finishing call.
 *   n_blocks_shard = 0 (an empty rank) writes zero roots only.
 *
 * qlora_quantize_nf4_shard_finish: mean, and the rank's q8 and step2.
 *   roots_all    device fp64 [n_roots_total], 16-byte aligned: the all-gathered
 *                roots in rank order.
 *   q8_shard, step2_shard, mean: 16-byte aligned (slices of a whole weight's
 *                arrays at the shard's first block are, since shards start on
 *                4096-block boundaries).
 *   q8_shard     device int8 [n_blocks_shard]                    (written)
 *   step2_shard  device fp32 [ceil(n_blocks_shard / 256)]        (written)
 *   mean         device fp32 [1]                                 (written)
 *   workspace    the same one the local call used.
 *
 * All device calls are asynchronous on `stream`; errors return before any
 * launch (QLORA_ERR_INVALID_ARG for bad pointers or sizes, QLORA_ERR_WORKSPACE
 * for a missing or short workspace).
 */
int qlora_quantize_shard_plan(int64_t n_blocks_total, int world, int rank,
                              int64_t* block_begin, int64_t* block_end,
                              int64_t* roots_per_rank);
size_t qlora_quantize_shard_workspace_size(int64_t n_blocks_shard, int64_t n_roots_total);
int qlora_quantize_nf4_shard_local(const float* W_shard, int64_t n_blocks_shard,
                                   uint8_t* codes_shard, double* roots, int64_t roots_per_rank,
                                   void* workspace, size_t workspace_bytes, void* stream);
int qlora_quantize_nf4_shard_finish(const double* roots_all, int64_t n_roots_total,
                                    int64_t n_blocks_total, int64_t n_blocks_shard,
                                    int8_t* q8_shard, float* step2_shard, float* mean,
                                    void* workspace, size_t workspace_bytes, void* stream);

/* qlora_status_string -- static English description of a status code. */
const char* qlora_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* QLORA_NF4_H_ */
