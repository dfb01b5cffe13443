/*
 * sharq.h -- C ABI of the SharQ sparse-dense FP4 linear layer for B200 (sm_100a).
 *
 * The method ("SharQ: Bridging Activation Sparsity and FP4 Quantization for LLM
 * Inference", Abstract): an online sparse-dense decomposition of each activation
 * tensor. An input-adaptive N:M mask extracts an outlier-dominated sparse
 * backbone, the backbone is quantized to FP4, a dense residual is defined
 * against the *quantized* backbone and quantized densely to FP4; a sparse FP4
 * GEMM on the backbone and a dense FP4 GEMM on the residual share one FP4
 * weight payload with path-specific scale views; a fused preparation kernel
 * absorbs mask generation, residual construction and layer normalization.
 * The README ("SharQ: Bridging Activation Sparsity and FP4 Quantization",
 * sections "Evaluation" and "Benchmarks") names the normalization RMSNorm and
 * the dense-FP4-only mode "NVFP4".
 *
 * Conventions for every call:
 *  - Pointers named *_dev are device pointers; the caller allocates and owns all
 *    of them (sizes from sharq_prep_buffer_sizes / sharq_wpack_buffer_sizes).
 *    The library allocates no memory and never synchronizes the stream.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *    Work is enqueued asynchronously on it.
 *  - Every argument is checked on the host before any launch. A call returns
 *    SHARQ_OK or an error status and launches nothing on error; the message is
 *    available from sharq_last_error() (per host thread). No exception crosses
 *    the ABI. A launch failure reported by the CUDA runtime returns SHARQ_ERR_CUDA.
 *  - Device pointers must be 16-byte aligned (the activation and RMSNorm weight given to
 *    sharq_prepare / sharq_quantize_dense: 32-byte aligned). bf16 values are raw 16-bit words.
 *  - Sizes: tokens >= 1; k a positive multiple of 256; n_out a positive multiple of 16.
 *
 * Formats. E2M1 element codes (2 per byte, the lower K index in the low nibble)
 * with block scales:
 *   SHARQ_NVFP4: 16-element blocks, E4M3 scale, plus one float32 second-level
 *                scale per token row (activations) or per tensor (weight).
 *   SHARQ_MXFP4: 32-element blocks, E8M0 scale, no second-level scale.
 *
 * Mask. Along K, `unit` consecutive elements form a unit and nm_m consecutive
 * units form a group; in each group the nm_n units with the largest key are
 * kept (key = largest |x| in the unit; equal keys go to the lower unit). The
 * sparse FP4 tensor-core MMA of sm_100a selects pairs, so the pattern
 * sharq_linear executes is (nm_n, nm_m, unit) = (2, 4, 2): two of every four
 * aligned pairs, i.e. 4 of 8 elements. sharq_prepare also computes the
 * element pattern (2, 4, 1).
 *
 * Scale layout ("128x4 atoms"). A scale tensor of R rows (R padded to a
 * multiple of 128; 256 for activations) and S scales per row (S a multiple of 4) is stored as atoms
 * of 512 bytes: atom (R/128 block rb, scale group sg = s/4) at byte offset
 * (rb * S/4 + sg) * 512, and inside it the scale of row r, index s at
 * (r%32)*16 + ((r%128)/32)*4 + s%4. This is the layout the tensor core's
 * scale-factor copy reads.
 *
 * Sparse metadata. One 4-bit entry per group, the two kept unit indices
 * (i0 < i1) as i0 | i1<<2, group g of a row at bits 4g..4g+3 of that row's
 * bit string. Stored in slabs of 128 bits per row: slab j holds groups
 * [32j, 32j+32) of every row, slab-major: byte offset (j * tokens_pad + row) * 16.
 */
#ifndef SHARQ_H
#define SHARQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { SHARQ_NVFP4 = 0, SHARQ_MXFP4 = 1 } sharq_fmt;
typedef enum { SHARQ_OUT_BF16 = 0, SHARQ_OUT_F32 = 1 } sharq_out;
typedef enum {
  SHARQ_OK = 0,
  SHARQ_ERR_INVALID_ARG = 1, /* bad size, null pointer, misalignment, mismatched operands */
  SHARQ_ERR_UNSUPPORTED = 2, /* valid request this build does not execute (e.g. a pattern) */
  SHARQ_ERR_CUDA = 3,        /* the CUDA runtime reported a launch or device error */
  SHARQ_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up (see sharq_device_status) */
} sharq_status;

/* The prepared activation of one call of sharq_prepare. Device buffers, caller-owned.
 *   sparse_codes  [tokens][k*nm_n/nm_m/2] bytes: kept values in K order, E2M1 pairs
 *   sparse_meta   metadata slabs (see above), k/(32*nm_m*unit) slabs of tokens_pad*16 bytes
 *   sparse_scales 128x4 atoms, tokens_pad rows, k*nm_n/nm_m/B scales per row; a backbone
 *                 block is B consecutive *stored* values (B = 16 NVFP4, 32 MXFP4)
 *   resid_codes   [tokens][k/2] bytes: the residual, E2M1 pairs
 *   resid_scales  128x4 atoms, tokens_pad rows, k/B scales per row
 *   row_scale     [tokens] float32: NVFP4 second-level scale s_x (1.0 for MXFP4)
 * tokens_pad = tokens rounded up to 256 (the GEMM's CTA pairs cover 256 rows). */
typedef struct {
  void *sparse_codes;
  void *sparse_meta;
  void *sparse_scales;
  void *resid_codes;
  void *resid_scales;
  float *row_scale;
  int tokens, k, nm_n, nm_m, unit;
  int fmt; /* sharq_fmt */
} sharq_prep;

/* One packed weight [n_out][k]: a single E2M1 code payload and two scale views.
 *   codes          [n_out][k/2] bytes
 *   scales_sparse  128x4 atoms, n_out_pad rows, k/(2B) scales per row: one scale per 2B
 *                  consecutive K, the span of one backbone block at density 1/2
 *   scales_dense   128x4 atoms, n_out_pad rows, k/B scales per row: scales_sparse with
 *                  each entry repeated for the two B-wide dense blocks it covers
 *   tensor_scale   float32[2]: [0] = s_w (NVFP4 per-tensor scale, 1.0 for MXFP4),
 *                  [1] = amax|W| (written by sharq_pack_weight)
 * n_out_pad = n_out rounded up to 128. */
typedef struct {
  void *codes;
  void *scales_sparse;
  void *scales_dense;
  float *tensor_scale;
  int n_out, k;
  int fmt; /* sharq_fmt */
} sharq_wpack;

/* Byte sizes of the six sharq_prep buffers, in struct order, written to sizes[0..5];
 * returns their sum, or 0 (with sharq_last_error set) for invalid arguments. */
size_t sharq_prep_buffer_sizes(int tokens, int k, int nm_n, int nm_m, int unit, int fmt,
                               size_t sizes[6]);

/* Byte sizes of codes, scales_sparse, scales_dense, tensor_scale; returns the sum or 0. */
size_t sharq_wpack_buffer_sizes(int n_out, int k, int fmt, size_t sizes[4]);

/* Pack a bf16 weight once (offline): per-tensor amax, block scales over 2B
 * consecutive K, E2M1 codes, and both scale views. The abstract: "The two paths
 * share a single FP4 weight payload with path-specific scale views."
 *   w_bf16_dev  [n_out][k] row-major bf16
 *   out         caller-filled struct of device buffers (fields n_out/k/fmt are set here)
 * Two launches (amax reduction, then quantization); tensor_scale is cleared first. */
int sharq_pack_weight(const void *w_bf16_dev, int n_out, int k, int fmt, sharq_wpack *out,
                      void *stream);

/* The fused preparation operator (one launch). The abstract: "a fused
 * preparation kernel absorbs mask generation, residual construction, and layer
 * normalization into one operator".
 *   x_bf16_dev      [tokens][k] row-major bf16 activations
 *   gamma_bf16_dev  [k] bf16 RMSNorm weight, or NULL for no normalization
 *   eps             RMSNorm epsilon (ignored without gamma)
 *   nm_n, nm_m, unit  the mask; (2,4,2) and (2,4,1) are executed
 *   out             caller-filled struct of device buffers (shape fields are set here)
 * RMSNorm: rstd = 1/sqrt(fp32(sum(x^2)/k) + eps), xh = (x*rstd)*gamma in float32.
 * NVFP4 row scale s_x = amax|xh|/2688 (1 for a zero row), shared by backbone
 * and residual. Codes are round-to-nearest-even with saturation. */
int sharq_prepare(const void *x_bf16_dev, int tokens, int k, const void *gamma_bf16_dev,
                  float eps, int nm_n, int nm_m, int unit, int fmt, sharq_prep *out,
                  void *stream);

/* The SharQ linear layer (one launch): Y = s_x * s_w * (A_sp (*) W^T + A_res . W^T),
 * the structured-sparse block-scaled FP4 MMA on the backbone and the dense one on
 * the residual accumulating into one tensor-memory accumulator, then one epilogue.
 *   a       a prepared activation (pattern (2,4,2); fmt equal to w->fmt; same k)
 *   w       a packed weight
 *   y_dev   [tokens][n_out] row-major, bf16 (round to nearest even) or float32
 *   out_dtype  SHARQ_OUT_BF16 or SHARQ_OUT_F32 */
int sharq_linear(const sharq_prep *a, const sharq_wpack *w, void *y_dev, int out_dtype,
                 void *stream);

/* The library's own dense FP4 baseline (the README's "NVFP4: dense FP4 baseline"):
 * optional RMSNorm + dense block quantization of xh with the same row-scale rule
 * (one launch), and a dense FP4 GEMM against the weight's dense view (one launch).
 *   codes_dev [tokens][k/2]; scales_dev 128x4 atoms (tokens_pad rows, k/B per row);
 *   row_scale_dev [tokens] float32. */
int sharq_quantize_dense(const void *x_bf16_dev, int tokens, int k, const void *gamma_bf16_dev,
                         float eps, int fmt, void *codes_dev, void *scales_dev,
                         float *row_scale_dev, void *stream);
int sharq_linear_dense(const void *codes_dev, const void *scales_dev, const float *row_scale_dev,
                       int tokens, int k, const sharq_wpack *w, void *y_dev, int out_dtype,
                       void *stream);

/* Synchronizes `stream`, then reports and clears the device-side status word that
 * bounded waits set when they give up: SHARQ_OK or SHARQ_ERR_TIMEOUT (or SHARQ_ERR_CUDA). */
int sharq_device_status(void *stream);

/* Test hook: time limit, in nanoseconds, of the GEMM's bounded waits (0 restores the
 * default of 4 s). Lowering it lets a test make a wait give up without faulting the device:
 * the kernel records SHARQ_ERR_TIMEOUT, drains its own copies and MMAs, frees its tensor
 * memory and returns; its output is then undefined. Applies to calls issued afterwards. */
void sharq_set_wait_limit(long long nanoseconds);

/* Message of the last error on this host thread ("" if none). */
const char *sharq_last_error(void);

/* ABI version (major*100 + minor). */
int sharq_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SHARQ_H */
