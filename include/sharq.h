/*
 * sharq.h -- C ABI of the SharQ sparse-dense FP4 linear layer for B200 (sm_100a).
 *
 * The method follows "SharQ: Bridging Activation Sparsity and FP4 Quantization for
 * LLM Inference" (Abstract). Every activation tensor is split at run time into two
 * FP4 operands: a structured-sparse one holding the N largest of every M values
 * along K (where the outliers end up), and a dense remainder computed against the
 * backbone *after* its FP4 rounding. The sparse operand feeds a sparse FP4 MMA, the
 * remainder a dense FP4 MMA; both multiply the same FP4 weight codes, each with its
 * own scale layout, and add into one output. Normalization, mask selection and both
 * quantizations happen in one preparation kernel. The README mirror ("SharQ:
 * Bridging Activation Sparsity and FP4 Quantization", sections "Evaluation" and
 * "Benchmarks") names the normalization RMSNorm and calls the dense-only mode NVFP4.
 *
 * Conventions for every call:
 *  - Pointers named *_dev are device pointers; the caller allocates and owns all
 *    of them (sizes from sharq_prep_buffer_sizes / sharq_wpack_buffer_sizes and the
 *    workspace-size queries). The library allocates no memory and never synchronizes the
 *    stream; its only device memory of its own is the 8 KB static array that
 *    sharq_prepare_tensor_scale_noalloc uses in place of a workspace.
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
 * aligned pairs, i.e. 4 of 8 elements. sharq_prepare (and only it) also computes
 * the element patterns (2, 4, 1) and (4, 8, 1), which no sparse FP4 MMA of sm_100a
 * executes: sharq_linear rejects them with SHARQ_ERR_UNSUPPORTED.
 *
 * Sparse metadata. 2:4: one 4-bit entry per group, the two kept unit indices
 * (i0 < i1) as i0 | i1<<2; group g of a row at bits 4g..4g+3 of that row's bit
 * string (per 256 K positions: 128 bits for pairs, 256 bits for elements).
 * 4:8 over elements: one 12-bit entry per group of 8, the four kept indices
 * ascending as i0 | i1<<3 | i2<<6 | i3<<9, group g at bits 12g..12g+11 (384 bits).
 *
 * Tiled operands. Activations and weights are stored as the tensor-core GEMM reads
 * them: chunks of 128 rows x 256 K positions, one contiguous chunk per (128-row block
 * rb, K step ks = k/256), chunk-major: chunk (rb, ks) at byte (rb * k/256 + ks) * C,
 * C the chunk size below. Inside a chunk, with r = row % 128:
 *   - codes with row pitch P (128 bytes for 256 codes, 64 bytes for 128 kept codes):
 *     byte b of row r's codes at r*P + ((b/16) XOR s(r))*16 + b%16, where the 16-byte
 *     unit is swizzled with s(r) = r%8 (P = 128) or (r/2)%4 (P = 64);
 *   - a scale run ("128x4 atoms"): scale s (0-based within the K step) of row r at
 *     (s/4)*512 + (r%32)*16 + (r/32)*4 + s%4;
 *   - metadata: row r's 16 bytes of bit string at r*16 (pairs); for elements, the two
 *     16-byte halves at h*2048 + r*16.
 * Rows past the tensor's end (up to the padded row count) are zero.
 *
 * Prepared activation chunk (sharq_prepare), B = 16 (NVFP4) or 32 (MXFP4):
 *   residual codes  offset 0,      128 rows x 128 bytes (256 codes)
 *   backbone codes  offset 16384,  128 rows x 64 bytes (the 128 kept codes, in K order)
 *   metadata        offset 24576,  2048 bytes (pairs), 4096 (elements 2:4) or 6144
 *                   (elements 4:8: byte b of row r's 48 at (b/16)*2048 + r*16 + b%16)
 *   backbone scales then residual scales, scale runs of 128/B and 256/B scales per row
 *   C = 29696 (NVFP4, pairs), 28672 (MXFP4, pairs), 31744 (NVFP4, elements 2:4),
 *       30720 (MXFP4, elements 2:4), 33792 (NVFP4, 4:8), 32768 (MXFP4, 4:8);
 *       padded rows: tokens_pad = tokens rounded up to 256.
 * Dense-quantized activation chunk (sharq_quantize_dense): codes at 0 (128 x 128 bytes),
 *   scale run at 16384 (256/B scales per row); C = 18432 (NVFP4) or 17408 (MXFP4).
 * Packed weight chunk, for 128 weight rows = one half of a 256-row block (n_out_pad =
 *   n_out rounded up to 256): codes at 0 (128 x 128 bytes); then the sparse-view scales
 *   (256/(2B) per row) and the dense-view scales (256/B per row) of ALL 256 rows of the
 *   block, each as two scale runs (rows 0..127 of the block, then rows 128..255), so the
 *   chunks of both halves carry the same scales; C = 22528 (NVFP4) or 19456 (MXFP4).
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
  SHARQ_ERR_UNSUPPORTED = 2, /* valid request the library does not execute (e.g. a pattern) */
  SHARQ_ERR_CUDA = 3,        /* the CUDA runtime reported a launch or device error */
  SHARQ_ERR_TIMEOUT = 4      /* a bounded device-side wait gave up (see sharq_device_status) */
} sharq_status;

/* The prepared activation of one call of sharq_prepare. Device buffers, caller-owned.
 *   tiles      prepared activation chunks (see "Tiled operands"): backbone codes,
 *              metadata and scales, residual codes and scales
 *   row_scale  [tokens] float32: NVFP4 second-level scale s_x (1.0 for MXFP4) */
typedef struct {
  void *tiles;
  float *row_scale;
  int tokens, k, nm_n, nm_m, unit;
  int fmt; /* sharq_fmt */
} sharq_prep;

/* One packed weight [n_out][k]: a single E2M1 code payload and two scale views.
 *   tiles          packed weight chunks (see "Tiled operands"): the codes, the sparse
 *                  view (one scale per 2B consecutive K, the span of one backbone
 *                  block at density 1/2) and the dense view (each sparse-view scale
 *                  repeated for the two B-wide dense blocks it covers)
 *   tensor_scale   float32[2]: [0] = s_w (NVFP4 per-tensor scale, 1.0 for MXFP4),
 *                  [1] = amax|W| (written by sharq_pack_weight) */
typedef struct {
  void *tiles;
  float *tensor_scale;
  int n_out, k;
  int fmt; /* sharq_fmt */
} sharq_wpack;

/* Byte sizes of the sharq_prep buffers (tiles, row_scale), written to sizes[0..1];
 * returns their sum, or 0 (with sharq_last_error set) for invalid arguments. */
size_t sharq_prep_buffer_sizes(int tokens, int k, int nm_n, int nm_m, int unit, int fmt,
                               size_t sizes[2]);

/* Byte sizes of the dense quantizer's buffers (tiles, row_scale); returns the sum or 0. */
size_t sharq_dense_buffer_sizes(int tokens, int k, int fmt, size_t sizes[2]);

/* Byte sizes of the sharq_wpack buffers (tiles, tensor_scale); returns the sum or 0. */
size_t sharq_wpack_buffer_sizes(int n_out, int k, int fmt, size_t sizes[2]);

/* Pack a bf16 weight once (offline): per-tensor amax, block scales over 2B
 * consecutive K, E2M1 codes, and both scale views (Abstract: the two GEMM paths read
 * the same weight codes, each with scales laid out for it).
 *   w_bf16_dev  [n_out][k] row-major bf16
 *   out         caller-filled struct of device buffers (fields n_out/k/fmt are set here)
 * Two launches (amax reduction, then quantization); tensor_scale is cleared first. */
int sharq_pack_weight(const void *w_bf16_dev, int n_out, int k, int fmt, sharq_wpack *out,
                      void *stream);

/* The fused preparation operator (one launch; Abstract: normalization, the mask and the
 * residual are computed by one kernel).
 *   x_bf16_dev      [tokens][k] row-major bf16 activations
 *   gamma_bf16_dev  [k] bf16 RMSNorm weight, or NULL for no normalization
 *   eps             RMSNorm epsilon (ignored without gamma)
 *   nm_n, nm_m, unit  the mask: (2,4,2), (2,4,1) or (4,8,1); only (2,4,2) feeds sharq_linear
 *   out             caller-filled struct of device buffers (shape fields are set here)
 * RMSNorm: rstd = 1/sqrt(fp32(sum(x^2)/k) + eps), xh = (x*rstd)*gamma in float32.
 * NVFP4 row scale s_x = amax|xh|/2688 (1 for a zero row), shared by backbone
 * and residual. Codes are round-to-nearest-even with saturation. */
int sharq_prepare(const void *x_bf16_dev, int tokens, int k, const void *gamma_bf16_dev,
                  float eps, int nm_n, int nm_m, int unit, int fmt, sharq_prep *out,
                  void *stream);

/* sharq_prepare with ONE NVFP4 second-level scale for the whole activation tensor instead
 * of one per row: s_x = fp32(amax|xh|/2688) over every row (the stricter reading of NVFP4's
 * "fp32 tensor scale"), shared by backbone and residual; row_scale receives that value in
 * every entry, so sharq_linear consumes the result unchanged. MXFP4 has no second-level
 * scale: same as sharq_prepare (the workspace is not touched).
 * One cooperative launch (every block resident): a first phase forms each row's rstd and
 * normalized amax (rstd is parked in row_scale), a grid-wide barrier exchanges the block maxima
 * through the workspace, a second phase quantizes. When every row fits on chip (about 2400
 * rows at k = 4096 on B200) x is read once; beyond that the rows not held in registers are
 * read again, the most recent first.
 *   workspace_dev  caller-owned device buffer of sharq_tensor_scale_workspace_size(tokens, k)
 *                  bytes, 16-byte aligned, ZEROED ONCE before its first use (e.g. by
 *                  cudaMemset when it is allocated). Each call leaves its barrier words ready
 *                  for the next, so it can be reused without clearing, across sizes too
 *                  (a buffer sized for the largest call serves all). Calls whose launches may
 *                  overlap on the GPU need distinct workspaces.
 * If the barrier's bounded wait gives up (only if blocks were not all resident), the call's
 * outputs are undefined, sharq_device_status reports SHARQ_ERR_TIMEOUT, and the workspace
 * must be zeroed again before it is reused. Other arguments, layouts and errors as
 * sharq_prepare. */
size_t sharq_tensor_scale_workspace_size(int tokens, int k);
int sharq_prepare_tensor_scale(const void *x_bf16_dev, int tokens, int k, const void *gamma_bf16_dev,
                               float eps, int nm_n, int nm_m, int unit, int fmt, sharq_prep *out,
                               void *workspace_dev, void *stream);

/* sharq_prepare_tensor_scale for callers that cannot allocate device memory. The paper has no
 * counterpart: this is an integration variant. Some callers may not call cudaMalloc at all --
 * a host framework or inference server that owns every byte of the GPU's memory and hands a
 * kernel library only its tensors, or a latency-critical path where cudaMalloc's implicit
 * device synchronization is not acceptable -- so they have no way to supply the workspace.
 * This entry point allocates nothing: the grid barrier's words and the block maxima live in a
 * static device array of 8192 bytes inside the library (held on every GPU that loads the
 * library until the process exits), enough for launches of up to 2044 blocks; a launch that
 * would need more (a GPU with more than 255 SMs) is rejected with SHARQ_ERR_UNSUPPORTED and a
 * message naming both sizes, and nothing is launched. The caller still passes the input and
 * the output struct; results are identical to sharq_prepare_tensor_scale's.
 *   - Every call on a device shares that array, and it keeps the last call's contents: each
 *     call clears its barrier words on `stream` first (an 8-byte memset, no allocation). Calls
 *     whose launches may overlap on the GPU race on the array: order them on one stream.
 *   - The first call on a device looks up the array's device address (with that device
 *     current) and caches it; make that first call before any stream capture.
 *   - MXFP4 has no second-level scale: as sharq_prepare, the array is not touched.
 * Arguments, layouts and errors otherwise as sharq_prepare_tensor_scale. */
int sharq_prepare_tensor_scale_noalloc(const void *x_bf16_dev, int tokens, int k, const void *gamma_bf16_dev,
                                       float eps, int nm_n, int nm_m, int unit, int fmt, sharq_prep *out,
                                       void *stream);

/* The preparation operator fed by a gate/up projection's output (one launch): the down
 * projection's input x = SiLU(g) * u is formed in registers from [g | u] and prepared as
 * by sharq_prepare without normalization, so x never goes through memory (the abstract's
 * preparation kernel folds the steps in front of the quantizer into itself).
 *   gate_up_bf16_dev  [tokens][2k] row-major bf16: g in columns [0, k), u in [k, 2k);
 *                     32-byte aligned
 *   x = bf16(fp32(silu(g) * u)) rounded to nearest even, silu(g) = g * sigma(g) in float32
 *   with sigma(g) = 1/(1+e) (g >= 0) or e/(1+e) (g < 0), e = exp(-|g|) evaluated by Cody-Waite
 *   range reduction and a degree-7 Taylor polynomial in correctly rounded float32 steps
 *   (|g| * log2(e) >= 126 gives e = 0); the division is correctly rounded.
 * Output, pattern, formats and errors as sharq_prepare. */
int sharq_prepare_swiglu(const void *gate_up_bf16_dev, int tokens, int k, int nm_n, int nm_m,
                         int unit, int fmt, sharq_prep *out, void *stream);

/* The SharQ linear layer (one launch): Y = s_x * s_w * (A_sp (*) W^T + A_res . W^T),
 * the structured-sparse block-scaled FP4 MMA on the backbone and the dense one on
 * the residual accumulating into one tensor-memory accumulator, then one epilogue.
 *   a       a prepared activation (pattern (2,4,2); fmt equal to w->fmt; same k)
 *   w       a packed weight
 *   y_dev   [tokens][n_out] row-major, bf16 (round to nearest even) or float32
 *   out_dtype  SHARQ_OUT_BF16 or SHARQ_OUT_F32 */
int sharq_linear(const sharq_prep *a, const sharq_wpack *w, void *y_dev, int out_dtype,
                 void *stream);

/* sharq_linear for launches with few output tiles (few tokens and a narrow output), where a
 * plain launch leaves most SM pairs idle while one pair walks all of K: with a caller
 * workspace the K range is cut into S slices (S from sharq_linear_workspace_size's shape
 * rule), run as S problems of one grouped launch that each write float32 partial outputs
 * already scaled by s_x * s_w, then summed in slice order by a second kernel into y (bf16
 * rounded once, at the end). The same two MMA paths and scales as sharq_linear; the result
 * differs from it only by float32 rounding order. When the shape does not call for slicing,
 * this is exactly sharq_linear and the workspace is not touched.
 *   workspace_dev    device buffer of at least sharq_linear_workspace_size(tokens, n_out, k)
 *                    bytes, 16-byte aligned, contents irrelevant; overwritten. Calls whose
 *                    launches may overlap on the GPU need distinct workspaces.
 * Errors as sharq_linear; SHARQ_ERR_INVALID_ARG if the workspace is smaller than needed. */
size_t sharq_linear_workspace_size(int tokens, int n_out, int k);
int sharq_linear_split(const sharq_prep *a, const sharq_wpack *w, void *y_dev, int out_dtype,
                       void *workspace_dev, size_t workspace_bytes, void *stream);

/* Grouped (mixture-of-experts) SharQ linear: n_groups independent problems
 * Y_e = sharq_linear(a[e], w[e]) computed by one launch per 64 groups, the persistent grid
 * working through the output tiles of all groups (no tile mixes experts). When the groups are
 * mostly at most 128 rows the launch runs on single-CTA 128-row tiles instead of CTA-pair
 * 256-row tiles (chosen per launch, same results up to float32 rounding order). The abstract
 * evaluates a mixture-of-experts model (Qwen3-30B-A3B) with the method; this is its expert
 * layer.
 *   a[e], w[e]  prepared activation and packed weight of group e; every weight has the same
 *               n_out, k and fmt; a[e].tokens == 0 marks an expert without tokens (skipped:
 *               its prep buffers and y_dev[e] are not used and may be NULL). a[e].tiles may
 *               point into a larger prepared buffer at any 128-row block (one sharq_prepare
 *               over all experts' rows laid out expert by expert): the GEMM reads up to
 *               round_up(tokens, 256) rows of chunks from there (rows past the expert's own are
 *               read, never written), so that many rows must lie inside the allocation.
 *   y_dev[e]    [a[e].tokens][n_out] output of group e (bf16 or float32 per out_dtype)
 * Checks and errors as sharq_linear, per group. */
int sharq_linear_grouped(const sharq_prep *a, const sharq_wpack *w, void *const *y_dev, int n_groups,
                         int out_dtype, void *stream);

/* The library's own dense FP4 baseline (the README mirror's dense-only NVFP4 mode):
 * optional RMSNorm + dense block quantization of xh with the same row-scale rule
 * (one launch), and a dense FP4 GEMM against the weight's dense view (one launch).
 *   tiles_dev      dense-quantized activation chunks (sharq_dense_buffer_sizes)
 *   row_scale_dev  [tokens] float32 */
int sharq_quantize_dense(const void *x_bf16_dev, int tokens, int k, const void *gamma_bf16_dev,
                         float eps, int fmt, void *tiles_dev, float *row_scale_dev, void *stream);
int sharq_linear_dense(const void *tiles_dev, const float *row_scale_dev, int tokens, int k,
                       const sharq_wpack *w, void *y_dev, int out_dtype, void *stream);

/* The separate normalization pass of the dense baseline pipeline (one launch):
 * y = bf16_RNE(fp32(fp32(x * rstd) * gamma)), rstd = 1/sqrt(fp32(sum(x^2)/k) + eps) with the
 * sum of squares in float64 -- the value the fused preparation operator normalizes to,
 * rounded to bf16 as an unfused pipeline passes it to the next kernel. The baseline then runs
 * sharq_quantize_dense on y without gamma and sharq_linear_dense. The fused preparation
 * operator replaces this pass (Abstract: normalization folded into the preparation kernel).
 *   x_bf16_dev, y_bf16_dev  [tokens][k] row-major bf16 (16-byte aligned); k <= 32768
 *   gamma_bf16_dev          [k] bf16 */
int sharq_rmsnorm(const void *x_bf16_dev, int tokens, int k, const void *gamma_bf16_dev, float eps,
                  void *y_bf16_dev, void *stream);

/* Diagnostic: the tensor-core ceiling that sharq_linear is measured against. The pages have no
 * counterpart; this is the measured denominator of the GEMM's tensor-pipe fraction. One
 * launch, one CTA pair per SM pair (or `clusters` pairs if 0 < clusters < SMs/2), each issuing
 * `iters` K steps of sharq_linear's MMAs (M = 256 rows over the pair, N = 256, 256 logical K
 * per step) from one resident shared-memory stage and one tensor-memory scale buffer, with no
 * loads, scale writes or epilogue. The caller times the launch (CUDA events on `stream`).
 *   mode   0: the four dense block-scaled MMAs of a K step (2*256*256*256 flops per step);
 *          1: the two structured-sparse MMAs (2*256*256*256 logical flops, half of them on
 *             kept values); 2: both, sharq_linear's K step
 *   fmt    SHARQ_NVFP4 (kind::mxf4nvf4, 16-element E4M3 scales) or SHARQ_MXFP4 (kind::mxf4)
 *   iters  1 .. 2^20 K steps per pair
 * Operands are pseudo-random; results are discarded. A completion wait that gives up is
 * reported by sharq_device_status. */
int sharq_mma_peak(int mode, int fmt, int iters, int clusters, void *stream);

/* Synchronizes `stream`, then reports and clears the device-side status word that
 * bounded waits set when they give up: SHARQ_OK or SHARQ_ERR_TIMEOUT (or SHARQ_ERR_CUDA). */
int sharq_device_status(void *stream);

/* Test hook: time limit, in nanoseconds, of the GEMM's bounded waits and of the per-tensor
 * preparation's grid barrier (0 restores the default of 4 s). Process-wide (one atomic value
 * shared by every host thread), read by each call when it launches. Lowering it lets a test make a wait give up without faulting the device:
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
