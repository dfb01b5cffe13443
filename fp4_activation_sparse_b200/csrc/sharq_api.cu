// C ABI of the SharQ library: argument checks, buffer sizes, launches.
// Every entry point validates on the host before it launches anything and returns a
// sharq_status; the message of the last failure is kept per host thread.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/sharq.h"
#include "sharq_common.cuh"
#include "sharq_internal.h"

namespace {

thread_local char g_err[512] = "";
// Time limit (ns) of the GEMM's bounded waits for calls issued from now on, process-wide;
// 0 = the kernel's default. Read once per launch.
std::atomic<long long> g_wait_limit{0};

int fail(int status, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return status;
}

int cuda_fail(cudaError_t e, const char *what) {
  return fail(SHARQ_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

bool valid_fmt(int fmt) { return fmt == SHARQ_NVFP4 || fmt == SHARQ_MXFP4; }

// Pattern checks shared by sizes and prepare. Returns 0 or a status.
int check_pattern(int nm_n, int nm_m, int unit) {
  if (nm_n < 1 || nm_m < 1 || nm_n > nm_m || (unit != 1 && unit != 2))
    return fail(SHARQ_ERR_INVALID_ARG, "invalid N:M pattern %d:%d unit %d", nm_n, nm_m, unit);
  if (!(nm_n == 2 && nm_m == 4))
    return fail(SHARQ_ERR_UNSUPPORTED, "pattern %d:%d (unit %d) is not executed; supported: 2:4 over units of 1 or 2",
                nm_n, nm_m, unit);
  return 0;
}

// sharq_prepare and the size query also take four of eight elements (4:8, unit 1); returns 0
// or a status and sets *code to the layout's pattern code (2 pairs, 1 elements 2:4, kPat48).
int check_prepare_pattern(int nm_n, int nm_m, int unit, int *code) {
  if (nm_n == 4 && nm_m == 8 && unit == 1) {
    *code = sharq::kPat48;
    return 0;
  }
  *code = unit;
  return check_pattern(nm_n, nm_m, unit);
}

int check_shape(int rows, int k, const char *rows_name) {
  if (rows < 1) return fail(SHARQ_ERR_INVALID_ARG, "%s must be >= 1 (got %d)", rows_name, rows);
  if (k < 256 || k % 256 != 0) return fail(SHARQ_ERR_INVALID_ARG, "k must be a positive multiple of 256 (got %d)", k);
  if ((long long)rows * k > (1ll << 40)) return fail(SHARQ_ERR_INVALID_ARG, "tensor too large");
  return 0;
}

}  // namespace

extern "C" {

const char *sharq_last_error(void) { return g_err; }

int sharq_version(void) { return 200; }

void sharq_set_wait_limit(long long nanoseconds) { g_wait_limit.store(nanoseconds, std::memory_order_relaxed); }

size_t sharq_prep_buffer_sizes(int tokens, int k, int nm_n, int nm_m, int unit, int fmt, size_t sizes[2]) {
  if (!sizes) { fail(SHARQ_ERR_INVALID_ARG, "sizes is null"); return 0; }
  if (!valid_fmt(fmt)) { fail(SHARQ_ERR_INVALID_ARG, "unknown fmt %d", fmt); return 0; }
  int code = 0;
  if (check_shape(tokens, k, "tokens") || check_prepare_pattern(nm_n, nm_m, unit, &code)) return 0;
  const sharq::ActTile A = sharq::act_tile(fmt, code, true);
  sizes[0] = (size_t)(sharq::round_up(tokens, 256) / 128) * (k / 256) * A.bytes;  // tiles
  sizes[1] = (size_t)tokens * 4;                                                    // row scales
  return sizes[0] + sizes[1];
}

size_t sharq_dense_buffer_sizes(int tokens, int k, int fmt, size_t sizes[2]) {
  if (!sizes) { fail(SHARQ_ERR_INVALID_ARG, "sizes is null"); return 0; }
  if (!valid_fmt(fmt)) { fail(SHARQ_ERR_INVALID_ARG, "unknown fmt %d", fmt); return 0; }
  if (check_shape(tokens, k, "tokens")) return 0;
  const sharq::ActTile A = sharq::act_tile(fmt, 2, false);
  sizes[0] = (size_t)(sharq::round_up(tokens, 256) / 128) * (k / 256) * A.bytes;
  sizes[1] = (size_t)tokens * 4;
  return sizes[0] + sizes[1];
}

size_t sharq_wpack_buffer_sizes(int n_out, int k, int fmt, size_t sizes[2]) {
  if (!sizes) { fail(SHARQ_ERR_INVALID_ARG, "sizes is null"); return 0; }
  if (!valid_fmt(fmt)) { fail(SHARQ_ERR_INVALID_ARG, "unknown fmt %d", fmt); return 0; }
  if (check_shape(n_out, k, "n_out")) return 0;
  if (n_out % 16) { fail(SHARQ_ERR_INVALID_ARG, "n_out must be a multiple of 16 (got %d)", n_out); return 0; }
  sizes[0] = (size_t)(sharq::round_up(n_out, 256) / 128) * (k / 256) * sharq::w_tile(fmt).bytes;
  sizes[1] = 2 * sizeof(float);
  return sizes[0] + sizes[1];
}

int sharq_pack_weight(const void *w, int n_out, int k, int fmt, sharq_wpack *out, void *stream) {
  if (!w || !out) return fail(SHARQ_ERR_INVALID_ARG, "null weight or output struct");
  size_t sz[2];
  if (!sharq_wpack_buffer_sizes(n_out, k, fmt, sz)) return SHARQ_ERR_INVALID_ARG;
  if (!out->tiles || !out->tensor_scale) return fail(SHARQ_ERR_INVALID_ARG, "null output buffer in sharq_wpack");
  if (!aligned16(w) || !aligned16(out->tiles) || !aligned16(out->tensor_scale))
    return fail(SHARQ_ERR_INVALID_ARG, "device buffers must be 16-byte aligned");
  out->n_out = n_out;
  out->k = k;
  out->fmt = fmt;
  sharq::PackParams p;
  p.w = static_cast<const uint16_t *>(w);
  p.N = n_out;
  p.K = k;
  p.N_pad = sharq::round_up(n_out, 256);
  p.tiles = static_cast<uint8_t *>(out->tiles);
  p.tensor_scale = out->tensor_scale;
  cudaError_t e = sharq::launch_pack(p, fmt, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "sharq_pack_weight");
  g_err[0] = 0;
  return SHARQ_OK;
}

static int prepare_common(const void *x, int tokens, int k, const void *gamma, float eps, int fmt, bool dense,
                          int unit, uint8_t *tiles, float *row_scale, cudaStream_t st, bool swiglu = false,
                          bool per_tensor = false, void *workspace = nullptr) {
  if (!x) return fail(SHARQ_ERR_INVALID_ARG, "x is null");
  if (!valid_fmt(fmt)) return fail(SHARQ_ERR_INVALID_ARG, "unknown fmt %d", fmt);
  if (int s = check_shape(tokens, k, "tokens")) return s;
  if (k > 32768) return fail(SHARQ_ERR_INVALID_ARG, "k must be <= 32768 for the preparation kernel (got %d)", k);
  if (((uintptr_t)x & 31u) || ((uintptr_t)gamma & 31u))
    return fail(SHARQ_ERR_INVALID_ARG, "x and gamma must be 32-byte aligned (256-bit loads)");
  if (!tiles || !row_scale) return fail(SHARQ_ERR_INVALID_ARG, "null output buffer");
  if (!aligned16(tiles) || !aligned16(row_scale)) return fail(SHARQ_ERR_INVALID_ARG, "output buffers must be 16-byte aligned");
  if (gamma && !(eps >= 0.f)) return fail(SHARQ_ERR_INVALID_ARG, "eps must be >= 0");
  sharq::PrepParams p;
  memset(&p, 0, sizeof p);
  p.x = static_cast<const uint16_t *>(x);
  p.x_stride = swiglu ? 2 * k : k;
  p.gamma = static_cast<const uint16_t *>(gamma);
  p.eps = eps;
  p.T = tokens;
  p.K = k;
  p.T_pad = sharq::round_up(tokens, 256);
  p.tiles = tiles;
  p.row_scale = row_scale;
  const long long lim = g_wait_limit.load(std::memory_order_relaxed);
  cudaError_t e = per_tensor && fmt == SHARQ_NVFP4
                      ? sharq::launch_prep_tensor_scale(p, unit, gamma != nullptr, workspace,
                                                        lim > 0 ? (unsigned long long)lim : 4000000000ull, st)
                      : sharq::launch_prep(p, fmt, unit, gamma != nullptr, dense, swiglu, st);
  if (e != cudaSuccess)
    return cuda_fail(e, dense ? "sharq_quantize_dense" : swiglu ? "sharq_prepare_swiglu" : "sharq_prepare");
  g_err[0] = 0;
  return SHARQ_OK;
}

int sharq_prepare(const void *x, int tokens, int k, const void *gamma, float eps, int nm_n, int nm_m, int unit,
                  int fmt, sharq_prep *out, void *stream) {
  if (!out) return fail(SHARQ_ERR_INVALID_ARG, "output struct is null");
  int code = 0;
  if (int s = check_prepare_pattern(nm_n, nm_m, unit, &code)) return s;
  int s = prepare_common(x, tokens, k, gamma, eps, fmt, false, code, static_cast<uint8_t *>(out->tiles),
                         out->row_scale, static_cast<cudaStream_t>(stream));
  if (s == SHARQ_OK) {
    out->tokens = tokens;
    out->k = k;
    out->nm_n = nm_n;
    out->nm_m = nm_m;
    out->unit = unit;
    out->fmt = fmt;
  }
  return s;
}

size_t sharq_tensor_scale_workspace_size(int tokens, int k) {
  if (check_shape(tokens, k, "tokens")) return 0;
  if (k > 32768) { fail(SHARQ_ERR_INVALID_ARG, "k must be <= 32768 (got %d)", k); return 0; }
  return 16 + 4 * (size_t)sharq::prep_tensor_groups(tokens, k);
}

int sharq_prepare_tensor_scale(const void *x, int tokens, int k, const void *gamma, float eps, int nm_n, int nm_m,
                               int unit, int fmt, sharq_prep *out, void *workspace, void *stream) {
  if (!out) return fail(SHARQ_ERR_INVALID_ARG, "output struct is null");
  if (int s = check_pattern(nm_n, nm_m, unit)) return s;
  if (fmt == SHARQ_NVFP4 && (!workspace || !aligned16(workspace)))
    return fail(SHARQ_ERR_INVALID_ARG, "workspace must be a 16-byte aligned device buffer");
  int s = prepare_common(x, tokens, k, gamma, eps, fmt, false, unit, static_cast<uint8_t *>(out->tiles),
                         out->row_scale, static_cast<cudaStream_t>(stream), false, true, workspace);
  if (s == SHARQ_OK) {
    out->tokens = tokens;
    out->k = k;
    out->nm_n = nm_n;
    out->nm_m = nm_m;
    out->unit = unit;
    out->fmt = fmt;
  }
  return s;
}

int sharq_prepare_tensor_scale_noalloc(const void *x, int tokens, int k, const void *gamma, float eps, int nm_n,
                                       int nm_m, int unit, int fmt, sharq_prep *out, void *stream) {
  if (!out) return fail(SHARQ_ERR_INVALID_ARG, "output struct is null");
  if (int s = check_pattern(nm_n, nm_m, unit)) return s;
  if (fmt != SHARQ_NVFP4)  // MXFP4 has no second-level scale: the per-row operator, no scratch
    return sharq_prepare(x, tokens, k, gamma, eps, nm_n, nm_m, unit, fmt, out, stream);
  if (!x) return fail(SHARQ_ERR_INVALID_ARG, "x is null");
  if (int s = check_shape(tokens, k, "tokens")) return s;
  if (k > 32768) return fail(SHARQ_ERR_INVALID_ARG, "k must be <= 32768 for the preparation kernel (got %d)", k);
  if (((uintptr_t)x & 31u) || ((uintptr_t)gamma & 31u))
    return fail(SHARQ_ERR_INVALID_ARG, "x and gamma must be 32-byte aligned (256-bit loads)");
  if (!out->tiles || !out->row_scale) return fail(SHARQ_ERR_INVALID_ARG, "null output buffer");
  if (!aligned16(out->tiles) || !aligned16(out->row_scale))
    return fail(SHARQ_ERR_INVALID_ARG, "output buffers must be 16-byte aligned");
  if (gamma && !(eps >= 0.f)) return fail(SHARQ_ERR_INVALID_ARG, "eps must be >= 0");
  sharq::PrepParams p;
  memset(&p, 0, sizeof p);
  p.x = static_cast<const uint16_t *>(x);
  p.x_stride = k;
  p.gamma = static_cast<const uint16_t *>(gamma);
  p.eps = eps;
  p.T = tokens;
  p.K = k;
  p.T_pad = sharq::round_up(tokens, 256);
  p.tiles = static_cast<uint8_t *>(out->tiles);
  p.row_scale = out->row_scale;
  const long long lim = g_wait_limit.load(std::memory_order_relaxed);
  size_t needed = 0, capacity = 0;
  cudaError_t e = sharq::launch_prep_tensor_scale_static(p, unit, gamma != nullptr,
                                                         lim > 0 ? (unsigned long long)lim : 4000000000ull,
                                                         static_cast<cudaStream_t>(stream), &needed, &capacity);
  if (e == cudaErrorInvalidValue && needed > capacity)
    return fail(SHARQ_ERR_UNSUPPORTED, "sharq_prepare_tensor_scale_noalloc: this launch needs %zu bytes of scratch, "
                "the library's static scratch holds %zu (use sharq_prepare_tensor_scale with a workspace)",
                needed, capacity);
  if (e != cudaSuccess) return cuda_fail(e, "sharq_prepare_tensor_scale_noalloc");
  out->tokens = tokens;
  out->k = k;
  out->nm_n = nm_n;
  out->nm_m = nm_m;
  out->unit = unit;
  out->fmt = fmt;
  g_err[0] = 0;
  return SHARQ_OK;
}

int sharq_prepare_swiglu(const void *gate_up, int tokens, int k, int nm_n, int nm_m, int unit, int fmt,
                         sharq_prep *out, void *stream) {
  if (!out) return fail(SHARQ_ERR_INVALID_ARG, "output struct is null");
  if (int s = check_pattern(nm_n, nm_m, unit)) return s;
  if (tokens > 0 && (long long)tokens * 2 * k > (1ll << 40)) return fail(SHARQ_ERR_INVALID_ARG, "tensor too large");
  int s = prepare_common(gate_up, tokens, k, nullptr, 0.f, fmt, false, unit, static_cast<uint8_t *>(out->tiles),
                         out->row_scale, static_cast<cudaStream_t>(stream), true);
  if (s == SHARQ_OK) {
    out->tokens = tokens;
    out->k = k;
    out->nm_n = nm_n;
    out->nm_m = nm_m;
    out->unit = unit;
    out->fmt = fmt;
  }
  return s;
}

int sharq_quantize_dense(const void *x, int tokens, int k, const void *gamma, float eps, int fmt, void *tiles,
                         float *row_scale, void *stream) {
  return prepare_common(x, tokens, k, gamma, eps, fmt, true, 2, static_cast<uint8_t *>(tiles), row_scale,
                        static_cast<cudaStream_t>(stream));
}

static int check_wpack(const sharq_wpack *w) {
  if (!w) return fail(SHARQ_ERR_INVALID_ARG, "weight pack is null");
  if (!valid_fmt(w->fmt)) return fail(SHARQ_ERR_INVALID_ARG, "weight pack has unknown fmt %d", w->fmt);
  if (int s = check_shape(w->n_out, w->k, "n_out")) return s;
  if (w->n_out % 16) return fail(SHARQ_ERR_INVALID_ARG, "n_out must be a multiple of 16");
  if (!w->tiles || !w->tensor_scale) return fail(SHARQ_ERR_INVALID_ARG, "null buffer in weight pack");
  if (!aligned16(w->tiles)) return fail(SHARQ_ERR_INVALID_ARG, "weight buffers must be 16-byte aligned");
  return 0;
}

static int run_gemm(sharq::GemmParams &g, const char *name, cudaStream_t st) {
  g.wait_limit = g_wait_limit.load(std::memory_order_relaxed);
  const char *why = nullptr;
  cudaError_t e = sharq::launch_gemm(g, st, &why);
  if (why) return fail(SHARQ_ERR_CUDA, "%s: %s", name, why);
  if (e != cudaSuccess) return cuda_fail(e, name);
  g_err[0] = 0;
  return SHARQ_OK;
}

// Checks one (prep, weight, output) problem of sharq_linear / sharq_linear_grouped.
static int check_linear(const sharq_prep *a, const sharq_wpack *w, const void *y, int out_dtype) {
  if (!a || !y) return fail(SHARQ_ERR_INVALID_ARG, "null prep or output");
  if (int s = check_wpack(w)) return s;
  if (!valid_fmt(a->fmt)) return fail(SHARQ_ERR_INVALID_ARG, "prep has unknown fmt %d", a->fmt);
  if (int s = check_shape(a->tokens, a->k, "tokens")) return s;
  if (a->fmt != w->fmt) return fail(SHARQ_ERR_INVALID_ARG, "format mismatch: prep %d, weight %d", a->fmt, w->fmt);
  if (a->k != w->k) return fail(SHARQ_ERR_INVALID_ARG, "k mismatch: prep %d, weight %d", a->k, w->k);
  if (out_dtype != SHARQ_OUT_BF16 && out_dtype != SHARQ_OUT_F32) return fail(SHARQ_ERR_INVALID_ARG, "bad out_dtype");
  if (!(a->nm_n == 2 && a->nm_m == 4 && a->unit == 2))
    return fail(SHARQ_ERR_UNSUPPORTED,
                "the sparse FP4 MMA executes pattern 2:4 over pairs (unit 2); got %d:%d unit %d", a->nm_n, a->nm_m,
                a->unit);
  if (!a->tiles || !a->row_scale) return fail(SHARQ_ERR_INVALID_ARG, "null buffer in prep");
  if (!aligned16(a->tiles) || !aligned16(a->row_scale) || !aligned16(y))
    return fail(SHARQ_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  return 0;
}

static void set_group(sharq::GemmGroup &G, const void *tiles, const float *row_scale, int tokens,
                      const sharq_wpack *w, void *y) {
  G.a_tiles = static_cast<const uint8_t *>(tiles);
  G.row_scale = row_scale;
  G.w_tiles = static_cast<const uint8_t *>(w->tiles);
  G.tensor_scale = w->tensor_scale;
  G.y = y;
  G.T = tokens;
  G.T_pad = sharq::round_up(tokens, 256);
}

int sharq_linear(const sharq_prep *a, const sharq_wpack *w, void *y, int out_dtype, void *stream) {
  if (int s = check_linear(a, w, y, out_dtype)) return s;
  sharq::GemmParams g;
  memset(&g, 0, sizeof g);
  set_group(g.grp[0], a->tiles, a->row_scale, a->tokens, w, y);
  g.n_groups = 1;
  g.N = w->n_out;
  g.K = a->k;
  g.N_pad = sharq::round_up(w->n_out, 256);
  g.fmt = a->fmt;
  g.out_f32 = out_dtype == SHARQ_OUT_F32;
  g.sparse = 1;
  return run_gemm(g, "sharq_linear", static_cast<cudaStream_t>(stream));
}

size_t sharq_linear_workspace_size(int tokens, int n_out, int k) {
  if (check_shape(tokens, k, "tokens")) return 0;
  if (n_out < 16 || n_out % 16) { fail(SHARQ_ERR_INVALID_ARG, "n_out must be a positive multiple of 16"); return 0; }
  const int S = sharq::gemm_split_count(tokens, n_out, k);
  g_err[0] = 0;
  return S > 1 ? (size_t)S * tokens * n_out * sizeof(float) : 0;
}

int sharq_linear_split(const sharq_prep *a, const sharq_wpack *w, void *y, int out_dtype, void *workspace,
                       size_t workspace_bytes, void *stream) {
  if (int s = check_linear(a, w, y, out_dtype)) return s;
  const int S = sharq::gemm_split_count(a->tokens, w->n_out, a->k);
  if (S <= 1) return sharq_linear(a, w, y, out_dtype, stream);
  const size_t plane = (size_t)a->tokens * w->n_out;
  const size_t need = (size_t)S * plane * sizeof(float);
  if (!workspace || workspace_bytes < need)
    return fail(SHARQ_ERR_INVALID_ARG, "sharq_linear_split: this launch needs a workspace of %zu bytes (got %zu)",
                need, workspace ? workspace_bytes : (size_t)0);
  if (!aligned16(workspace)) return fail(SHARQ_ERR_INVALID_ARG, "workspace must be 16-byte aligned");
  sharq::GemmParams g;
  memset(&g, 0, sizeof g);
  const int ks = a->k / 256, q = (ks + S - 1) / S;
  for (int s = 0; s < S; ++s) {
    set_group(g.grp[s], a->tiles, a->row_scale, a->tokens, w, static_cast<float *>(workspace) + s * plane);
    g.grp[s].k0 = s * q;
    g.grp[s].num_k = ks - s * q < q ? ks - s * q : q;
  }
  g.n_groups = S;
  g.N = w->n_out;
  g.K = a->k;
  g.N_pad = sharq::round_up(w->n_out, 256);
  g.fmt = a->fmt;
  g.out_f32 = 1;  // partial outputs
  g.sparse = 1;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (int s = run_gemm(g, "sharq_linear_split", st)) return s;
  cudaError_t e = sharq::launch_splitk_reduce(static_cast<const float *>(workspace), S, a->tokens, w->n_out, y,
                                              out_dtype == SHARQ_OUT_F32, st);
  if (e != cudaSuccess) return cuda_fail(e, "sharq_linear_split (reduction)");
  g_err[0] = 0;
  return SHARQ_OK;
}

int sharq_linear_grouped(const sharq_prep *a, const sharq_wpack *w, void *const *y, int n_groups, int out_dtype,
                         void *stream) {
  if (!a || !w || !y) return fail(SHARQ_ERR_INVALID_ARG, "null group arrays");
  if (n_groups < 1) return fail(SHARQ_ERR_INVALID_ARG, "n_groups must be >= 1 (got %d)", n_groups);
  for (int e = 0; e < n_groups; ++e) {
    if (a[e].tokens == 0) continue;  // an expert without tokens: nothing to do (y[e] may be null)
    if (int s = check_linear(&a[e], &w[e], y[e], out_dtype)) return s;
    if (w[e].n_out != w[0].n_out || w[e].k != w[0].k || w[e].fmt != w[0].fmt)
      return fail(SHARQ_ERR_INVALID_ARG, "group %d: every weight must have the shape and format of group 0", e);
  }
  if (int s = check_wpack(&w[0])) return s;
  for (int e0 = 0; e0 < n_groups; e0 += sharq::kMaxGroups) {  // one launch per kMaxGroups groups
    sharq::GemmParams g;
    memset(&g, 0, sizeof g);
    const int n = n_groups - e0 < sharq::kMaxGroups ? n_groups - e0 : sharq::kMaxGroups;
    for (int i = 0; i < n; ++i) {
      const sharq_prep &ae = a[e0 + i];
      set_group(g.grp[i], ae.tiles, ae.row_scale, ae.tokens > 0 ? ae.tokens : 0, &w[e0 + i], y[e0 + i]);
    }
    g.n_groups = n;
    g.N = w[0].n_out;
    g.K = w[0].k;
    g.N_pad = sharq::round_up(w[0].n_out, 256);
    g.fmt = w[0].fmt;
    g.out_f32 = out_dtype == SHARQ_OUT_F32;
    g.sparse = 1;
    if (int s = run_gemm(g, "sharq_linear_grouped", static_cast<cudaStream_t>(stream))) return s;
  }
  return SHARQ_OK;
}

int sharq_linear_dense(const void *tiles, const float *row_scale, int tokens, int k, const sharq_wpack *w, void *y,
                       int out_dtype, void *stream) {
  if (!tiles || !row_scale || !y) return fail(SHARQ_ERR_INVALID_ARG, "null buffer");
  if (int s = check_wpack(w)) return s;
  if (int s = check_shape(tokens, k, "tokens")) return s;
  if (k != w->k) return fail(SHARQ_ERR_INVALID_ARG, "k mismatch: activation %d, weight %d", k, w->k);
  if (out_dtype != SHARQ_OUT_BF16 && out_dtype != SHARQ_OUT_F32) return fail(SHARQ_ERR_INVALID_ARG, "bad out_dtype");
  if (!aligned16(tiles) || !aligned16(row_scale) || !aligned16(y))
    return fail(SHARQ_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  sharq::GemmParams g;
  memset(&g, 0, sizeof g);
  set_group(g.grp[0], tiles, row_scale, tokens, w, y);
  g.n_groups = 1;
  g.N = w->n_out;
  g.K = k;
  g.N_pad = sharq::round_up(w->n_out, 256);
  g.fmt = w->fmt;
  g.out_f32 = out_dtype == SHARQ_OUT_F32;
  g.sparse = 0;
  return run_gemm(g, "sharq_linear_dense", static_cast<cudaStream_t>(stream));
}

int sharq_rmsnorm(const void *x, int tokens, int k, const void *gamma, float eps, void *y, void *stream) {
  if (!x || !gamma || !y) return fail(SHARQ_ERR_INVALID_ARG, "null x, gamma or output");
  if (int s = check_shape(tokens, k, "tokens")) return s;
  if (k > 32768) return fail(SHARQ_ERR_INVALID_ARG, "k must be <= 32768 (got %d)", k);
  if (!aligned16(x) || !aligned16(gamma) || !aligned16(y)) return fail(SHARQ_ERR_INVALID_ARG, "buffers must be 16-byte aligned");
  if (!(eps >= 0.f)) return fail(SHARQ_ERR_INVALID_ARG, "eps must be >= 0");
  cudaError_t e = sharq::launch_rmsnorm(static_cast<const uint16_t *>(x), static_cast<const uint16_t *>(gamma), eps,
                                        tokens, k, static_cast<uint16_t *>(y), static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "sharq_rmsnorm");
  g_err[0] = 0;
  return SHARQ_OK;
}

int sharq_mma_peak(int mode, int fmt, int iters, int clusters, void *stream) {
  if (mode < 0 || mode > 2) return fail(SHARQ_ERR_INVALID_ARG, "mode must be 0 (dense), 1 (sparse) or 2 (both)");
  if (!valid_fmt(fmt)) return fail(SHARQ_ERR_INVALID_ARG, "bad fmt %d", fmt);
  if (iters < 1 || iters > (1 << 20)) return fail(SHARQ_ERR_INVALID_ARG, "iters must be in [1, 2^20] (got %d)", iters);
  if (clusters < 0) return fail(SHARQ_ERR_INVALID_ARG, "clusters must be >= 0");
  cudaError_t e = sharq::launch_mma_peak(mode, fmt, iters, clusters, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "sharq_mma_peak");
  g_err[0] = 0;
  return SHARQ_OK;
}

int sharq_device_status(void *stream) {
  int st = 0;
  uint32_t prep_st = 0;
  cudaError_t e = sharq::read_and_clear_device_status(&st, static_cast<cudaStream_t>(stream));
  if (e == cudaSuccess) e = sharq::read_and_clear_prep_status(&prep_st);
  if (e != cudaSuccess) return cuda_fail(e, "sharq_device_status");
  st |= (int)(prep_st << 1);
  if (st) return fail(SHARQ_ERR_TIMEOUT, "a bounded device wait gave up (code 0x%x)", st);
  g_err[0] = 0;
  return SHARQ_OK;
}

}  // extern "C"
