// C ABI entry points: argument checks, kernel selection, launches.
#include <math.h>
#include <stdlib.h>
#include <string.h>

#include <cmath>

#include <nvtx3/nvToolsExt.h>

#include "internal.cuh"

using namespace mla;

namespace {

int from_cuda(cudaError_t e) { return e == cudaSuccess ? MLA_OK : MLA_ERR_CUDA; }

// An NVTX range around an entry point, named after it, so that profilers can
// attribute the kernels each call launches (e.g. ncu --nvtx).  Without an
// attached tool the push and pop are no-ops.
struct Range {
  explicit Range(const char *name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
  Range(const Range &) = delete;
  Range &operator=(const Range &) = delete;
};

bool dtype_ok(int dt) { return dt == MLA_BF16 || dt == MLA_FP32; }

// Attention kernel for a configuration.  The tensor-core kernels exist for the
// DeepSeek-V2 attention shapes in bf16; everything else runs the generic
// CUDA-core kernel.
int choose_attn(const mla_config &c) {
  if (c.dtype != MLA_BF16) return kAttnSimt;
  if (c.d_c != 512 || c.d_r != 64) return kAttnSimt;
  if (c.page_size != 0 && c.page_size != kTile) return kAttnSimt;
  if (c.n_h == 128) return kAttnTcPair;
  if (c.n_h <= 32 && c.n_h % 16 == 0) return kAttnTcSmallH;
  return kAttnSimt;
}

int choose_gemm(const mla_config &c) {
  if (c.dtype != MLA_BF16) return kGemmSimt;
  // TMA needs 16-byte row pitches and the kernels tile d_c, d_h and d_model by 64.
  if (c.d_c % 128 != 0 || c.d_h % 64 != 0 || c.d_h > 256 || c.d_model % 64 != 0) return kGemmSimt;
  if (c.d_r % 16 != 0 || c.d_r > 128) return kGemmSimt;
  return kGemmTc;
}

int default_parts(const mla_handle *h) {
  switch (h->attn_kind) {
    case kAttnTcPair: return h->num_sms / 2;       // one CTA pair per two SMs
    case kAttnTcSmallH: return h->num_sms;         // one CTA per SM
    default: return h->num_sms * 4;
  }
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

// Tokens per tile of the split plan: the MMA tile of the attention kernel the
// handle runs (a share then never pays for a partial tile inside a sequence).
int plan_tile_of(const mla_handle *h, bool fp8) {
  if (h->attn_kind == kAttnTcPair && !fp8) return 256;
  if (h->attn_kind == kAttnTcSmallH) return 128;
  return kTile;
}

// Appends to theta[0 .. nth) (double) the float pairs (hi, lo) with
// hi + lo = theta[k] to about 2^-48 (the second half of the table).
void split_theta(double *theta, int nth) {
  float *pairs = reinterpret_cast<float *>(theta + nth);
  for (int k = 0; k < nth; ++k) {
    const float hi = (float)theta[k];
    pairs[2 * k] = hi;
    pairs[2 * k + 1] = (float)(theta[k] - (double)hi);
  }
}

// Strict mode: a tensor-core kernel that exists for the configuration but
// could not take the call's arguments is not replaced by a CUDA-core kernel.
bool strict_refuses(const mla_handle *h, bool tc_exists, cudaError_t e) {
  return h->strict && tc_exists && e == cudaErrorNotSupported;
}

}  // namespace

extern "C" {

const char *mla_status_string(int status) {
  switch (status) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_WORKSPACE: return "MLA_ERR_WORKSPACE";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
    case MLA_ERR_DEVICE_BOUNDS: return "MLA_ERR_DEVICE_BOUNDS";
    default: return "MLA_ERR_UNKNOWN";
  }
}

int mla_config_validate(const mla_config *c) {
  if (!c) return MLA_ERR_INVALID_ARG;
  if (c->n_h <= 0 || c->d_h <= 0 || c->d_c <= 0 || c->d_r <= 0 || c->d_model <= 0)
    return MLA_ERR_INVALID_ARG;
  if (c->d_r % 2 != 0 || c->page_size < 0 || !(c->rope_base > 0.0) || !dtype_ok(c->dtype))
    return MLA_ERR_INVALID_ARG;
  // Limits of the generic kernels (register tiles and shared-memory rows).
  if (c->d_c > 512 || c->d_c + c->d_r > 576 || c->d_model > 12288 || c->d_h > 4096)
    return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

int mla_create(const mla_config *cfg, mla_handle **out) {
  if (!out) return MLA_ERR_INVALID_ARG;
  *out = nullptr;
  int st = mla_config_validate(cfg);
  if (st != MLA_OK) return st;
  mla_handle *h = (mla_handle *)calloc(1, sizeof(mla_handle));
  if (!h) return MLA_ERR_CUDA;
  h->cfg = *cfg;
  if (cudaGetDevice(&h->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->num_sms, cudaDevAttrMultiProcessorCount, h->device) != cudaSuccess) {
    free(h);
    return MLA_ERR_CUDA;
  }
  h->attn_kind = choose_attn(*cfg);
  h->gemm_kind = choose_gemm(*cfg);
  h->score_mult = 1.0;
  if ((h->attn_kind != kAttnSimt || h->gemm_kind != kGemmSimt) && !tma_available()) {
    free(h);
    return MLA_ERR_CUDA;
  }
  if (noalloc_scratch_lookup(&h->noalloc_scratch) != MLA_OK) {
    free(h);
    return MLA_ERR_CUDA;
  }
  const int nth = cfg->d_r / 2;
  double *theta = (double *)malloc(2 * sizeof(double) * nth);
  for (int k = 0; k < nth; ++k) theta[k] = pow(cfg->rope_base, -2.0 * k / (double)cfg->d_r);
  split_theta(theta, nth);
  cudaError_t e = cudaMalloc(&h->d_status, sizeof(unsigned));
  if (e == cudaSuccess) e = cudaMalloc(&h->d_theta, 2 * sizeof(double) * nth);
  if (e == cudaSuccess) e = cudaMemset(h->d_status, 0, sizeof(unsigned));
  if (e == cudaSuccess) e = cudaMemcpy(h->d_theta, theta, 2 * sizeof(double) * nth, cudaMemcpyHostToDevice);
  free(theta);
  if (e != cudaSuccess) {
    mla_destroy(h);
    return MLA_ERR_CUDA;
  }
  *out = h;
  return MLA_OK;
}

void mla_destroy(mla_handle *h) {
  if (!h) return;
  if (h->d_status) cudaFree(h->d_status);
  if (h->d_theta) cudaFree(h->d_theta);
  free(h);
}

int mla_set_rope_scaling(mla_handle *h, double factor, int original_ctx, double alpha, double beta,
                         double mscale_coef) {
  if (!h || !(factor >= 1.0) || original_ctx <= 0 || !(alpha >= 0.0) || !(beta > alpha) ||
      !(mscale_coef >= 0.0) || !std::isfinite(factor) || !std::isfinite(beta) || !std::isfinite(mscale_coef))
    return MLA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev != h->device) return MLA_ERR_INVALID_ARG;
  const int d_r = h->cfg.d_r, nth = d_r / 2;
  double *theta = (double *)malloc(2 * sizeof(double) * (nth > 0 ? nth : 1));
  if (!theta) return MLA_ERR_CUDA;
  for (int k = 0; k < nth; ++k) {
    const double th = pow(h->cfg.rope_base, -2.0 * k / (double)d_r);
    double keep = 1.0;   // share of the original frequency (1: unchanged, 0: slowed by the factor)
    if (factor > 1.0) {
      const double turns = (double)original_ctx * th / (2.0 * 3.14159265358979323846);
      keep = (turns - alpha) / (beta - alpha);
      keep = keep < 0.0 ? 0.0 : (keep > 1.0 ? 1.0 : keep);
    }
    theta[k] = keep * th + (1.0 - keep) * th / factor;
  }
  split_theta(theta, nth);
  const cudaError_t e = cudaMemcpy(h->d_theta, theta, 2 * sizeof(double) * nth, cudaMemcpyHostToDevice);
  free(theta);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  const double m = factor > 1.0 ? mscale_coef * log(factor) + 1.0 : 1.0;
  h->score_mult = m * m;
  return MLA_OK;
}

int mla_set_strict(mla_handle *h, int strict) {
  if (!h) return MLA_ERR_INVALID_ARG;
  h->strict = strict ? 1 : 0;
  return MLA_OK;
}

int mla_cache_append(mla_handle *h, const void *x, int B, int T, const int *start_pos,
                     const void *w_dkv, const void *w_kr, void *cache, long long cache_len,
                     const int *block_table, int max_blocks_per_seq, mla_stream_t stream) {
  Range range("mla_cache_append");
  if (!h || B < 0 || T < 0 || cache_len < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return MLA_OK;
  if (!x || !start_pos || !w_dkv || !w_kr || !cache) return MLA_ERR_INVALID_ARG;
  const mla_config &c = h->cfg;
  if (c.page_size > 0 && (!block_table || max_blocks_per_seq <= 0)) return MLA_ERR_INVALID_ARG;
  if (c.page_size == 0 && block_table) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaErrorNotSupported;
  if (h->gemm_kind == kGemmTc)
    e = launch_append_tc(c, x, B, T, start_pos, w_dkv, w_kr, cache, cache_len, block_table,
                         max_blocks_per_seq, h->d_theta, h->d_status, s);
  if (strict_refuses(h, h->gemm_kind == kGemmTc, e)) return MLA_ERR_UNSUPPORTED;
  if (e == cudaErrorNotSupported)
    e = launch_append_simt(c, x, B, T, start_pos, w_dkv, w_kr, cache, cache_len, block_table,
                           max_blocks_per_seq, h->d_theta, h->d_status, s);
  if (e == cudaErrorNotSupported) return MLA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

int mla_absorb_q(mla_handle *h, const void *q_nope, const void *q_rope, const int *pos,
                 const void *w_uk, void *q_abs, int B, mla_stream_t stream) {
  Range range("mla_absorb_q");
  if (!h || B < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!q_nope || !q_rope || !pos || !w_uk || !q_abs) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaErrorNotSupported;
  if (h->gemm_kind == kGemmTc)
    e = launch_absorb_tc(h->cfg, q_nope, q_rope, pos, w_uk, q_abs, B, h->d_theta, h->d_status, s);
  if (strict_refuses(h, h->gemm_kind == kGemmTc, e)) return MLA_ERR_UNSUPPORTED;
  if (e == cudaErrorNotSupported)
    e = launch_absorb_simt(h->cfg, q_nope, q_rope, pos, w_uk, q_abs, B, h->d_theta, s);
  if (e == cudaErrorNotSupported) return MLA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

int mla_default_num_parts(const mla_handle *h) { return h ? default_parts(h) : 0; }

size_t mla_decode_workspace_size(const mla_handle *h, int B, int num_parts) {
  if (!h || B < 0 || num_parts < 0) return 0;
  const int P = num_parts == 0 ? default_parts(h) : num_parts;
  return ws_layout(h->cfg, B, P).total;
}

namespace {
// Decode attention over a cache in cfg.dtype (kv_scale NULL) or of FP8 codes
// with their group scales.
int decode_attn(mla_handle *h, const void *q_abs, const void *cache, const float *kv_scale,
                long long cache_len, const int *block_table, int max_blocks_per_seq, const int *ctx_begin,
                const int *ctx_len, int B, int num_parts, void *workspace, size_t ws_bytes,
                mla_stream_t stream) {
  if (!h || B < 0 || num_parts < 0 || cache_len < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!q_abs || !cache || !ctx_len) return MLA_ERR_INVALID_ARG;
  const mla_config &c = h->cfg;
  if (c.page_size > 0 && (!block_table || max_blocks_per_seq <= 0)) return MLA_ERR_INVALID_ARG;
  if (c.page_size == 0 && block_table) return MLA_ERR_INVALID_ARG;
  const int P = num_parts == 0 ? default_parts(h) : num_parts;
  const WsLayout L = ws_layout(c, B, P);
  if (!workspace || ((uintptr_t)workspace & 255u) || ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  // Tokens one sequence can address: the contiguous cache's capacity, or the
  // pages of its block-table row.
  const long long cap = c.page_size > 0 ? (long long)max_blocks_per_seq * c.page_size : cache_len;
  const long long cap_i = cap < 0x7fffffffLL ? cap : 0x7fffffffLL;
  const int tile = plan_tile_of(h, kv_scale != nullptr);
  cudaError_t e = launch_plan(ctx_begin, ctx_len, B, P, cap_i, tile, (char *)workspace, L, h->d_status, s);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  AttnArgs a;
  a.q_abs = q_abs;
  a.cache = cache;
  a.cache_len = cache_len;
  a.block_table = block_table;
  a.max_blocks = max_blocks_per_seq;
  a.page_size = c.page_size;
  a.B = B;
  a.n_h = c.n_h;
  a.d_c = c.d_c;
  a.d_r = c.d_r;
  a.scale_log2 = (float)(1.4426950408889634 * h->score_mult / sqrt((double)(c.d_h + c.d_r)));
  a.kv_scale = kv_scale;
  a.n_groups = fp8_num_groups(c.d_c, c.d_r);
  a.ws = (char *)workspace;
  a.L = L;
  a.plan_tile = tile;
  a.status = h->d_status;
  e = cudaErrorNotSupported;
  if (h->attn_kind == kAttnTcPair && !kv_scale && aligned16(q_abs) && aligned16(cache))
    e = launch_attn_tc_pair(a, P, s);
  else if (h->attn_kind == kAttnTcSmallH && aligned16(q_abs) && aligned16(cache))
    e = launch_attn_tc_smallh(a, P, s);
  const bool tc_exists = (h->attn_kind == kAttnTcPair && !kv_scale) || h->attn_kind == kAttnTcSmallH;
  if (strict_refuses(h, tc_exists, e)) return MLA_ERR_UNSUPPORTED;
  if (e == cudaErrorNotSupported) e = launch_attn_simt(a, P, c.dtype == MLA_FP32, s);
  if (e == cudaErrorNotSupported) return MLA_ERR_UNSUPPORTED;
  return from_cuda(e);
}
}  // namespace

int mla_decode_attn(mla_handle *h, const void *q_abs, const void *cache, long long cache_len,
                    const int *block_table, int max_blocks_per_seq, const int *ctx_len, int B,
                    int num_parts, void *workspace, size_t ws_bytes, mla_stream_t stream) {
  Range range("mla_decode_attn");
  return decode_attn(h, q_abs, cache, nullptr, cache_len, block_table, max_blocks_per_seq, nullptr, ctx_len, B,
                     num_parts, workspace, ws_bytes, stream);
}

int mla_decode_attn_fp8(mla_handle *h, const void *q_abs, const void *cache, const float *kv_scale,
                        long long cache_len, const int *block_table, int max_blocks_per_seq,
                        const int *ctx_len, int B, int num_parts, void *workspace, size_t ws_bytes,
                        mla_stream_t stream) {
  Range range("mla_decode_attn_fp8");
  if (!kv_scale && h && B > 0) return MLA_ERR_INVALID_ARG;
  return decode_attn(h, q_abs, cache, kv_scale, cache_len, block_table, max_blocks_per_seq, nullptr, ctx_len, B,
                     num_parts, workspace, ws_bytes, stream);
}

int mla_decode_attn_range(mla_handle *h, const void *q_abs, const void *cache, long long cache_len,
                          const int *block_table, int max_blocks_per_seq, const int *ctx_begin, const int *ctx_len,
                          int B, int num_parts, void *workspace, size_t ws_bytes, mla_stream_t stream) {
  Range range("mla_decode_attn_range");
  if (!ctx_begin && h && B > 0) return MLA_ERR_INVALID_ARG;
  return decode_attn(h, q_abs, cache, nullptr, cache_len, block_table, max_blocks_per_seq, ctx_begin, ctx_len, B,
                     num_parts, workspace, ws_bytes, stream);
}

int mla_fp8_scale_groups(const mla_handle *h) { return h ? fp8_num_groups(h->cfg.d_c, h->cfg.d_r) : 0; }

size_t mla_cache_append_fp8_workspace_size(const mla_handle *h, int B, int T) {
  if (!h || B < 0 || T < 0) return 0;
  const size_t n = (size_t)B * (size_t)T * (size_t)(h->cfg.d_c + h->cfg.d_r) * sizeof(float);
  return align_up(n > 0 ? n : 1, 256);
}

int mla_cache_append_fp8(mla_handle *h, const void *x, int B, int T, const int *start_pos,
                         const void *w_dkv, const void *w_kr, void *cache, float *kv_scale,
                         long long cache_len, const int *block_table, int max_blocks_per_seq,
                         void *workspace, size_t ws_bytes, mla_stream_t stream) {
  Range range("mla_cache_append_fp8");
  if (!h || B < 0 || T < 0 || cache_len < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0 || T == 0) return MLA_OK;
  if (!x || !start_pos || !w_dkv || !w_kr || !cache || !kv_scale) return MLA_ERR_INVALID_ARG;
  const mla_config &c = h->cfg;
  if (c.page_size > 0 && (!block_table || max_blocks_per_seq <= 0)) return MLA_ERR_INVALID_ARG;
  if (c.page_size == 0 && block_table) return MLA_ERR_INVALID_ARG;
  if (!workspace || ((uintptr_t)workspace & 255u) || ws_bytes < mla_cache_append_fp8_workspace_size(h, B, T))
    return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  float *rows = (float *)workspace;
  cudaError_t e = cudaErrorNotSupported;
  if (h->gemm_kind == kGemmTc)
    e = launch_append_tc(c, x, B, T, start_pos, w_dkv, w_kr, nullptr, 0, nullptr, 0, h->d_theta,
                         h->d_status, s, rows);
  if (strict_refuses(h, h->gemm_kind == kGemmTc, e)) return MLA_ERR_UNSUPPORTED;
  if (e == cudaErrorNotSupported)
    e = launch_append_simt(c, x, B, T, start_pos, w_dkv, w_kr, nullptr, 0, nullptr, 0, h->d_theta,
                           h->d_status, s, rows);
  if (e == cudaErrorNotSupported) return MLA_ERR_UNSUPPORTED;
  if (e != cudaSuccess) return from_cuda(e);
  e = launch_quantize_fp8(c, rows, true, (long long)B * T, T, start_pos, (uint8_t *)cache, kv_scale,
                          cache_len, block_table, max_blocks_per_seq, h->d_status, s);
  if (e == cudaErrorNotSupported) return MLA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

int mla_quantize_rows_fp8(mla_handle *h, const void *rows, long long n_rows, void *codes, float *kv_scale,
                          mla_stream_t stream) {
  Range range("mla_quantize_rows_fp8");
  if (!h || n_rows < 0) return MLA_ERR_INVALID_ARG;
  if (n_rows == 0) return MLA_OK;
  if (!rows || !codes || !kv_scale) return MLA_ERR_INVALID_ARG;
  const cudaError_t e = launch_quantize_fp8(h->cfg, rows, false, n_rows, 1, nullptr, (uint8_t *)codes,
                                            kv_scale, 0, nullptr, 0, h->d_status, (cudaStream_t)stream);
  if (e == cudaErrorNotSupported) return MLA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

int mla_combine_splits(mla_handle *h, const void *workspace, size_t ws_bytes, int B, int num_parts,
                       void *ctx_lat, float *lse, mla_stream_t stream) {
  Range range("mla_combine_splits");
  if (!h || B < 0 || num_parts < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!ctx_lat) return MLA_ERR_INVALID_ARG;
  const int P = num_parts == 0 ? default_parts(h) : num_parts;
  const WsLayout L = ws_layout(h->cfg, B, P);
  if (!workspace || ((uintptr_t)workspace & 255u) || ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  return from_cuda(launch_combine(h->cfg, (const char *)workspace, L, B, ctx_lat, lse,
                                  (cudaStream_t)stream));
}

int mla_combine_splits_f32(mla_handle *h, const void *workspace, size_t ws_bytes, int B, int num_parts,
                           float *ctx_lat, float *lse, mla_stream_t stream) {
  Range range("mla_combine_splits_f32");
  if (!h || B < 0 || num_parts < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!ctx_lat || !lse) return MLA_ERR_INVALID_ARG;
  const int P = num_parts == 0 ? default_parts(h) : num_parts;
  const WsLayout L = ws_layout(h->cfg, B, P);
  if (!workspace || ((uintptr_t)workspace & 255u) || ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  return from_cuda(launch_combine(h->cfg, (const char *)workspace, L, B, ctx_lat, lse, (cudaStream_t)stream,
                                  true));
}

int mla_merge_ranges(mla_handle *h, const float *ctx_parts, const float *lse_parts, int R, int B, void *ctx_lat,
                     float *lse, mla_stream_t stream) {
  Range range("mla_merge_ranges");
  if (!h || R < 0 || B < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (R == 0 || !ctx_parts || !lse_parts || !ctx_lat) return MLA_ERR_INVALID_ARG;
  return from_cuda(launch_merge_ranges(h->cfg, ctx_parts, lse_parts, R, B, ctx_lat, lse, (cudaStream_t)stream));
}

int mla_out_proj(mla_handle *h, const void *ctx_lat, const void *w_uv, const void *w_o, void *o,
                 void *u, int B, mla_stream_t stream) {
  Range range("mla_out_proj");
  if (!h || B < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!ctx_lat || !w_uv || !o || (w_o && !u)) return MLA_ERR_INVALID_ARG;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaErrorNotSupported;
  if (h->gemm_kind == kGemmTc) e = launch_outproj_tc(h->cfg, ctx_lat, w_uv, o, B, h->d_status, s);
  if (strict_refuses(h, h->gemm_kind == kGemmTc, e)) return MLA_ERR_UNSUPPORTED;
  if (e == cudaErrorNotSupported) e = launch_outproj_simt(h->cfg, ctx_lat, w_uv, o, B, s);
  if (e != cudaSuccess) return e == cudaErrorNotSupported ? MLA_ERR_UNSUPPORTED : MLA_ERR_CUDA;
  if (w_o) {
    e = cudaErrorNotSupported;
    if (h->gemm_kind == kGemmTc) e = launch_wo_tc(h->cfg, o, w_o, u, B, h->d_status, s);
    if (strict_refuses(h, h->gemm_kind == kGemmTc, e)) return MLA_ERR_UNSUPPORTED;
    if (e == cudaErrorNotSupported) e = launch_wo_simt(h->cfg, o, w_o, u, B, s);
    if (e != cudaSuccess) return e == cudaErrorNotSupported ? MLA_ERR_UNSUPPORTED : MLA_ERR_CUDA;
  }
  return MLA_OK;
}

int mla_combine_out_proj(mla_handle *h, const void *workspace, size_t ws_bytes, int B, int num_parts,
                         const void *w_uv, const void *w_o, void *o, void *u, void *ctx_lat, float *lse,
                         mla_stream_t stream) {
  Range range("mla_combine_out_proj");
  if (!h || B < 0 || num_parts < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!w_uv || !o || (w_o && !u)) return MLA_ERR_INVALID_ARG;
  const int P = num_parts == 0 ? default_parts(h) : num_parts;
  const WsLayout L = ws_layout(h->cfg, B, P);
  if (!workspace || ((uintptr_t)workspace & 255u) || ws_bytes < L.total) return MLA_ERR_WORKSPACE;
  cudaStream_t s = (cudaStream_t)stream;
  const char *ws = (const char *)workspace;
  cudaError_t e = cudaErrorNotSupported;
  if (h->gemm_kind == kGemmTc)
    e = launch_combine_outproj_tc(h->cfg, ws, L, B, w_uv, o, ctx_lat, lse, h->d_status, s);
  if (strict_refuses(h, h->gemm_kind == kGemmTc, e)) return MLA_ERR_UNSUPPORTED;
  if (e == cudaErrorNotSupported) e = launch_combine_outproj_simt(h->cfg, ws, L, B, w_uv, o, ctx_lat, lse, s);
  if (e != cudaSuccess) return e == cudaErrorNotSupported ? MLA_ERR_UNSUPPORTED : MLA_ERR_CUDA;
  if (w_o) {
    e = cudaErrorNotSupported;
    if (h->gemm_kind == kGemmTc) e = launch_wo_tc(h->cfg, o, w_o, u, B, h->d_status, s);
    if (strict_refuses(h, h->gemm_kind == kGemmTc, e)) return MLA_ERR_UNSUPPORTED;
    if (e == cudaErrorNotSupported) e = launch_wo_simt(h->cfg, o, w_o, u, B, s);
    if (e != cudaSuccess) return e == cudaErrorNotSupported ? MLA_ERR_UNSUPPORTED : MLA_ERR_CUDA;
  }
  return MLA_OK;
}

namespace {
// y[N, M] = x[N, K] w[M, K]^T on the handle's GEMM path, CUDA cores when the
// tensor-core kernel lacks the shape (or for fp32).
cudaError_t linear(const mla_handle *h, const void *x, const void *w, void *y, int M, int K, int N,
                   cudaStream_t s) {
  cudaError_t e = cudaErrorNotSupported;
  if (h->gemm_kind == kGemmTc) e = launch_linear_tc(x, w, y, M, K, N, h->d_status, s);
  if (strict_refuses(h, h->gemm_kind == kGemmTc, e)) return e;   // reported as MLA_ERR_UNSUPPORTED
  if (e == cudaErrorNotSupported) e = launch_linear_simt(x, w, y, M, K, N, h->cfg.dtype == MLA_FP32, s);
  return e;
}
}  // namespace

int mla_query_proj(mla_handle *h, const void *x, int B, const void *w_dq, int d_cq, const void *w_uq,
                   const void *w_qr, void *c_q, void *q_nope, void *q_rope, mla_stream_t stream) {
  Range range("mla_query_proj");
  if (!h || B < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!x || !w_uq || !w_qr || !q_nope || !q_rope) return MLA_ERR_INVALID_ARG;
  if (w_dq && (!c_q || d_cq <= 0)) return MLA_ERR_INVALID_ARG;
  const mla_config &c = h->cfg;
  cudaStream_t s = (cudaStream_t)stream;
  const void *src = x;
  int K = c.d_model;
  cudaError_t e = cudaSuccess;
  if (w_dq) {
    e = linear(h, x, w_dq, c_q, d_cq, c.d_model, B, s);
    src = c_q;
    K = d_cq;
  }
  if (e == cudaSuccess) e = linear(h, src, w_uq, q_nope, c.n_h * c.d_h, K, B, s);
  if (e == cudaSuccess) e = linear(h, src, w_qr, q_rope, c.n_h * c.d_r, K, B, s);
  if (e != cudaSuccess) return e == cudaErrorNotSupported ? MLA_ERR_UNSUPPORTED : MLA_ERR_CUDA;
  return MLA_OK;
}

int mla_selftest_wait_timeout(mla_handle *h, long long limit_ns, mla_stream_t stream) {
  if (!h || limit_ns < 1000 || limit_ns > 1000000000LL) return MLA_ERR_INVALID_ARG;
  return from_cuda(launch_wait_timeout_selftest(h->d_status, (unsigned long long)limit_ns,
                                                (cudaStream_t)stream));
}

int mla_get_device_status(mla_handle *h, mla_stream_t stream) {
  if (!h) return MLA_ERR_INVALID_ARG;
  unsigned v = 0;
  cudaStream_t s = (cudaStream_t)stream;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MLA_ERR_CUDA;
  if (cudaMemcpy(&v, h->d_status, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
  if (v && cudaMemset(h->d_status, 0, sizeof(unsigned)) != cudaSuccess) return MLA_ERR_CUDA;
  if (v & kStatusTimeout) return MLA_ERR_TIMEOUT;
  if (v & kStatusBounds) return MLA_ERR_DEVICE_BOUNDS;
  return MLA_OK;
}

long long mla_plan_pieces_tiled(const int *ctx_len, int B, int num_parts, int tile_tokens, long long *piece_base) {
  if (!ctx_len || !piece_base || B < 0 || num_parts <= 0 || tile_tokens < kTile || tile_tokens % kTile != 0)
    return -1;
  const int tile = tile_tokens;
  long long Ttot = 0;
  for (int b = 0; b < B; ++b) {
    if (ctx_len[b] < 0) return -1;
    Ttot += ceil_div_ll(ctx_len[b], tile);
  }
  const long long P = Ttot < num_parts ? Ttot : num_parts;
  long long s = 0, n = 0;
  for (int b = 0; b < B; ++b) {
    piece_base[b] = n;
    const long long t = ceil_div_ll(ctx_len[b], tile);
    if (t > 0) n += plan_share_of_tile(s + t - 1, P, Ttot) - plan_share_of_tile(s, P, Ttot) + 1;
    s += t;
  }
  piece_base[B] = n;
  return n;
}

long long mla_plan_pieces(const int *ctx_len, int B, int num_parts, long long *piece_base) {
  return mla_plan_pieces_tiled(ctx_len, B, num_parts, kTile, piece_base);
}

int mla_plan_tile(const mla_handle *h, int fp8) { return h ? plan_tile_of(h, fp8 != 0) : -1; }

}  // extern "C"
