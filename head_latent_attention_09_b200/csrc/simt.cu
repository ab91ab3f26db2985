// CUDA-core kernels: the split plan, the log-sum-exp combine, and generic
// (any shape, fp32 or bf16) versions of append / absorb / attention /
// output projection.  The fp32 configuration runs entirely here; bf16 shapes
// with a tensor-core kernel use those instead (see api.cu).
#include <cuda_fp8.h>
#include <math_constants.h>

#include "internal.cuh"

namespace mla {
namespace {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Row index (in units of D-element rows) of token p of sequence b, or -1 when
// the position is outside the cache / unmapped (the caller flags it).
__device__ __forceinline__ long long cache_row(int b, long long p, long long cache_len,
                                               const int *block_table, int max_blocks,
                                               int page_size) {
  if (p < 0) return -1;
  if (page_size == 0) {
    if (p >= cache_len) return -1;
    return (long long)b * cache_len + p;
  }
  long long bi = p / page_size;
  if (bi >= max_blocks) return -1;
  int blk = block_table[(long long)b * max_blocks + bi];
  if (blk < 0 || blk >= cache_len) return -1;
  return (long long)blk * page_size + (p % page_size);
}

// ---------------------------------------------------------------------------
// plan: one block of up to 1024 threads (a multiple of 32)
// ---------------------------------------------------------------------------
// Exclusive prefix sum over the block (thread order), and the total: a
// shuffle scan within each warp, then one warp scans the warp totals.
// `smem` holds 32 values.
__device__ long long block_exclusive_scan(long long v, long long *smem, long long *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) smem[warp] = x;
  __syncthreads();
  if (warp == 0) {
    long long t = lane < nw ? smem[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    if (lane < nw) smem[lane] = t;   // inclusive prefix of the warp totals
  }
  __syncthreads();
  const long long before = warp > 0 ? smem[warp - 1] : 0;
  *total = smem[nw - 1];
  __syncthreads();   // smem is reused by the next scan
  return before + x - v;
}

__global__ void __launch_bounds__(1024) plan_kernel(const int *ctx_begin, const int *ctx_len, int B, int P_req,
                                                    long long cap, int tile, char *ws, WsLayout L,
                                                    unsigned *status) {
  pdl_trigger();
  pdl_wait();   // the workspace may still be read by the previous step's combine
  __shared__ long long scan[32];
  long long *tile_prefix = reinterpret_cast<long long *>(ws + L.tile_prefix_off);
  long long *piece_base = reinterpret_cast<long long *>(ws + L.piece_base_off);
  int *ctx_eff = reinterpret_cast<int *>(ws + L.ctx_off);   // [B] ends, then [B] first tokens
  int *beg_eff = ctx_eff + B;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (B + nt - 1) / nt;
  const int b0 = min(B, tid * per), b1 = min(B, b0 + per);

  long long local = 0;
  for (int b = b0; b < b1; ++b) {
    // A length outside [0, cap] is flagged and clamped; the tiles below and
    // every attention kernel use the clamped length.
    long long c = ctx_len[b];
    if (c < 0 || c > cap) {
      atomicOr(status, kStatusBounds);
      c = c < 0 ? 0 : cap;
    }
    long long g = ctx_begin ? ctx_begin[b] : 0;
    if (g < 0 || g > c || g % kTile != 0) {
      atomicOr(status, kStatusBounds);
      g = g < 0 ? 0 : (g > c ? c : g);
      g -= g % kTile;
    }
    ctx_eff[b] = (int)c;
    beg_eff[b] = (int)g;
    local += ceil_div_ll(c - g, tile);
  }
  long long Ttot;
  long long run = block_exclusive_scan(local, scan, &Ttot);
  for (int b = b0; b < b1; ++b) {
    tile_prefix[b] = run;
    run += ceil_div_ll(ctx_eff[b] - beg_eff[b], tile);
  }
  if (tid == 0) tile_prefix[B] = Ttot;
  const long long P = Ttot < (long long)P_req ? Ttot : (long long)P_req;

  long long local_pieces = 0;
  for (int b = b0; b < b1; ++b) {
    long long s = tile_prefix[b];
    long long t = ceil_div_ll(ctx_eff[b] - beg_eff[b], tile);
    if (t > 0) local_pieces += plan_share_of_tile(s + t - 1, P, Ttot) - plan_share_of_tile(s, P, Ttot) + 1;
  }
  long long n_pieces;
  long long prun = block_exclusive_scan(local_pieces, scan, &n_pieces);
  for (int b = b0; b < b1; ++b) {
    piece_base[b] = prun;
    long long s = tile_prefix[b];
    long long t = ceil_div_ll(ctx_eff[b] - beg_eff[b], tile);
    if (t > 0) prun += plan_share_of_tile(s + t - 1, P, Ttot) - plan_share_of_tile(s, P, Ttot) + 1;
  }
  // Each share's first sequence (the first whose tiles reach past the share's
  // first tile), so that the attention kernels need no search; tile_prefix is
  // complete here (the scan above synchronised the block).
  int *share_first = reinterpret_cast<int *>(ws + L.share_first_off);
  for (long long w = tid; w < P; w += nt) {
    const long long t0 = plan_begin(w, P, Ttot);
    int lo = 0, hi = B;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (tile_prefix[mid + 1] <= t0) lo = mid + 1; else hi = mid;
    }
    share_first[w] = lo;
  }
  if (tid == 0) {
    piece_base[B] = n_pieces;
    WsHeader *hd = reinterpret_cast<WsHeader *>(ws);
    hd->B = B;
    hd->P = P;
    hd->Ttot = Ttot;
    hd->n_pieces = n_pieces;
    if (n_pieces > L.max_pieces) atomicOr(status, kStatusBounds);  // cannot happen by construction
  }
}

// ---------------------------------------------------------------------------
// generic attention: one warp per head, lanes split the row's features
// ---------------------------------------------------------------------------
constexpr int kSimtMaxD = 576;      // d_c + d_r
constexpr int kSimtMaxC = 512;      // d_c
constexpr int kQPerLane = kSimtMaxD / 32;
constexpr int kOPerLane = kSimtMaxC / 32;

__device__ __forceinline__ float e4m3_value(uint8_t c) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3)));
}

// Group of channel f of a cached row (see fp8_group_range).
__device__ __forceinline__ int fp8_group_of(int f, int d_c) {
  return f < d_c ? f / kFp8Group : (d_c + kFp8Group - 1) / kFp8Group + (f - d_c) / kFp8Group;
}

// T: element type of the query; F8: the cache holds E4M3 codes with group
// scales (else elements of type T).
template <typename T, bool F8>
__global__ void __launch_bounds__(256) attn_simt_kernel(AttnArgs a) {
  const WsHeader *hd = reinterpret_cast<const WsHeader *>(a.ws);
  const long long P = hd->P, Ttot = hd->Ttot;
  const int w = blockIdx.x;
  if (w >= P) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.y * (blockDim.x >> 5) + warp;
  if (h >= a.n_h) return;
  const int D = a.d_c + a.d_r;
  const long long *tp = reinterpret_cast<const long long *>(a.ws + a.L.tile_prefix_off);
  const long long *pb = reinterpret_cast<const long long *>(a.ws + a.L.piece_base_off);
  float *opart = reinterpret_cast<float *>(a.ws + a.L.opart_off);
  float *lse = reinterpret_cast<float *>(a.ws + a.L.lse_off);
  const T *cache = reinterpret_cast<const T *>(a.cache);
  const uint8_t *cache8 = reinterpret_cast<const uint8_t *>(a.cache);
  const T *qg = reinterpret_cast<const T *>(a.q_abs);

  const long long t0 = plan_begin(w, P, Ttot), t1 = plan_begin(w + 1, P, Ttot);
  // first sequence whose tiles reach past t0 (found by the plan)
  const int lo = reinterpret_cast<const int *>(a.ws + a.L.share_first_off)[w];
  for (int b = lo; b < a.B && tp[b] < t1; ++b) {
    const long long s0 = t0 > tp[b] ? t0 : tp[b];
    const long long s1 = t1 < tp[b + 1] ? t1 : tp[b + 1];
    if (s0 >= s1) continue;
    const long long piece = pb[b] + (w - plan_share_of_tile(tp[b], P, Ttot));
    const int ctx = plan_ctx(a.ws, a.L, b);
    const long long beg = plan_begin_tok(a.ws, a.L, b, a.B);
    const long long p_begin = beg + (s0 - tp[b]) * a.plan_tile;
    const long long p_end = min((long long)ctx, beg + (s1 - tp[b]) * a.plan_tile);

    float q[kQPerLane];
#pragma unroll
    for (int j = 0; j < kQPerLane; ++j) {
      const int f = lane + 32 * j;
      q[j] = f < D ? to_f(qg[((long long)b * a.n_h + h) * D + f]) : 0.f;
    }
    float o[kOPerLane];
#pragma unroll
    for (int j = 0; j < kOPerLane; ++j) o[j] = 0.f;
    float m = -CUDART_INF_F, l = 0.f;

    for (long long p = p_begin; p < p_end; ++p) {
      const long long row = cache_row(b, p, a.cache_len, a.block_table, a.max_blocks, a.page_size);
      if (row < 0) {
        if (lane == 0) atomicOr(a.status, kStatusBounds);
        continue;
      }
      float val[kQPerLane];
#pragma unroll
      for (int j = 0; j < kQPerLane; ++j) {
        const int f = lane + 32 * j;
        val[j] = 0.f;
        if (f < D) {
          if (F8) val[j] = e4m3_value(cache8[row * D + f]) * a.kv_scale[row * a.n_groups + fp8_group_of(f, a.d_c)];
          else val[j] = to_f(cache[row * D + f]);
        }
      }
      float part = 0.f;
#pragma unroll
      for (int j = 0; j < kQPerLane; ++j) part += q[j] * val[j];
      const float s = warp_sum(part) * a.scale_log2;   // score in log2 units
      const float m_new = fmaxf(m, s);
      const float corr = exp2f(m - m_new);
      const float pr = exp2f(s - m_new);
      l = l * corr + pr;
#pragma unroll
      for (int j = 0; j < kOPerLane; ++j) {
        const int f = lane + 32 * j;
        if (f < a.d_c) o[j] = o[j] * corr + pr * val[j];
      }
      m = m_new;
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float *dst = opart + part_row(a.L, piece, h) * (long long)a.d_c;
#pragma unroll
    for (int j = 0; j < kOPerLane; ++j) {
      const int f = lane + 32 * j;
      if (f < a.d_c) dst[f] = o[j] * inv;
    }
    if (lane == 0)
      lse[part_row(a.L, piece, h)] = l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
  }
}

// ---------------------------------------------------------------------------
// log-sum-exp combine, generic form: one block per (sequence, head)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(128) combine_kernel(const char *ws, WsLayout L, int n_h, int d_c,
                                                      T *ctx_lat, float *lse_out) {
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, h = blockIdx.y;
  const long long *pb = reinterpret_cast<const long long *>(ws + L.piece_base_off);
  const float *lse = reinterpret_cast<const float *>(ws + L.lse_off);
  const float *op = reinterpret_cast<const float *>(ws + L.opart_off);
  const long long p0 = pb[b], p1 = pb[b + 1];
  float m = -CUDART_INF_F;
  for (long long p = p0; p < p1; ++p) m = fmaxf(m, lse[part_row(L, p, h)]);
  T *dst = ctx_lat + ((long long)b * n_h + h) * d_c;
  if (m == -CUDART_INF_F) {
    for (int f = threadIdx.x; f < d_c; f += blockDim.x) dst[f] = from_f<T>(0.f);
    if (lse_out && threadIdx.x == 0) lse_out[(long long)b * n_h + h] = -CUDART_INF_F;
    return;
  }
  float tot = 0.f;
  for (long long p = p0; p < p1; ++p) tot += expf(lse[part_row(L, p, h)] - m);
  const float inv = 1.f / tot;
  for (int f = threadIdx.x; f < d_c; f += blockDim.x) {
    float acc = 0.f;
    for (long long p = p0; p < p1; ++p)
      acc += expf(lse[part_row(L, p, h)] - m) * op[part_row(L, p, h) * (long long)d_c + f];
    dst[f] = from_f<T>(acc * inv);
  }
  if (lse_out && threadIdx.x == 0) lse_out[(long long)b * n_h + h] = m + logf(tot);
}

// ---------------------------------------------------------------------------
// cache append: one block per token; each warp computes a pair of features
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) append_simt_kernel(
    const T *h, int T_new, int d, int d_c, int d_r, const int *start_pos, const T *w_dkv,
    const T *w_kr, T *cache, long long cache_len, const int *block_table, int max_blocks,
    int page_size, const double *theta, unsigned *status, float *rows_out) {
  extern __shared__ float sh[];
  const long long tok = blockIdx.x;
  const int b = (int)(tok / T_new), t = (int)(tok % T_new);
  for (int k = threadIdx.x; k < d; k += blockDim.x) sh[k] = to_f(h[tok * d + k]);
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int D = d_c + d_r;
  const int f0 = 2 * (blockIdx.y * (blockDim.x >> 5) + warp);
  if (f0 >= D) return;
  const T *w0 = f0 < d_c ? w_dkv + (long long)f0 * d : w_kr + (long long)(f0 - d_c) * d;
  const T *w1 = w0 + d;
  float a0 = 0.f, a1 = 0.f;
  for (int k = lane; k < d; k += 32) {
    a0 += to_f(w0[k]) * sh[k];
    a1 += to_f(w1[k]) * sh[k];
  }
  a0 = warp_sum(a0);
  a1 = warp_sum(a1);
  if (lane != 0) return;
  const long long p = (long long)start_pos[b] + t;
  if (f0 >= d_c) {
    double sn, cs;
    sincos((double)p * theta[(f0 - d_c) >> 1], &sn, &cs);
    const float c = (float)cs, s = (float)sn;
    const float r0 = a0 * c - a1 * s, r1 = a0 * s + a1 * c;
    a0 = r0;
    a1 = r1;
  }
  if (rows_out) {
    rows_out[tok * D + f0] = a0;
    rows_out[tok * D + f0 + 1] = a1;
    return;
  }
  const long long row = cache_row(b, p, cache_len, block_table, max_blocks, page_size);
  if (row < 0) {
    atomicOr(status, kStatusBounds);
    return;
  }
  cache[row * D + f0] = from_f<T>(a0);
  cache[row * D + f0 + 1] = from_f<T>(a1);
}

// ---------------------------------------------------------------------------
// FP8 E4M3 quantisation of cached rows: one warp per row; per 128-channel
// group (over c^KV, then over k^R) sigma = amax / 448 and the codes of
// x / sigma, both divisions rounded to nearest in float32, the conversion
// rounding to nearest even and saturating at 448.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ void fp8_group_range(int g, int d_c, int d_r, int &a, int &e) {
  const int gc = (d_c + kFp8Group - 1) / kFp8Group;
  if (g < gc) {
    a = g * kFp8Group;
    e = min(a + kFp8Group, d_c);
  } else {
    a = d_c + (g - gc) * kFp8Group;
    e = min(a + kFp8Group, d_c + d_r);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) quantize_fp8_kernel(
    const T *src, long long n_rows, int d_c, int d_r, int T_new, const int *start_pos,
    uint8_t *codes, float *scales, long long cache_len, const int *block_table, int max_blocks,
    int page_size, unsigned *status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long r = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  if (r >= n_rows) return;
  long long dst = r;
  if (start_pos) {
    const int b = (int)(r / T_new), t = (int)(r % T_new);
    dst = cache_row(b, (long long)start_pos[b] + t, cache_len, block_table, max_blocks, page_size);
    if (dst < 0) {
      if (lane == 0) atomicOr(status, kStatusBounds);
      return;
    }
  }
  const int D = d_c + d_r, G = fp8_num_groups(d_c, d_r);
  const T *x = src + r * D;
  uint8_t *out = codes + dst * D;
  for (int g = 0; g < G; ++g) {
    int a, e;
    fp8_group_range(g, d_c, d_r, a, e);
    float amax = 0.f;
    for (int f = a + lane; f < e; f += 32) amax = fmaxf(amax, fabsf(to_f(x[f])));
    amax = warp_max(amax);
    const float sigma = __fdiv_rn(amax, 448.f);
    for (int f = a + lane; f < e; f += 32)
      out[f] = sigma > 0.f ? (uint8_t)__nv_cvt_float_to_fp8(__fdiv_rn(to_f(x[f]), sigma), __NV_SATFINITE, __NV_E4M3)
                           : (uint8_t)0;
    if (lane == 0) scales[dst * G + g] = sigma;
  }
}

// ---------------------------------------------------------------------------
// query absorption: one block per (sequence, head)
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) absorb_simt_kernel(const T *q_nope, const T *q_rope,
                                                          const int *pos, const T *w_uk, T *q_abs,
                                                          int n_h, int d_h, int d_c, int d_r,
                                                          const double *theta) {
  extern __shared__ float sq[];
  const int b = blockIdx.x, i = blockIdx.y;
  const long long bi = (long long)b * n_h + i;
  for (int r = threadIdx.x; r < d_h; r += blockDim.x) sq[r] = to_f(q_nope[bi * d_h + r]);
  __syncthreads();
  const int D = d_c + d_r;
  for (int m = threadIdx.x; m < d_c; m += blockDim.x) {
    float acc = 0.f;
    for (int r = 0; r < d_h; ++r) acc += to_f(w_uk[((long long)i * d_h + r) * d_c + m]) * sq[r];
    q_abs[bi * D + m] = from_f<T>(acc);
  }
  const double p = (double)pos[b];
  for (int k = threadIdx.x; k < d_r / 2; k += blockDim.x) {
    const float x0 = to_f(q_rope[bi * d_r + 2 * k]), x1 = to_f(q_rope[bi * d_r + 2 * k + 1]);
    double sn, cs;
    sincos(p * theta[k], &sn, &cs);
    const float c = (float)cs, s = (float)sn;
    q_abs[bi * D + d_c + 2 * k] = from_f<T>(x0 * c - x1 * s);
    q_abs[bi * D + d_c + 2 * k + 1] = from_f<T>(x0 * s + x1 * c);
  }
}

// ---------------------------------------------------------------------------
// output projection: one block per (sequence, head), one warp per output
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) outproj_simt_kernel(const T *ctx, const T *w_uv, T *o,
                                                           int n_h, int d_h, int d_c) {
  const int b = blockIdx.x, i = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const T *c = ctx + ((long long)b * n_h + i) * d_c;
  for (int r = warp; r < d_h; r += nw) {
    const T *wr = w_uv + ((long long)i * d_h + r) * d_c;
    float acc = 0.f;
    for (int k = lane; k < d_c; k += 32) acc += to_f(wr[k]) * to_f(c[k]);
    acc = warp_sum(acc);
    if (lane == 0) o[((long long)b * n_h + i) * d_h + r] = from_f<T>(acc);
  }
}

// Split combine fused with the output projection, CUDA-core form: one block
// per (sequence, head).  The merge is the vectorised combine's arithmetic per
// element (weights exp(lse_p - max) / sum, accumulated in piece order), the
// merged row is rounded to the dtype as ctx_lat would be, and the projection
// is the output-projection kernel's, reading the row from shared memory.
template <typename T>
__global__ void __launch_bounds__(256) combine_outproj_simt_kernel(const char *ws, WsLayout L, int n_h, int d_h,
                                                                   int d_c, const T *w_uv, T *o, T *ctx_lat,
                                                                   float *lse_out) {
  extern __shared__ float sctx[];   // [d_c]
  __shared__ float s_m, s_inv;
  pdl_trigger();
  pdl_wait();
  const int b = blockIdx.x, h = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
  const long long row = (long long)b * n_h + h;
  const long long *pb = reinterpret_cast<const long long *>(ws + L.piece_base_off);
  const float *lse = reinterpret_cast<const float *>(ws + L.lse_off);
  const float *op = reinterpret_cast<const float *>(ws + L.opart_off);
  const long long p0 = pb[b], p1 = pb[b + 1];
  if (warp == 0) {
    float m = -CUDART_INF_F;
    for (long long p = p0 + lane; p < p1; p += 32) m = fmaxf(m, lse[part_row(L, p, h)]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
    float tot = 0.f;
    if (m != -CUDART_INF_F)
      for (long long p = p0 + lane; p < p1; p += 32) tot += expf(lse[part_row(L, p, h)] - m);
    tot = warp_sum(tot);
    if (lane == 0) {
      s_m = m;
      s_inv = m == -CUDART_INF_F ? 0.f : 1.f / tot;
      if (lse_out) lse_out[row] = m == -CUDART_INF_F ? -CUDART_INF_F : m + logf(tot);
    }
  }
  __syncthreads();
  const float m = s_m, inv = s_inv;
  for (int c = threadIdx.x; c < d_c; c += blockDim.x) {
    float acc = 0.f;
    if (m != -CUDART_INF_F)
      for (long long p = p0; p < p1; ++p) {
        const float w = expf(lse[part_row(L, p, h)] - m) * inv;
        acc += w * op[part_row(L, p, h) * (long long)d_c + c];
      }
    const T v = from_f<T>(acc);
    if (ctx_lat) ctx_lat[row * d_c + c] = v;
    sctx[c] = to_f(v);
  }
  __syncthreads();
  for (int r = warp; r < d_h; r += nw) {
    const T *wr = w_uv + ((long long)h * d_h + r) * d_c;
    float acc = 0.f;
    for (int k = lane; k < d_c; k += 32) acc += to_f(wr[k]) * sctx[k];
    acc = warp_sum(acc);
    if (lane == 0) o[row * d_h + r] = from_f<T>(acc);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) linear_simt_kernel(const T *o, const T *w_o, T *u, int K, int d) {
  const int b = blockIdx.x;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j = blockIdx.y * (blockDim.x >> 5) + warp;
  if (j >= d) return;
  const T *wr = w_o + (long long)j * K;
  const T *x = o + (long long)b * K;
  float acc = 0.f;
  for (int k = lane; k < K; k += 32) acc += to_f(wr[k]) * to_f(x[k]);
  acc = warp_sum(acc);
  if (lane == 0) u[(long long)b * d + j] = from_f<T>(acc);
}

}  // namespace

// ---------------------------------------------------------------------------
// launchers
// ---------------------------------------------------------------------------
cudaError_t launch_plan(const int *ctx_begin, const int *ctx_len, int B, int P, long long cap, int tile, char *ws,
                        const WsLayout &L, unsigned *status, cudaStream_t s) {
  if (tile < kTile || tile % kTile != 0) return cudaErrorInvalidValue;
  // one thread per sequence up to 1024 (each thread takes a run of sequences beyond)
  const int threads = B >= 1024 ? 1024 : (B <= 32 ? 32 : (B + 31) / 32 * 32);
  return launch_pdl(plan_kernel, dim3(1), dim3(threads), 0, s, 1, ctx_begin, ctx_len, B, P, cap, tile, ws, L,
                    status);
}

cudaError_t launch_attn_simt(const AttnArgs &a, int P, bool fp32, cudaStream_t s) {
  if (a.d_c + a.d_r > kSimtMaxD || a.d_c > kSimtMaxC) return cudaErrorNotSupported;
  const int warps = a.n_h < 8 ? a.n_h : 8;
  dim3 grid(P, (a.n_h + warps - 1) / warps);
  const bool f8 = a.kv_scale != nullptr;
  if (fp32 && f8) attn_simt_kernel<float, true><<<grid, warps * 32, 0, s>>>(a);
  else if (fp32) attn_simt_kernel<float, false><<<grid, warps * 32, 0, s>>>(a);
  else if (f8) attn_simt_kernel<__nv_bfloat16, true><<<grid, warps * 32, 0, s>>>(a);
  else attn_simt_kernel<__nv_bfloat16, false><<<grid, warps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

// Vectorised combine for d_c a multiple of 4 and at most 512: one warp per
// (sequence, head), 8 per block.  The warp reduces the pieces' log-sum-exps
// across its lanes, then each lane accumulates up to four float4 columns of
// the weighted partials, with the loads of several pieces in flight at once.
template <typename T>
__device__ __forceinline__ void store4(T *dst, float4 v);
template <>
__device__ __forceinline__ void store4<float>(float *dst, float4 v) {
  *reinterpret_cast<float4 *>(dst) = v;
}
template <>
__device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16 *dst, float4 v) {
  __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y), hi = __floats2bfloat162_rn(v.z, v.w);
  uint2 u;
  u.x = *reinterpret_cast<uint32_t *>(&lo);
  u.y = *reinterpret_cast<uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(dst) = u;
}

template <typename T>
__global__ void __launch_bounds__(256) combine_vec_kernel(const char *ws, WsLayout L, int B, int n_h, int d_c,
                                                          T *ctx_lat, float *lse_out) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + warp;   // = b * n_h + h
  if (row >= (long long)B * n_h) return;
  const int b = (int)(row / n_h), h = (int)(row % n_h);
  const long long *pb = reinterpret_cast<const long long *>(ws + L.piece_base_off);
  const float *lse = reinterpret_cast<const float *>(ws + L.lse_off);
  const float *op = reinterpret_cast<const float *>(ws + L.opart_off);
  const long long p0 = pb[b], p1 = pb[b + 1];
  float m = -CUDART_INF_F;
  for (long long p = p0 + lane; p < p1; p += 32) m = fmaxf(m, lse[part_row(L, p, h)]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  T *dst = ctx_lat + row * d_c;
  const int n4 = d_c / 4;
  if (m == -CUDART_INF_F) {
    for (int f = lane; f < n4; f += 32) store4<T>(dst + 4 * f, make_float4(0.f, 0.f, 0.f, 0.f));
    if (lse_out && lane == 0) lse_out[row] = -CUDART_INF_F;
    return;
  }
  float tot = 0.f;
  for (long long p = p0 + lane; p < p1; p += 32) tot += expf(lse[part_row(L, p, h)] - m);
  tot = warp_sum(tot);
  const float inv = 1.f / tot;
  float4 acc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
  for (long long p = p0; p < p1; ++p) {
    const float w = expf(lse[part_row(L, p, h)] - m) * inv;
    const float4 *src = reinterpret_cast<const float4 *>(op + part_row(L, p, h) * (long long)d_c);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int f = lane + 32 * i;
      if (f < n4) {
        const float4 v = __ldg(src + f);
        acc[i].x += w * v.x;
        acc[i].y += w * v.y;
        acc[i].z += w * v.z;
        acc[i].w += w * v.w;
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int f = lane + 32 * i;
    if (f < n4) store4<T>(dst + 4 * f, acc[i]);
  }
  if (lse_out && lane == 0) lse_out[row] = m + logf(tot);
}

cudaError_t launch_combine(const mla_config &cfg, const char *ws, const WsLayout &L, int B,
                           void *ctx_lat, float *lse, cudaStream_t s, bool out_f32) {
  const bool f32 = out_f32 || cfg.dtype == MLA_FP32;
  const size_t esz = f32 ? 4 : 2;
  if (cfg.d_c % 4 == 0 && cfg.d_c <= 512 && ((uintptr_t)ctx_lat % (4 * esz)) == 0 &&
      ((uintptr_t)ws % 16) == 0) {
    const long long rows = (long long)B * cfg.n_h;
    const unsigned blocks = (unsigned)((rows + 7) / 8);
    if (f32)
      return launch_pdl(combine_vec_kernel<float>, dim3(blocks), dim3(256), 0, s, 1, ws, L, B, cfg.n_h, cfg.d_c,
                        (float *)ctx_lat, lse);
    else
      return launch_pdl(combine_vec_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, s, 1, ws, L, B, cfg.n_h,
                        cfg.d_c, (__nv_bfloat16 *)ctx_lat, lse);
  }
  dim3 grid(B, cfg.n_h);
  if (f32)
    return launch_pdl(combine_kernel<float>, grid, dim3(128), 0, s, 1, ws, L, cfg.n_h, cfg.d_c, (float *)ctx_lat, lse);
  else
    return launch_pdl(combine_kernel<__nv_bfloat16>, grid, dim3(128), 0, s, 1, ws, L, cfg.n_h, cfg.d_c,
                      (__nv_bfloat16 *)ctx_lat, lse);
}

// ---------------------------------------------------------------------------
// merge of R token-range results (split-KV across devices): one warp per
// (sequence, head) row; the same log-sum-exp algebra as the combine, over the
// R float32 results [R, B, n_h, d_c] and their log-sum-exps [R, B, n_h], in
// range order.
// ---------------------------------------------------------------------------
template <typename T>
__global__ void __launch_bounds__(256) merge_ranges_kernel(const float *parts, const float *lse_parts, int R,
                                                           int B, int n_h, int d_c, T *ctx_lat, float *lse_out) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * 8 + warp;   // = b * n_h + h
  const long long rows = (long long)B * n_h;
  if (row >= rows) return;
  float m = -CUDART_INF_F;
  for (int r = lane; r < R; r += 32) m = fmaxf(m, lse_parts[r * rows + row]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  T *dst = ctx_lat + row * d_c;
  if (m == -CUDART_INF_F) {
    for (int f = lane; f < d_c; f += 32) dst[f] = from_f<T>(0.f);
    if (lse_out && lane == 0) lse_out[row] = -CUDART_INF_F;
    return;
  }
  float tot = 0.f;
  for (int r = lane; r < R; r += 32) tot += expf(lse_parts[r * rows + row] - m);
  tot = warp_sum(tot);
  const float inv = 1.f / tot;
  for (int f = lane; f < d_c; f += 32) {
    float acc = 0.f;
    for (int r = 0; r < R; ++r) acc += expf(lse_parts[r * rows + row] - m) * inv * parts[(r * rows + row) * d_c + f];
    dst[f] = from_f<T>(acc);
  }
  if (lse_out && lane == 0) lse_out[row] = m + logf(tot);
}

cudaError_t launch_merge_ranges(const mla_config &cfg, const float *parts, const float *lse_parts, int R, int B,
                                void *ctx_lat, float *lse, cudaStream_t s) {
  const long long rows = (long long)B * cfg.n_h;
  const unsigned blocks = (unsigned)((rows + 7) / 8);
  if (cfg.dtype == MLA_FP32)
    return launch_pdl(merge_ranges_kernel<float>, dim3(blocks), dim3(256), 0, s, 1, parts, lse_parts, R, B,
                      cfg.n_h, cfg.d_c, (float *)ctx_lat, lse);
  return launch_pdl(merge_ranges_kernel<__nv_bfloat16>, dim3(blocks), dim3(256), 0, s, 1, parts, lse_parts, R, B,
                    cfg.n_h, cfg.d_c, (__nv_bfloat16 *)ctx_lat, lse);
}

cudaError_t launch_append_simt(const mla_config &cfg, const void *h, int B, int T,
                               const int *start_pos, const void *w_dkv, const void *w_kr,
                               void *cache, long long cache_len, const int *block_table,
                               int max_blocks, const double *theta, unsigned *status,
                               cudaStream_t s, float *rows_out) {
  const int D = cfg.d_c + cfg.d_r;
  dim3 grid((unsigned)((long long)B * T), (D / 2 + 7) / 8);
  const size_t smem = sizeof(float) * cfg.d_model;
  if (smem > 48 * 1024) return cudaErrorNotSupported;
  if (cfg.dtype == MLA_FP32)
    append_simt_kernel<float><<<grid, 256, smem, s>>>(
        (const float *)h, T, cfg.d_model, cfg.d_c, cfg.d_r, start_pos, (const float *)w_dkv,
        (const float *)w_kr, (float *)cache, cache_len, block_table, max_blocks, cfg.page_size,
        theta, status, rows_out);
  else
    append_simt_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(
        (const __nv_bfloat16 *)h, T, cfg.d_model, cfg.d_c, cfg.d_r, start_pos,
        (const __nv_bfloat16 *)w_dkv, (const __nv_bfloat16 *)w_kr, (__nv_bfloat16 *)cache,
        cache_len, block_table, max_blocks, cfg.page_size, theta, status, rows_out);
  return cudaGetLastError();
}

cudaError_t launch_quantize_fp8(const mla_config &cfg, const void *src, bool src_f32, long long n_rows,
                                int T, const int *start_pos, uint8_t *codes, float *scales,
                                long long cache_len, const int *block_table, int max_blocks,
                                unsigned *status, cudaStream_t s) {
  if (n_rows <= 0) return cudaSuccess;
  const long long blocks = (n_rows + 7) / 8;
  if (blocks > 0x7fffffffLL) return cudaErrorNotSupported;
  if (src_f32 || cfg.dtype == MLA_FP32)
    quantize_fp8_kernel<float><<<(unsigned)blocks, 256, 0, s>>>(
        (const float *)src, n_rows, cfg.d_c, cfg.d_r, T, start_pos, codes, scales, cache_len,
        block_table, max_blocks, cfg.page_size, status);
  else
    quantize_fp8_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, s>>>(
        (const __nv_bfloat16 *)src, n_rows, cfg.d_c, cfg.d_r, T, start_pos, codes, scales, cache_len,
        block_table, max_blocks, cfg.page_size, status);
  return cudaGetLastError();
}

cudaError_t launch_absorb_simt(const mla_config &cfg, const void *q_nope, const void *q_rope,
                               const int *pos, const void *w_uk, void *q_abs, int B,
                               const double *theta, cudaStream_t s) {
  dim3 grid(B, cfg.n_h);
  const size_t smem = sizeof(float) * cfg.d_h;
  if (cfg.dtype == MLA_FP32)
    absorb_simt_kernel<float><<<grid, 256, smem, s>>>(
        (const float *)q_nope, (const float *)q_rope, pos, (const float *)w_uk, (float *)q_abs,
        cfg.n_h, cfg.d_h, cfg.d_c, cfg.d_r, theta);
  else
    absorb_simt_kernel<__nv_bfloat16><<<grid, 256, smem, s>>>(
        (const __nv_bfloat16 *)q_nope, (const __nv_bfloat16 *)q_rope, pos,
        (const __nv_bfloat16 *)w_uk, (__nv_bfloat16 *)q_abs, cfg.n_h, cfg.d_h, cfg.d_c, cfg.d_r,
        theta);
  return cudaGetLastError();
}

cudaError_t launch_outproj_simt(const mla_config &cfg, const void *ctx_lat, const void *w_uv,
                                void *o, int B, cudaStream_t s) {
  dim3 grid(B, cfg.n_h);
  if (cfg.dtype == MLA_FP32)
    outproj_simt_kernel<float><<<grid, 256, 0, s>>>((const float *)ctx_lat, (const float *)w_uv,
                                                    (float *)o, cfg.n_h, cfg.d_h, cfg.d_c);
  else
    outproj_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(
        (const __nv_bfloat16 *)ctx_lat, (const __nv_bfloat16 *)w_uv, (__nv_bfloat16 *)o, cfg.n_h,
        cfg.d_h, cfg.d_c);
  return cudaGetLastError();
}

cudaError_t launch_combine_outproj_simt(const mla_config &cfg, const char *ws, const WsLayout &L, int B,
                                        const void *w_uv, void *o, void *ctx_lat, float *lse, cudaStream_t s) {
  if (B > 0x7fffffff || cfg.n_h > 65535) return cudaErrorNotSupported;
  const dim3 grid(B, cfg.n_h);
  const size_t smem = sizeof(float) * cfg.d_c;
  if (cfg.dtype == MLA_FP32)
    return launch_pdl(combine_outproj_simt_kernel<float>, grid, dim3(256), smem, s, 1, ws, L, cfg.n_h, cfg.d_h,
                      cfg.d_c, (const float *)w_uv, (float *)o, (float *)ctx_lat, lse);
  return launch_pdl(combine_outproj_simt_kernel<__nv_bfloat16>, grid, dim3(256), smem, s, 1, ws, L, cfg.n_h,
                    cfg.d_h, cfg.d_c, (const __nv_bfloat16 *)w_uv, (__nv_bfloat16 *)o, (__nv_bfloat16 *)ctx_lat,
                    lse);
}

cudaError_t launch_linear_simt(const void *x, const void *w, void *y, int M, int K, int N, bool fp32,
                               cudaStream_t s) {
  // y[N, M] = x[N, K] w[M, K]^T: one warp per output element.
  if (M <= 0 || N <= 0 || K <= 0 || (M + 7) / 8 > 65535) return cudaErrorNotSupported;
  dim3 grid(N, (M + 7) / 8);
  if (fp32)
    linear_simt_kernel<float><<<grid, 256, 0, s>>>((const float *)x, (const float *)w, (float *)y, K, M);
  else
    linear_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>((const __nv_bfloat16 *)x, (const __nv_bfloat16 *)w,
                                                       (__nv_bfloat16 *)y, K, M);
  return cudaGetLastError();
}

cudaError_t launch_wo_simt(const mla_config &cfg, const void *o, const void *w_o, void *u, int B,
                           cudaStream_t s) {
  return launch_linear_simt(o, w_o, u, cfg.d_model, cfg.n_h * cfg.d_h, B, cfg.dtype == MLA_FP32, s);
}

}  // namespace mla
