// Internal declarations shared by the host runtime and the kernels of the MLA
// decode library.  Nothing here is part of the public ABI (see include/mla.h).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "mla.h"

namespace mla {

// Devices a process may drive (per-device launch set-up is kept per index).
constexpr int kMaxDevices = 64;

// KV tokens per page of the paged fast paths (page_size == kTile), the
// granularity of a token range's first token, and the smallest tile of the
// split plan.
constexpr int kTile = 64;

// FP8 latent cache: channels per scale group (over c^KV, then over k^R).
constexpr int kFp8Group = 128;
__host__ __device__ inline int fp8_num_groups(int d_c, int d_r) {
  return (d_c + kFp8Group - 1) / kFp8Group + (d_r + kFp8Group - 1) / kFp8Group;
}

// Bits of the device status word.
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusBounds = 2u;

// Attention kernel chosen for a configuration at mla_create time.
enum AttnKind : int {
  kAttnSimt = 0,      // generic CUDA-core kernel (any shape, fp32 or bf16)
  kAttnTcPair = 1,    // bf16, n_h == 128, d_c == 512, d_r == 64: tcgen05, CTA pair
  kAttnTcSmallH = 2,  // bf16, n_h <= 32 (multiple of 16), d_c == 512, d_r == 64
};

enum GemmKind : int { kGemmSimt = 0, kGemmTc = 1 };

}  // namespace mla

namespace mla {

// cos and sin of the rotary angle pos * theta in single precision, accurate
// at positions up to 2^24.  theta is given as an unevaluated float sum
// hi + lo (its double value split in two); the product pos * hi is kept with
// its exact rounding error (fma), so the angle carries ~2^-48 relative error
// (a plain float product would err by ~1e-2 rad near position 131072), and it
// is reduced to [-pi, pi] with a three-part split of 2 pi (Cody and Waite).
// Error of the reduced angle: a few 1e-7 rad; the hardware sine and cosine on
// [-pi, pi] add at most ~4e-7 (far below the bf16 rounding of the results).
__device__ __forceinline__ void rope_sincos(int pos, float2 theta, float *s, float *c) {
  const float p = (float)pos;                                   // exact below 2^24
  const float a_hi = p * theta.x;
  const float a_lo = fmaf(p, theta.x, -a_hi) + p * theta.y;
  const float k = rintf(a_hi * 0.15915494309189535f);          // whole turns
  float r = fmaf(-k, 6.28125f, a_hi);                           // 2 pi = 6.28125 + 1.93548e-3 - 1.74846e-7
  r = fmaf(-k, 1.9354820251464844e-3f, r);
  r = fmaf(-k, -1.7484555314695172e-7f, r);
  __sincosf(r + a_lo, s, c);
}

// The handle's frequency table: theta_k in double [d_r / 2], then the same
// values split into float pairs (hi, lo) [d_r / 2], in one allocation.
__host__ __device__ inline const float2 *theta_pairs(const double *theta, int d_r) {
  return reinterpret_cast<const float2 *>(theta + d_r / 2);
}

// Programmatic dependent launch.  Kernels of this library are launched so
// that the next kernel in the stream may begin while the current one
// finishes (its set-up overlapping the tail); each kernel signals that its
// dependents may launch, and waits for the kernels before it to complete
// before it touches memory they write or read.
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Launches kern(args...) with programmatic stream serialization (and a
// cluster shape when cluster_x > 1).  Only kernels that call pdl_wait()
// before their first dependent memory access may be launched this way.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, int cluster_x,
                       Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  int n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster_x > 1) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster_x;
    attr[n].val.clusterDim.y = 1;
    attr[n].val.clusterDim.z = 1;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<Args &&>(args)...);
}

}  // namespace mla

struct mla_handle {
  mla_config cfg;
  int device;
  int num_sms;
  unsigned *d_status;  // device status word (kStatus* bits)
  double *d_theta;     // device RoPE frequencies theta_k: [d_r/2] double, then [d_r/2] float (hi, lo) pairs
  double score_mult;   // YaRN temperature t multiplying every score (1 without scaling)
  int attn_kind;       // mla::AttnKind
  int gemm_kind;       // mla::GemmKind
  int strict;          // 1: no CUDA-core substitute for a tensor-core kernel (mla_set_strict)
  void *noalloc_scratch;  // device address of the allocation-free entry point's array
};

namespace mla {

// ---------------------------------------------------------------------------
// Split plan.  Sequence b contributes T_b = ceil((end_b - begin_b) / tile)
// tiles of `tile` tokens (the MMA tile of the attention kernel that runs:
// 256 for 128 heads, 128 for 16/32 heads, 64 on the CUDA cores, so that a
// share never pays for a partial tile in the middle of a sequence); the
// batch's Ttot tiles, in sequence order, are cut into P equal shares
// [begin(w), begin(w+1)).  A (share, sequence) intersection is a piece: it
// yields one partial ctx_lat and log-sum-exp.  P is clamped to Ttot so that no
// share is empty, which makes the pieces of one sequence a run of consecutive
// shares.
// ---------------------------------------------------------------------------
__host__ __device__ inline long long plan_begin(long long w, long long P, long long Ttot) {
  return w * Ttot / P;
}
// Largest share index whose range starts at or before tile t (0 <= t < Ttot).
__host__ __device__ inline long long plan_share_of_tile(long long t, long long P, long long Ttot) {
  return ((t + 1) * P - 1) / Ttot;
}
__host__ __device__ inline long long ceil_div_ll(long long a, long long b) { return (a + b - 1) / b; }

// Workspace header written by the plan kernel; the per-sequence arrays follow.
struct WsHeader {
  long long B;
  long long P;           // effective number of shares (<= requested, <= Ttot)
  long long Ttot;        // total tiles
  long long n_pieces;    // total pieces
};

struct WsLayout {
  size_t tile_prefix_off;  // int64 [B+1]
  size_t piece_base_off;   // int64 [B+1]
  size_t ctx_off;          // int32 [2][B]: each sequence's end and first token as attended (clamped by the plan)
  size_t share_first_off;  // int32 [P]: the first sequence whose tiles reach into each share
  size_t opart_off;        // float [n_h, max_pieces, d_c]: a head's pieces are consecutive rows
  size_t lse_off;          // float [n_h, max_pieces]
  size_t total;
  long long max_pieces;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Row of (piece, head) in the partials (units of d_c floats) and index of its
// log-sum-exp.
__host__ __device__ inline long long part_row(const WsLayout &L, long long piece, int head) {
  return (long long)head * L.max_pieces + piece;
}

inline WsLayout ws_layout(const mla_config &cfg, int B, int P) {
  WsLayout L;
  L.max_pieces = (long long)P + B;
  size_t off = align_up(sizeof(WsHeader), 256);
  L.tile_prefix_off = off;
  off = align_up(off + sizeof(long long) * (size_t)(B + 1), 256);
  L.piece_base_off = off;
  off = align_up(off + sizeof(long long) * (size_t)(B + 1), 256);
  L.ctx_off = off;
  off = align_up(off + 2 * sizeof(int) * (size_t)(B > 0 ? B : 1), 256);
  L.share_first_off = off;
  off = align_up(off + sizeof(int) * (size_t)(P > 0 ? P : 1), 256);
  L.opart_off = off;
  off = align_up(off + sizeof(float) * (size_t)L.max_pieces * cfg.n_h * cfg.d_c, 256);
  L.lse_off = off;
  off = align_up(off + sizeof(float) * (size_t)L.max_pieces * cfg.n_h, 256);
  L.total = off;
  return L;
}

// Arguments shared by the attention kernels.
struct AttnArgs {
  const void *q_abs;
  const void *cache;
  long long cache_len;
  const int *block_table;
  int max_blocks;
  int page_size;
  int B;
  int n_h, d_c, d_r;
  float scale_log2;  // log2(e) / sqrt(d_h + d_r)
  // FP8 cache: the rows are E4M3 codes and kv_scale [rows, n_groups] holds
  // each row's group scales; NULL for a cache in cfg.dtype
  const float *kv_scale;
  int n_groups;
  char *ws;
  WsLayout L;
  int plan_tile;     // tokens per tile of the split plan
  unsigned *status;
};

// ---------------------------------------------------------------------------
// Launchers (return cudaGetLastError() of the launch).
// ---------------------------------------------------------------------------
// The plan attends tokens [begin_b, end_b) of sequence b: end_b = ctx_len[b]
// clamped to [0, cap] (cap: the tokens the cache can address for one
// sequence), begin_b = ctx_begin[b] (0 when ctx_begin is NULL) rounded down to
// a multiple of kTile and clamped to [0, end_b].  Any value it has to change
// is flagged in the status word.  It stores both in the workspace; every
// attention kernel reads those instead of the caller's arrays, so that the
// plan's tiles and the kernels' token ranges agree.  `tile` (a multiple of
// kTile) is the plan's tile in tokens.
cudaError_t launch_plan(const int *ctx_begin, const int *ctx_len, int B, int P, long long cap, int tile, char *ws,
                        const WsLayout &L, unsigned *status, cudaStream_t s);

// The clamped end (context length) of sequence b, as the plan stored it.
__device__ __forceinline__ int plan_ctx(const char *ws, const WsLayout &L, int b) {
  return reinterpret_cast<const int *>(ws + L.ctx_off)[b];
}
// The first attended token of sequence b (a multiple of kTile).
__device__ __forceinline__ int plan_begin_tok(const char *ws, const WsLayout &L, int b, int B) {
  return reinterpret_cast<const int *>(ws + L.ctx_off)[B + b];
}

cudaError_t launch_attn_simt(const AttnArgs &a, int P, bool fp32, cudaStream_t s);
// With out_f32, ctx_lat is written in float32 whatever cfg.dtype.
cudaError_t launch_combine(const mla_config &cfg, const char *ws, const WsLayout &L, int B,
                           void *ctx_lat, float *lse, cudaStream_t s, bool out_f32 = false);
// Merge of R float32 token-range results [R, B, n_h, d_c] with their
// log-sum-exps [R, B, n_h] into ctx_lat [B, n_h, d_c] (cfg.dtype) and lse.
cudaError_t launch_merge_ranges(const mla_config &cfg, const float *parts, const float *lse_parts, int R, int B,
                                void *ctx_lat, float *lse, cudaStream_t s);

cudaError_t launch_append_simt(const mla_config &cfg, const void *h, int B, int T,
                               const int *start_pos, const void *w_dkv, const void *w_kr,
                               void *cache, long long cache_len, const int *block_table,
                               int max_blocks, const double *theta, unsigned *status,
                               cudaStream_t s, float *rows_out = nullptr);
// FP8 E4M3 quantisation of n_rows rows [n_rows, d_c + d_r] (cfg.dtype, or
// float32 when src_f32): per row and 128-channel group, sigma = amax / 448 and
// codes E4M3(x / sigma).  With start_pos, row r is token r % T of sequence
// r / T and goes to its cache row (bounds flagged); without, to row r.
cudaError_t launch_quantize_fp8(const mla_config &cfg, const void *src, bool src_f32, long long n_rows,
                                int T, const int *start_pos, uint8_t *codes, float *scales,
                                long long cache_len, const int *block_table, int max_blocks,
                                unsigned *status, cudaStream_t s);
cudaError_t launch_absorb_simt(const mla_config &cfg, const void *q_nope, const void *q_rope,
                               const int *pos, const void *w_uk, void *q_abs, int B,
                               const double *theta, cudaStream_t s);
cudaError_t launch_outproj_simt(const mla_config &cfg, const void *ctx_lat, const void *w_uv,
                                void *o, int B, cudaStream_t s);
// CUDA-core form of the fused combine and output projection (any dtype/shape).
cudaError_t launch_combine_outproj_simt(const mla_config &cfg, const char *ws, const WsLayout &L, int B,
                                        const void *w_uv, void *o, void *ctx_lat, float *lse, cudaStream_t s);
cudaError_t launch_wo_simt(const mla_config &cfg, const void *o, const void *w_o, void *u, int B,
                           cudaStream_t s);
// y[N, M] = x[N, K] w[M, K]^T (row-major, the config's dtype).
cudaError_t launch_linear_simt(const void *x, const void *w, void *y, int M, int K, int N, bool fp32,
                               cudaStream_t s);

// tcgen05 paths (bf16 only); return cudaErrorNotSupported for shapes they lack.
// With rows_out set, the rotated rows go to rows_out [B*T, d_c + d_r] in
// float32 instead of to the cache (the cache arguments are then unused).
cudaError_t launch_append_tc(const mla_config &cfg, const void *h, int B, int T,
                             const int *start_pos, const void *w_dkv, const void *w_kr,
                             void *cache, long long cache_len, const int *block_table,
                             int max_blocks, const double *theta, unsigned *status,
                             cudaStream_t s, float *rows_out = nullptr);
cudaError_t launch_absorb_tc(const mla_config &cfg, const void *q_nope, const void *q_rope,
                             const int *pos, const void *w_uk, void *q_abs, int B,
                             const double *theta, unsigned *status, cudaStream_t s);
cudaError_t launch_outproj_tc(const mla_config &cfg, const void *ctx_lat, const void *w_uv,
                              void *o, int B, unsigned *status, cudaStream_t s);
cudaError_t launch_wo_tc(const mla_config &cfg, const void *o, const void *w_o, void *u, int B,
                         unsigned *status, cudaStream_t s);
cudaError_t launch_linear_tc(const void *x, const void *w, void *y, int M, int K, int N, unsigned *status,
                             cudaStream_t s);
// Split combine fused with the output projection: o[b, i] = W^UV_i ctx_lat[b, i]
// with ctx_lat merged from the workspace's partials inside the kernel
// (written out too when ctx_lat is set; lse likewise).
cudaError_t launch_combine_outproj_tc(const mla_config &cfg, const char *ws, const WsLayout &L, int B,
                                      const void *w_uv, void *o, void *ctx_lat, float *lse, unsigned *status,
                                      cudaStream_t s);
cudaError_t launch_attn_tc_pair(const AttnArgs &a, int P, cudaStream_t s);
cudaError_t launch_attn_tc_smallh(const AttnArgs &a, int P, cudaStream_t s);

// One bounded wait on a barrier that nothing completes, giving up after
// limit_ns: sets the status word's time-out bit (self-test of that path).
cudaError_t launch_wait_timeout_selftest(unsigned *status, unsigned long long limit_ns, cudaStream_t s);

// Resolve the driver entry point for tensor-map encoding (no libcuda link).
bool tma_available();

// Device address, on the current device, of the fixed scratch array of the
// allocation-free entry point (noalloc.cu).  MLA_OK or MLA_ERR_CUDA.
int noalloc_scratch_lookup(void **out);

// Once-per-device launch set-up (the dynamic shared-memory opt-in, which
// applies per device): runs `fn` the first time it is called for the current
// device and caches its result; concurrent callers wait for the first.
template <typename Fn>
cudaError_t once_per_device(std::atomic<int> (&state)[kMaxDevices], Fn fn) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorNotSupported;
  if (state[dev].load(std::memory_order_acquire) == 2) return cudaSuccess;
  static std::mutex mu;
  std::lock_guard<std::mutex> g(mu);
  if (state[dev].load(std::memory_order_relaxed) == 2) return cudaSuccess;
  e = fn();
  if (e == cudaSuccess) state[dev].store(2, std::memory_order_release);
  return e;
}

}  // namespace mla
