// tcgen05 GEMMs of the decode step: cache append (W_DKV / W_KR), query
// absorption (W_UK^T per head) and output projection (W_UV per head, W_O).
//
// All four are "weight times a few activations": the weight is the MMA's A
// operand (M = 128 output features per tile, streamed by TMA), the
// activations are B (N = tokens or sequences, padded to a multiple of 16 by
// TMA zero fill), and the fp32 accumulator lives in tensor memory.  The
// epilogue reads it back with tcgen05.ld (one thread per output feature) and
// writes bf16 results, applying RoPE where the step calls for it.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 allocates tensor
// memory and issues MMAs, warps 2-5 run the epilogue.
#include <math_constants.h>
#include <string.h>

#include "ptx.cuh"

namespace mla {

// ---------------------------------------------------------------------------
// tensor-map encoding through the driver entry point (no libcuda link)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn resolve_encode() {
  static EncodeTiledFn fn = [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return (EncodeTiledFn)p;
  }();
  return fn;
}

bool tma_available() { return resolve_encode() != nullptr; }

static bool encode_map(CUtensorMap *map, CUtensorMapDataType type, const void *base, int rank,
                       const uint64_t *dims, const uint64_t *strides, const uint32_t *box,
                       CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = resolve_encode();
  if (!fn) return false;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides[i];
  CUresult r = fn(map, type, (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_map_bf16(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                     const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swz) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, rank, dims, strides, box, swz);
}

bool encode_map_u8(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                   const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swz) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, rank, dims, strides, box, swz);
}

namespace {

constexpr int kGemmThreads = 192;
constexpr int kMaxStages = 8;           // pipeline depth is chosen per launch (<= this)
constexpr int kKChunk = 64;           // bf16 elements per 128-byte swizzled row
constexpr int kABytes = 128 * kKChunk * 2;

enum EpiMode : int { kEpiAbsorb = 0, kEpiOutProj = 1, kEpiWo = 2, kEpiAppend = 3 };

struct GemmParams {
  int mode;
  int num_k_chunks;   // K / 64 of the whole product
  int stages;         // pipeline stages of this launch (<= kMaxStages)
  int ksplit;         // K slices per output tile (1, or a cluster of ksplit CTAs along x)
  int mt_per_cta;     // 128-row m tiles one CTA computes, sharing its B tiles (1 when ksplit > 1)
  int m_tiles;        // m tiles of the whole product
  int M_valid;        // valid output features (rows of the product)
  int N;              // valid columns (tokens or sequences)
  int a_split_tile;   // m-tiles >= a_split_tile read map A1 (append: W_KR)
  int a1_rows;        // rows of map A1's box (bytes of that A tile = a1_rows * 128)
  int a_row_per_z;    // added to A's row coordinate per blockIdx.z
  int b_is_3d;        // B map is [N][Z][K] with the head index as middle coordinate
  __nv_bfloat16 *out;
  long long out_ld;   // elements between consecutive columns n
  long long out_z;    // elements between consecutive z
  // absorb: rotary part of the query
  const __nv_bfloat16 *q_rope;
  const int *pos;
  const double *theta;
  int d_c, d_r, n_h;
  // append: destination rows
  int T;
  const int *start_pos;
  long long cache_len;
  const int *block_table;
  int max_blocks;
  int page_size;
  // append: when set, token n's row goes to out_f32[n * (d_c + d_r) ..] in
  // float32 (for a later FP8 quantisation) instead of to the cache
  float *out_f32;
  unsigned *status;
};

__device__ __forceinline__ long long dest_row(int b, long long p, const GemmParams &g) {
  if (p < 0) return -1;
  if (g.page_size == 0) return p < g.cache_len ? (long long)b * g.cache_len + p : -1;
  const long long bi = p / g.page_size;
  if (bi >= g.max_blocks) return -1;
  const int blk = g.block_table[(long long)b * g.max_blocks + bi];
  if (blk < 0 || blk >= g.cache_len) return -1;
  return (long long)blk * g.page_size + p % g.page_size;
}

template <int BN, bool A_MN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap mapA0, const __grid_constant__ CUtensorMap mapA1,
                   const __grid_constant__ CUtensorMap mapB, const GemmParams g) {
  constexpr int kBBytes = BN * kKChunk * 2;
  static_assert(kBBytes % 1024 == 0, "stage buffers must stay 1024-byte aligned");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int S = g.stages;
  const int MT = g.mt_per_cta;
  const int kStage = MT * kABytes + kBBytes;   // one K chunk: MT A tiles, then the shared B tile
  const bool split = g.ksplit > 1;
  // The stage ring; with a K split it is reused afterwards for this CTA's fp32 partial.
  const int region = split && 128 * BN * 4 > S * kStage ? 128 * BN * 4 : S * kStage;
  uint64_t *full = reinterpret_cast<uint64_t *>(base + region);
  uint64_t *empty = full + kMaxStages;
  uint64_t *accf = empty + kMaxStages;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accf + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  long long *s_row = reinterpret_cast<long long *>(base + region + 256);
  int *s_pos = reinterpret_cast<int *>(s_row + BN);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // blockIdx.x = m-tile group * ksplit + K slice; a K split runs as one
  // cluster of ksplit CTAs along x, so the slice index is also the CTA's
  // cluster rank.  A group is MT consecutive m tiles (MT = 1 with a split).
  const int mt = ((int)blockIdx.x / g.ksplit) * MT, zs = (int)blockIdx.x % g.ksplit;
  const int mcount = min(MT, g.m_tiles - mt);
  const int nt = blockIdx.y, z = blockIdx.z;
  const int per = (g.num_k_chunks + g.ksplit - 1) / g.ksplit;
  const int kc0 = zs * per;
  const int nk = max(0, min(g.num_k_chunks, kc0 + per) - kc0);   // K chunks of this CTA
  const int m0 = mt * 128, n0 = nt * BN;
  const bool use_a1 = mt >= g.a_split_tile;   // (only with MT = 1)
  uint32_t tmem_cols = 32;
  while (tmem_cols < (uint32_t)(MT * BN)) tmem_cols <<= 1;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accf, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, tmem_cols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      const CUtensorMap *mA = use_a1 ? &mapA1 : &mapA0;
      const int a_m0 = use_a1 ? m0 - g.a_split_tile * 128 : m0;
      const uint32_t a_bytes = use_a1 ? (uint32_t)g.a1_rows * 128u : (uint32_t)kABytes;
      ptx::tma_prefetch_desc(mA);
      ptx::tma_prefetch_desc(&mapB);
      // The weights (A) never depend on earlier kernels: the first stages'
      // A tiles are requested before waiting for those kernels, the
      // activations (B) after.
      const int pre = nk < S ? nk : S;
      auto load_a = [&](int kl) {
        const int s = kl % S, kc = kc0 + kl;
        uint8_t *sa = base + s * kStage;
        ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)mcount * a_bytes + (uint32_t)kBBytes);
        for (int t = 0; t < mcount; ++t) {
          uint8_t *st = sa + t * kABytes;
          if (A_MN) {
            const int krow = z * g.a_row_per_z + kc * kKChunk;
            ptx::tma_load_2d(st, mA, &full[s], a_m0 + 128 * t, krow);
            ptx::tma_load_2d(st + kABytes / 2, mA, &full[s], a_m0 + 128 * t + 64, krow);
          } else {
            ptx::tma_load_2d(st, mA, &full[s], kc * kKChunk, z * g.a_row_per_z + a_m0 + 128 * t);
          }
        }
      };
      auto load_b = [&](int kl) {
        const int s = kl % S, kc = kc0 + kl;
        uint8_t *sb = base + s * kStage + MT * kABytes;
        if (g.b_is_3d) ptx::tma_load_3d(sb, &mapB, &full[s], kc * kKChunk, z, n0);
        else ptx::tma_load_2d(sb, &mapB, &full[s], kc * kKChunk, n0);
      };
      for (int kl = 0; kl < pre; ++kl) load_a(kl);
      pdl_wait();
      for (int kl = 0; kl < pre; ++kl) load_b(kl);
      int issued = pre;
      for (int kl = pre; kl < nk; ++kl) {
        const int s = kl % S;
        if (!ptx::mbar_wait(&empty[s], ((kl / S) - 1) & 1, g.status, abort_flag)) break;
        ++issued;
        load_a(kl);
        load_b(kl);
      }
      // Drain: do not leave while loads into this CTA's shared memory are in flight.
      for (int kl = issued - S > 0 ? issued - S : 0; kl < issued; ++kl) {
        volatile int no_abort = 0;
        ptx::mbar_wait(&full[kl % S], (kl / S) & 1, g.status, &no_abort);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BN, A_MN, false);
      for (int kl = 0; kl < nk; ++kl) {
        const int s = kl % S;
        if (!ptx::mbar_wait(&full[s], (kl / S) & 1, g.status, abort_flag)) break;
        ptx::tc_fence_after();
        const uint32_t sa = ptx::smem_u32(base + s * kStage);
        const uint32_t sb = sa + MT * kABytes;
        for (int t = 0; t < mcount; ++t) {
          const uint32_t st = sa + t * kABytes;
#pragma unroll
          for (int j = 0; j < kKChunk / 16; ++j) {
            // A: K-major rows of 128 B (advance 32 B per 16-element k step), or
            //    MN-major: 64-wide m chunks 8 KB apart, k rows 128 B apart.
            const uint64_t ad = A_MN ? ptx::sdesc(st + j * 2048, kABytes / 2, 1024, 2)
                                     : ptx::sdesc(st + j * 32, 16, 1024, 2);
            const uint64_t bd = ptx::sdesc(sb + j * 32, 16, 1024, 2);
            ptx::mma_bf16_ss(tmem + t * BN, ad, bd, idesc, (kl | j) != 0 ? 1u : 0u);
          }
        }
        ptx::mma_commit(&empty[s]);
      }
      ptx::mma_commit(accf);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    pdl_wait();
    const int et = threadIdx.x - 64;  // 0..127
    if (g.mode == kEpiAppend) {
      for (int j = et; j < BN; j += 128) {
        const int n = n0 + j;
        long long row = -1;
        int p = 0;
        if (n < g.N) {
          const int b = n / g.T, t = n % g.T;
          p = g.start_pos[b] + t;
          if (g.out_f32) {
            row = n;
          } else {
            row = dest_row(b, p, g);
            if (row < 0) atomicOr(g.status, kStatusBounds);
          }
        }
        s_row[j] = row;
        s_pos[j] = p;
      }
      asm volatile("bar.sync 1, 128;" ::: "memory");
    }
    const bool ok = ptx::mbar_wait(accf, 0, g.status, abort_flag);
    ptx::tc_fence_after();
    const int q = warp & 3;
    const int m_local = q * 32 + lane;
    const int m = m0 + m_local;
    const bool rope_tile = g.mode == kEpiAppend && use_a1;
    if (split) {
      // Partial of this K slice, [BN columns][128 rows] fp32, read by the whole cluster below.
      float *red = reinterpret_cast<float *>(base);
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t r[16];
        const bool have = ok && nk > 0;   // a slice with no K chunks contributes zero
        if (have) {
          ptx::tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, r);
          ptx::tmem_ld_wait();
        }
#pragma unroll
        for (int j = 0; j < 16; ++j) red[(c0 + j) * 128 + m_local] = have ? __uint_as_float(r[j]) : 0.f;
      }
    } else if (ok) {
#pragma unroll 1
      for (int t = 0; t < mcount; ++t) {
        // m tile mt + t: rows m0 + 128 t .., accumulator columns t * BN ..
        const int mm = m + 128 * t;
        const bool mm_ok = mm < g.M_valid;
#pragma unroll 1
        for (int c0 = 0; c0 < BN; c0 += 16) {
          uint32_t r[16];
          ptx::tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(t * BN + c0), r);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int n = n0 + c0 + j;
            float v = __uint_as_float(r[j]);
            if (rope_tile) {
              const float partner = __shfl_xor_sync(0xffffffffu, v, 1);
              const int k = m_local >> 1;
              if (mm_ok && n < g.N && k < g.d_r / 2) {
                double sn, cs;
                sincos((double)s_pos[c0 + j] * g.theta[k], &sn, &cs);
                const float c = (float)cs, s = (float)sn;
                v = (lane & 1) ? partner * s + v * c : v * c - partner * s;
              }
            }
            if (!mm_ok || n >= g.N) continue;
            if (g.mode == kEpiAppend) {
              const long long row = s_row[c0 + j];
              if (row >= 0) {
                if (g.out_f32) g.out_f32[row * (long long)(g.d_c + g.d_r) + mm] = v;
                else g.out[row * (long long)(g.d_c + g.d_r) + mm] = __float2bfloat16_rn(v);
              }
            } else {
              g.out[(long long)n * g.out_ld + (long long)z * g.out_z + mm] = __float2bfloat16_rn(v);
            }
          }
        }
      }
    }
    if (g.mode == kEpiAbsorb && mt == 0 && zs == 0) {
      // rotary part of the absorbed query: q_abs[b, z, d_c + 2k (+1)] = RoPE(q_rope[b, z], pos[b])
      const int npair = g.d_r / 2;
      const int ncol = min(BN, g.N - n0);
      for (int idx = et; idx < ncol * npair; idx += 128) {
        const int n = n0 + idx / npair, k = idx % npair;
        const long long src = ((long long)n * g.n_h + z) * g.d_r + 2 * k;
        const float x0 = __bfloat162float(g.q_rope[src]), x1 = __bfloat162float(g.q_rope[src + 1]);
        double sn, cs;
        sincos((double)g.pos[n] * g.theta[k], &sn, &cs);
        const float c = (float)cs, s = (float)sn;
        __nv_bfloat16 *dst = g.out + (long long)n * g.out_ld + (long long)z * g.out_z + g.d_c + 2 * k;
        dst[0] = __float2bfloat16_rn(x0 * c - x1 * s);
        dst[1] = __float2bfloat16_rn(x0 * s + x1 * c);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, tmem_cols);
  }

  if (split) {
    // Every CTA of the cluster reaches this point (all waits above are
    // bounded), so the two cluster barriers always complete.
    pdl_wait();                // every thread below writes outputs
    ptx::cluster_sync_all();   // partials of all K slices are written
    const int ks = g.ksplit;
    if (ptx::cluster_nctarank() == (uint32_t)ks) {
      // This CTA sums rows [zs*R, zs*R + R) of the tile over the cluster's
      // partials, 4 rows (one float4) per item, and writes them out.
      const int R = 128 / ks, R4 = R / 4;
      const uint32_t red = ptx::smem_u32(base);
      for (int idx = threadIdx.x; idx < BN * R4; idx += kGemmThreads) {
        const int c = idx / R4, ml = zs * R + 4 * (idx % R4);
        const uint32_t off = (uint32_t)((c * 128 + ml) * 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int p = 0; p < ks; ++p) {
          const float4 v = ptx::ld_shared_cluster_v4f(ptx::mapa_peer(red + off, (uint32_t)p));
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
        const int n = n0 + c;
        if (n >= g.N) continue;
        float v[4] = {acc.x, acc.y, acc.z, acc.w};
        if (g.mode == kEpiAppend && use_a1) {
          // rows (ml, ml+1) and (ml+2, ml+3) are rotary pairs k = ml/2, ml/2 + 1
#pragma unroll
          for (int e = 0; e < 4; e += 2) {
            const int k = (ml + e) >> 1;
            if (k < g.d_r / 2) {
              double sn, cs;
              sincos((double)s_pos[c] * g.theta[k], &sn, &cs);
              const float co = (float)cs, si = (float)sn;
              const float x0 = v[e], x1 = v[e + 1];
              v[e] = x0 * co - x1 * si;
              v[e + 1] = x0 * si + x1 * co;
            }
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int m = m0 + ml + e;
          if (m >= g.M_valid) continue;
          if (g.mode == kEpiAppend) {
            const long long row = s_row[c];
            if (row >= 0) {
              if (g.out_f32) g.out_f32[row * (long long)(g.d_c + g.d_r) + m] = v[e];
              else g.out[row * (long long)(g.d_c + g.d_r) + m] = __float2bfloat16_rn(v[e]);
            }
          } else {
            g.out[(long long)n * g.out_ld + (long long)z * g.out_z + m] = __float2bfloat16_rn(v[e]);
          }
        }
      }
    } else if (threadIdx.x == 0) {
      atomicOr(g.status, kStatusBounds);   // launched without the cluster shape it needs
    }
    ptx::cluster_sync_all();   // no CTA leaves while others still read its partial
  }
}

constexpr size_t kSmemLimit = 232448;   // opt-in shared memory per block on sm_100

template <int BN>
constexpr int b_bytes() { return BN * kKChunk * 2; }

template <int BN>
constexpr size_t smem_tail() { return 256 + (size_t)BN * (8 + 4); }

template <int BN, bool A_MN>
cudaError_t launch_gemm(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b, GemmParams g,
                        int mtiles, int ntiles, int nz, cudaStream_t s) {
  if (g.mt_per_cta < 1 || (g.ksplit > 1 && g.mt_per_cta != 1) || g.mt_per_cta * BN > 512)
    return cudaErrorNotSupported;
  g.m_tiles = mtiles;
  const int stage = g.mt_per_cta * kABytes + b_bytes<BN>();
  const int per = (g.num_k_chunks + g.ksplit - 1) / g.ksplit;
  int max_st = (int)((kSmemLimit - 1024 - smem_tail<BN>()) / stage);
  if (max_st > kMaxStages) max_st = kMaxStages;
  if (max_st < 1) return cudaErrorNotSupported;
  g.stages = per < max_st ? (per > 0 ? per : 1) : max_st;
  size_t region = (size_t)g.stages * stage;
  if (g.ksplit > 1 && (size_t)128 * BN * 4 > region) region = (size_t)128 * BN * 4;
  const size_t smem = 1024 + region + smem_tail<BN>();
  if (smem > kSmemLimit) return cudaErrorNotSupported;
  auto kern = gemm_tc_kernel<BN, A_MN>;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = once_per_device(configured, [kern] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
  });
  if (e != cudaSuccess) return e;
  const int groups = (mtiles + g.mt_per_cta - 1) / g.mt_per_cta;
  const dim3 grid(groups * g.ksplit, ntiles, nz);
  return launch_pdl(kern, grid, dim3(kGemmThreads), smem, s, g.ksplit, a0, a1, b, g);
}

// K split: the smallest power of two (<= 8, the portable cluster size) that
// gives at least one CTA per SM, while every slice keeps >= 2 K chunks.
int pick_ksplit(long long ctas, int num_k_chunks) {
  int sms = 148, dev = 0;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int ks = 1;
  while (ks < 8 && ctas * ks < sms && num_k_chunks >= 4 * ks) ks *= 2;
  return ks;
}

template <bool A_MN>
cudaError_t dispatch_bn(int N, const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b,
                        GemmParams g, int mtiles, int z, cudaStream_t s, int bn) {
  const int ntiles = (N + bn - 1) / bn;
  if (g.mt_per_cta == 0) g.mt_per_cta = 1;
  if (g.ksplit == 0)
    g.ksplit = g.mt_per_cta > 1 ? 1 : pick_ksplit((long long)mtiles * ntiles * z, g.num_k_chunks);
  switch (bn) {
    case 16: return launch_gemm<16, A_MN>(a0, a1, b, g, mtiles, ntiles, z, s);
    case 32: return launch_gemm<32, A_MN>(a0, a1, b, g, mtiles, ntiles, z, s);
    case 64: return launch_gemm<64, A_MN>(a0, a1, b, g, mtiles, ntiles, z, s);
    case 128: return launch_gemm<128, A_MN>(a0, a1, b, g, mtiles, ntiles, z, s);
    default: return launch_gemm<256, A_MN>(a0, a1, b, g, mtiles, ntiles, z, s);
  }
}

int pick_bn(long long N) {
  if (N <= 16) return 16;
  if (N <= 32) return 32;
  if (N <= 64) return 64;
  if (N <= 128) return 128;
  return 256;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }

GemmParams blank_params() {
  GemmParams g;
  memset(&g, 0, sizeof(g));
  g.a_split_tile = 1 << 30;
  g.a1_rows = 128;
  return g;
}

}  // namespace

// ---------------------------------------------------------------------------
cudaError_t launch_absorb_tc(const mla_config &c, const void *q_nope, const void *q_rope, const int *pos,
                             const void *w_uk, void *q_abs, int B, const double *theta, cudaStream_t s) {
  if (!aligned16(q_nope) || !aligned16(w_uk)) return cudaErrorNotSupported;
  const int bn = pick_bn(B);
  CUtensorMap ma, mb;
  const uint64_t da[2] = {(uint64_t)c.d_c, (uint64_t)c.n_h * c.d_h};
  const uint64_t sa[1] = {(uint64_t)c.d_c * 2};
  const uint32_t ba[2] = {64, 64};
  const uint64_t db[3] = {(uint64_t)c.d_h, (uint64_t)c.n_h, (uint64_t)B};
  const uint64_t sb[2] = {(uint64_t)c.d_h * 2, (uint64_t)c.n_h * c.d_h * 2};
  const uint32_t bb[3] = {64, 1, (uint32_t)bn};
  if (!encode_map_bf16(&ma, w_uk, 2, da, sa, ba, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_bf16(&mb, q_nope, 3, db, sb, bb, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  GemmParams g = blank_params();
  g.mode = kEpiAbsorb;
  // One m tile per CTA: 512 short CTAs measured faster here (30.7 us at B=64)
  // than 256 or 128 CTAs that share q^C across 2 or 4 tiles (32.9 / 41.0 us),
  // whose single TMA-issuing thread then streams twice or four times as many
  // boxes.
  g.mt_per_cta = 1;
  g.num_k_chunks = c.d_h / kKChunk;
  g.M_valid = c.d_c;
  g.N = B;
  g.a_row_per_z = c.d_h;
  g.b_is_3d = 1;
  g.out = (__nv_bfloat16 *)q_abs;
  g.out_ld = (long long)c.n_h * (c.d_c + c.d_r);
  g.out_z = c.d_c + c.d_r;
  g.q_rope = (const __nv_bfloat16 *)q_rope;
  g.pos = pos;
  g.theta = theta;
  g.d_c = c.d_c;
  g.d_r = c.d_r;
  g.n_h = c.n_h;
  return dispatch_bn<true>(B, ma, ma, mb, g, c.d_c / 128, c.n_h, s, bn);
}

cudaError_t launch_outproj_tc(const mla_config &c, const void *ctx_lat, const void *w_uv, void *o, int B,
                              cudaStream_t s) {
  if (!aligned16(ctx_lat) || !aligned16(w_uv) || c.d_h % 128 != 0) return cudaErrorNotSupported;
  const int bn = pick_bn(B);
  CUtensorMap ma, mb;
  const uint64_t da[2] = {(uint64_t)c.d_c, (uint64_t)c.n_h * c.d_h};
  const uint64_t sa[1] = {(uint64_t)c.d_c * 2};
  const uint32_t ba[2] = {64, 128};
  const uint64_t db[3] = {(uint64_t)c.d_c, (uint64_t)c.n_h, (uint64_t)B};
  const uint64_t sb[2] = {(uint64_t)c.d_c * 2, (uint64_t)c.n_h * c.d_c * 2};
  const uint32_t bb[3] = {64, 1, (uint32_t)bn};
  if (!encode_map_bf16(&ma, w_uv, 2, da, sa, ba, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_bf16(&mb, ctx_lat, 3, db, sb, bb, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  GemmParams g = blank_params();
  g.mode = kEpiOutProj;
  g.num_k_chunks = c.d_c / kKChunk;
  g.M_valid = c.d_h;
  g.N = B;
  g.a_row_per_z = c.d_h;
  g.b_is_3d = 1;
  g.out = (__nv_bfloat16 *)o;
  g.out_ld = (long long)c.n_h * c.d_h;
  g.out_z = c.d_h;
  return dispatch_bn<false>(B, ma, ma, mb, g, c.d_h / 128, c.n_h, s, bn);
}

cudaError_t launch_linear_tc(const void *x, const void *w, void *y, int M, int K, int N, cudaStream_t s) {
  // y[N, M] = x[N, K] w[M, K]^T, bf16 in and out, fp32 accumulation.
  if (!aligned16(x) || !aligned16(w) || K % 64 != 0 || M <= 0 || N <= 0) return cudaErrorNotSupported;
  const int bn = pick_bn(N);
  CUtensorMap ma, mb;
  const uint64_t da[2] = {(uint64_t)K, (uint64_t)M};
  const uint64_t sa[1] = {(uint64_t)K * 2};
  const uint32_t ba[2] = {64, 128};
  const uint64_t db[2] = {(uint64_t)K, (uint64_t)N};
  const uint64_t sb[1] = {(uint64_t)K * 2};
  const uint32_t bb[2] = {64, (uint32_t)bn};
  if (!encode_map_bf16(&ma, w, 2, da, sa, ba, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_bf16(&mb, x, 2, db, sb, bb, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  GemmParams g = blank_params();
  g.mode = kEpiWo;
  g.num_k_chunks = K / kKChunk;
  g.M_valid = M;
  g.N = N;
  g.out = (__nv_bfloat16 *)y;
  g.out_ld = M;
  return dispatch_bn<false>(N, ma, ma, mb, g, (M + 127) / 128, 1, s, bn);
}

cudaError_t launch_wo_tc(const mla_config &c, const void *o, const void *w_o, void *u, int B, cudaStream_t s) {
  return launch_linear_tc(o, w_o, u, c.d_model, c.n_h * c.d_h, B, s);
}

cudaError_t launch_append_tc(const mla_config &c, const void *h, int B, int T, const int *start_pos,
                             const void *w_dkv, const void *w_kr, void *cache, long long cache_len,
                             const int *block_table, int max_blocks, const double *theta,
                             unsigned *status, cudaStream_t s, float *rows_out) {
  if (!aligned16(h) || !aligned16(w_dkv) || !aligned16(w_kr)) return cudaErrorNotSupported;
  const long long N = (long long)B * T;
  if (N > 65535LL * 256) return cudaErrorNotSupported;
  const int bn = pick_bn(N);
  const int a1_rows = c.d_r < 128 ? c.d_r : 128;
  CUtensorMap m0, m1, mb;
  const uint64_t d0[2] = {(uint64_t)c.d_model, (uint64_t)c.d_c};
  const uint64_t d1[2] = {(uint64_t)c.d_model, (uint64_t)c.d_r};
  const uint64_t sw[1] = {(uint64_t)c.d_model * 2};
  const uint32_t b0[2] = {64, 128};
  const uint32_t b1[2] = {64, (uint32_t)a1_rows};
  const uint64_t db[2] = {(uint64_t)c.d_model, (uint64_t)N};
  const uint32_t bb[2] = {64, (uint32_t)bn};
  if (!encode_map_bf16(&m0, w_dkv, 2, d0, sw, b0, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_bf16(&m1, w_kr, 2, d1, sw, b1, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_bf16(&mb, h, 2, db, sw, bb, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  GemmParams g = blank_params();
  g.mode = kEpiAppend;
  g.num_k_chunks = c.d_model / kKChunk;
  g.M_valid = c.d_c + c.d_r;
  g.N = (int)N;
  g.a_split_tile = c.d_c / 128;
  g.a1_rows = a1_rows;
  g.out = (__nv_bfloat16 *)cache;
  g.theta = theta;
  g.d_c = c.d_c;
  g.d_r = c.d_r;
  g.T = T;
  g.start_pos = start_pos;
  g.cache_len = cache_len;
  g.block_table = block_table;
  g.max_blocks = max_blocks;
  g.page_size = c.page_size;
  g.out_f32 = rows_out;
  g.status = status;
  const int mtiles = c.d_c / 128 + (c.d_r + 127) / 128;
  return dispatch_bn<false>((int)N, m0, m1, mb, g, mtiles, 1, s, bn);
}

}  // namespace mla
