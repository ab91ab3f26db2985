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
//
// Loads come in groups of G consecutive 64-wide K chunks, one TMA box of G
// chunks per operand and m tile (3D/4D boxes whose outer dimension steps
// through the chunks): a thread issuing cp.async.bulk.tensor copies sustains
// about two copies per microsecond (measured), so these short, weight-
// streaming GEMMs need few and large copies.
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

bool encode_map_f32(CUtensorMap *map, const void *base, int rank, const uint64_t *dims,
                    const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle swz) {
  return encode_map(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, rank, dims, strides, box, swz);
}

namespace {

constexpr int kGemmThreads = 192;
constexpr int kMaxStages = 8;           // K-chunk slots of the ring (<= this), a multiple of the group
constexpr int kMaxGroups = kMaxStages;  // load groups of the ring
constexpr int kKChunk = 64;           // bf16 elements per 128-byte swizzled row
constexpr int kABytes = 128 * kKChunk * 2;

enum EpiMode : int { kEpiAbsorb = 0, kEpiOutProj = 1, kEpiWo = 2, kEpiAppend = 3 };

struct GemmParams {
  int mode;
  int num_k_chunks;   // K / 64 of the whole product
  int stages;         // K-chunk slots of the ring (<= kMaxStages, a multiple of group)
  int group;          // K chunks per TMA load group (1, 2 or 4)
  int ksplit;         // K slices per output tile (1, or a cluster of ksplit CTAs along x)
  int mt_per_cta;     // 128-row m tiles one CTA computes, sharing its B tiles (1 when ksplit > 1)
  int m_tiles;        // m tiles of the whole product
  int M_valid;        // valid output features (rows of the product)
  int N;              // valid columns (tokens or sequences)
  int a_split_tile;   // m-tiles >= a_split_tile read map A1 (append: W_KR)
  int a1_rows;        // rows of map A1's box (<= 128; its chunks are a1_rows * 128 B apart)
  int a_row_per_z;    // added to A's row coordinate per blockIdx.z
  int b_is_3d;        // B map is [N][Z][K] with the head index as middle coordinate
  __nv_bfloat16 *out;
  long long out_ld;   // elements between consecutive columns n
  long long out_z;    // elements between consecutive z
  // absorb: rotary part of the query
  const __nv_bfloat16 *q_rope;
  const int *pos;
  const float2 *theta;   // rotary frequencies as float (hi, lo) pairs
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
  int vec_out;        // bf16 outputs aligned for 16-byte stores (rows of 128 contiguous features)
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
  const int G = g.group;
  const int NG = S / G;                          // load groups in the ring
  const int MT = g.mt_per_cta;
  // Ring layout, per load group gs: MT A blocks of G chunks (G x 16 KB each),
  // then the shared B block of G chunks (G x kBBytes).
  const int kGroupBytes = G * (MT * kABytes + kBBytes);
  const bool split = g.ksplit > 1;
  // The ring; with a K split it is reused afterwards for this CTA's fp32 partial.
  const int region = split && 128 * BN * 4 > NG * kGroupBytes ? 128 * BN * 4 : NG * kGroupBytes;
  uint64_t *full = reinterpret_cast<uint64_t *>(base + region);
  uint64_t *empty = full + kMaxGroups;
  uint64_t *accf = empty + kMaxGroups;
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
  const int ngrp = (nk + G - 1) / G;                               // load groups of this CTA
  const int m0 = mt * 128, n0 = nt * BN;
  const bool use_a1 = mt >= g.a_split_tile;   // (only with MT = 1)
  uint32_t tmem_cols = 32;
  while (tmem_cols < (uint32_t)(MT * BN)) tmem_cols <<= 1;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < NG; ++s) {
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
      // The weights (A) never depend on earlier kernels: the first groups'
      // A blocks are requested before waiting for those kernels, the
      // activations (B) after.  A group always loads G whole chunks (a last
      // group past the slice's end loads chunks its MMAs skip).
      const int pre = ngrp < NG ? ngrp : NG;
      auto load_a = [&](int gi) {
        const int s = gi % NG, kc = kc0 + gi * G;
        uint8_t *sa = base + s * kGroupBytes;
        ptx::mbar_arrive_expect_tx(&full[s], (uint32_t)G * ((uint32_t)mcount * a_bytes + (uint32_t)kBBytes));
        for (int t = 0; t < mcount; ++t) {
          uint8_t *st = sa + t * G * kABytes;
          if (A_MN) {
            // [2 m halves][64 G k rows][64 m]: m chunks 2 (mt + t), +1
            ptx::tma_load_3d(st, mA, &full[s], 0, z * g.a_row_per_z + kc * kKChunk, 2 * (a_m0 / 128 + t));
          } else {
            // [G chunks][rows][64 k]
            ptx::tma_load_3d(st, mA, &full[s], 0, z * g.a_row_per_z + a_m0 + 128 * t, kc);
          }
        }
      };
      auto load_b = [&](int gi) {
        const int s = gi % NG, kc = kc0 + gi * G;
        uint8_t *sb = base + s * kGroupBytes + MT * G * kABytes;
        if (g.b_is_3d) ptx::tma_load_4d(sb, &mapB, &full[s], 0, n0, kc, z);
        else ptx::tma_load_3d(sb, &mapB, &full[s], 0, n0, kc);
      };
      for (int gi = 0; gi < pre; ++gi) load_a(gi);
      pdl_wait();
      for (int gi = 0; gi < pre; ++gi) load_b(gi);
      int issued = pre;
      for (int gi = pre; gi < ngrp; ++gi) {
        const int s = gi % NG;
        if (!ptx::mbar_wait(&empty[s], ((gi / NG) - 1) & 1, g.status, abort_flag)) break;
        ++issued;
        load_a(gi);
        load_b(gi);
      }
      // Drain: do not leave while loads into this CTA's shared memory are in flight.
      for (int gi = issued - NG > 0 ? issued - NG : 0; gi < issued; ++gi) {
        volatile int no_abort = 0;
        ptx::mbar_wait(&full[gi % NG], (gi / NG) & 1, g.status, &no_abort);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, BN, A_MN, false);
      for (int gi = 0; gi < ngrp; ++gi) {
        const int s = gi % NG;
        if (!ptx::mbar_wait(&full[s], (gi / NG) & 1, g.status, abort_flag)) break;
        ptx::tc_fence_after();
        const uint32_t sa = ptx::smem_u32(base + s * kGroupBytes);
        const uint32_t sb = sa + MT * G * kABytes;
        // K-major A chunks lie a box's rows x 128 B apart (a shorter A1 box
        // leaves the tile's last rows holding other data: those output rows
        // are past M_valid and never written)
        const uint32_t a_step = use_a1 ? (uint32_t)g.a1_rows * 128u : (uint32_t)kABytes;
        for (int j = 0; j < G && gi * G + j < nk; ++j) {
          const int kl = gi * G + j;
          for (int t = 0; t < mcount; ++t) {
            const uint32_t st = sa + t * G * kABytes;
#pragma unroll
            for (int kk = 0; kk < kKChunk / 16; ++kk) {
              // A: K-major rows of 128 B (advance 32 B per 16-element k step), or
              //    MN-major: 64-wide m halves G * 8 KB apart, k rows 128 B apart.
              const uint64_t ad = A_MN ? ptx::sdesc(st + j * 8192 + kk * 2048, G * 8192, 1024, 2)
                                       : ptx::sdesc(st + j * a_step + kk * 32, 16, 1024, 2);
              const uint64_t bd = ptx::sdesc(sb + j * kBBytes + kk * 32, 16, 1024, 2);
              ptx::mma_bf16_ss(tmem + t * BN, ad, bd, idesc, (kl | kk) != 0 ? 1u : 0u);
            }
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
    if (g.mode == kEpiAbsorb && zs == 0) {
      // Rotary part of the absorbed query, q_abs[b, z, d_c + 2k (+1)] =
      // RoPE(q_rope[b, z], pos[b]): independent of the product, so done while
      // the MMAs run, shared out over the head's m-tile CTAs.  Eight elements
      // per thread at a time, all their loads issued before any use.
      const int npair = g.d_r / 2;
      const int ncol = min(BN, g.N - n0);
      const int total = ncol * npair;
      const int stride = 128 * g.m_tiles;
      for (int idx0 = et + 128 * mt; idx0 < total; idx0 += stride * 8) {
        __nv_bfloat162 xr[8];
        int pp[8];
        float2 th[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int idx = idx0 + stride * u;
          if (idx < total) {
            const int n = n0 + idx / npair, k = idx % npair;
            xr[u] = *reinterpret_cast<const __nv_bfloat162 *>(g.q_rope + ((long long)n * g.n_h + z) * g.d_r + 2 * k);
            pp[u] = g.pos[n];
            th[u] = g.theta[k];
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int idx = idx0 + stride * u;
          if (idx < total) {
            const int n = n0 + idx / npair, k = idx % npair;
            const float x0 = __low2float(xr[u]), x1 = __high2float(xr[u]);
            float s, c;
            rope_sincos(pp[u], th[u], &s, &c);
            *reinterpret_cast<__nv_bfloat162 *>(g.out + (long long)n * g.out_ld + (long long)z * g.out_z + g.d_c +
                                                2 * k) = __floats2bfloat162_rn(x0 * c - x1 * s, x0 * s + x1 * c);
          }
        }
      }
    }
    // One thread polls the accumulator barrier and the other epilogue threads
    // wait on a named barrier, which takes no issue slots: with every
    // epilogue warp polling, the polls of the CTAs sharing an SM slowed each
    // other's epilogues several-fold (measured).
    if (et == 0) ptx::mbar_wait(accf, 0, g.status, abort_flag);
    asm volatile("bar.sync 2, 128;" ::: "memory");
    const bool ok = !*abort_flag;   // the same for every epilogue thread
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
    } else {
      const bool go = ok;
      // With vec_out, bf16 outputs go through shared memory (the ring, free
      // once the accumulator is complete): each warp writes its 32 rows of a
      // block of up to 64 columns as [column][128 rows], then the four warps
      // store 16-byte pieces of each column's 128 contiguous output rows.
      const bool vec = go && g.vec_out && g.out_f32 == nullptr;
      __nv_bfloat16 *stg = reinterpret_cast<__nv_bfloat16 *>(base);
#pragma unroll 1
      for (int t = 0; t < mcount && go; ++t) {
        // m tile mt + t: rows m0 + 128 t .., accumulator columns t * BN ..
        const int mm = m + 128 * t;
        const bool mm_ok = mm < g.M_valid;
#pragma unroll 1
        for (int cb = 0; cb < BN; cb += 64) {
          const int ncb = BN < 64 ? BN : 64;
#pragma unroll 1
          for (int c0 = cb; c0 < cb + ncb; c0 += 16) {
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
                  float s, c;
                  rope_sincos(s_pos[c0 + j], g.theta[k], &s, &c);
                  v = (lane & 1) ? partner * s + v * c : v * c - partner * s;
                }
              }
              if (vec) {
                stg[(c0 - cb + j) * 128 + m_local] = __float2bfloat16_rn(v);
                continue;
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
          if (vec) {
            asm volatile("bar.sync 1, 128;" ::: "memory");
            const int mt0 = m0 + 128 * t;
            for (int idx = et; idx < ncb * 16; idx += 128) {
              const int cl = idx >> 4, u = idx & 15, n = n0 + cb + cl, mrow = mt0 + 8 * u;
              if (n >= g.N || mrow >= g.M_valid) continue;
              __nv_bfloat16 *dst;
              if (g.mode == kEpiAppend) {
                const long long row = s_row[cb + cl];
                if (row < 0) continue;
                dst = g.out + row * (long long)(g.d_c + g.d_r) + mrow;
              } else {
                dst = g.out + (long long)n * g.out_ld + (long long)z * g.out_z + mrow;
              }
              *reinterpret_cast<uint4 *>(dst) = *reinterpret_cast<const uint4 *>(stg + cl * 128 + 8 * u);
            }
            asm volatile("bar.sync 1, 128;" ::: "memory");   // the staging block is reused
          }
        }
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
        // every peer's float4 in flight at once, summed in cluster-rank order
        float4 pv[8];
#pragma unroll
        for (int p = 0; p < 8; ++p)
          if (p < ks) pv[p] = ptx::ld_shared_cluster_v4f(ptx::mapa_peer(red + off, (uint32_t)p));
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          if (p < ks) {
            acc.x += pv[p].x;
            acc.y += pv[p].y;
            acc.z += pv[p].z;
            acc.w += pv[p].w;
          }
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
              float si, co;
              rope_sincos(s_pos[c], g.theta[k], &si, &co);
              const float x0 = v[e], x1 = v[e + 1];
              v[e] = x0 * co - x1 * si;
              v[e + 1] = x0 * si + x1 * co;
            }
          }
        }
        __nv_bfloat16 *dst = nullptr;
        float *dst32 = nullptr;
        if (g.mode == kEpiAppend) {
          const long long row = s_row[c];
          if (row < 0) continue;
          if (g.out_f32) dst32 = g.out_f32 + row * (long long)(g.d_c + g.d_r) + m0 + ml;
          else dst = g.out + row * (long long)(g.d_c + g.d_r) + m0 + ml;
        } else {
          dst = g.out + (long long)n * g.out_ld + (long long)z * g.out_z + m0 + ml;
        }
        if (dst && g.vec_out && m0 + ml + 4 <= g.M_valid) {
          // four consecutive rows: one 8-byte store
          const __nv_bfloat162 lo = __floats2bfloat162_rn(v[0], v[1]), hi = __floats2bfloat162_rn(v[2], v[3]);
          uint2 pk;
          pk.x = *reinterpret_cast<const uint32_t *>(&lo);
          pk.y = *reinterpret_cast<const uint32_t *>(&hi);
          *reinterpret_cast<uint2 *>(dst) = pk;
          continue;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (m0 + ml + e >= g.M_valid) continue;
          if (dst32) dst32[e] = v[e];
          else dst[e] = __float2bfloat16_rn(v[e]);
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

size_t smem_tail_of(int bn) { return 256 + (size_t)bn * (8 + 4); }

// Group G (K chunks per TMA box): G divides the slice's chunk count when it
// can, and the ring holds two groups (or the whole slice) in shared memory.
int pick_group(int per, int bn, int mt) {
  const int chunk = mt * kABytes + bn * kKChunk * 2;
  int max_chunks = (int)((kSmemLimit - 1024 - smem_tail_of(bn)) / chunk);
  if (max_chunks > kMaxStages) max_chunks = kMaxStages;
  for (int cand : {4, 2})
    if (per % cand == 0 && (2 * cand <= max_chunks || (per == cand && cand <= max_chunks))) return cand;
  return 1;
}

template <int BN, bool A_MN>
cudaError_t launch_gemm(const CUtensorMap &a0, const CUtensorMap &a1, const CUtensorMap &b, GemmParams g,
                        int mtiles, int ntiles, int nz, cudaStream_t s) {
  if (g.mt_per_cta < 1 || (g.ksplit > 1 && g.mt_per_cta != 1) || g.mt_per_cta * BN > 512)
    return cudaErrorNotSupported;
  g.m_tiles = mtiles;
  const int chunk = g.mt_per_cta * kABytes + b_bytes<BN>();   // one K chunk's A and B
  const int per = (g.num_k_chunks + g.ksplit - 1) / g.ksplit;
  int max_chunks = (int)((kSmemLimit - 1024 - smem_tail<BN>()) / chunk);
  if (max_chunks > kMaxStages) max_chunks = kMaxStages;
  const int G = g.group;
  if (G < 1 || max_chunks < G) return cudaErrorNotSupported;
  int ng = max_chunks / G;
  const int need = (per + G - 1) / G;
  if (ng > need) ng = need > 0 ? need : 1;
  g.stages = ng * G;
  size_t region = (size_t)g.stages * chunk;
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

int pick_bn(long long N) {
  if (N <= 16) return 16;
  if (N <= 32) return 32;
  if (N <= 64) return 64;
  if (N <= 128) return 128;
  return 256;
}

// Tensor maps of one launch: A (two, for a product whose rows come from two
// weights) and B, built for the chosen group G and N tile bn.
struct Maps {
  CUtensorMap a0, a1, b;
};

// Chooses bn, the K split and the group, lets `encode(G, bn, maps)` build the
// tensor maps, and launches.
template <bool A_MN, typename Encode>
cudaError_t dispatch(int N, GemmParams g, int mtiles, int z, cudaStream_t s, Encode encode) {
  const int bn = pick_bn(N);
  const int ntiles = (N + bn - 1) / bn;
  if (g.mt_per_cta == 0) g.mt_per_cta = 1;
  if (g.ksplit == 0)
    g.ksplit = g.mt_per_cta > 1 ? 1 : pick_ksplit((long long)mtiles * ntiles * z, g.num_k_chunks);
  const int per = (g.num_k_chunks + g.ksplit - 1) / g.ksplit;
  g.group = pick_group(per, bn, g.mt_per_cta);
  Maps m;
  if (!encode(g.group, bn, m)) return cudaErrorNotSupported;
  switch (bn) {
    case 16: return launch_gemm<16, A_MN>(m.a0, m.a1, m.b, g, mtiles, ntiles, z, s);
    case 32: return launch_gemm<32, A_MN>(m.a0, m.a1, m.b, g, mtiles, ntiles, z, s);
    case 64: return launch_gemm<64, A_MN>(m.a0, m.a1, m.b, g, mtiles, ntiles, z, s);
    case 128: return launch_gemm<128, A_MN>(m.a0, m.a1, m.b, g, mtiles, ntiles, z, s);
    default: return launch_gemm<256, A_MN>(m.a0, m.a1, m.b, g, mtiles, ntiles, z, s);
  }
}

// A, K-major: a row-major weight [rows][K] viewed as [K/64 chunks][rows][64];
// a box of G chunks x box_rows rows (rows past the weight are zero-filled).
bool map_a_kmajor(CUtensorMap *m, const void *w, uint64_t K, uint64_t rows, int G, uint32_t box_rows = 128) {
  const uint64_t d[3] = {64, rows, K / 64};
  const uint64_t st[2] = {K * 2, 128};
  const uint32_t box[3] = {64, box_rows, (uint32_t)G};
  return encode_map_bf16(m, w, 3, d, st, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// A, MN-major: a row-major weight [K rows][M] viewed as [M/64 chunks][K][64];
// a box of 2 m chunks (one 128-row m tile) x 64 G k rows.
bool map_a_mnmajor(CUtensorMap *m, const void *w, uint64_t M, uint64_t krows, int G) {
  const uint64_t d[3] = {64, krows, M / 64};
  const uint64_t st[2] = {M * 2, 128};
  const uint32_t box[3] = {64, (uint32_t)(64 * G), 2};
  return encode_map_bf16(m, w, 3, d, st, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// B: row-major activations [N][K] viewed as [K/64][N][64]; a box of G chunks x bn rows.
bool map_b(CUtensorMap *m, const void *x, uint64_t K, uint64_t N, int bn, int G) {
  const uint64_t d[3] = {64, N, K / 64};
  const uint64_t st[2] = {K * 2, 128};
  const uint32_t box[3] = {64, (uint32_t)bn, (uint32_t)G};
  return encode_map_bf16(m, x, 3, d, st, box, CU_TENSOR_MAP_SWIZZLE_128B);
}
// B per head: activations [N][Z][K] viewed as [Z][K/64][N][64]; a box of G chunks x bn rows of one head.
bool map_b_heads(CUtensorMap *m, const void *x, uint64_t K, uint64_t Z, uint64_t N, int bn, int G) {
  const uint64_t d[4] = {64, N, K / 64, Z};
  const uint64_t st[3] = {Z * K * 2, 128, K * 2};
  const uint32_t box[4] = {64, (uint32_t)bn, (uint32_t)G, 1};
  return encode_map_bf16(m, x, 4, d, st, box, CU_TENSOR_MAP_SWIZZLE_128B);
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
                             const void *w_uk, void *q_abs, int B, const double *theta, unsigned *status,
                             cudaStream_t s) {
  if (!aligned16(q_nope) || !aligned16(w_uk) || c.d_h % 64 != 0) return cudaErrorNotSupported;
  GemmParams g = blank_params();
  g.mode = kEpiAbsorb;
  // One m tile per CTA (512 CTAs at DeepSeek-V2 shapes).
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
  g.theta = theta_pairs(theta, c.d_r);
  g.d_c = c.d_c;
  g.d_r = c.d_r;
  g.n_h = c.n_h;
  g.status = status;
  g.vec_out = aligned16(q_abs) && c.d_c % 8 == 0 && c.d_r % 8 == 0;
  return dispatch<true>(B, g, c.d_c / 128, c.n_h, s, [&](int G, int bn, Maps &m) {
    // W^UK [n_h d_h, d_c]: row k of head z is k-row z d_h + k, the d_c columns are m.
    if (!map_a_mnmajor(&m.a0, w_uk, c.d_c, (uint64_t)c.n_h * c.d_h, G)) return false;
    m.a1 = m.a0;
    return map_b_heads(&m.b, q_nope, c.d_h, c.n_h, B, bn, G);
  });
}

cudaError_t launch_outproj_tc(const mla_config &c, const void *ctx_lat, const void *w_uv, void *o, int B,
                              unsigned *status, cudaStream_t s) {
  if (!aligned16(ctx_lat) || !aligned16(w_uv) || c.d_h % 128 != 0) return cudaErrorNotSupported;
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
  g.status = status;
  g.vec_out = aligned16(o);
  return dispatch<false>(B, g, c.d_h / 128, c.n_h, s, [&](int G, int bn, Maps &m) {
    if (!map_a_kmajor(&m.a0, w_uv, c.d_c, (uint64_t)c.n_h * c.d_h, G)) return false;
    m.a1 = m.a0;
    return map_b_heads(&m.b, ctx_lat, c.d_c, c.n_h, B, bn, G);
  });
}

cudaError_t launch_linear_tc(const void *x, const void *w, void *y, int M, int K, int N, unsigned *status,
                             cudaStream_t s) {
  // y[N, M] = x[N, K] w[M, K]^T, bf16 in and out, fp32 accumulation.
  if (!aligned16(x) || !aligned16(w) || K % 64 != 0 || M <= 0 || N <= 0) return cudaErrorNotSupported;
  GemmParams g = blank_params();
  g.mode = kEpiWo;
  g.num_k_chunks = K / kKChunk;
  g.M_valid = M;
  g.N = N;
  g.out = (__nv_bfloat16 *)y;
  g.out_ld = M;
  g.status = status;
  g.vec_out = aligned16(y) && M % 8 == 0;
  return dispatch<false>(N, g, (M + 127) / 128, 1, s, [&](int G, int bn, Maps &m) {
    if (!map_a_kmajor(&m.a0, w, K, M, G)) return false;
    m.a1 = m.a0;
    return map_b(&m.b, x, K, N, bn, G);
  });
}

cudaError_t launch_wo_tc(const mla_config &c, const void *o, const void *w_o, void *u, int B, unsigned *status,
                         cudaStream_t s) {
  return launch_linear_tc(o, w_o, u, c.d_model, c.n_h * c.d_h, B, status, s);
}

cudaError_t launch_append_tc(const mla_config &c, const void *h, int B, int T, const int *start_pos,
                             const void *w_dkv, const void *w_kr, void *cache, long long cache_len,
                             const int *block_table, int max_blocks, const double *theta,
                             unsigned *status, cudaStream_t s, float *rows_out) {
  if (!aligned16(h) || !aligned16(w_dkv) || !aligned16(w_kr)) return cudaErrorNotSupported;
  const long long N = (long long)B * T;
  if (N > 65535LL * 256) return cudaErrorNotSupported;
  GemmParams g = blank_params();
  g.mode = kEpiAppend;
  g.num_k_chunks = c.d_model / kKChunk;
  g.M_valid = c.d_c + c.d_r;
  g.N = (int)N;
  g.a_split_tile = c.d_c / 128;
  g.a1_rows = c.d_r < 128 ? c.d_r : 128;
  g.out = (__nv_bfloat16 *)cache;
  g.theta = theta_pairs(theta, c.d_r);
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
  g.vec_out = aligned16(cache) && (c.d_c + c.d_r) % 8 == 0;
  const int mtiles = c.d_c / 128 + (c.d_r + 127) / 128;
  return dispatch<false>((int)N, g, mtiles, 1, s, [&](int G, int bn, Maps &m) {
    // W^DKV rows form the c^KV tiles, W^KR (d_r rows) the last tile
    return map_a_kmajor(&m.a0, w_dkv, c.d_model, c.d_c, G) &&
           map_a_kmajor(&m.a1, w_kr, c.d_model, c.d_r, G, (uint32_t)g.a1_rows) &&
           map_b(&m.b, h, c.d_model, N, bn, G);
  });
}

}  // namespace mla
