// Split-KV decode attention over the latent cache for few heads (n_h = 16 or
// 32; DeepSeek-V2-Lite shapes: d_c = 512, d_h^R = 64, bf16), one CTA per SM.
//
// Same result as the 128-head kernel (per piece: ctx_i = softmax(q_abs_i .
// rows / sqrt(d_h + d_h^R)) . c and its log-sum-exp), but with few heads the
// tensor core's M dimension is taken by tokens instead (the transposed form):
//   S^T = K Q^T      M = 64 tokens, N = n_h heads, K = 576 (nine 64-col chunks)
//   O^T += V^T P^T   M = 64 latent columns per MMA (eight blocks), N = n_h,
//                    K = 64 tokens
// A 64-token tile of the cache is read from HBM once into nine 8 KB chunks of
// a 24-slot ring; each chunk serves both products.  This path is HBM-bound
// (30 flop/byte), so the tile is small and the ring deep.  Per-head softmax
// statistics are reductions across tokens, i.e. across threads: warp shuffles
// over the 16 lanes of each M=64 accumulator quarter, then shared memory.
//
// Warp roles (192 threads): warp 0 TMA producer, warp 1 tensor-memory
// allocation and MMA issue, warps 2-5 softmax / rescale / epilogue.
//
// FP8 cache (E4M3 codes, a float32 scale per token and 128-channel group):
// the producer stages each 64 x 64 chunk of codes (4 KB) by TMA, and four
// more warps (6-9) widen it into the bf16 ring slot the MMAs read, applying
// the group scale on the way (code * sigma rounded to bf16).  HBM then
// carries 576 B + 20 B of scales per token instead of 1152 B; the products,
// the softmax and the epilogue are those of the bf16 cache.
#include <cuda_fp8.h>
#include <math_constants.h>

#include "ptx.cuh"

namespace mla {
namespace {

constexpr int kChunk = 8192;               // [64 rows x 128 B]
constexpr int kChunk8 = 4096;              // FP8 staging: [64 rows x 64 B]
constexpr int kTileTok = 64;
constexpr float kRescale = 8.0f;
constexpr int kGroups8 = 5;                // scale groups of a 576-wide row

#ifndef MLA_F8_CONV_WARPS
#define MLA_F8_CONV_WARPS 4
#endif
#ifndef MLA_F8_RING
#define MLA_F8_RING 21
#endif
#ifndef MLA_F8_STAGE16
#define MLA_F8_STAGE16 6
#endif

template <int H, bool F8>
struct Cfg {
  static constexpr int kConvWarps = F8 ? MLA_F8_CONV_WARPS : 0;   // FP8 converter warps (4 or 8)
  static constexpr int kThreads = 192 + 32 * kConvWarps;
  // Ring chunk slots.  A tile holds its nine slots until its P.V is done,
  // which is issued after the next tile's S: at least two tiles' worth.
  static constexpr int kNS = F8 ? (H <= 16 ? MLA_F8_RING : 18) : (H <= 16 ? 24 : 18);
  static constexpr int kNSt = F8 ? (H <= 16 ? MLA_F8_STAGE16 : 8) : 0;  // FP8 staging chunks
  static_assert(!F8 || kNS >= 18, "the ring must hold two tiles");
  static constexpr int kQ = 9 * H * 128;                    // H rows x 576
  static constexpr int kPT = H * 128;                       // P^T: H rows x 64 tokens
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = (kQ + 1023) / 1024 * 1024;
  static constexpr int kOffStage = kOffRing + kNS * kChunk;
  static constexpr int kOffP = kOffStage + kNSt * kChunk8;
  static constexpr int kOffRed = kOffP + 2 * ((kPT + 1023) / 1024 * 1024);  // float [2][4][H] max, [4][H] sum
  static constexpr int kOffBar = kOffRed + 12 * H * 4;
  // barriers
  static constexpr int bFull = 0, bEmpty = kNS, bQFull = 2 * kNS, bQEmpty = bQFull + 1, bSFull = bQEmpty + 1,
                       bPFull = bSFull + 2, bPFree = bPFull + 2, bODone = bPFree + 2, bOFree = bODone + 2,
                       bXchg = bOFree + 1, bLsum = bXchg + 2, bStFull = bLsum + 1, bStEmpty = bStFull + kNSt,
                       kNumBars = bStEmpty + kNSt;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 16 + 1024;
  static constexpr uint32_t kTmemCols = 10 * H <= 256 ? 256 : 512;  // S^T 2 x H, O^T 8 x H
  static constexpr uint32_t kColO = 2 * H;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

// Two E4M3 codes (low byte first) times sigma, as a bf16 pair.
__device__ __forceinline__ uint32_t e4m3x2_to_bf16x2(uint32_t two, float sigma) {
  const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(two & 0xffffu), __NV_E4M3);
  float2 f = __half22float2(__half2(hr));
  f.x *= sigma;
  f.y *= sigma;
  const __nv_bfloat162 b = __float22bfloat162_rn(f);
  return *reinterpret_cast<const uint32_t *>(&b);
}

struct Piece {
  int b;
  long long piece;
  int tok_begin, tok_end, ctx, ntiles;
};

struct Walk {
  const long long *tp, *pb;
  long long P, Ttot, t0, t1;
  int b, B;
};

__device__ __forceinline__ void walk_init(Walk &w, const AttnArgs &a, int share) {
  const WsHeader *hd = reinterpret_cast<const WsHeader *>(a.ws);
  w.P = hd->P;
  w.Ttot = hd->Ttot;
  w.tp = reinterpret_cast<const long long *>(a.ws + a.L.tile_prefix_off);
  w.pb = reinterpret_cast<const long long *>(a.ws + a.L.piece_base_off);
  w.B = a.B;
  if (share >= w.P) {
    w.b = a.B;
    return;
  }
  w.t0 = plan_begin(share, w.P, w.Ttot);
  w.t1 = plan_begin(share + 1, w.P, w.Ttot);
  int lo = 0, hi = a.B;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (w.tp[mid + 1] <= w.t0) lo = mid + 1; else hi = mid;
  }
  w.b = lo;
}

__device__ __forceinline__ bool walk_next(Walk &w, const AttnArgs &a, int share, Piece &pc) {
  while (w.b < w.B && w.tp[w.b] < w.t1) {
    const int b = w.b++;
    const long long s0 = w.t0 > w.tp[b] ? w.t0 : w.tp[b];
    const long long s1 = w.t1 < w.tp[b + 1] ? w.t1 : w.tp[b + 1];
    if (s0 >= s1) continue;
    const int ctx = plan_ctx(a.ws, a.L, b);
    const int beg = plan_begin_tok(a.ws, a.L, b, a.B);
    pc.b = b;
    pc.piece = w.pb[b] + (share - plan_share_of_tile(w.tp[b], w.P, w.Ttot));
    pc.tok_begin = beg + (int)((s0 - w.tp[b]) * kTile);
    const long long e = beg + (s1 - w.tp[b]) * kTile;
    pc.tok_end = (int)(e < ctx ? e : ctx);
    pc.ctx = ctx;
    pc.ntiles = (pc.tok_end - pc.tok_begin + kTileTok - 1) / kTileTok;
    return true;
  }
  return false;
}

__device__ __forceinline__ long long kv_row(const AttnArgs &a, int b, int t) {
  if (a.page_size == 0) return (long long)b * a.cache_len + t;
  const int bi = t / kTile;
  if (bi >= a.max_blocks) return -1;
  const int blk = a.block_table[(long long)b * a.max_blocks + bi];
  if (blk < 0 || blk >= a.cache_len) return -1;
  return (long long)blk * kTile + (t % kTile);
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, unsigned *status, volatile int *abort) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait(bar, parity, status, abort);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok && (threadIdx.x & 31) != 0) ptx::mbar_test_wait(bar, parity);
  __syncwarp();
  return ok;
}

template <int H, bool F8>
__global__ void __launch_bounds__(Cfg<H, F8>::kThreads, 1)
    attn_smallh_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapKV,
                       const AttnArgs a, const long long kv_rows) {
  using C = Cfg<H, F8>;
  constexpr int NS = C::kNS;
  // Staging chunks as a divisor for the FP8 code paths; without FP8 those
  // paths never run and there are no staging barriers (C::kNSt = 0).
  constexpr int NSt = C::kNSt > 0 ? C::kNSt : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = sm + C::kOffQ;
  uint8_t *sRing = sm + C::kOffRing;
  uint8_t *sP = sm + C::kOffP;
  uint8_t *sStage = sm + C::kOffStage;
  constexpr int kPStride = (C::kPT + 1023) / 1024 * 1024;
  float *red_m = reinterpret_cast<float *>(sm + C::kOffRed);  // [2][4][H]
  float *red_s = red_m + 8 * H;                                // [4][H]
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + C::kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int share = blockIdx.x;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      ptx::mbar_init(bar + C::bFull + s, F8 ? C::kConvWarps : 1);   // FP8: every converter warp
      ptx::mbar_init(bar + C::bEmpty + s, 1);
    }
    for (int s = 0; s < C::kNSt; ++s) {
      ptx::mbar_init(bar + C::bStFull + s, 1);
      ptx::mbar_init(bar + C::bStEmpty + s, C::kConvWarps);
    }
    ptx::mbar_init(bar + C::bQFull, 1);
    ptx::mbar_init(bar + C::bQEmpty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bar + C::bSFull + i, 1);
      ptx::mbar_init(bar + C::bPFull + i, 4);
      ptx::mbar_init(bar + C::bPFree + i, 1);
      ptx::mbar_init(bar + C::bXchg + i, 4);
    }
    ptx::mbar_init(bar + C::bODone, 1);
    ptx::mbar_init(bar + C::bODone + 1, 1);
    ptx::mbar_init(bar + C::bOFree, 4);
    ptx::mbar_init(bar + C::bLsum, 4);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, C::kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The set-up above overlaps the previous kernel; from here on the plan,
  // the query and the cache it wrote are read.
  pdl_wait();

  if (warp == 0) {
    // -------------------------------------------------------------- producer
    Walk w;
    walk_init(w, a, share);
    Piece pc;
    int sc = 0, npc = 0;
    bool ok = true;
    if (lane == 0) {
      ptx::tma_prefetch_desc(&mapQ);
      ptx::tma_prefetch_desc(&mapKV);
    }
    while (ok && walk_next(w, a, share, pc)) {
      if (npc > 0 && !warp_wait(bar + C::bQEmpty, (npc - 1) & 1, a.status, abort_flag)) { ok = false; break; }
      if (lane == 0) {
        ptx::mbar_arrive_expect_tx(bar + C::bQFull, C::kQ);
        for (int c = 0; c < 9; ++c)
          ptx::tma_load_2d(sQ + c * H * 128, &mapQ, bar + C::bQFull, 64 * c, pc.b * H);
      }
      for (int k = 0; k < pc.ntiles && ok; ++k) {
        const int tok0 = pc.tok_begin + kTileTok * k;
        const bool manual = tok0 + kTileTok > pc.ctx;     // tile runs past the sequence end
        int y = (int)kv_rows;
        if (!manual) {
          const long long r = kv_row(a, pc.b, tok0);
          if (r >= 0) y = (int)r;
          else if (lane == 0) atomicOr(a.status, kStatusBounds);
        }
        for (int c = 0; c < 9 && F8; ++c) {
          // FP8: stage the 64 x 64 chunk of codes for the converter warps
          const int s = sc % NSt;
          if (sc >= NSt && !warp_wait(bar + C::bStEmpty + s, ((sc / NSt) - 1) & 1, a.status, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *dst = sStage + s * kChunk8;
          if (manual) {
            for (int u = lane; u < 64 * 4; u += 32) {
              const int row = u >> 2, cc = u & 3;
              const int t = tok0 + row;
              uint4 v = make_uint4(0, 0, 0, 0);
              if (t < pc.ctx) {
                const long long r = kv_row(a, pc.b, t);
                if (r >= 0)
                  v = *reinterpret_cast<const uint4 *>(reinterpret_cast<const uint8_t *>(a.cache) + r * 576 +
                                                       64 * c + 16 * cc);
                else
                  atomicOr(a.status, kStatusBounds);
              }
              *reinterpret_cast<uint4 *>(dst + row * 64 + 16 * cc) = v;
            }
            ptx::fence_proxy_async_smem();   // later TMA writes to this slot come after these
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar + C::bStFull + s);
          } else if (lane == 0) {
            ptx::mbar_arrive_expect_tx(bar + C::bStFull + s, kChunk8);
            ptx::tma_load_2d(dst, &mapKV, bar + C::bStFull + s, 64 * c, y);
          }
          ++sc;
        }
        for (int c = 0; c < 9 && !F8; ++c) {
          const int s = sc % NS;
          if (sc >= NS && !warp_wait(bar + C::bEmpty + s, ((sc / NS) - 1) & 1, a.status, abort_flag)) {
            ok = false;
            break;
          }
          uint8_t *dst = sRing + s * kChunk;
          if (manual) {
            // copy valid rows by hand, zero the rest (no unwritten row reaches P V)
            for (int u = lane; u < 64 * 8; u += 32) {
              const int row = u >> 3, cc = u & 7;
              const int t = tok0 + row;
              uint4 v = make_uint4(0, 0, 0, 0);
              if (t < pc.ctx) {
                const long long r = kv_row(a, pc.b, t);
                if (r >= 0)
                  v = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.cache) +
                                                       r * 576 + 64 * c + 8 * cc);
                else
                  atomicOr(a.status, kStatusBounds);
              }
              *reinterpret_cast<uint4 *>(dst + row * 128 + ((cc ^ (row & 7)) << 4)) = v;
            }
            ptx::fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(bar + C::bFull + s);
          } else if (lane == 0) {
            ptx::mbar_arrive_expect_tx(bar + C::bFull + s, kChunk);
            ptx::tma_load_2d(dst, &mapKV, bar + C::bFull + s, 64 * c, y);
          }
          ++sc;
        }
      }
      ++npc;
    }
    if (*abort_flag) {
      const unsigned long long t0 = ptx::globaltimer();
      while (ptx::globaltimer() - t0 < 100000ull) {}
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(64, H, false, false);
      constexpr uint32_t idO = idesc_bf16(64, H, true, false);
      Walk w;
      walk_init(w, a, share);
      Piece pc;
      int sc = 0, npc = 0, i = 0;
      bool ok = true;
      struct Prev { int i, first, npc, slot0; } prev{0, 0, 0, 0};
      bool have_prev = false;
      const uint32_t q0 = ptx::smem_u32(sQ), r0 = ptx::smem_u32(sRing), p0 = ptx::smem_u32(sP);
      auto pv = [&](const Prev &t) -> bool {
        if (t.first && t.npc > 0 && !ptx::mbar_wait(bar + C::bOFree, (t.npc - 1) & 1, a.status, abort_flag))
          return false;
        if (!ptx::mbar_wait(bar + C::bPFull + (t.i & 1), (t.i >> 1) & 1, a.status, abort_flag)) return false;
        ptx::tc_fence_after();
        const uint32_t pt = p0 + (t.i & 1) * kPStride;
        for (int f = 0; f < 8; ++f) {
          const uint32_t slot = r0 + ((t.slot0 + f) % NS) * kChunk;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t ad = ptx::sdesc(slot + j * 2048, kChunk, 1024, 2);   // V^T, MN-major
            const uint64_t bd = ptx::sdesc(pt + j * 32, 16, 1024, 2);          // P^T, K-major
            ptx::mma_bf16_ss(tmem + C::kColO + f * H, ad, bd, idO, (t.first && j == 0) ? 0u : 1u);
          }
        }
        for (int c = 0; c < 9; ++c) ptx::mma_commit(bar + C::bEmpty + (t.slot0 + c) % NS);
        ptx::mma_commit(bar + C::bPFree + (t.i & 1));
        ptx::mma_commit(bar + C::bODone + (t.i & 1));
        return true;
      };
      while (ok && walk_next(w, a, share, pc)) {
        if (!ptx::mbar_wait(bar + C::bQFull, npc & 1, a.status, abort_flag)) { ok = false; break; }
        for (int k = 0; k < pc.ntiles && ok; ++k) {
          const int slot0 = sc % NS;
          for (int c = 0; c < 9; ++c) {
            const int s = sc % NS;
            if (!ptx::mbar_wait(bar + C::bFull + s, (sc / NS) & 1, a.status, abort_flag)) { ok = false; break; }
            ptx::tc_fence_after();
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint64_t ad = ptx::sdesc(r0 + s * kChunk + 32 * j, 16, 1024, 2);       // K rows
              const uint64_t bd = ptx::sdesc(q0 + c * H * 128 + 32 * j, 16, 1024, 2);      // Q rows
              ptx::mma_bf16_ss(tmem + (i & 1) * H, ad, bd, idS, (c | j) != 0 ? 1u : 0u);
            }
            ++sc;
          }
          if (!ok) break;
          ptx::mma_commit(bar + C::bSFull + (i & 1));
          if (k == pc.ntiles - 1) ptx::mma_commit(bar + C::bQEmpty);
          if (have_prev && !pv(prev)) { ok = false; break; }
          prev = {i, k == 0 ? 1 : 0, npc, slot0};
          have_prev = true;
          ++i;
        }
        ++npc;
      }
      if (ok && have_prev) pv(prev);
    }
  } else if (warp < 6) {
    // --------------------------------------- softmax, rescale and epilogue
    // M = 64 accumulators live in lanes 0-15 of each 32-lane quarter: this
    // thread's token (S^T row) or latent column within a block (O^T row) is
    // 16 * q + lane for lane < 16.
    const int q = warp & 3;
    const bool act = lane < 16;
    const int row = 16 * q + (lane & 15);
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
    float *opart = reinterpret_cast<float *>(a.ws + a.L.opart_off);
    float *lse_out = reinterpret_cast<float *>(a.ws + a.L.lse_off);
    Walk w;
    walk_init(w, a, share);
    Piece pc;
    int i = 0, npc = 0;
    bool ok = true;
    while (ok && walk_next(w, a, share, pc)) {
      float m_run[H], l_part[H];
#pragma unroll
      for (int hh = 0; hh < H; ++hh) {
        m_run[hh] = -CUDART_INF_F;
        l_part[hh] = 0.f;
      }
      for (int k = 0; k < pc.ntiles; ++k, ++i) {
        const int tok = pc.tok_begin + kTileTok * k + row;
        const bool valid = act && tok < pc.tok_end;
        if (!warp_wait(bar + C::bSFull + (i & 1), (i >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        float s[H];
#pragma unroll
        for (int c = 0; c < H / 16; ++c) {
          uint32_t r[16];
          ptx::tmem_ld16(lane_addr + (i & 1) * H + 16 * c, r);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) s[16 * c + j] = valid ? __uint_as_float(r[j]) * a.scale_log2 : -CUDART_INF_F;
        }
        // per-head maximum over the tile's 64 tokens
        float mx[H];
#pragma unroll
        for (int hh = 0; hh < H; ++hh) {
          float v = s[hh];
#pragma unroll
          for (int o = 8; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          mx[hh] = v;
        }
        float *rm = red_m + (i & 1) * 4 * H;
        if (lane < 16) {
#pragma unroll
          for (int hb = 0; hb < H; hb += 16) {
            float v = mx[hb];
#pragma unroll
            for (int j = 1; j < 16; ++j) v = lane == j ? mx[hb + j] : v;
            rm[q * H + hb + lane] = v;
          }
        }
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar + C::bXchg + (i & 1));
        if (!warp_wait(bar + C::bXchg + (i & 1), (i >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
        bool any_rescale = false;
        float alpha[H];
#pragma unroll
        for (int hh = 0; hh < H; ++hh) {
          const float mt = fmaxf(fmaxf(rm[hh], rm[H + hh]), fmaxf(rm[2 * H + hh], rm[3 * H + hh]));
          alpha[hh] = 1.f;
          if (mt > m_run[hh] + kRescale) {
            alpha[hh] = exp2f(m_run[hh] - mt);
            any_rescale |= k > 0;
            m_run[hh] = mt;
            l_part[hh] *= alpha[hh];
          }
        }
        float p[H];
#pragma unroll
        for (int hh = 0; hh < H; ++hh) {
          p[hh] = exp2f(s[hh] - m_run[hh]);
          l_part[hh] += p[hh];
        }
        if (i >= 2 && !warp_wait(bar + C::bPFree + (i & 1), ((i >> 1) - 1) & 1, a.status, abort_flag)) {
          ok = false;
          break;
        }
        if (act) {
          // P^T: K-major rows of 64 tokens (128 B) per head, 16-byte units swizzled by row
          uint8_t *pt = sP + (i & 1) * kPStride;
          const int unit = row >> 3, inunit = (row & 7) * 2;
#pragma unroll
          for (int hh = 0; hh < H; ++hh)
            *reinterpret_cast<__nv_bfloat16 *>(pt + hh * 128 + ((unit ^ (hh & 7)) << 4) + inunit) =
                __float2bfloat16_rn(p[hh]);
        }
        if (any_rescale) {
          // P.V of the previous tile must be complete before O^T is rescaled.
          // o_done[b] completes for the P.V of tiles b, b+2, ...; S^T of this
          // tile being complete implies every P.V up to tile i-2 is (MMAs of
          // one thread complete in order), so this wait is never more than
          // one phase away from the barrier's state.
          if (!warp_wait(bar + C::bODone + ((i - 1) & 1), ((i - 1) >> 1) & 1, a.status, abort_flag)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll 1
          for (int f = 0; f < 8; ++f) {
#pragma unroll
            for (int c = 0; c < H / 16; ++c) {
              uint32_t r[16];
              ptx::tmem_ld16(lane_addr + C::kColO + f * H + 16 * c, r);
              ptx::tmem_ld_wait();
#pragma unroll
              for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha[16 * c + j]);
              ptx::tmem_st16(lane_addr + C::kColO + f * H + 16 * c, r);
            }
          }
          ptx::tmem_st_wait();
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bar + C::bPFull + (i & 1));
      }
      if (!ok) break;
      // ---- epilogue: per-head sums across the 64 token rows, then O^T / l
#pragma unroll
      for (int hh = 0; hh < H; ++hh) {
        float v = act ? l_part[hh] : 0.f;
#pragma unroll
        for (int o = 8; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        l_part[hh] = v;
      }
      if (lane < 16) {
#pragma unroll
        for (int hb = 0; hb < H; hb += 16) {
          float v = l_part[hb];
#pragma unroll
          for (int j = 1; j < 16; ++j) v = lane == j ? l_part[hb + j] : v;
          red_s[q * H + hb + lane] = v;
        }
      }
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar + C::bLsum);
      if (!warp_wait(bar + C::bLsum, npc & 1, a.status, abort_flag)) { ok = false; break; }
      float inv[H];
#pragma unroll
      for (int hh = 0; hh < H; ++hh) {
        const float l = red_s[hh] + red_s[H + hh] + red_s[2 * H + hh] + red_s[3 * H + hh];
        inv[hh] = l > 0.f ? 1.f / l : 0.f;
        if (q == 0 && lane == 0)
          lse_out[pc.piece * a.n_h + hh] = l > 0.f ? (m_run[hh] + log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
      }
      if (!warp_wait(bar + C::bODone + ((i - 1) & 1), ((i - 1) >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
      ptx::tc_fence_after();
#pragma unroll 1
      for (int f = 0; f < 8; ++f) {
#pragma unroll
        for (int c = 0; c < H / 16; ++c) {
          uint32_t r[16];
          ptx::tmem_ld16(lane_addr + C::kColO + f * H + 16 * c, r);
          ptx::tmem_ld_wait();
          if (act) {
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const int hh = 16 * c + j;
              opart[(pc.piece * a.n_h + hh) * (long long)a.d_c + 64 * f + row] = __uint_as_float(r[j]) * inv[hh];
            }
          }
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bar + C::bOFree);
      ++npc;
    }
  } else if (F8) {
    // ------------------------------------------ FP8 converters (warps 6 ..)
    // A chunk is 64 rows x 4 units of 16 codes.  Thread ct handles unit ct%4
    // of rows ct/4, ct/4 + RS, ... (RS = rows covered by all converters at
    // once): 16 codes become 32 bytes of bf16, two 16-byte units of the
    // 128-byte-swizzled ring row.
    constexpr int RS = (C::kConvWarps > 0 ? C::kConvWarps : 4) * 8, NR = 64 / RS;
    const int ct = (warp - 6) * 32 + lane;
    const int r0 = ct >> 2, u = ct & 3;
    Walk w;
    walk_init(w, a, share);
    Piece pc;
    int sc = 0;
    bool ok = true;
    while (ok && walk_next(w, a, share, pc)) {
      for (int k = 0; k < pc.ntiles && ok; ++k) {
        const int tok0 = pc.tok_begin + kTileTok * k;
        float sig[NR][kGroups8];
#pragma unroll
        for (int rr = 0; rr < NR; ++rr) {
          const int t = tok0 + r0 + RS * rr;
          const long long r = t < pc.ctx ? kv_row(a, pc.b, t) : -1;
#pragma unroll
          for (int g = 0; g < kGroups8; ++g) sig[rr][g] = r >= 0 ? a.kv_scale[r * kGroups8 + g] : 0.f;
        }
        for (int c = 0; c < 9; ++c) {
          const int st = sc % NSt, s = sc % NS;
          if (!warp_wait(bar + C::bStFull + st, (sc / NSt) & 1, a.status, abort_flag)) { ok = false; break; }
          if (sc >= NS && !warp_wait(bar + C::bEmpty + s, ((sc / NS) - 1) & 1, a.status, abort_flag)) {
            ok = false;
            break;
          }
          const int g = c >> 1;   // chunks 0-7: c^KV groups 0-3; chunk 8: the k^R group
#pragma unroll
          for (int rr = 0; rr < NR; ++rr) {
            const int row = r0 + RS * rr;
            // select the group's scale without indexing the array at run time
            float sg = sig[rr][0];
#pragma unroll
            for (int gg = 1; gg < kGroups8; ++gg) sg = g == gg ? sig[rr][gg] : sg;
            const uint4 raw = *reinterpret_cast<const uint4 *>(sStage + st * kChunk8 + row * 64 + 16 * u);
            uint4 lo, hi;
            lo.x = e4m3x2_to_bf16x2(raw.x, sg);
            lo.y = e4m3x2_to_bf16x2(raw.x >> 16, sg);
            lo.z = e4m3x2_to_bf16x2(raw.y, sg);
            lo.w = e4m3x2_to_bf16x2(raw.y >> 16, sg);
            hi.x = e4m3x2_to_bf16x2(raw.z, sg);
            hi.y = e4m3x2_to_bf16x2(raw.z >> 16, sg);
            hi.z = e4m3x2_to_bf16x2(raw.w, sg);
            hi.w = e4m3x2_to_bf16x2(raw.w >> 16, sg);
            uint8_t *dst = sRing + s * kChunk + row * 128;
            *reinterpret_cast<uint4 *>(dst + (((2 * u) ^ (row & 7)) << 4)) = lo;
            *reinterpret_cast<uint4 *>(dst + (((2 * u + 1) ^ (row & 7)) << 4)) = hi;
          }
          ptx::fence_proxy_async_smem();   // the MMAs read the slot through the async proxy
          __syncwarp();
          if (lane == 0) {
            ptx::mbar_arrive(bar + C::bFull + s);
            ptx::mbar_arrive(bar + C::bStEmpty + st);
          }
          ++sc;
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int H, bool F8>
cudaError_t launch_h(const AttnArgs &a, int P, cudaStream_t s) {
  using C = Cfg<H, F8>;
  const long long rows = a.page_size ? a.cache_len * kTile : (long long)a.B * a.cache_len;
  if (rows <= 0 || rows >= (1ll << 31) - 256) return cudaErrorNotSupported;
  CUtensorMap mq, mkv;
  const uint64_t dq[2] = {576, (uint64_t)a.B * H};
  const uint64_t dkv[2] = {576, (uint64_t)rows};
  const uint64_t st[1] = {576 * 2};
  const uint64_t st8[1] = {576};
  const uint32_t bq[2] = {64, (uint32_t)H}, bkv[2] = {64, 64};
  if (!encode_map_bf16(&mq, a.q_abs, 2, dq, st, bq, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorNotSupported;
  const bool kv_ok = F8 ? encode_map_u8(&mkv, a.cache, 2, dkv, st8, bkv, CU_TENSOR_MAP_SWIZZLE_NONE)
                        : encode_map_bf16(&mkv, a.cache, 2, dkv, st, bkv, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!kv_ok) return cudaErrorNotSupported;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = once_per_device(configured, [] {
    return cudaFuncSetAttribute(attn_smallh_kernel<H, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  });
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_smallh_kernel<H, F8>, dim3(P), dim3(C::kThreads), C::kSmem, s, 1, mq, mkv, a, rows);
}

}  // namespace

cudaError_t launch_attn_tc_smallh(const AttnArgs &a, int P, cudaStream_t s) {
  if (a.d_c != 512 || a.d_r != 64) return cudaErrorNotSupported;
  if (a.page_size != 0 && a.page_size != kTile) return cudaErrorNotSupported;
  if (a.kv_scale) {
    if (a.n_groups != kGroups8) return cudaErrorNotSupported;
    if (a.n_h == 16) return launch_h<16, true>(a, P, s);
    if (a.n_h == 32) return launch_h<32, true>(a, P, s);
    return cudaErrorNotSupported;
  }
  if (a.n_h == 16) return launch_h<16, false>(a, P, s);
  if (a.n_h == 32) return launch_h<32, false>(a, P, s);
  return cudaErrorNotSupported;
}

}  // namespace mla
