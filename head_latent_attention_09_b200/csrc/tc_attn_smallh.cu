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
#include <math_constants.h>

#include "ptx.cuh"

namespace mla {
namespace {

constexpr int kThreads = 192;
constexpr int kChunk = 8192;               // [64 rows x 128 B]
constexpr int kTileTok = 64;
constexpr float kRescale = 8.0f;

template <int H>
struct Cfg {
  static constexpr int kNS = H <= 16 ? 24 : 18;             // ring chunk slots
  static constexpr int kQ = 9 * H * 128;                    // H rows x 576
  static constexpr int kPT = H * 128;                       // P^T: H rows x 64 tokens
  static constexpr int kOffQ = 0;
  static constexpr int kOffRing = (kQ + 1023) / 1024 * 1024;
  static constexpr int kOffP = kOffRing + kNS * kChunk;
  static constexpr int kOffRed = kOffP + 2 * ((kPT + 1023) / 1024 * 1024);  // float [2][4][H] max, [4][H] sum
  static constexpr int kOffBar = kOffRed + 12 * H * 4;
  // barriers
  static constexpr int bFull = 0, bEmpty = kNS, bQFull = 2 * kNS, bQEmpty = bQFull + 1, bSFull = bQEmpty + 1,
                       bPFull = bSFull + 2, bPFree = bPFull + 2, bODone = bPFree + 2, bOFree = bODone + 2,
                       bXchg = bOFree + 1, bLsum = bXchg + 2, kNumBars = bLsum + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 16 + 1024;
  static constexpr uint32_t kTmemCols = 10 * H <= 256 ? 256 : 512;  // S^T 2 x H, O^T 8 x H
  static constexpr uint32_t kColO = 2 * H;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
};

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
    int ctx = a.ctx_len[b];
    if (a.page_size == 0 && ctx > a.cache_len) ctx = (int)a.cache_len;
    pc.b = b;
    pc.piece = w.pb[b] + (share - plan_share_of_tile(w.tp[b], w.P, w.Ttot));
    pc.tok_begin = (int)((s0 - w.tp[b]) * kTile);
    const long long e = (s1 - w.tp[b]) * kTile;
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

template <int H>
__global__ void __launch_bounds__(kThreads, 1)
    attn_smallh_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapKV,
                       const AttnArgs a, const long long kv_rows) {
  using C = Cfg<H>;
  constexpr int NS = C::kNS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = sm + C::kOffQ;
  uint8_t *sRing = sm + C::kOffRing;
  uint8_t *sP = sm + C::kOffP;
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
      ptx::mbar_init(bar + C::bFull + s, 1);
      ptx::mbar_init(bar + C::bEmpty + s, 1);
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
        for (int c = 0; c < 9; ++c) {
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
  } else {
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
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int H>
cudaError_t launch_h(const AttnArgs &a, int P, cudaStream_t s) {
  using C = Cfg<H>;
  const long long rows = a.page_size ? a.cache_len * kTile : (long long)a.B * a.cache_len;
  if (rows <= 0 || rows >= (1ll << 31) - 256) return cudaErrorNotSupported;
  CUtensorMap mq, mkv;
  const uint64_t dq[2] = {576, (uint64_t)a.B * H};
  const uint64_t dkv[2] = {576, (uint64_t)rows};
  const uint64_t st[1] = {576 * 2};
  const uint32_t bq[2] = {64, (uint32_t)H}, bkv[2] = {64, 64};
  if (!encode_map_bf16(&mq, a.q_abs, 2, dq, st, bq, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_bf16(&mkv, a.cache, 2, dkv, st, bkv, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_smallh_kernel<H>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  return launch_pdl(attn_smallh_kernel<H>, dim3(P), dim3(kThreads), C::kSmem, s, 1, mq, mkv, a, rows);
}

}  // namespace

cudaError_t launch_attn_tc_smallh(const AttnArgs &a, int P, cudaStream_t s) {
  if (a.d_c != 512 || a.d_r != 64) return cudaErrorNotSupported;
  if (a.page_size != 0 && a.page_size != kTile) return cudaErrorNotSupported;
  if (a.n_h == 16) return launch_h<16>(a, P, s);
  if (a.n_h == 32) return launch_h<32>(a, P, s);
  return cudaErrorNotSupported;
}

}  // namespace mla
