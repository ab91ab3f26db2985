// Split-KV decode attention over the latent cache for few heads (n_h = 16 or
// 32; DeepSeek-V2-Lite shapes: d_c = 512, d_h^R = 64), one CTA per SM.
//
// Same result as the 128-head kernel (per piece: ctx_i = softmax(q_abs_i .
// rows / sqrt(d_h + d_h^R)) . c and its log-sum-exp), but with few heads the
// tensor core's M dimension is taken by tokens and latent columns instead
// (the transposed form), 128 at a time:
//   S^T = K Q^T      M = 128 tokens, N = n_h heads, K = 576 (nine 64-col chunks)
//   O^T += V^T P^T   M = 128 latent columns per MMA (four blocks), N = n_h,
//                    K = 128 tokens
// A tcgen05.mma instruction takes at least ~124 cycles however little it
// computes (measured), so this path is bound by the number of MMA
// instructions per cached token: M = 128 needs 68 per 128 tokens, half of
// what M = 64 needs.
//
// A 128-token tile of the cache is read from HBM once, as nine 16 KB chunks
// (128 rows x 64 columns): the rotary chunk into a ring of its own (it only
// feeds S), and the eight latent chunks as four pairs into a ring of 32 KB
// pair slots, where each pair is the MN-major A operand of one O^T block (the
// two chunks 16 KB apart).  Both products read the same staged chunks.  A
// tile holds its pair slots until its P.V; the MMAs of the next tile's S that
// have their data already (its rotary chunk, and one pair where the ring has a
// fifth slot) are issued before that P.V, so that the tensor core works
// while the softmax runs.
//
// Per-head softmax statistics are reductions across tokens, i.e. across
// threads: warp shuffles over 32 lanes, then shared memory across the warps.
//
// Warp roles: warps 0 and 6 TMA producers (bf16; FP8 has warp 0 only), warp 1
// tensor-memory allocation and MMA issue, warps 2-5 softmax / rescale /
// epilogue.
//
// FP8 cache (E4M3 codes, a float32 scale per token and 128-channel group):
// the producer stages the codes by TMA (16 heads: per 64-row half of a tile,
// one box of three 64-code chunks), and six more warps (6-11) widen each
// 128 x 64 chunk into the bf16 chunk the MMAs read, applying the group scale
// on the way (code * sigma rounded to bf16).  HBM then carries 576 B + 20 B
// of scales per token instead of 1152 B; the products, the softmax and the
// epilogue are those of the bf16 cache, with the rotary chunk taken last.
// The widening sets the pace: a tile's chunks are widened one after another
// into the pair slots as P.V of the previous tile frees them, at about 0.6 us
// a chunk inside the kernel (a clock trace of one CTA), so the FP8 tile takes
// longer than the bf16 one although it reads half the bytes.
//
// Every wait is bounded; a wait that runs out flags MLA_ERR_TIMEOUT and the
// kernel winds down without further waits.
#include <cuda_fp8.h>
#include <math_constants.h>

#include "ptx.cuh"

namespace mla {
namespace {

constexpr int kTileTok = 128;              // tokens per tile (MMA M of S^T)
constexpr int kChunk = 16384;              // bf16 chunk: 128 rows x 128 B
constexpr int kPair = 2 * kChunk;          // latent pair slot: chunks 2b, 2b + 1
constexpr int kChunk8 = 8192;              // FP8 staging chunk: 128 rows x 64 B
constexpr float kRescale = 8.0f;
constexpr int kGroups8 = 5;                // scale groups of a 576-wide row

template <int H, bool F8>
struct Cfg {
  // FP8 converter warps: six make 12 warps, three per sub-partition, which
  // leaves the 168-register cap of ten warps unchanged (measured 2 % faster
  // than four).
  static constexpr int kConvWarps = F8 ? 6 : 0;
  // bf16: a second TMA producer, warp 6 (the rotary chunk and latent pairs
  // 2-3 of every tile; warp 0 the query and pairs 0-1).  A thread issuing
  // cp.async.bulk.tensor copies sustains about two per microsecond, and a
  // paged tile takes 18 of them (two 64-token pages x nine chunks).
  static constexpr int kProducers = F8 ? 1 : 2;
  static constexpr int kProd1Warp = 6;
  static constexpr int kThreads = 192 + 32 * kConvWarps + 32 * (kProducers - 1);
  // Latent pair slots: a tile takes 4; with a fifth (bf16, 16 heads) the
  // next tile's first pair is staged, and its S^T chunks issued, before P.V
  // of this tile frees a slot.  (FP8 has no room for one beside a staging
  // ring deep enough to cover the TMA latency.)
  static constexpr int kNL = (!F8 && H <= 16) ? 5 : 4;
  static constexpr int kNR = F8 ? 1 : 2;                        // rotary chunk slots
  // FP8 staging: slots of kStCh chunks of codes, laid out [64-row half]
  // [chunk][64 rows][64 B] so that one 3D box brings a half's kStCh chunks
  // (kStCh = 1: a 2D box per half).  16 heads: two slots of three chunks,
  // six copies per tile in place of eighteen.
  static constexpr int kStCh = (F8 && H <= 16) ? 3 : 1;
  static constexpr int kNSt = F8 ? (H <= 16 ? 2 : 3) : 0;       // FP8 staging slots
  static constexpr int kStBytes = kStCh * kChunk8;
  static constexpr int kEarlyPairs = kNL - 4;                   // next tile's pairs issued before P.V
  static constexpr bool kEarlyRope = kNR >= 2;                  // next tile's rotary chunk likewise
  // FP8: S^T takes the latent chunks first and the rotary chunk last, the
  // order in which the converters fill them (chunk indices consecutive, as
  // a multi-chunk staging box needs).
  static constexpr bool kRopeLast = F8;
  static constexpr int kQ = 9 * H * 128;                        // H rows x 576, nine 64-column chunks
  static constexpr int kPT = 2 * H * 128;                       // P^T: H rows x 128 tokens, two 64-token chunks
  static constexpr int kOffQ = 0;
  static constexpr int kOffLat = (kQ + 1023) / 1024 * 1024;
  static constexpr int kOffRope = kOffLat + kNL * kPair;
  static constexpr int kOffStage = kOffRope + kNR * kChunk;
  static constexpr int kOffP = kOffStage + kNSt * kStBytes;
  static constexpr int kPStride = (kPT + 1023) / 1024 * 1024;
  static constexpr int kOffRed = kOffP + 2 * kPStride;          // float [2][4][H] max, [4][H] sum
  static constexpr int kOffBar = kOffRed + 12 * H * 4;
  // barriers
  static constexpr int bLatFull = 0, bLatEmpty = kNL, bRopeFull = 2 * kNL, bRopeEmpty = bRopeFull + kNR,
                       bStFull = bRopeEmpty + kNR, bStEmpty = bStFull + kNSt, bQFull = bStEmpty + kNSt,
                       bQEmpty = bQFull + 1, bSFull = bQEmpty + 1, bPFull = bSFull + 2, bPFree = bPFull + 2,
                       bODone = bPFree + 2, bOFree = bODone + 2, bXchg = bOFree + 1, bLsum = bXchg + 2,
                       kNumBars = bLsum + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmem = kOffMisc + 16 + 1024;
  static constexpr uint32_t kTmemCols = 6 * H <= 128 ? 128 : 256;   // S^T 2 x H, O^T 4 x H
  static constexpr uint32_t kColO = 2 * H;
  static_assert(kSmem <= 227 * 1024, "shared memory budget");
  static_assert(kNL >= 4, "a tile takes four pair slots");
  static_assert(9 % kStCh == 0, "staging slots hold whole thirds or ninths of a row");
  static_assert(!kRopeLast || !kEarlyRope, "the rotary chunk is either first (and may be early) or last");
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
  w.b = reinterpret_cast<const int *>(a.ws + a.L.share_first_off)[share];   // found by the plan
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
    pc.tok_begin = beg + (int)((s0 - w.tp[b]) * a.plan_tile);
    const long long e = beg + (s1 - w.tp[b]) * a.plan_tile;
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

// Row coordinate of the 64-row block of cache rows starting at token t0 of the
// piece's sequence, or an out-of-range row (TMA then fills zeros) when the
// block starts at or past the piece's end.
__device__ __forceinline__ int block_row(const AttnArgs &a, const Piece &p, int t0, long long kv_rows) {
  if (t0 >= p.tok_end) return (int)kv_rows;
  const long long r = kv_row(a, p.b, t0);
  if (r < 0) {
    atomicOr(a.status, kStatusBounds);
    return (int)kv_rows;
  }
  return (int)r;
}

__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, unsigned *status, volatile int *abort) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait(bar, parity, status, abort);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok && (threadIdx.x & 31) != 0) ptx::mbar_test_wait(bar, parity);
  __syncwarp();
  return ok;
}

// A ring of slots consumed in fill order: slot and phase parity of the next use.
struct RingPos {
  int slot = 0;
  uint32_t phase = 0;
  int round = 0;
  __device__ void advance(int n) {
    if (++slot == n) {
      slot = 0;
      phase ^= 1u;
      ++round;
    }
  }
};

// Hand copy of the 64-row half of a tile that holds the sequence's end: rows
// [t0, ctx) of columns [64c, 64c + 64), zeros for rows [ctx, t0 + 64), so
// that no unwritten cache row (possibly NaN) reaches P.V.  bf16: 128-byte
// rows with the 128-byte swizzle; FP8: 64-byte rows, no swizzle.  The whole
// warp copies, every lane issuing all its loads before its stores (a half
// lies inside one 64-token page, so its rows are consecutive).
template <bool F8>
__device__ __forceinline__ void hand_copy_half(const AttnArgs &a, const Piece &p, int t0, int c, uint8_t *dst) {
  const int lane = threadIdx.x & 31;
  constexpr int kUnits = F8 ? 4 : 8;          // 16-byte units per row
  constexpr int kPer = 64 * kUnits / 32;      // units per lane
  const long long r0 = kv_row(a, p.b, t0);
  if (r0 < 0 && lane == 0) atomicOr(a.status, kStatusBounds);
  uint4 v[kPer];
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int u = lane + 32 * k, row = u / kUnits, cc = u % kUnits;
    v[k] = make_uint4(0, 0, 0, 0);
    if (r0 >= 0 && t0 + row < p.ctx)
      v[k] = *reinterpret_cast<const uint4 *>(reinterpret_cast<const uint8_t *>(a.cache) +
                                              (r0 + row) * (F8 ? 576 : 1152) + (F8 ? 64 * c : 128 * c) + 16 * cc);
  }
#pragma unroll
  for (int k = 0; k < kPer; ++k) {
    const int u = lane + 32 * k, row = u / kUnits, cc = u % kUnits;
    const int off = F8 ? row * 64 + 16 * cc : row * 128 + ((cc ^ (row & 7)) << 4);
    *reinterpret_cast<uint4 *>(dst + off) = v[k];
  }
}

template <int H, bool F8>
__global__ void __launch_bounds__(Cfg<H, F8>::kThreads, 1)
    attn_smallh_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapKV,
                       const __grid_constant__ CUtensorMap mapKV64, const __grid_constant__ CUtensorMap mapPair,
                       const AttnArgs a, const long long kv_rows) {
  using C = Cfg<H, F8>;
  constexpr int NL = C::kNL, NR = C::kNR;
  // Staging slots as a divisor for the FP8 code paths; without FP8 those
  // paths never run and there are no staging barriers (C::kNSt = 0).
  constexpr int NSt = C::kNSt > 0 ? C::kNSt : 1;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = sm + C::kOffQ;
  uint8_t *sLat = sm + C::kOffLat;
  uint8_t *sRope = sm + C::kOffRope;
  uint8_t *sStage = sm + C::kOffStage;
  uint8_t *sP = sm + C::kOffP;
  float *red_m = reinterpret_cast<float *>(sm + C::kOffRed);  // [2][4][H]
  float *red_s = red_m + 8 * H;                                // [4][H]
  uint64_t *bar = reinterpret_cast<uint64_t *>(sm + C::kOffBar);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + C::kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int share = blockIdx.x;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < NL; ++s) {
      ptx::mbar_init(bar + C::bLatFull + s, F8 ? 2 * C::kConvWarps : 1);   // FP8: both chunks, every converter
      ptx::mbar_init(bar + C::bLatEmpty + s, 1);
    }
    for (int s = 0; s < NR; ++s) {
      ptx::mbar_init(bar + C::bRopeFull + s, F8 ? C::kConvWarps : 1);
      ptx::mbar_init(bar + C::bRopeEmpty + s, 1);
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
      ptx::mbar_init(bar + C::bODone + i, 1);
      ptx::mbar_init(bar + C::bXchg + i, 4);
    }
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

  if (warp == 0 || (C::kProducers > 1 && warp == C::kProd1Warp)) {
    // ------------------------------------------------------------- producers
    // Per tile, in the order the MMAs consume them: the rotary chunk, then
    // the four latent pairs (bf16), or the nine chunks of codes into the
    // staging ring (FP8: latent chunks 0-7, then the rotary chunk).  With
    // two producers each walks every tile and ring position but fills only
    // its own slots: producer 0 the query and pairs 0-1, producer 1 the
    // rotary chunk and pairs 2-3.
    const int pid = warp == 0 ? 0 : 1;
    const bool own_rope = pid == C::kProducers - 1;
    Walk w;
    walk_init(w, a, share);
    Piece pc;
    RingPos lat, rope, stg;
    int npc = 0;
    bool ok = true;
    if (lane == 0) {
      ptx::tma_prefetch_desc(&mapQ);
      ptx::tma_prefetch_desc(&mapKV);
      ptx::tma_prefetch_desc(&mapKV64);
      if (!F8) ptx::tma_prefetch_desc(&mapPair);
    }
    // Waits (lane 0) for a slot's previous use to be released; warp-uniform.
    auto slot_free = [&](uint64_t *empty, const RingPos &r) -> bool {
      if (r.round == 0) return true;
      return warp_wait(empty, r.phase ^ 1u, a.status, abort_flag);
    };
    while (ok && walk_next(w, a, share, pc)) {
      if (pid == 0) {
        if (npc > 0 && !warp_wait(bar + C::bQEmpty, (npc - 1) & 1, a.status, abort_flag)) { ok = false; break; }
        if (lane == 0) {
          ptx::mbar_arrive_expect_tx(bar + C::bQFull, C::kQ);
          for (int c = 0; c < 9; ++c)
            ptx::tma_load_2d(sQ + c * H * 128, &mapQ, bar + C::bQFull, 64 * c, pc.b * H);
        }
      }
      for (int k = 0; k < pc.ntiles && ok; ++k) {
        const int tok0 = pc.tok_begin + kTileTok * k;
        // Each 64-row half of the tile: wholly inside the sequence (TMA from
        // its rows), wholly past its end (TMA from an out-of-range row: zeros),
        // or holding its end (hand copy).
        int kind[2], yy[2];
#pragma unroll
        for (int h2 = 0; h2 < 2; ++h2) {
          const int t = tok0 + 64 * h2;
          kind[h2] = t + 64 <= pc.ctx ? 0 : (t >= pc.ctx ? 1 : 2);
          int y = (int)kv_rows;
          if (kind[h2] == 0 && lane == 0) y = block_row(a, pc, t, kv_rows);
          yy[h2] = __shfl_sync(0xffffffffu, y, 0);
        }
        const bool whole = a.page_size == 0 && kind[0] == 0 && kind[1] == 0 && yy[0] < kv_rows &&
                           yy[1] == yy[0] + 64;
        const bool partial = kind[0] == 2 || kind[1] == 2;
        // One chunk (column block c) into `dst` as two 64-row halves `half`
        // bytes apart; the barrier is armed with the bytes the TMA brings.
        auto stage_chunk = [&](uint8_t *dst, int c, int half, uint32_t &tx) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2)
            if (kind[h2] == 2) hand_copy_half<F8>(a, pc, tok0 + 64 * h2, c, dst + h2 * half);
          tx += (kind[0] != 2 ? half : 0) + (kind[1] != 2 ? half : 0);
        };
        auto issue_chunk = [&](uint8_t *dst, int c, int half, const CUtensorMap *m64, uint64_t *full) {
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2)
            if (kind[h2] != 2) ptx::tma_load_2d(dst + h2 * half, m64, full, 64 * c, yy[h2]);
        };
        // After any hand copy: make it visible to the tensor core, then arm.
        auto arm = [&](uint64_t *full, uint32_t tx) {
          if (partial) {
            ptx::fence_proxy_async_smem();
            __syncwarp();
          }
          if (lane == 0) ptx::mbar_arrive_expect_tx(full, tx);
        };
        if (F8) {
          // The nine chunks of codes in index order (the rotary chunk last),
          // kStCh to a staging slot: per 64-row half one box of kStCh chunks
          // (3D map) or of one chunk (2D map), or the hand copy of the half
          // that holds the sequence's end.
          constexpr int SC = C::kStCh, kHalfSt = SC * kChunk8 / 2;
          for (int g = 0; g < 9 / SC && ok; ++g) {
            uint64_t *full = bar + C::bStFull + stg.slot;
            if (!slot_free(bar + C::bStEmpty + stg.slot, stg)) { ok = false; break; }
            uint8_t *dst = sStage + stg.slot * C::kStBytes;
            uint32_t tx = 0;
#pragma unroll 1
            for (int h2 = 0; h2 < 2; ++h2) {
              if (kind[h2] == 2) {
#pragma unroll 1
                for (int cc = 0; cc < SC; ++cc)
                  hand_copy_half<true>(a, pc, tok0 + 64 * h2, SC * g + cc, dst + h2 * kHalfSt + cc * (kChunk8 / 2));
              } else {
                tx += kHalfSt;
              }
            }
            arm(full, tx);
            if (lane == 0) {
#pragma unroll
              for (int h2 = 0; h2 < 2; ++h2) {
                if (kind[h2] == 2) continue;
                if (SC == 1) ptx::tma_load_2d(dst + h2 * kHalfSt, &mapKV64, full, 64 * g, yy[h2]);
                else ptx::tma_load_3d(dst + h2 * kHalfSt, &mapKV, full, 0, yy[h2], SC * g);
              }
            }
            stg.advance(NSt);
          }
          continue;
        }
        // bf16: the rotary chunk
        if (!own_rope) {
          rope.advance(NR);
        } else {
          uint64_t *full = bar + C::bRopeFull + rope.slot;
          if (!slot_free(bar + C::bRopeEmpty + rope.slot, rope)) { ok = false; break; }
          uint8_t *dst = sRope + rope.slot * kChunk;
          if (whole) {
            if (lane == 0) {
              ptx::mbar_arrive_expect_tx(full, kChunk);
              ptx::tma_load_2d(dst, &mapKV, full, 512, yy[0]);
            }
          } else {
            uint32_t tx = 0;
            stage_chunk(dst, 8, kChunk / 2, tx);
            arm(full, tx);
            if (lane == 0) issue_chunk(dst, 8, kChunk / 2, &mapKV64, full);
          }
          rope.advance(NR);
        }
        // the four latent pairs
        for (int pb = 0; pb < 4 && ok; ++pb) {
          if (C::kProducers > 1 && (pb >> 1) != pid) {
            lat.advance(NL);
            continue;
          }
          uint64_t *full = bar + C::bLatFull + lat.slot;
          if (!slot_free(bar + C::bLatEmpty + lat.slot, lat)) { ok = false; break; }
          uint8_t *dst = sLat + lat.slot * kPair;
          if (whole) {
            if (lane == 0) {
              // one 3D box: 128 rows x chunks 2pb, 2pb + 1
              ptx::mbar_arrive_expect_tx(full, kPair);
              ptx::tma_load_3d(dst, &mapPair, full, 0, yy[0], 2 * pb);
            }
          } else {
            uint32_t tx = 0;
            stage_chunk(dst, 2 * pb, kChunk / 2, tx);
            stage_chunk(dst + kChunk, 2 * pb + 1, kChunk / 2, tx);
            arm(full, tx);
            if (lane == 0) {
              issue_chunk(dst, 2 * pb, kChunk / 2, &mapKV64, full);
              issue_chunk(dst + kChunk, 2 * pb + 1, kChunk / 2, &mapKV64, full);
            }
          }
          lat.advance(NL);
        }
      }
      ++npc;
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issue
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(128, H, false, false);
      constexpr uint32_t idO = idesc_bf16(128, H, true, false);
      Walk w;
      walk_init(w, a, share);
      Piece pc;
      RingPos lat, rope;   // next slot to consume
      int npc = 0, i = 0;
      bool ok = true;
      const uint32_t q0 = ptx::smem_u32(sQ), l0 = ptx::smem_u32(sLat), r0 = ptx::smem_u32(sRope),
                     p0 = ptx::smem_u32(sP);
      // S^T chunk c of tile i from the staged rows at address `src`.
      auto s_chunk = [&](uint32_t src, int c, uint32_t dS, bool first) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const uint64_t ad = ptx::sdesc(src + 32 * j, 16, 1024, 2);                   // K rows
          const uint64_t bd = ptx::sdesc(q0 + c * H * 128 + 32 * j, 16, 1024, 2);     // Q rows
          ptx::mma_bf16_ss(dS, ad, bd, idS, (first && j == 0) ? 0u : 1u);
        }
      };
      // Chunks of S^T(i) issued ahead of P.V(i-1) (count of pairs, rotary chunk done).
      int early_pairs = 0;
      bool early_rope = false;
      int lat_first = 0;        // pair slots of the tile whose S is being issued start here
      auto wait_full = [&](uint64_t *b, uint32_t ph) -> bool {
        if (!ptx::mbar_wait(b, ph, a.status, abort_flag)) return false;
        ptx::tc_fence_after();
        return true;
      };
      struct Tile { int i, first, npc, lat0; };
      auto pv = [&](const Tile &t) -> bool {
        if (t.first && t.npc > 0 && !ptx::mbar_wait(bar + C::bOFree, (t.npc - 1) & 1, a.status, abort_flag))
          return false;
        if (!wait_full(bar + C::bPFull + (t.i & 1), (t.i >> 1) & 1)) return false;
        const uint32_t pt = p0 + (t.i & 1) * C::kPStride;
        for (int pb = 0; pb < 4; ++pb) {
          const int slot = (t.lat0 + pb) % NL;
          const uint32_t src = l0 + slot * kPair;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            // A = V^T: chunks 2pb, 2pb + 1 (16 KB apart, MN-major) x tokens 16j..;
            // B = P^T: H rows x the same tokens (K-major, 64-token chunks)
            const uint64_t ad = ptx::sdesc(src + 2048 * j, kChunk, 1024, 2);
            const uint64_t bd = ptx::sdesc(pt + (j >> 2) * H * 128 + 32 * (j & 3), 16, 1024, 2);
            ptx::mma_bf16_ss(tmem + C::kColO + pb * H, ad, bd, idO, (t.first && j == 0) ? 0u : 1u);
          }
          ptx::mma_commit(bar + C::bLatEmpty + slot);
        }
        ptx::mma_commit(bar + C::bPFree + (t.i & 1));
        ptx::mma_commit(bar + C::bODone + (t.i & 1));
        return true;
      };
      while (ok && walk_next(w, a, share, pc)) {
        if (!ptx::mbar_wait(bar + C::bQFull, npc & 1, a.status, abort_flag)) { ok = false; break; }
        for (int k = 0; k < pc.ntiles && ok; ++k) {
          const uint32_t dS = tmem + (i & 1) * H;
          // the rest of S^T(i): the rotary chunk and pairs not issued early
          if (!early_rope && !C::kRopeLast) {
            if (!wait_full(bar + C::bRopeFull + rope.slot, rope.phase)) { ok = false; break; }
            s_chunk(r0 + rope.slot * kChunk, 8, dS, true);
          }
          const int rope_slot = rope.slot;
          const uint32_t rope_phase = rope.phase;
          rope.advance(NR);
          for (int pb = early_pairs; pb < 4; ++pb) {
            if (!wait_full(bar + C::bLatFull + lat.slot, lat.phase)) { ok = false; break; }
            const uint32_t src = l0 + lat.slot * kPair;
            s_chunk(src, 2 * pb, dS, C::kRopeLast && pb == 0);
            s_chunk(src + kChunk, 2 * pb + 1, dS, false);
            lat.advance(NL);
          }
          if (!ok) break;
          if (C::kRopeLast) {
            if (!wait_full(bar + C::bRopeFull + rope_slot, rope_phase)) { ok = false; break; }
            s_chunk(r0 + rope_slot * kChunk, 8, dS, false);
          }
          ptx::mma_commit(bar + C::bRopeEmpty + rope_slot);   // the rotary chunk only feeds S
          ptx::mma_commit(bar + C::bSFull + (i & 1));
          if (k == pc.ntiles - 1) ptx::mma_commit(bar + C::bQEmpty);
          const int this_lat0 = lat_first;
          // S^T(i+1) chunks whose data needs no slot of tile i, within the piece
          early_pairs = 0;
          early_rope = false;
          if (k + 1 < pc.ntiles) {
            const uint32_t dN = tmem + ((i + 1) & 1) * H;
            if (C::kEarlyRope) {
              if (!wait_full(bar + C::bRopeFull + rope.slot, rope.phase)) { ok = false; break; }
              s_chunk(r0 + rope.slot * kChunk, 8, dN, true);
              early_rope = true;
            }
            for (int pb = 0; pb < C::kEarlyPairs; ++pb) {
              if (!wait_full(bar + C::bLatFull + lat.slot, lat.phase)) { ok = false; break; }
              const uint32_t src = l0 + lat.slot * kPair;
              s_chunk(src, 2 * pb, dN, !early_rope && pb == 0);
              s_chunk(src + kChunk, 2 * pb + 1, dN, false);
              lat.advance(NL);
              ++early_pairs;
            }
            if (!ok) break;
          }
          lat_first = (this_lat0 + 4) % NL;
          // P.V of this tile (its pairs are released as they are consumed)
          if (!pv({i, k == 0 ? 1 : 0, npc, this_lat0})) { ok = false; break; }
          ++i;
        }
        ++npc;
      }
    }
  } else if (warp < 6) {
    // --------------------------------------- softmax, rescale and epilogue
    // S^T row (token) and O^T row (latent column within a block) of this
    // thread: 32 q + lane.
    const int q = warp & 3;
    const int row = 32 * q + lane;
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
        const bool valid = tok < pc.tok_end;
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
        // per-head maximum over the tile's 128 tokens: 32 lanes, then 4 warps
        float *rm = red_m + (i & 1) * 4 * H;
#pragma unroll
        for (int hh = 0; hh < H; ++hh) {
          float v = s[hh];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
          if (lane == (hh & 31)) rm[q * H + hh] = v;
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
          p[hh] = ptx::exp2_approx(s[hh] - m_run[hh]);
          l_part[hh] += p[hh];
        }
        if (i >= 2 && !warp_wait(bar + C::bPFree + (i & 1), ((i >> 1) - 1) & 1, a.status, abort_flag)) {
          ok = false;
          break;
        }
        {
          // P^T: K-major rows of 64 tokens (128 B) per head in two chunks,
          // 16-byte units swizzled by row
          uint8_t *pt = sP + (i & 1) * C::kPStride + (row >> 6) * H * 128;
          const int rr = row & 63, unit = rr >> 3, inunit = (rr & 7) * 2;
#pragma unroll
          for (int hh = 0; hh < H; ++hh)
            *reinterpret_cast<__nv_bfloat16 *>(pt + hh * 128 + ((unit ^ (hh & 7)) << 4) + inunit) =
                __float2bfloat16_rn(p[hh]);
        }
        if (__any_sync(0xffffffffu, any_rescale)) {
          // P.V of the previous tile must be complete before O^T is rescaled
          // (o_done[(i-1)&1] completes with it; nothing later is issued before
          // this tile's P is full).
          if (!warp_wait(bar + C::bODone + ((i - 1) & 1), ((i - 1) >> 1) & 1, a.status, abort_flag)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
#pragma unroll 1
          for (int f = 0; f < 4; ++f) {
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
      // ---- epilogue: per-head sums across the 128 token rows, then O^T / l
#pragma unroll
      for (int hh = 0; hh < H; ++hh) {
        float v = l_part[hh];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == (hh & 31)) red_s[q * H + hh] = v;
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
          lse_out[part_row(a.L, pc.piece, hh)] = l > 0.f ? (m_run[hh] + log2f(l)) * 0.69314718055994531f : -CUDART_INF_F;
      }
      if (!warp_wait(bar + C::bODone + ((i - 1) & 1), ((i - 1) >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
      ptx::tc_fence_after();
#pragma unroll 1
      for (int f = 0; f < 4; ++f) {
#pragma unroll
        for (int c = 0; c < H / 16; ++c) {
          uint32_t r[16];
          ptx::tmem_ld16(lane_addr + C::kColO + f * H + 16 * c, r);
          ptx::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int hh = 16 * c + j;
            opart[part_row(a.L, pc.piece, hh) * (long long)a.d_c + 128 * f + row] = __uint_as_float(r[j]) * inv[hh];
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
    // A staged chunk is 128 rows x 4 units of 16 codes (each 64-row half of a
    // staging slot holds its kStCh chunks one after another).  Converter
    // thread ct handles units ct + kCT rr of the chunk (unit n: row n / 4,
    // 16 codes n % 4): 16 codes become 32 bytes of bf16, two 16-byte units of
    // the 128-byte-swizzled chunk.  Chunks come in index order: latent
    // chunks 0-7, then the rotary chunk.
    constexpr int kCT = 32 * (C::kConvWarps > 0 ? C::kConvWarps : 1), kUnitsCh = kTileTok * 4;   // (bf16: never runs)
    constexpr int RS = kCT / 4, NRR = (kUnitsCh + kCT - 1) / kCT;
    static_assert(kCT % 4 == 0 && kCT % 32 == 0, "converter rows");
    constexpr int SC = C::kStCh, kHalfSt = SC * kChunk8 / 2;
    const int ct = (warp - 6) * 32 + lane;
    const int r0 = ct >> 2, u = ct & 3;
    // unit rr of this thread lies in the chunk (warp-uniform: kCT and the
    // chunk's unit count are multiples of 32)
    auto has = [&](int rr) { return ct + kCT * rr < kUnitsCh; };
    Walk w;
    walk_init(w, a, share);
    Piece pc;
    RingPos stg, lat, rope;
    bool ok = true;
    auto slot_free = [&](uint64_t *empty, const RingPos &r) -> bool {
      if (r.round == 0) return true;
      return warp_wait(empty, r.phase ^ 1u, a.status, abort_flag);
    };
    while (ok && walk_next(w, a, share, pc)) {
      for (int k = 0; k < pc.ntiles && ok; ++k) {
        const int tok0 = pc.tok_begin + kTileTok * k;
        float sig[NRR][kGroups8];
#pragma unroll
        for (int rr = 0; rr < NRR; ++rr) {
          const int t = tok0 + r0 + RS * rr;
          const long long r = has(rr) && t < pc.ctx ? kv_row(a, pc.b, t) : -1;
#pragma unroll
          for (int g = 0; g < kGroups8; ++g) sig[rr][g] = r >= 0 ? a.kv_scale[r * kGroups8 + g] : 0.f;
        }
        for (int g = 0; g < 9 / SC && ok; ++g) {
          if (!warp_wait(bar + C::bStFull + stg.slot, stg.phase, a.status, abort_flag)) { ok = false; break; }
          const uint8_t *src = sStage + stg.slot * C::kStBytes;
          for (int cc = 0; cc < SC; ++cc) {
            const int c = SC * g + cc;
            uint8_t *dst;
            uint64_t *full;
            if (c == 8) {
              if (!slot_free(bar + C::bRopeEmpty + rope.slot, rope)) { ok = false; break; }
              dst = sRope + rope.slot * kChunk;
              full = bar + C::bRopeFull + rope.slot;
            } else {
              if ((c & 1) == 0 && !slot_free(bar + C::bLatEmpty + lat.slot, lat)) { ok = false; break; }
              dst = sLat + lat.slot * kPair + (c & 1) * kChunk;
              full = bar + C::bLatFull + lat.slot;
            }
            const int gi = c >> 1;   // chunks 0-7: c^KV groups 0-3; chunk 8: the k^R group
#pragma unroll
            for (int rr = 0; rr < NRR; ++rr) {
              if (!has(rr)) continue;
              const int rw = r0 + RS * rr;
              // select the group's scale without indexing the array at run time
              float sg = sig[rr][0];
#pragma unroll
              for (int gg = 1; gg < kGroups8; ++gg) sg = gi == gg ? sig[rr][gg] : sg;
              const uint4 raw = *reinterpret_cast<const uint4 *>(src + (rw >> 6) * kHalfSt + cc * (kChunk8 / 2) +
                                                                 (rw & 63) * 64 + 16 * u);
              uint4 lo, hi;
              lo.x = e4m3x2_to_bf16x2(raw.x, sg);
              lo.y = e4m3x2_to_bf16x2(raw.x >> 16, sg);
              lo.z = e4m3x2_to_bf16x2(raw.y, sg);
              lo.w = e4m3x2_to_bf16x2(raw.y >> 16, sg);
              hi.x = e4m3x2_to_bf16x2(raw.z, sg);
              hi.y = e4m3x2_to_bf16x2(raw.z >> 16, sg);
              hi.z = e4m3x2_to_bf16x2(raw.w, sg);
              hi.w = e4m3x2_to_bf16x2(raw.w >> 16, sg);
              uint8_t *d = dst + rw * 128;
              *reinterpret_cast<uint4 *>(d + (((2 * u) ^ (rw & 7)) << 4)) = lo;
              *reinterpret_cast<uint4 *>(d + (((2 * u + 1) ^ (rw & 7)) << 4)) = hi;
            }
            ptx::fence_proxy_async_smem();   // the MMAs read the slot through the async proxy
            __syncwarp();
            if (lane == 0) ptx::mbar_arrive(full);
            if (c == 8) rope.advance(NR);
            else if (c & 1) lat.advance(NL);
          }
          if (!ok) break;
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(bar + C::bStEmpty + stg.slot);
          stg.advance(NSt);
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
  CUtensorMap mq, mkv, mkv64, mpair;
  const uint64_t dq[2] = {576, (uint64_t)a.B * H};
  const uint64_t dkv[2] = {576, (uint64_t)rows};
  const uint64_t st[1] = {576 * 2};
  const uint64_t st8[1] = {576};
  const uint32_t bq[2] = {64, (uint32_t)H}, bkv[2] = {64, kTileTok}, bkv64[2] = {64, 64};
  if (!encode_map_bf16(&mq, a.q_abs, 2, dq, st, bq, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorNotSupported;
  if (F8) {
    // codes: 64-byte rows, no swizzle (the converters swizzle the bf16 they write)
    if (!encode_map_u8(&mkv64, a.cache, 2, dkv, st8, bkv64, CU_TENSOR_MAP_SWIZZLE_NONE)) return cudaErrorNotSupported;
    mkv = mkv64;
    mpair = mkv64;
    if (C::kStCh > 1) {
      // The codes viewed as [9 chunks][rows][64 codes]: one box of 64 rows x
      // kStCh chunks is one half of a staging slot.
      const uint64_t d3[3] = {64, (uint64_t)rows, 9};
      const uint64_t s3[2] = {576, 64};
      const uint32_t b3[3] = {64, 64, (uint32_t)C::kStCh};
      if (!encode_map_u8(&mkv, a.cache, 3, d3, s3, b3, CU_TENSOR_MAP_SWIZZLE_NONE)) return cudaErrorNotSupported;
    }
  } else {
    // The cache viewed as [9 chunks][rows][64 columns]: one box of 128 rows x 2
    // chunks lands as two 16 KB row-major chunks, a latent pair slot.
    const uint64_t dkv3[3] = {64, (uint64_t)rows, 9};
    const uint64_t st3[2] = {576 * 2, 64 * 2};
    const uint32_t bpair[3] = {64, kTileTok, 2};
    if (!encode_map_bf16(&mkv, a.cache, 2, dkv, st, bkv, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map_bf16(&mkv64, a.cache, 2, dkv, st, bkv64, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !encode_map_bf16(&mpair, a.cache, 3, dkv3, st3, bpair, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorNotSupported;
  }
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = once_per_device(configured, [] {
    return cudaFuncSetAttribute(attn_smallh_kernel<H, F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  });
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_smallh_kernel<H, F8>, dim3(P), dim3(C::kThreads), C::kSmem, s, 1, mq, mkv, mkv64, mpair,
                    a, rows);
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
