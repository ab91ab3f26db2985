// Split-KV decode attention over the latent cache for 128 heads (DeepSeek-V2
// shapes: d_c = 512, d_h^R = 64, bf16), on pairs of SMs.
//
// What it computes (absorbed MLA, "DeepSeek-V2", Appendix C; softmax of the
// "DeepSeek-V3" note's o_{t,i}): for every (sequence, share) piece,
//   s_j   = q_abs_i . [c_j ; k^R_j] / sqrt(d_h + d_h^R)
//   ctx_i = sum_j softmax_j(s) c_j      and   lse_i = log sum_j e^{s_j}
// over the piece's tokens, written as fp32 partials for the log-sum-exp merge.
//
// Why a pair: the output accumulator of 128 heads x 512 latent columns in fp32
// is 256 KB -- all of one SM's tensor memory -- so it is split across the two
// SMs of a cluster, 64 heads each, and the MMAs are pair MMAs
// (tcgen05.mma.cta_group::2, M = 128).  A pair MMA takes half of A's rows and
// half of B's columns from each CTA's shared memory.  Per 256-token tile:
//   S = Q K^T  (N = 256 tokens): CTA r holds Q rows 64r.. and tokens 128r..
//               of the tile; each CTA receives S for its 64 heads x 256 tokens,
//               folded into 128 lanes x 128 columns (lanes 64.. = tokens 128..).
//   O += P V   (N = 256 latent columns per MMA, two MMAs): CTA r holds P for
//               its heads and columns 128r.. of each 256-column group; each CTA
//               accumulates O for its 64 heads x 512 columns in 256 columns.
// The cache is therefore staged twice per CTA -- once token-split for S, once
// column-split for O -- which raises L2->SM traffic but reads HBM once and
// needs no exchange of partial scores between the SMs.
//
// Why 256-token tiles: one thread issues the MMAs, and back-to-back
// tcgen05.mma instructions cost ~55 cycles each however little work they
// carry; a pair MMA with N = 256 carries 64 cycles of work, so only N = 256
// keeps the tensor pipe busy.  A 256-token tile does not fit in shared memory
// beside the resident query (72 KB), so it is streamed: S = Q K^T in nine
// chunks of 64 columns (this CTA's 128 tokens, 16 KB each), O += P V in eight
// sub-stages of 64 tokens x 128 columns (16 KB each), all through one ring of
// 16 KB slots filled in the order the MMAs consume them.
//
// Warp roles per CTA (224 threads): warps 0 and 6 producers (TMA, and the
// hand copy of a sequence's last partial block; each owns half the ring's
// slots), warp 1 tensor-memory allocation and (leader CTA only) MMA issue,
// warps 2-5 softmax, O rescale and epilogue (one thread per tensor-memory
// lane).
//
// Every wait is bounded; a wait that runs out flags MLA_ERR_TIMEOUT and the
// kernel winds down without further waits.
#include <math_constants.h>

#include "ptx.cuh"

namespace mla {
namespace {

constexpr int kThreads = 224;
// TMA producer warps 0 and 6.  A thread that issues cp.async.bulk.tensor
// copies sustains about two copies per microsecond (about 31 GB/s of 16 KB
// boxes, measured, from L2 or HBM alike), so two threads issue: each owns the
// ring slots s with s % 2 == its index.  Warp 0 also loads Q.  (A third
// producer warp measured slightly slower: it shares a sub-partition with a
// softmax warp.)
constexpr int kProducers = 2;
__device__ __forceinline__ int producer_index(int warp) { return warp == 0 ? 0 : (warp == 6 ? 1 : -1); }
constexpr int kTileTok = 256;           // tokens per pair tile (MMA N of S = Q K^T)
constexpr int kHalfTok = 128;           // tokens of a tile each CTA stages for S
constexpr int kSubTok = 64;             // tokens per O += P V sub-stage
constexpr int kSlot = 16384;            // ring slot: a K chunk (128 rows x 128 B) or a V sub-stage
constexpr int kSlots = 7;               // 112 KB of ring: what is left beside Q (72 KB) and P (32 KB)
constexpr int kQBytes = 9 * 8192;       // 64 heads x 576 bf16, nine 64-column chunks
constexpr int kPBytes = 4 * 8192;       // 64 heads x 256 tokens bf16, four 64-token chunks
constexpr float kRescale = 8.0f;        // rescale O only when the running max grows by > 2^8

// The evict-first L2 hint on a row's last read (the column-split V staging).
#ifndef MLA_PAIR_EVICT
#define MLA_PAIR_EVICT 1
#endif

constexpr int kOffQ = 0;
constexpr int kOffRing = kOffQ + kQBytes;
constexpr int kOffP = kOffRing + kSlots * kSlot;
constexpr int kOffRed = kOffP + kPBytes;                // float red_m[2][128], red_l[128]
constexpr int kOffBar = kOffRed + 3 * 128 * 4;
// barriers
constexpr int kBarFull = 0;                     // [7] leader: 1 arrival + tx bytes of both CTAs
constexpr int kBarEmpty = kBarFull + kSlots;    // [7] both: pair commit
constexpr int kBarQFull = kBarEmpty + kSlots;   // leader: 1 arrival + tx
constexpr int kBarQEmpty = kBarQFull + 1;       // both: pair commit
constexpr int kBarSFull = kBarQEmpty + 1;       // [2] both: pair commit
constexpr int kBarPFull = kBarSFull + 2;        // leader: 8 warp arrivals per tile
constexpr int kBarPFree = kBarPFull + 1;        // both: pair commit after each tile's P.V
constexpr int kBarODone = kBarPFree + 1;        // [2] both: pair commit after P.V of even / odd tiles
constexpr int kBarOFree = kBarODone + 2;        // leader: 8 warp arrivals
constexpr int kBarXchg = kBarOFree + 1;         // [2] local: 4 softmax-warp arrivals (row-max exchange)
constexpr int kBarLsum = kBarXchg + 2;          // local: 4 softmax-warp arrivals (row-sum exchange)
constexpr int kNumBars = kBarLsum + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget");
static_assert(kOffRing % 1024 == 0 && kOffP % 1024 == 0 && kSlot % 1024 == 0,
              "128-byte-swizzled buffers must be 1024-byte aligned");

constexpr uint32_t kTmemCols = 512;         // S: 2 x 128 columns, O: columns 256..511
constexpr uint32_t kColS = 128;
constexpr uint32_t kColO = 256;

constexpr uint32_t kIdescQK = idesc_bf16(128, kTileTok, false, false);
constexpr uint32_t kIdescPV = idesc_bf16(128, 256, false, true);

struct Piece {
  int b;
  long long piece;     // global piece index
  int tok_begin;       // first token of the piece in sequence b
  int tok_end;         // one past the last token attended by this piece
  int ctx;             // the sequence's context length (clamped to the cache)
  int ntiles;          // 256-token MMA tiles
};

struct Walk {
  const long long *tp;
  const long long *pb;
  long long P, Ttot, t0, t1;
  int b;
  int B;
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

// Next piece of this share; false when done.
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

// Cache row of token t of sequence b, or -1 (unmapped / outside the cache).
__device__ __forceinline__ long long kv_row(const AttnArgs &a, int b, int t) {
  if (a.page_size == 0) return (long long)b * a.cache_len + t;
  const int bi = t / kTile;
  if (bi >= a.max_blocks) return -1;
  const int blk = a.block_table[(long long)b * a.max_blocks + bi];
  if (blk < 0 || blk >= a.cache_len) return -1;
  return (long long)blk * kTile + (t % kTile);
}

struct Bars {
  uint64_t *b;
  __device__ uint64_t *full(int s) { return b + kBarFull + s; }
  __device__ uint64_t *empty(int s) { return b + kBarEmpty + s; }
  __device__ uint64_t *qfull() { return b + kBarQFull; }
  __device__ uint64_t *qempty() { return b + kBarQEmpty; }
  __device__ uint64_t *sfull(int i) { return b + kBarSFull + i; }
  __device__ uint64_t *pfull() { return b + kBarPFull; }
  __device__ uint64_t *pfree() { return b + kBarPFree; }
  __device__ uint64_t *odone(int i) { return b + kBarODone + i; }
  __device__ uint64_t *ofree() { return b + kBarOFree; }
  __device__ uint64_t *xchg(int i) { return b + kBarXchg + i; }
  __device__ uint64_t *lsum() { return b + kBarLsum; }
};

// Warp-uniform bounded wait: lane 0 waits, the result is broadcast, the other
// lanes then observe the completed phase themselves (acquire).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, unsigned *status,
                                          volatile int *abort) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = ptx::mbar_wait(bar, parity, status, abort);
  ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
  if (ok && (threadIdx.x & 31) != 0) ptx::mbar_test_wait(bar, parity);
  __syncwarp();
  return ok;
}

// Row coordinate of a block of cache rows starting at token t0 of the piece's
// sequence, or an out-of-range row (TMA then fills zeros) when the block
// starts past the piece.
__device__ __forceinline__ int block_row(const AttnArgs &a, const Piece &p, int t0, long long kv_rows) {
  if (t0 >= p.tok_end) return (int)kv_rows;
  const long long r = kv_row(a, p.b, t0);
  if (r < 0) {
    atomicOr(a.status, kStatusBounds);
    return (int)kv_rows;
  }
  return (int)r;
}

// O += P V sub-stages of a tile that starts at token t0 of the piece (the
// sub-stages past the piece's end are skipped by the producer and the MMAs).
__device__ __forceinline__ int tile_subs(const Piece &p, int t0) {
  const int n = min(p.tok_end - t0, kTileTok);
  return (n + kSubTok - 1) / kSubTok;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    attn_pair_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                     const __grid_constant__ CUtensorMap mapV, const __grid_constant__ CUtensorMap mapV2,
                     const AttnArgs a, const long long kv_rows) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *sQ = sm + kOffQ;
  uint8_t *sRing = sm + kOffRing;
  uint8_t *sP = sm + kOffP;
  float *red_m = reinterpret_cast<float *>(sm + kOffRed);   // [2][128]
  float *red_l = red_m + 256;                                // [128]
  Bars bars{reinterpret_cast<uint64_t *>(sm + kOffBar)};
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(sm + kOffMisc);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(sm + kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = ptx::cluster_ctarank();
  const bool leader = rank == 0;
  const int share = blockIdx.x >> 1;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSlots; ++s) {
      ptx::mbar_init(bars.full(s), 1);
      ptx::mbar_init(bars.empty(s), 1);
    }
    ptx::mbar_init(bars.qfull(), 1);
    ptx::mbar_init(bars.qempty(), 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(bars.sfull(i), 1);
      ptx::mbar_init(bars.odone(i), 1);
      ptx::mbar_init(bars.xchg(i), 4);
    }
    ptx::mbar_init(bars.pfull(), 8);
    ptx::mbar_init(bars.pfree(), 1);
    ptx::mbar_init(bars.ofree(), 8);
    ptx::mbar_init(bars.lsum(), 4);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc_pair(tmem_slot, kTmemCols);
    ptx::tmem_relinquish_pair();
  }
  ptx::tc_fence_before();
  ptx::cluster_sync_all();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // The set-up above overlaps the previous kernel; from here on the plan,
  // the query and the cache it wrote are read.
  pdl_wait();

  if (producer_index(warp) >= 0) {
    // -------------------------------------------------------------- producers
    // Fill the ring in the order the MMAs consume it: the nine K chunks of
    // tile i, then the V sub-stages of tile i-1 (tiles counted across the
    // share's pieces).  Job j goes to slot j % kSlots, owned by producer
    // (j % kSlots) % kProducers, so two threads keep TMA loads in flight at
    // once, while every slot still has one producer that visits its jobs in
    // order: its empty barrier is never more than one phase behind the phase
    // waited for (a parity wait cannot tell one phase behind from three).  Lane 0 issues TMA; the
    // leader arms each slot with the bytes both CTAs' loads bring (the peer's
    // loads count on the leader's barrier directly).  Warp 0 also loads Q.
    const int pid = producer_index(warp);
    const uint32_t lq = ptx::leader_addr(bars.qfull());
    const uint32_t lf0 = ptx::leader_addr(bars.full(0));
    if (lane == 0) {
      ptx::tma_prefetch_desc(&mapQ);
      ptx::tma_prefetch_desc(&mapK);
      ptx::tma_prefetch_desc(&mapV);
      ptx::tma_prefetch_desc(&mapV2);
    }
    Walk w;
    walk_init(w, a, share);
#if MLA_PAIR_EVICT
    const uint64_t last_read = ptx::l2_policy_evict_first();
#endif
    Piece pc, vpc;            // vpc/vt0: the tile whose V sub-stages are pending
    int vt0 = 0;
    bool vpending = false;
    int sc = 0, npc = 0;
    bool ok = true;
    int ws_ = 0;               // ring slot of the next job
    int wround = 0;            // how many times the ring has been filled before
    // Next ring job: returns its slot if this warp owns it (after waiting,
    // in round r >= 1, until the MMAs of round r-1 released it), -2 if the
    // other producer owns it, -1 on a failed wait.  Warp-uniform.
    auto acquire = [&]() -> int {
      const int s = ws_;
      const int r = wround;
      if (++ws_ == kSlots) {
        ws_ = 0;
        ++wround;
      }
      if (s % kProducers != pid) return -2;
      bool got = true;
      if (lane == 0 && r > 0) got = ptx::mbar_wait(bars.empty(s), (r - 1) & 1, a.status, abort_flag);
      got = __shfl_sync(0xffffffffu, got ? 1 : 0, 0) != 0;
      __syncwarp();
      return got ? s : -1;
    };
    // V sub-stages of the tile at token t0 of piece p: tokens t0 + 64t..,
    // latent columns 256g + 128 * rank .. +128.
    auto issue_v = [&](const Piece &p, int t0) -> bool {
      const int nsub = tile_subs(p, t0);
      for (int t = 0; t < nsub; ++t) {
        for (int g = 0; g < 2; ++g) {
          const int s = acquire();
          if (s == -2) continue;
          if (s < 0) return false;
          uint8_t *dst = sRing + s * kSlot;
          const int tok0 = t0 + kSubTok * t;
          if (tok0 + kSubTok > p.ctx) {
            // The block runs past the sequence: the leader copies the valid
            // rows of both CTAs' column halves by hand and zeroes the rest,
            // so that no unwritten cache row (possibly NaN) reaches P.V.
            // 128-byte rows, 16-byte units swizzled by row (the layout a
            // 128-byte-swizzled TMA load produces).  The peer skips it.
            if (leader) {
              const uint32_t own = ptx::smem_u32(dst), peer = ptx::mapa_peer(own, 1);
              for (int u = lane; u < 2 * 2 * 64 * 8; u += 32) {
                const int cta = u >> 10, half = (u >> 9) & 1, row = (u >> 3) & 63, c = u & 7;
                const int tk = tok0 + row;
                uint4 v = make_uint4(0, 0, 0, 0);
                if (tk < p.ctx) {
                  const long long r = kv_row(a, p.b, tk);
                  if (r >= 0)
                    v = *reinterpret_cast<const uint4 *>(reinterpret_cast<const __nv_bfloat16 *>(a.cache) +
                                                         r * 576 + 256 * g + 128 * cta + 64 * half + 8 * c);
                  else
                    atomicOr(a.status, kStatusBounds);
                }
                const uint32_t off = half * 8192 + row * 128 + ((c ^ (row & 7)) << 4);
                ptx::st_shared_cluster_v4(cta ? peer + off : own + off, v);
              }
              ptx::fence_acq_rel_cluster();
              ptx::fence_proxy_async_cluster();
              __syncwarp();
              if (lane == 0) ptx::mbar_arrive(bars.full(s));
            }
          } else if (lane == 0) {
            const int y = block_row(a, p, tok0, kv_rows);
            if (leader) ptx::mbar_arrive_expect_tx(bars.full(s), 2 * kSlot);
            const int feat0 = 256 * g + 128 * (int)rank;
            // one 3D box: 64 rows x both 64-column chunks (chunk index feat0 / 64)
#if MLA_PAIR_EVICT
            ptx::tma_load_3d_pair_hint(dst, &mapV2, lf0 + 8 * s, 0, y, feat0 / 64, last_read);
#else
            ptx::tma_load_3d_pair(dst, &mapV2, lf0 + 8 * s, 0, y, feat0 / 64);
#endif
          }
          ++sc;
        }
      }
      return true;
    };
    while (ok && walk_next(w, a, share, pc)) {
      bool qok = true;
      if (lane == 0) {
        if (pid == 0 && npc > 0) qok = ptx::mbar_wait(bars.qempty(), (npc - 1) & 1, a.status, abort_flag);
        if (pid == 0 && qok) {
          if (leader) ptx::mbar_arrive_expect_tx(bars.qfull(), 2 * kQBytes);
          for (int c = 0; c < 9; ++c)
            ptx::tma_load_2d_pair(sQ + c * 8192, &mapQ, lq, 64 * c, pc.b * 128 + 64 * (int)rank);
        }
      }
      if (!__shfl_sync(0xffffffffu, qok ? 1 : 0, 0)) break;
      for (int k = 0; k < pc.ntiles && ok; ++k) {
        // K chunks of this tile: this CTA's 128 tokens x 64 columns each.
        const int t0 = pc.tok_begin + kTileTok * k;
        const int tr = t0 + kHalfTok * (int)rank;
        int y0 = 0, y1 = 0;
        if (lane == 0) {
          y0 = block_row(a, pc, tr, kv_rows);
          if (a.page_size) y1 = block_row(a, pc, tr + kSubTok, kv_rows);
        }
        for (int c = 0; c < 9; ++c) {
          const int s = acquire();
          if (s == -2) continue;
          if (s < 0) { ok = false; break; }
          if (lane == 0) {
            uint8_t *dst = sRing + s * kSlot;
            if (leader) ptx::mbar_arrive_expect_tx(bars.full(s), 2 * kSlot);
            if (a.page_size == 0) {
              ptx::tma_load_2d_pair(dst, &mapK, lf0 + 8 * s, 64 * c, y0);
            } else {
              // 64-token pages: two 64-row boxes.
              ptx::tma_load_2d_pair(dst, &mapV, lf0 + 8 * s, 64 * c, y0);
              ptx::tma_load_2d_pair(dst + 8192, &mapV, lf0 + 8 * s, 64 * c, y1);
            }
          }
          ++sc;
        }
        if (!ok) break;
        if (vpending && !issue_v(vpc, vt0)) { ok = false; break; }
        vpc = pc;
        vt0 = t0;
        vpending = true;
      }
      ++npc;
    }
    if (ok && vpending) issue_v(vpc, vt0);
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issue
    if (leader && lane == 0) {
      Walk w;
      walk_init(w, a, share);
      Piece pc;
      int npc = 0, i = 0;
      int rs = 0;                 // ring slot of the next job
      uint32_t rph = 0;           // its full-barrier phase parity
      bool ok = true;
      struct PrevTile { int i, first, npc, nsub; } prev{0, 0, 0, 0};
      bool have_prev = false;
      // Descriptors are built once; the start address (bits 0-13, 16-byte
      // units) is advanced by adding offsets.  The issue loop is kept lean:
      // one thread issues every MMA, and its own instruction latency, not the
      // tensor pipe, bounds the rate when the loop does more than it must.
      const uint64_t dQ = ptx::sdesc(ptx::smem_u32(sQ), 16, 1024, 2);
      const uint64_t dK = ptx::sdesc(ptx::smem_u32(sRing), 16, 1024, 2);
      const uint64_t dV = ptx::sdesc(ptx::smem_u32(sRing), 8192, 1024, 2);
      const uint64_t dP = ptx::sdesc(ptx::smem_u32(sP), 16, 1024, 2);
      // Waits for the next ring job; returns its slot or -1.
      auto slot_wait = [&]() -> int {
        const int s = rs;
        if (!ptx::mbar_wait(bars.full(s), rph, a.status, abort_flag)) return -1;
        ptx::tc_fence_after();
        if (++rs == kSlots) {
          rs = 0;
          rph ^= 1u;
        }
        return s;
      };
      auto pv = [&](const PrevTile &t) -> bool {
        if (t.first && t.npc > 0 && !ptx::mbar_wait(bars.ofree(), (t.npc - 1) & 1, a.status, abort_flag))
          return false;
        if (!ptx::mbar_wait(bars.pfull(), t.i & 1, a.status, abort_flag)) return false;
        ptx::tc_fence_after();
        for (int tt = 0; tt < t.nsub; ++tt) {
          const uint64_t ad = dP + (uint64_t)((tt * 8192) >> 4);
          const uint32_t acc0 = (t.first && tt == 0) ? 0u : 1u;
#pragma unroll
          for (int g = 0; g < 2; ++g) {
            const int s = slot_wait();
            if (s < 0) return false;
            // A = P rows (heads) x tokens 64tt + 16j.. (K-major); B = V rows
            // (tokens 16j.. of the sub-stage) x 128 columns in two 64-column
            // chunks 8 KB apart.
            const uint64_t bd = dV + (uint64_t)((s * kSlot) >> 4);
            const uint32_t d = tmem + kColO + 128 * g;
            ptx::mma_bf16_ss_pair(d, ad, bd, kIdescPV, acc0);
            ptx::mma_bf16_ss_pair(d, ad + 2, bd + 128, kIdescPV, 1u);
            ptx::mma_bf16_ss_pair(d, ad + 4, bd + 256, kIdescPV, 1u);
            ptx::mma_bf16_ss_pair(d, ad + 6, bd + 384, kIdescPV, 1u);
            ptx::mma_commit_pair_both(bars.empty(s));
          }
        }
        ptx::mma_commit_pair_both(bars.pfree());
        ptx::mma_commit_pair_both(bars.odone(t.i & 1));
        return true;
      };
      while (ok && walk_next(w, a, share, pc)) {
        if (!ptx::mbar_wait(bars.qfull(), npc & 1, a.status, abort_flag)) { ok = false; break; }
        for (int k = 0; k < pc.ntiles && ok; ++k) {
          const uint32_t dS = tmem + (i & 1) * kColS;
#pragma unroll
          for (int c = 0; c < 9; ++c) {
            const int s = slot_wait();
            if (s < 0) { ok = false; break; }
            // A = Q chunk c (64-column chunks 8 KB apart), B = this slot's
            // 128 tokens x 64 columns; k steps of 16 columns are 32 B apart.
            const uint64_t ad = dQ + (uint64_t)((c * 8192) >> 4);
            const uint64_t bd = dK + (uint64_t)((s * kSlot) >> 4);
            ptx::mma_bf16_ss_pair(dS, ad, bd, kIdescQK, c != 0 ? 1u : 0u);
            ptx::mma_bf16_ss_pair(dS, ad + 2, bd + 2, kIdescQK, 1u);
            ptx::mma_bf16_ss_pair(dS, ad + 4, bd + 4, kIdescQK, 1u);
            ptx::mma_bf16_ss_pair(dS, ad + 6, bd + 6, kIdescQK, 1u);
            ptx::mma_commit_pair_both(bars.empty(s));
          }
          if (!ok) break;
          ptx::mma_commit_pair_both(bars.sfull(i & 1));
          if (k == pc.ntiles - 1) ptx::mma_commit_pair_both(bars.qempty());
          if (have_prev && !pv(prev)) { ok = false; break; }
          prev = {i, k == 0 ? 1 : 0, npc, tile_subs(pc, pc.tok_begin + kTileTok * k)};
          have_prev = true;
          ++i;
        }
        ++npc;
      }
      if (ok && have_prev) pv(prev);
    }
  } else {
    // ------------------------------------------- softmax, rescale, epilogue
    const int q = warp & 3;
    const int l = q * 32 + lane;          // tensor-memory lane of this thread
    const int h = l & 63, th = l >> 6;    // local head, token half
    const uint32_t lane_addr = tmem + ((uint32_t)(q * 32) << 16);
    const uint32_t leader_pfull = ptx::leader_addr(bars.pfull());
    const uint32_t leader_ofree = ptx::leader_addr(bars.ofree());
    float *opart = reinterpret_cast<float *>(a.ws + a.L.opart_off);
    float *lse_out = reinterpret_cast<float *>(a.ws + a.L.lse_off);
    uint8_t *prow = sP + h * 128;         // row h of each 64-token P chunk
    Walk w;
    walk_init(w, a, share);
    Piece pc;
    int i = 0, npc_s = 0;
    bool ok = true;
    while (ok && walk_next(w, a, share, pc)) {
      float m_run = -CUDART_INF_F, l_part = 0.f;
      for (int k = 0; k < pc.ntiles; ++k, ++i) {
        const int base = pc.tok_begin + kTileTok * k + kHalfTok * th;
        const int nvalid = min(max(pc.tok_end - base, 0), kHalfTok);
        const uint32_t scol = lane_addr + (i & 1) * kColS;
        if (!warp_wait(bars.sfull(i & 1), (i >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
        ptx::tc_fence_after();
        // This row's 128 scores, in log2 units, invalid tokens at -inf.
        float v[kHalfTok];
        ptx::tmem_ld64_sync(scol, reinterpret_cast<uint32_t *>(v));
        ptx::tmem_ld64_sync(scol + 64, reinterpret_cast<uint32_t *>(v) + 64);
        float mx[4] = {-CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F, -CUDART_INF_F};
#pragma unroll
        for (int j = 0; j < kHalfTok; ++j) {
          v[j] = j < nvalid ? v[j] * a.scale_log2 : -CUDART_INF_F;
          mx[j & 3] = fmaxf(mx[j & 3], v[j]);
        }
        const float mloc = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
        red_m[(i & 1) * 128 + l] = mloc;
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bars.xchg(i & 1));
        if (!warp_wait(bars.xchg(i & 1), (i >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
        const float m_tile = fmaxf(mloc, red_m[(i & 1) * 128 + (l ^ 64)]);
        bool rescale = false;
        float alpha = 1.f;
        if (m_tile > m_run + kRescale) {
          alpha = exp2f(m_run - m_tile);       // 0 when m_run = -inf
          m_run = m_tile;
          l_part *= alpha;
          rescale = k > 0;
        }
        // Probabilities (bf16 pairs) and their sum, before waiting for the
        // previous tile's P.V, so that only the store below waits for it.
        uint32_t pk[kHalfTok / 2];
        float ps[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < kHalfTok / 2; ++j) {
          const float p0 = ptx::exp2_approx(v[2 * j] - m_run), p1 = ptx::exp2_approx(v[2 * j + 1] - m_run);
          ps[j & 7] += p0 + p1;
          __nv_bfloat162 b2 = __floats2bfloat162_rn(p0, p1);
          pk[j] = *reinterpret_cast<uint32_t *>(&b2);
        }
        const float sum = ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        // P of the previous tile must have been read by its P.V.
        if (i >= 1 && !warp_wait(bars.pfree(), (i - 1) & 1, a.status, abort_flag)) { ok = false; break; }
        // Tokens 128 th + 16c.. are 16-byte units 2(c&3), 2(c&3)+1 of row h of
        // P chunk 2 th + (c >> 2) (128-byte swizzle by row).
#pragma unroll
        for (int c = 0; c < kHalfTok / 16; ++c) {
          uint8_t *chunk = prow + (2 * th + (c >> 2)) * 8192;
          const int u0 = 2 * (c & 3);
          *reinterpret_cast<uint4 *>(chunk + ((u0 ^ (h & 7)) << 4)) =
              make_uint4(pk[8 * c], pk[8 * c + 1], pk[8 * c + 2], pk[8 * c + 3]);
          *reinterpret_cast<uint4 *>(chunk + (((u0 + 1) ^ (h & 7)) << 4)) =
              make_uint4(pk[8 * c + 4], pk[8 * c + 5], pk[8 * c + 6], pk[8 * c + 7]);
        }
        l_part += sum;
        // The rescale (tensor-memory loads and stores, .sync.aligned) is done by
        // the whole warp when any of its rows needs it; other rows use alpha = 1.
        if (__any_sync(0xffffffffu, rescale)) {
          // P.V of the previous tile must be complete before O is rescaled.
          // o_done[b] completes for the P.V of tiles b, b+2, ...; since S of
          // this tile is complete, every P.V up to tile i-2 is too (MMAs of
          // one thread complete in order), so the wait below is never more
          // than one phase away from the barrier's state.
          if (!warp_wait(bars.odone((i - 1) & 1), ((i - 1) >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
          ptx::tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 16; ++c) {
            uint32_t r[16];
            ptx::tmem_ld16(lane_addr + kColO + 16 * c, r);
            ptx::tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) r[j] = __float_as_uint(__uint_as_float(r[j]) * alpha);
            ptx::tmem_st16(lane_addr + kColO + 16 * c, r);
          }
          ptx::tmem_st_wait();
        }
        ptx::fence_proxy_async_smem();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive_remote_addr(leader_pfull);
      }
      if (!ok) break;
      // ---- epilogue of the piece: O / l and the log-sum-exp
      red_l[l] = l_part;
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(bars.lsum());
      if (!warp_wait(bars.lsum(), npc_s & 1, a.status, abort_flag)) { ok = false; break; }
      ++npc_s;
      const float lsum = l_part + red_l[l ^ 64];
      if (!warp_wait(bars.odone((i - 1) & 1), ((i - 1) >> 1) & 1, a.status, abort_flag)) { ok = false; break; }
      ptx::tc_fence_after();
      const float inv = lsum > 0.f ? 1.f / lsum : 0.f;
      const int head = 64 * (int)rank + h;
      float *dst = opart + part_row(a.L, pc.piece, head) * (long long)a.d_c + 128 * th;
#pragma unroll 1
      for (int c = 0; c < 16; ++c) {
        uint32_t r[16];
        ptx::tmem_ld16(lane_addr + kColO + 16 * c, r);
        ptx::tmem_ld_wait();
        float *d = dst + (c >> 3) * 256 + (c & 7) * 16;
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          *reinterpret_cast<float4 *>(d + j) =
              make_float4(__uint_as_float(r[j]) * inv, __uint_as_float(r[j + 1]) * inv,
                          __uint_as_float(r[j + 2]) * inv, __uint_as_float(r[j + 3]) * inv);
      }
      if (th == 0)
        lse_out[part_row(a.L, pc.piece, head)] =
            lsum > 0.f ? (m_run + log2f(lsum)) * 0.69314718055994531f : -CUDART_INF_F;
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive_remote_addr(leader_ofree);
      // red_l is rewritten only after the next piece's per-tile exchanges
    }
  }

  // ---------------------------------------------------------------- teardown
  ptx::tc_fence_before();
  __syncwarp();
  ptx::cluster_sync_all();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc_pair(tmem, kTmemCols);
  }
}

}  // namespace

cudaError_t launch_attn_tc_pair(const AttnArgs &a, int P, cudaStream_t s) {
  if (a.n_h != 128 || a.d_c != 512 || a.d_r != 64) return cudaErrorNotSupported;
  if (a.page_size != 0 && a.page_size != kTile) return cudaErrorNotSupported;
  const long long rows = a.page_size ? a.cache_len * kTile : (long long)a.B * a.cache_len;
  if (rows <= 0 || rows >= (1ll << 31) - 256) return cudaErrorNotSupported;
  CUtensorMap mq, mk, mv, mv2;
  const uint64_t dq[2] = {576, (uint64_t)a.B * 128};
  const uint64_t dkv[2] = {576, (uint64_t)rows};
  const uint64_t st[1] = {576 * 2};
  const uint32_t boxq[2] = {64, 64};
  const uint32_t boxk[2] = {64, kHalfTok};
  const uint32_t boxv[2] = {64, kSubTok};
  // The cache viewed as [9 chunks][rows][64 columns]: one box of 64 rows x 2
  // chunks lands as two 8 KB row-major chunks, the V sub-stage layout.
  const uint64_t dkv3[3] = {64, (uint64_t)rows, 9};
  const uint64_t st3[2] = {576 * 2, 64 * 2};
  const uint32_t boxv3[3] = {64, kSubTok, 2};
  if (!encode_map_bf16(&mq, a.q_abs, 2, dq, st, boxq, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_bf16(&mk, a.cache, 2, dkv, st, boxk, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_bf16(&mv, a.cache, 2, dkv, st, boxv, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_map_bf16(&mv2, a.cache, 3, dkv3, st3, boxv3, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = once_per_device(configured, [] {
    return cudaFuncSetAttribute(attn_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemAlloc);
  });
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_pair_kernel, dim3(2 * P), dim3(kThreads), kSmemAlloc, s, 1, mq, mk, mv, mv2, a, rows);
}

}  // namespace mla
