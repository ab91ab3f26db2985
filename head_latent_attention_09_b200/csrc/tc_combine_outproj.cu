// Split combine fused with the output projection, on the tensor cores
// ("DeepSeek-V2" Appendix C: W^UV is applied after the softmax-weighted sum of
// latents; the merge is the log-sum-exp algebra of the split combine).
//
// One CTA per (head i, 128-row m tile of d_h, tile of <= 64 sequences):
//   ctx[n, i, :] = sum_p e^(lse_p - max) O_p[i, :] / sum_p e^(lse_p - max)
//   o[n, i, m]   = sum_c W^UV_i[m, c] ctx[n, i, c]
// over sequence n's pieces p.  The merged latents never leave the SM: they
// are formed in 128-column phases straight into the MMA's B operand
// (K-major, 128-byte swizzle), rounded to bf16 as ctx_lat would be, and once
// every warp has finished a phase, warp 0 issues that phase's MMAs, so the
// tensor core works while the next phase's partials load.
//
// W^UV_i's 128 rows (128 KB) come by TMA, requested before the kernel waits
// for the attention kernel.  The partials are read with plain vector loads,
// software-pipelined: each warp issues the next step's loads (two pieces of
// each of its sequences) before it accumulates the current ones.  (Staging
// the partials by TMA instead, one {64 columns x pieces} box per phase, was
// measured slower: boxes of 256-byte rows arrived at ~9 GB/s per SM.)
//
// All 16 warps merge (sequences r = warp + 16 j); warp 0 also issues the
// loads and the MMAs, warps 4-7 then read the accumulator back and write o.
// Every wait is bounded.
#include <math_constants.h>

#include "ptx.cuh"

namespace mla {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxPhases = 4;          // d_c <= 512, 128 latent columns per phase
constexpr int kW = 8;                  // pieces per row whose merge weights are kept in shared memory
constexpr int kAChunk = 128 * 64 * 2;  // one 64-wide K chunk of 128 weight rows, bf16
constexpr size_t kSmemLimit = 232448;

struct Params {
  const char *ws;
  WsLayout L;
  int B, n_h, d_h, d_c;
  __nv_bfloat16 *ctx_lat;   // optional
  float *lse;               // optional
  __nv_bfloat16 *o;
  unsigned *status;
};

size_t smem_bytes(int bn, int d_c) {
  return 1024 + (size_t)(d_c / 64) * (kAChunk + bn * 128) + (size_t)bn * kW * 4 + (2 * kMaxPhases + 1) * 8 + 16;
}

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    combine_outproj_kernel(const __grid_constant__ CUtensorMap mapA, const Params g) {
  constexpr int RW = BN / kWarps;      // sequences per warp (1, 2 or 4)
  constexpr int kBChunk = BN * 128;    // one 64-wide K chunk of B: BN rows x 64 bf16
  constexpr uint32_t kTmemCols = BN < 32 ? 32 : BN;
  static_assert(RW >= 1 && BN % kWarps == 0, "tile of 16, 32 or 64 sequences");

  extern __shared__ uint8_t smem_raw[];
  uint8_t *base = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int nchunks = g.d_c / 64, nph = g.d_c / 128;
  uint8_t *sa = base;                        // [nchunks][128 rows][64] bf16, swizzled
  uint8_t *sb = base + nchunks * kAChunk;    // [nchunks][BN rows][64] bf16, swizzled
  float *s_w = reinterpret_cast<float *>(sb + nchunks * kBChunk);   // [BN][kW]
  uint64_t *afull = reinterpret_cast<uint64_t *>(s_w + BN * kW);
  uint64_t *bready = afull + kMaxPhases;
  uint64_t *accf = bready + kMaxPhases;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(accf + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * BN, z = blockIdx.z;
  const int n_h = g.n_h;
  pdl_trigger();

  if (threadIdx.x == 0) {
    for (int i = 0; i < kMaxPhases; ++i) {
      ptx::mbar_init(&afull[i], 1);
      ptx::mbar_init(&bready[i], kWarps);
    }
    ptx::mbar_init(accf, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (threadIdx.x == 0) {
    // The weight does not depend on earlier kernels: all of W^UV_i's rows of
    // this m tile are requested before waiting for them.
    ptx::tma_prefetch_desc(&mapA);
    for (int ph = 0; ph < nph; ++ph) {
      ptx::mbar_arrive_expect_tx(&afull[ph], 2u * (uint32_t)kAChunk);
      ptx::tma_load_3d(sa + ph * 2 * kAChunk, &mapA, &afull[ph], 0, z * g.d_h + m0, 2 * ph);
    }
  }
  pdl_wait();   // the partials come from the attention kernel

  const long long *pb = reinterpret_cast<const long long *>(g.ws + g.L.piece_base_off);
  const float *lse = reinterpret_cast<const float *>(g.ws + g.L.lse_off);
  const float *op = reinterpret_cast<const float *>(g.ws + g.L.opart_off);

  // Row statistics of this warp's sequences r = warp + 16 j, all rows at once
  // (one round trip for the piece ranges, one for the first 32 pieces' log-sum-
  // exps): the pieces' largest log-sum-exp, 1 / sum e^(lse - max) (lane-strided,
  // then across lanes, as the combine kernel sums) and the first kW pieces'
  // weights e^(lse - max) / sum, kept in shared memory.
  long long p0[RW];
  int np[RW];
  float mx[RW], inv[RW];
  {
    long long a = 0, e = 0;
    if (lane < RW) {
      const int n = n0 + warp + kWarps * lane;
      if (n < g.B) {
        a = pb[n];
        e = pb[n + 1];
      }
    }
    long long p1[RW];
    float l0[RW];
#pragma unroll
    for (int j = 0; j < RW; ++j) {
      p0[j] = __shfl_sync(0xffffffffu, a, j);
      p1[j] = __shfl_sync(0xffffffffu, e, j);
    }
#pragma unroll
    for (int j = 0; j < RW; ++j) {
      const long long p = p0[j] + lane;
      l0[j] = p < p1[j] ? lse[part_row(g.L, p, z)] : -CUDART_INF_F;
    }
#pragma unroll
    for (int j = 0; j < RW; ++j) {
      float m = l0[j];
      for (long long p = p0[j] + 32 + lane; p < p1[j]; p += 32) m = fmaxf(m, lse[part_row(g.L, p, z)]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      const bool empty = m == -CUDART_INF_F;
      float tot = 0.f;
      if (!empty) {
        if (p0[j] + lane < p1[j]) tot += expf(l0[j] - m);
        for (long long p = p0[j] + 32 + lane; p < p1[j]; p += 32) tot += expf(lse[part_row(g.L, p, z)] - m);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
      const int r = warp + kWarps * j, n = n0 + r;
      mx[j] = m;
      inv[j] = empty ? 0.f : 1.f / tot;
      np[j] = empty ? 0 : (int)(p1[j] - p0[j]);
      if (lane < kW && lane < np[j]) s_w[r * kW + lane] = expf(l0[j] - m) * inv[j];
      if (lane == 0 && g.lse && n < g.B && blockIdx.x == 0)
        g.lse[(long long)n * n_h + z] = empty ? -CUDART_INF_F : m + logf(tot);
    }
  }
  __syncwarp();
  int kmax = 0;
#pragma unroll
  for (int j = 0; j < RW; ++j) kmax = max(kmax, np[j]);
  // Partial row of (piece p0[j], head i); the piece's columns follow.
  const float *src[RW];
#pragma unroll
  for (int j = 0; j < RW; ++j) src[j] = op + part_row(g.L, p0[j], z) * (long long)g.d_c;

  constexpr uint32_t idesc = idesc_bf16(128, BN, false, false);
  bool ok = true;
  // Steps (phase ph, pieces k, k + 1 of every row), software-pipelined: the
  // next step's loads are issued before this step's are accumulated.  Every
  // phase has at least one step.
  const int KG = kmax > 2 ? (kmax + 1) / 2 : 1;
  const int nsteps = nph * KG;
  auto load_step = [&](int st, float4(&v)[RW][2]) {
    const int k = 2 * (st % KG), f = (st / KG) * 32 + lane;
#pragma unroll
    for (int j = 0; j < RW; ++j)
#pragma unroll
      for (int u = 0; u < 2; ++u)
        if (k + u < np[j]) v[j][u] = __ldg(reinterpret_cast<const float4 *>(src[j] + (long long)(k + u) * g.d_c) + f);
  };
  float4 cur[RW][2], nxt[RW][2];
  float4 acc[RW];
#pragma unroll
  for (int j = 0; j < RW; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
  load_step(0, cur);
#pragma unroll 1
  for (int st = 0; st < nsteps; ++st) {
    const int ph = st / KG, k = 2 * (st % KG);
    if (st + 1 < nsteps) load_step(st + 1, nxt);
#pragma unroll
    for (int j = 0; j < RW; ++j) {
      const int r = warp + kWarps * j;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int kk = k + u;
        if (kk < np[j]) {
          const float w = kk < kW ? s_w[r * kW + kk] : expf(lse[part_row(g.L, p0[j] + kk, z)] - mx[j]) * inv[j];
          acc[j].x += w * cur[j][u].x;
          acc[j].y += w * cur[j][u].y;
          acc[j].z += w * cur[j][u].z;
          acc[j].w += w * cur[j][u].w;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < RW; ++j)
#pragma unroll
      for (int u = 0; u < 2; ++u) cur[j][u] = nxt[j][u];
    if (st % KG != KG - 1) continue;
    // End of phase ph: lane's latent columns 128 ph + 4 lane .. + 3 go to B
    // chunk 2 ph + lane / 16, row r, 16-byte unit (lane % 16) / 2 swizzled
    // with r % 8, half lane % 2.
    const int f = ph * 32 + lane;
    const int chunk = 2 * ph + (lane >> 4), unit = (lane & 15) >> 1;
#pragma unroll
    for (int j = 0; j < RW; ++j) {
      const int r = warp + kWarps * j, n = n0 + r;
      const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[j].x, acc[j].y);
      const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[j].z, acc[j].w);
      uint2 pk;
      pk.x = *reinterpret_cast<const uint32_t *>(&lo);
      pk.y = *reinterpret_cast<const uint32_t *>(&hi);
      *reinterpret_cast<uint2 *>(sb + chunk * kBChunk + r * 128 + ((unit ^ (r & 7)) << 4) + ((lane & 1) << 3)) = pk;
      if (g.ctx_lat && n < g.B && blockIdx.x == 0)
        *reinterpret_cast<uint2 *>(g.ctx_lat + ((long long)n * n_h + z) * g.d_c + 4 * f) = pk;
      acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    ptx::fence_proxy_async_smem();   // the MMAs read B through the async proxy
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(&bready[ph]);
    if (warp == 0) {
      // Phase ph's MMAs, once every warp has written its rows and the
      // weight's two chunks have landed.
      if (lane == 0) {
        ok = ok && ptx::mbar_wait(&bready[ph], 0, g.status, abort_flag) &&
             ptx::mbar_wait(&afull[ph], 0, g.status, abort_flag);
        if (ok) {
          ptx::tc_fence_after();
#pragma unroll
          for (int jj = 0; jj < 2; ++jj) {
            const int kc = 2 * ph + jj;
            const uint32_t a_s = ptx::smem_u32(sa + kc * kAChunk), b_s = ptx::smem_u32(sb + kc * kBChunk);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              ptx::mma_bf16_ss(tmem, ptx::sdesc(a_s + kk * 32, 16, 1024, 2), ptx::sdesc(b_s + kk * 32, 16, 1024, 2),
                               idesc, (kc | kk) != 0 ? 1u : 0u);
          }
        }
      }
      __syncwarp();
    }
  }
  if (threadIdx.x == 0) ptx::mma_commit(accf);   // arrives once every issued MMA is done

  if (warp >= 4 && warp < 8) {
    // Epilogue: warp w reads tensor-memory lanes 32 (w % 4) .. (output rows
    // m0 + 32 (w % 4) ..), stages them as [sequence][128 rows] bf16 over B
    // (free once the accumulator is complete), and the four warps then write
    // o with 16-byte stores.
    const bool acc_ok = ptx::mbar_wait(accf, 0, g.status, abort_flag) && !*abort_flag;
    ptx::tc_fence_after();
    const int q = warp & 3, ml = q * 32 + lane;
    __nv_bfloat16 *ot = reinterpret_cast<__nv_bfloat16 *>(sb);
    if (acc_ok) {
#pragma unroll
      for (int c0 = 0; c0 < BN; c0 += 16) {
        uint32_t rr[16];
        ptx::tmem_ld16(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, rr);
        ptx::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) ot[(c0 + j) * 128 + ml] = __float2bfloat16_rn(__uint_as_float(rr[j]));
      }
    }
    ptx::named_bar_sync(1, 128);
    if (acc_ok) {
      const int et = threadIdx.x - 128;   // 0 .. 127
      for (int idx = et; idx < BN * 16; idx += 128) {
        const int nl = idx >> 4, u = idx & 15, n = n0 + nl;
        if (n < g.B)
          *reinterpret_cast<uint4 *>(g.o + ((long long)n * n_h + z) * g.d_h + m0 + 8 * u) =
              *reinterpret_cast<const uint4 *>(ot + nl * 128 + 8 * u);
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    // Do not leave with weight loads still landing in shared memory.
    if (lane == 0)
      for (int ph = 0; ph < nph; ++ph) {
        volatile int no_abort = 0;
        ptx::mbar_wait(&afull[ph], 0, g.status, &no_abort);
      }
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap &mA, const Params &g, cudaStream_t s) {
  const size_t smem = smem_bytes(BN, g.d_c);
  if (smem > kSmemLimit) return cudaErrorNotSupported;
  auto kern = combine_outproj_kernel<BN>;
  static std::atomic<int> configured[kMaxDevices];
  cudaError_t e = once_per_device(configured, [kern] {
    return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemLimit);
  });
  if (e != cudaSuccess) return e;
  const dim3 grid(g.d_h / 128, (g.B + BN - 1) / BN, g.n_h);
  return launch_pdl(kern, grid, dim3(kThreads), smem, s, 1, mA, g);
}

}  // namespace

cudaError_t launch_combine_outproj_tc(const mla_config &c, const char *ws, const WsLayout &L, int B,
                                      const void *w_uv, void *o, void *ctx_lat, float *lse, unsigned *status,
                                      cudaStream_t s) {
  const uintptr_t opart = (uintptr_t)(ws + L.opart_off);
  if (c.dtype != MLA_BF16 || ((uintptr_t)w_uv & 15u) != 0 || (opart & 15u) != 0 || ((uintptr_t)o & 15u) != 0 ||
      c.d_h % 128 != 0 || c.d_c % 128 != 0 || c.d_c > 128 * kMaxPhases || c.n_h > 65535 ||
      ((uintptr_t)ctx_lat & 7u) != 0)
    return cudaErrorNotSupported;
  Params g;
  g.ws = ws;
  g.L = L;
  g.B = B;
  g.n_h = c.n_h;
  g.d_h = c.d_h;
  g.d_c = c.d_c;
  g.ctx_lat = (__nv_bfloat16 *)ctx_lat;
  g.lse = lse;
  g.o = (__nv_bfloat16 *)o;
  g.status = status;
  // W^UV [n_h d_h][d_c] viewed as [d_c / 64 chunks][rows][64]; a box of two chunks x 128 rows.
  CUtensorMap mA;
  const uint64_t da[3] = {64, (uint64_t)c.n_h * c.d_h, (uint64_t)c.d_c / 64};
  const uint64_t sta[2] = {(uint64_t)c.d_c * 2, 128};
  const uint32_t ba[3] = {64, 128, 2};
  if (!encode_map_bf16(&mA, w_uv, 3, da, sta, ba, CU_TENSOR_MAP_SWIZZLE_128B)) return cudaErrorNotSupported;
  if (B <= 16) return launch_bn<16>(mA, g, s);
  if (B <= 32) return launch_bn<32>(mA, g, s);
  return launch_bn<64>(mA, g, s);
}

}  // namespace mla
