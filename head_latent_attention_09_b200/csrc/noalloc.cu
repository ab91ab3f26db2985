// Decode attention plus split combine without any device allocation: the
// split partials live in a fixed scratch array that is part of the library's
// device image, instead of in a workspace the caller allocates.
//
// Who needs this: callers that cannot call cudaMalloc (or any allocating
// routine) on the path that runs attention -- for example code running inside
// a custom allocator or memory-pool callback, a runtime that forbids device
// allocation after start-up, or an embedding that only hands the library
// buffers it already owns.  They still pass the inputs and outputs.
//
// Limits and sharing:
//  * the scratch array holds kStaticScratchBytes (32 MiB); every GPU that
//    loads the library keeps that much device memory until the process exits;
//  * every call on a device uses the same array and leaves its contents
//    behind; calls whose work overlaps on the GPU (different streams without
//    ordering) race on it;
//  * nothing in the array needs to start at zero: each call writes the split
//    plan and every partial it later reads.
#include <mutex>

#include "internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;

// The scratch array.  In host code this name is only a stand-in for the
// device array, never a device address; the address is looked up per device.
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_lock;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of the scratch array on `dev` (which must be current).
// Looked up once per device, on the first call there.
int scratch_address(int dev, void **out) {
  if (dev < 0 || dev >= kMaxDevices) return MLA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) return MLA_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MLA_OK;
}

}  // namespace

extern "C" size_t mla_noalloc_scratch_bytes(void) { return kStaticScratchBytes; }

extern "C" int mla_decode_attn_combine_noalloc(mla_handle *h, const void *q_abs, const void *cache,
                                               long long cache_len, const int *block_table,
                                               int max_blocks_per_seq, const int *ctx_len, int B,
                                               int num_parts, void *ctx_lat, float *lse,
                                               mla_stream_t stream) {
  if (!h || B < 0 || num_parts < 0) return MLA_ERR_INVALID_ARG;
  if (B == 0) return MLA_OK;
  if (!q_abs || !cache || !ctx_len || !ctx_lat) return MLA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLA_ERR_CUDA;
  if (dev != h->device) return MLA_ERR_INVALID_ARG;
  int P = num_parts ? num_parts : mla_default_num_parts(h);
  if (num_parts == 0) {
    // The default split count may not fit; use the largest that does.
    while (P > 1 && mla::ws_layout(h->cfg, B, P).total > kStaticScratchBytes) --P;
  }
  if (mla::ws_layout(h->cfg, B, P).total > kStaticScratchBytes) return MLA_ERR_WORKSPACE;
  void *scratch = nullptr;
  const int st = scratch_address(dev, &scratch);
  if (st != MLA_OK) return st;
  const int a = mla_decode_attn(h, q_abs, cache, cache_len, block_table, max_blocks_per_seq, ctx_len, B, P,
                                scratch, kStaticScratchBytes, stream);
  if (a != MLA_OK) return a;
  return mla_combine_splits(h, scratch, kStaticScratchBytes, B, P, ctx_lat, lse, stream);
}
