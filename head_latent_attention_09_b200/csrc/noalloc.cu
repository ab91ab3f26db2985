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
//  * the array's device address is looked up by mla_create (once per handle,
//    with the handle's device current).  Under lazy module loading that lookup
//    is what loads this file's part of the device image, i.e. what reserves
//    the array on the device, so the entry point itself allocates nothing;
//  * every call on a device uses the same array and leaves its contents
//    behind; calls whose work overlaps on the GPU (different streams without
//    ordering) race on it;
//  * nothing in the array needs to start at zero: each call writes the split
//    plan and every partial it later reads.
#include "internal.cuh"

namespace {

constexpr size_t kStaticScratchBytes = size_t(32) << 20;

// The scratch array.  In host code this name is only a stand-in for the
// device array, never a device address; the address comes from
// cudaGetSymbolAddress on the device in question.
__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

}  // namespace

namespace mla {

// Device address of the scratch array on the current device (set-up step of
// mla_create).  Returns MLA_OK or MLA_ERR_CUDA.
int noalloc_scratch_lookup(void **out) {
  void *p = nullptr;
  if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || !p) {
    *out = nullptr;
    return MLA_ERR_CUDA;
  }
  *out = p;
  return MLA_OK;
}

}  // namespace mla

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
  if (!h->noalloc_scratch) return MLA_ERR_CUDA;
  int P = num_parts ? num_parts : mla_default_num_parts(h);
  if (num_parts == 0) {
    // The default split count may not fit; use the largest that does.
    while (P > 1 && mla::ws_layout(h->cfg, B, P).total > kStaticScratchBytes) --P;
  }
  if (mla::ws_layout(h->cfg, B, P).total > kStaticScratchBytes) return MLA_ERR_WORKSPACE;
  const int a = mla_decode_attn(h, q_abs, cache, cache_len, block_table, max_blocks_per_seq, ctx_len, B, P,
                                h->noalloc_scratch, kStaticScratchBytes, stream);
  if (a != MLA_OK) return a;
  return mla_combine_splits(h, h->noalloc_scratch, kStaticScratchBytes, B, P, ctx_lat, lse, stream);
}
