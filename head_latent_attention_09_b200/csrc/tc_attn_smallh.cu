#include "internal.cuh"
namespace mla {
cudaError_t launch_attn_tc_smallh(const AttnArgs &, int, cudaStream_t) { return cudaErrorNotSupported; }
}
