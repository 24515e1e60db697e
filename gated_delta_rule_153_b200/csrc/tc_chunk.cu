// tc_chunk.cu -- tensor-core chunkwise kernels (placeholder until written).
#include "common.cuh"
#include "internal.h"

namespace gdn {
bool tc_supported(const gdn_dims&) { return false; }
size_t tc_fwd_workspace(const gdn_dims&) { return 0; }
size_t tc_bwd_workspace(const gdn_dims&) { return 0; }
void launch_tc_fwd(const gdn_dims&, const void*, const void*, const void*, const float*,
                   const float*, const float*, void*, float*, void*, cudaStream_t) {}
void launch_tc_bwd(const gdn_dims&, const void*, const void*, const void*, const float*,
                   const float*, const float*, const void*, const float*, void*, void*, void*,
                   float*, float*, float*, void*, cudaStream_t) {}
}  // namespace gdn
