// Internal declarations of the entropy-routed selection scope (select.cu),
// used by the C ABI layer.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "lbsa_internal.h"

namespace lbsa {

// Scratch: fp64 partial sums of the row entropies ([B*H*ceil(nB/8)]), per-head
// pool ids and pool tables.  Dynamic shared memory of the pool kernel for
// pools of min(group, H) heads.
size_t select_routed_workspace_bytes(int B, int H, int nB);
size_t select_routed_smem_bytes(int H, int nB, int group);
cudaError_t launch_select_routed(const float* scores, int B, int H, int nB, double p, double threshold, int group,
                                 double* ent_out, int32_t* dom_out, lbsa_blockset* bs, void* workspace,
                                 cudaStream_t s);

}  // namespace lbsa
