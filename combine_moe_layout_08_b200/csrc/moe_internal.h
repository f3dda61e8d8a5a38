// Host-side launchers shared between the C entry points and the kernels'
// translation units.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "moe_layout.h"

namespace moe {

// Tokens per layout tile: about one tile per SM, at least 64 tokens, a
// multiple of 32.
int layout_tile_tokens(int M);
int layout_num_tiles(int M);
size_t layout_workspace_bytes(const moe_problem_t& p);

cudaError_t launch_layout(const moe_problem_t& p, const int32_t* topk_idx,
                          const int32_t* part_of, const moe_layout_t& lay,
                          void* workspace, cudaStream_t stream);

cudaError_t launch_dispatch(const moe_problem_t& p, const void* x,
                            const moe_layout_t& lay, void* recv_x,
                            float* recv_scale, cudaStream_t stream);

cudaError_t launch_combine(const moe_problem_t& p, const void* y,
                           const float* w, const moe_layout_t& lay, void* out,
                           cudaStream_t stream);

}  // namespace moe
