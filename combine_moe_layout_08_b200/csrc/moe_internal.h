// Host-side launchers shared between the C entry points and the kernels'
// translation units.  Not part of the public ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include <utility>

#include "moe_layout.h"

namespace moe {
struct TileOut;  // layout_device.cuh
}

#ifndef MOE_USE_PDL
#define MOE_USE_PDL 1  // programmatic dependent launch between the path's kernels
#endif

namespace moe {

// Resident blocks of `kernel` at `threads` per block and `smem` bytes of
// dynamic shared memory on the whole current device (SM count x blocks per
// SM), looked up once per device and configuration.  Grids of persistent
// kernels are sized with it.
int device_block_slots(const void* kernel, int threads, size_t smem = 0);

// Launch `kernel` with programmatic stream serialisation (it may start while
// the previous kernel in `stream` runs; it must pdl_wait() before reading
// anything that kernel writes).
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = MOE_USE_PDL;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Unique id of the CUDA context current on this thread (cuCtxGetId; ids are
// never reused within a process, so a context destroyed and re-created gets
// a new one).  Makes the current device's primary context current if none is.
cudaError_t current_context_id(unsigned long long* id);

// Raise `kernel`'s dynamic shared-memory limit in the current context to at
// least `bytes` (once per context and kernel; no-op up to 48 KB).
cudaError_t allow_dynamic_smem(const void* kernel, size_t bytes);

// Tokens per layout tile: about one tile per SM, at least
// MOE_TILE_MIN_TOKENS, a multiple of 32 (so at most 148 tiles).
int layout_tile_tokens(int M);
int layout_num_tiles(int M);
size_t layout_workspace_bytes(const moe_problem_t& p);

// tiles: grouped-GEMM tile metadata to emit as well (tiles.block_m = 0: none)
cudaError_t launch_layout(const moe_problem_t& p, const int32_t* topk_idx,
                          const int32_t* part_of, const moe_layout_t& lay,
                          void* workspace, cudaStream_t stream, const TileOut& tiles);

cudaError_t launch_dispatch(const moe_problem_t& p, const void* x,
                            const moe_layout_t& lay, void* recv_x,
                            float* recv_scale, cudaStream_t stream);

// One-kernel layout + dispatch: taken for 1 <= M * topk <= MOE_FUSED_ITEMS.
bool layout_dispatch_fused(const moe_problem_t& p);
cudaError_t launch_layout_dispatch(const moe_problem_t& p, const int32_t* topk_idx,
                                   const int32_t* part_of, const moe_layout_t& lay,
                                   const void* x, void* recv_x, float* recv_scale,
                                   const TileOut& tiles, cudaStream_t stream);

// Grouped-GEMM tile metadata of a finished layout, as its own kernel
// (entries per tile array: capacity).
int64_t expert_tiles_capacity(const moe_problem_t& p, int block_m);
cudaError_t launch_expert_tiles(const moe_problem_t& p, const int32_t* part_of,
                                const moe_layout_t& lay, const moe_tiles_t& tiles,
                                cudaStream_t stream);

cudaError_t launch_combine_partial(const moe_problem_t& p, const void* y, const float* w,
                                   const moe_layout_t& lay, void* z, cudaStream_t stream);

cudaError_t launch_combine_reduce(const moe_problem_t& p, const void* z, const moe_layout_t& lay,
                                  void* out, cudaStream_t stream);

cudaError_t launch_ep_plan(int world, int rank, int G, const int32_t* part_counts,
                           const int32_t* expert_counts, const int32_t* part_of,
                           const moe_ep_plan_t& plan, cudaStream_t stream);

cudaError_t launch_ep_dispatch(const moe_problem_t& p, const void* x, const moe_layout_t& lay,
                               const int32_t* send_offset, const moe_ep_peers_t& peers,
                               cudaStream_t stream);
cudaError_t launch_ep_combine(const moe_problem_t& p, const moe_ep_peers_t& y, const float* w,
                              const moe_layout_t& lay, const int32_t* send_offset, void* out,
                              cudaStream_t stream);
cudaError_t launch_ep_reduce(const moe_problem_t& p, const moe_ep_peers_t& z,
                             const moe_layout_t& lay, const int32_t* send_offset, void* out,
                             cudaStream_t stream);

cudaError_t launch_combine(const moe_problem_t& p, const void* y,
                           const float* w, const moe_layout_t& lay, void* out,
                           cudaStream_t stream);

}  // namespace moe
