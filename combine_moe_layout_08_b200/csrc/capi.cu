// extern "C" entry points of libmoe_layout.so: argument validation (before
// any CUDA call, so that a bad call costs nothing on the device) and the
// launches.  See include/moe_layout.h for the contract of each call.
#include <cstdint>

#include "layout_device.cuh"
#include "moe_internal.h"
#include "moe_layout.h"

namespace {

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool valid_problem(const moe_problem_t* p) {
  if (!p) return false;
  if (p->M < 0 || p->N <= 0 || p->N > MOE_MAX_N || (p->N % 8) != 0) return false;
  if (p->G < 1 || p->G > MOE_MAX_G) return false;
  if (p->topk < 1 || p->topk > MOE_MAX_TOPK) return false;
  if (p->E_part < 1 || p->E_part > MOE_MAX_E_PART) return false;
  if ((p->dedup != 0 && p->dedup != 1) || (p->fp8 != 0 && p->fp8 != 1)) return false;
  if (p->fp8 && (p->N % 128) != 0) return false;
  if ((int64_t)p->M * p->topk >= ((int64_t)1 << 31)) return false;
  if ((int64_t)p->M * p->E_part >= ((int64_t)1 << 31)) return false;
  return true;
}

// device int32 array: present and 4-byte aligned
bool arr(const void* q) { return q != nullptr && aligned(q, 4); }

bool valid_layout(const moe_problem_t* p, const moe_layout_t* l) {
  if (!l) return false;
  if (!arr(l->expert_count) || !arr(l->expert_offset) || !arr(l->part_count) ||
      !arr(l->part_offset) || !arr(l->exp_row) || !arr(l->disp_token) || !arr(l->status))
    return false;
  if (p->dedup && (!arr(l->disp_row) || !arr(l->exp_to_disp))) return false;
  return true;
}

int cuda_rc(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

// tile metadata request: block_m >= 1, arrays present and aligned, capacity
// below 2^31 entries
bool valid_tiles(const moe_problem_t* p, const moe_tiles_t* t) {
  if (!t || t->block_m < 1) return false;
  if (!arr(t->tile_first) || !arr(t->tile_expert) || !arr(t->tile_row) || !arr(t->tile_rows))
    return false;
  return moe::expert_tiles_capacity(*p, t->block_m) < ((int64_t)1 << 31);
}

moe::TileOut tile_out(const moe_tiles_t* t) {
  moe::TileOut o{};
  if (t) {
    o.block_m = t->block_m;
    o.tile_first = t->tile_first;
    o.tile_expert = t->tile_expert;
    o.tile_row = t->tile_row;
    o.tile_rows = t->tile_rows;
  }
  return o;
}

}  // namespace

extern "C" {

int moe_abi_version(void) { return MOE_ABI_VERSION; }

const char* moe_status_string(int code) {
  switch (code) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "invalid argument (sizes, null or misaligned pointer)";
    case MOE_ERR_WORKSPACE: return "workspace missing or smaller than moe_layout_workspace_size()";
    case MOE_ERR_CUDA: return "CUDA launch failed";
    default: return "unknown status code";
  }
}

size_t moe_layout_workspace_size(const moe_problem_t* prob) {
  if (!valid_problem(prob)) return 0;
  return moe::layout_workspace_bytes(*prob);
}

int moe_layout(const moe_problem_t* prob, const int32_t* topk_idx, const int32_t* part_of,
               const moe_layout_t* lay, void* workspace, size_t workspace_bytes,
               moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay)) return MOE_ERR_ARG;
  if (!arr(part_of) || (prob->M > 0 && !arr(topk_idx))) return MOE_ERR_ARG;
  const size_t need = moe::layout_workspace_bytes(*prob);
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < need) return MOE_ERR_WORKSPACE;
  return cuda_rc(moe::launch_layout(*prob, topk_idx, part_of, *lay, workspace,
                                    reinterpret_cast<cudaStream_t>(stream), moe::TileOut{}));
}

int moe_dispatch(const moe_problem_t* prob, const void* x, const moe_layout_t* lay,
                 void* recv_x, float* recv_scale, moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay)) return MOE_ERR_ARG;
  if (prob->M > 0) {
    if (!x || !aligned(x, 16) || !recv_x || !aligned(recv_x, 16)) return MOE_ERR_ARG;
    if (prob->fp8 && (!recv_scale || !aligned(recv_scale, 16))) return MOE_ERR_ARG;
  }
  return cuda_rc(moe::launch_dispatch(*prob, x, *lay, recv_x, recv_scale,
                                      reinterpret_cast<cudaStream_t>(stream)));
}

int moe_layout_dispatch_fused(const moe_problem_t* prob) {
  return valid_problem(prob) && moe::layout_dispatch_fused(*prob) ? 1 : 0;
}

int moe_layout_dispatch(const moe_problem_t* prob, const int32_t* topk_idx,
                        const int32_t* part_of, const moe_layout_t* lay, void* workspace,
                        size_t workspace_bytes, const void* x, void* recv_x, float* recv_scale,
                        const moe_tiles_t* tiles, moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay)) return MOE_ERR_ARG;
  if (tiles && !valid_tiles(prob, tiles)) return MOE_ERR_ARG;
  if (!arr(part_of) || (prob->M > 0 && !arr(topk_idx))) return MOE_ERR_ARG;
  if (prob->M > 0) {
    if (!x || !aligned(x, 16) || !recv_x || !aligned(recv_x, 16)) return MOE_ERR_ARG;
    if (prob->fp8 && (!recv_scale || !aligned(recv_scale, 16))) return MOE_ERR_ARG;
  }
  const size_t need = moe::layout_workspace_bytes(*prob);
  if (!workspace || !aligned(workspace, 16) || workspace_bytes < need) return MOE_ERR_WORKSPACE;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const moe::TileOut t = tile_out(tiles);
  if (moe::layout_dispatch_fused(*prob))
    return cuda_rc(moe::launch_layout_dispatch(*prob, topk_idx, part_of, *lay, x, recv_x,
                                               recv_scale, t, s));
  cudaError_t e = moe::launch_layout(*prob, topk_idx, part_of, *lay, workspace, s, t);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_rc(moe::launch_dispatch(*prob, x, *lay, recv_x, recv_scale, s));
}

size_t moe_expert_tiles_capacity(const moe_problem_t* prob, int32_t block_m) {
  if (!valid_problem(prob) || block_m < 1) return 0;
  return (size_t)moe::expert_tiles_capacity(*prob, block_m);
}

int moe_expert_tiles(const moe_problem_t* prob, const int32_t* part_of, const moe_layout_t* lay,
                     const moe_tiles_t* tiles, moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay) || !arr(part_of)) return MOE_ERR_ARG;
  if (!valid_tiles(prob, tiles)) return MOE_ERR_ARG;
  return cuda_rc(moe::launch_expert_tiles(*prob, part_of, *lay, *tiles,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

int moe_combine(const moe_problem_t* prob, const void* y, const float* topk_weights,
                const moe_layout_t* lay, void* out, moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay)) return MOE_ERR_ARG;
  if (prob->M > 0) {
    if (!y || !aligned(y, 16) || !out || !aligned(out, 16)) return MOE_ERR_ARG;
    if (!arr(topk_weights)) return MOE_ERR_ARG;
  }
  return cuda_rc(moe::launch_combine(*prob, y, topk_weights, *lay, out,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

int moe_combine_partial(const moe_problem_t* prob, const void* y, const float* topk_weights,
                        const moe_layout_t* lay, void* z, moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay) || !prob->dedup) return MOE_ERR_ARG;
  if (prob->M > 0) {
    if (!y || !aligned(y, 16) || !z || !aligned(z, 16)) return MOE_ERR_ARG;
    if (!arr(topk_weights)) return MOE_ERR_ARG;
  }
  return cuda_rc(moe::launch_combine_partial(*prob, y, topk_weights, *lay, z,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

int moe_combine_reduce(const moe_problem_t* prob, const void* z, const moe_layout_t* lay,
                       void* out, moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay) || !prob->dedup) return MOE_ERR_ARG;
  if (prob->M > 0) {
    if (!z || !aligned(z, 16) || !out || !aligned(out, 16)) return MOE_ERR_ARG;
  }
  return cuda_rc(moe::launch_combine_reduce(*prob, z, *lay, out,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

int moe_ep_plan(int32_t world, int32_t rank, int32_t G, const int32_t* part_counts,
                const int32_t* expert_counts, const int32_t* part_of, const moe_ep_plan_t* plan,
                moe_stream_t stream) {
  if (world < 1 || world > MOE_MAX_E_PART || rank < 0 || rank >= world) return MOE_ERR_ARG;
  if (!plan || !arr(part_counts)) return MOE_ERR_ARG;
  if (!arr(plan->send_offset) || !arr(plan->src_offset) || !arr(plan->recv_count) ||
      !arr(plan->recv_offset) || !arr(plan->status))
    return MOE_ERR_ARG;
  if (expert_counts) {
    if (G < 1 || G > MOE_MAX_G || !arr(expert_counts) || !arr(part_of)) return MOE_ERR_ARG;
    if (!arr(plan->recv_expert_count) || !arr(plan->recv_block_offset)) return MOE_ERR_ARG;
  }
  return cuda_rc(moe::launch_ep_plan(world, rank, expert_counts ? G : 0, part_counts,
                                     expert_counts, part_of, *plan,
                                     reinterpret_cast<cudaStream_t>(stream)));
}

// the pointer array and its capacity (the pointers themselves are device
// data, checked by the kernels)
static bool valid_peers(const moe_problem_t* p, const moe_ep_peers_t* peers, bool scales) {
  if (!peers || !peers->rows || !aligned(peers->rows, 8) || peers->capacity < 0) return false;
  if (scales && (!peers->scales || !aligned(peers->scales, 8))) return false;
  (void)p;
  return true;
}

int moe_ep_dispatch(const moe_problem_t* prob, const void* x, const moe_layout_t* lay,
                    const int32_t* send_offset, const moe_ep_peers_t* peers, moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay) || !arr(send_offset)) return MOE_ERR_ARG;
  if (!valid_peers(prob, peers, prob->fp8 != 0)) return MOE_ERR_ARG;
  if (prob->M > 0 && (!x || !aligned(x, 16))) return MOE_ERR_ARG;
  return cuda_rc(moe::launch_ep_dispatch(*prob, x, *lay, send_offset, *peers,
                                         reinterpret_cast<cudaStream_t>(stream)));
}

int moe_ep_combine(const moe_problem_t* prob, const moe_ep_peers_t* y_peers,
                   const float* topk_weights, const moe_layout_t* lay, const int32_t* send_offset,
                   void* out, moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay) || prob->dedup) return MOE_ERR_ARG;
  if (!arr(send_offset) || !valid_peers(prob, y_peers, false)) return MOE_ERR_ARG;
  if (prob->M > 0 && (!out || !aligned(out, 16) || !arr(topk_weights))) return MOE_ERR_ARG;
  return cuda_rc(moe::launch_ep_combine(*prob, *y_peers, topk_weights, *lay, send_offset, out,
                                        reinterpret_cast<cudaStream_t>(stream)));
}

int moe_ep_combine_reduce(const moe_problem_t* prob, const moe_ep_peers_t* z_peers,
                          const moe_layout_t* lay, const int32_t* send_offset, void* out,
                          moe_stream_t stream) {
  if (!valid_problem(prob) || !valid_layout(prob, lay) || !prob->dedup) return MOE_ERR_ARG;
  if (!arr(send_offset) || !valid_peers(prob, z_peers, false)) return MOE_ERR_ARG;
  if (prob->M > 0 && (!out || !aligned(out, 16))) return MOE_ERR_ARG;
  return cuda_rc(moe::launch_ep_reduce(*prob, *z_peers, *lay, send_offset, out,
                                       reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
