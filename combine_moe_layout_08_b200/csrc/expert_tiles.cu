// Grouped-GEMM tile metadata of a layout, on the device: a grouped GEMM over
// the expert rows maps each of its row tiles to an expert without a
// device -> host copy of the offsets (DeepSpeed PR #8180, "Key points":
// per-tile -> group mapping computed on device from offs).
//
// Tiles hold block_m rows and never straddle two experts; expert e owns
// ceil(expert_count[e] / block_m) of them and tiles are numbered in row
// order, i.e. in the (partition, id) order of the experts that the layout
// gives the rows.  One block of 1024 threads:
//   1. warp 0 orders the experts by (partition, id) from the placement map
//      (the layout's own order); the other warps read the counts;
//   2. the tiles per expert are scanned in that order (64-bit, so that even
//      inconsistent counts cannot overflow) -> tile_first[e], total;
//   3. tile i (all threads, strided) finds its expert by binary search in the
//      scan and writes expert, first row and rows.
// The tile arrays hold max_tiles = ceil(M * topk / block_m) + G entries, the
// most a consistent layout needs; a larger total (counts that do not come
// from a layout of this problem) writes only max_tiles tiles and raises
// MOE_STATUS_BAD_ROW.
#include <climits>

#include "layout_device.cuh"
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kXThreads = 1024;

struct TilesArgs {
  int G, E, block_m;
  long long max_tiles;
  const int* __restrict__ part_of;
  const int* expert_count;
  const int* expert_offset;
  int* tile_first;   // [G + 1]
  int* tile_expert;  // [max_tiles]
  int* tile_row;
  int* tile_rows;
  int* status;
};

// One warp: in-place exclusive scan of data[0..n) in 64 bits; returns the total.
__device__ long long warp_exclusive_scan64(long long* data, int n) {
  const int lane = lane_id();
  const int per = (n + kWarp - 1) / kWarp;
  const int beg = min(n, lane * per), end = min(n, beg + per);
  long long s = 0;
  for (int i = beg; i < end; ++i) s += data[i];
  long long x = s;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const long long y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  long long run = x - s;
  for (int i = beg; i < end; ++i) {
    const long long v = data[i];
    data[i] = run;
    run += v;
  }
  return __shfl_sync(kFull, x, kWarp - 1);
}

__global__ void __launch_bounds__(kXThreads, 1) expert_tiles_kernel(TilesArgs a) {
  __shared__ int part_s[MOE_MAX_G];
  __shared__ int pos[MOE_MAX_G];
  __shared__ int order[MOE_MAX_G];
  __shared__ long long scan[MOE_MAX_G];
  __shared__ int kcnt[MOE_MAX_E_PART + 1];
  __shared__ long long total_s;
  const int tid = threadIdx.x, G = a.G;
  pdl_wait();
  pdl_trigger();
  if (warp_id() == 0) {
    for (int e = lane_id(); e < G; e += kWarp) part_s[e] = __ldg(a.part_of + e);
    __syncwarp();
    expert_order_warp(part_s, G, a.E, pos, kcnt);
  }
  long long n[(MOE_MAX_G + kXThreads - 1) / kXThreads];
#pragma unroll
  for (int j = 0; j < (MOE_MAX_G + kXThreads - 1) / kXThreads; ++j) {
    const int e = tid + j * kXThreads;
    const int c = e < G ? a.expert_count[e] : 0;
    n[j] = c > 0 ? ((long long)c + a.block_m - 1) / a.block_m : 0;
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < (MOE_MAX_G + kXThreads - 1) / kXThreads; ++j) {
    const int e = tid + j * kXThreads;
    if (e < G) {
      scan[pos[e]] = n[j];
      order[pos[e]] = e;
    }
  }
  __syncthreads();
  if (warp_id() == 0) {
    const long long total = warp_exclusive_scan64(scan, G);
    if (lane_id() == 0) total_s = total;
  }
  __syncthreads();
  const long long total = total_s;
  for (int e = tid; e < G; e += kXThreads) a.tile_first[e] = (int)min(scan[pos[e]], (long long)INT_MAX);
  if (tid == 0) {
    a.tile_first[G] = (int)min(total, (long long)INT_MAX);
    if (total > a.max_tiles) raise_status(a.status, MOE_STATUS_BAD_ROW);
  }
  const long long n_write = min(total, a.max_tiles);
  for (long long i = tid; i < n_write; i += kXThreads) {
    int lo = 0, hi = G - 1;  // largest q with scan[q] <= i (its expert has a tile there)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (scan[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int e = order[lo];
    const long long j = i - scan[lo];
    const long long rest = (long long)a.expert_count[e] - j * a.block_m;
    a.tile_expert[i] = e;
    a.tile_row[i] = (int)((long long)a.expert_offset[e] + j * a.block_m);
    a.tile_rows[i] = (int)min(rest, (long long)a.block_m);
  }
}

}  // namespace

int64_t expert_tiles_capacity(const moe_problem_t& p, int block_m) {
  return ((int64_t)p.M * p.topk + block_m - 1) / block_m + p.G;
}

cudaError_t launch_expert_tiles(const moe_problem_t& p, const int32_t* part_of,
                                const moe_layout_t& lay, const moe_tiles_t& tiles,
                                cudaStream_t stream) {
  TilesArgs a;
  a.G = p.G;
  a.E = p.E_part;
  a.block_m = tiles.block_m;
  a.max_tiles = expert_tiles_capacity(p, tiles.block_m);
  a.part_of = part_of;
  a.expert_count = lay.expert_count;
  a.expert_offset = lay.expert_offset;
  a.tile_first = tiles.tile_first;
  a.tile_expert = tiles.tile_expert;
  a.tile_row = tiles.tile_row;
  a.tile_rows = tiles.tile_rows;
  a.status = lay.status;
  cudaError_t e = launch_pdl(expert_tiles_kernel, dim3(1), dim3(kXThreads), 0, stream, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
