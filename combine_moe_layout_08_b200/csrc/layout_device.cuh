// Warp-level building blocks of the routing layout, shared by the tiled
// layout kernels and the one-kernel layout + dispatch of small batches.
#pragma once

#include "moe_device.cuh"

namespace moe {

__device__ __forceinline__ bool valid_part(int p, int E) { return p >= 0 && p < E; }

// One warp: in-place exclusive scan of data[0..n); returns the total.
__device__ __forceinline__ int warp_exclusive_scan(int* data, int n) {
  const int lane = lane_id();
  const int per = (n + kWarp - 1) / kWarp;
  const int beg = min(n, lane * per), end = min(n, beg + per);
  int s = 0;
  for (int i = beg; i < end; ++i) s += data[i];
  int x = s;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  int run = x - s;
  for (int i = beg; i < end; ++i) {
    const int v = data[i];
    data[i] = run;
    run += v;
  }
  return __shfl_sync(kFull, x, kWarp - 1);
}

// One warp: pos[e] = position of expert e in (partition, id) order, the
// experts with an invalid placement last.  kcnt has room for E + 1 ints.
// Reads only the placement map part_s[0..G).
__device__ __forceinline__ void expert_order_warp(const int* part_s, int G, int E, int* pos,
                                                  int* kcnt) {
  const int lane = lane_id();
  for (int k = lane; k <= E; k += kWarp) kcnt[k] = 0;
  __syncwarp();
  const int nbits = key_bits(E + 1);
  const unsigned lt = lanemask_lt();
  for (int c = 0; c < G; c += kWarp) {
    const int e = c + lane;
    int key = -1;
    if (e < G) key = valid_part(part_s[e], E) ? part_s[e] : E;
    const unsigned peers = match_peers(key, nbits);
    const int base = key >= 0 ? kcnt[key] : 0;
    __syncwarp();
    if (key >= 0) {
      pos[e] = base + __popc(peers & lt);  // rank among the experts of its key
      if (lane == __ffs(peers) - 1) kcnt[key] = base + __popc(peers);
    }
    __syncwarp();
  }
  (void)warp_exclusive_scan(kcnt, E + 1);  // start of each key
  __syncwarp();
  for (int e = lane; e < G; e += kWarp) {
    const int key = valid_part(part_s[e], E) ? part_s[e] : E;
    pos[e] += kcnt[key];
  }
  __syncwarp();
}

}  // namespace moe
