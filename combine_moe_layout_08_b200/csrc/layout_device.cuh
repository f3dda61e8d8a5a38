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

// Block-wide version of expert_order_warp: every warp orders 32-expert chunks
// at once.  The lanes of a chunk holding the same key (partition, or E for an
// invalid placement) are ranked with a ballot match; an exclusive scan of the
// per-(key, chunk) counts in key-major order (one warp) gives each (key,
// chunk) its first position.  wcnt has room for (E + 1) * ceil(G / 32) ints
// and must be zero on entry.  Reads only part_s[0..G).  Every thread of the
// block calls it (block barriers inside; pos is complete on return).
template <int kThreads>
__device__ __forceinline__ void expert_order_block(const int* part_s, int G, int E, int* pos,
                                                   int* wcnt) {
  constexpr int kWarps = kThreads / kWarp;
  const int lane = lane_id();
  const int nw = (G + kWarp - 1) / kWarp;
  const int nbits = key_bits(E + 1);
  const unsigned lt = lanemask_lt();
  for (int w = warp_id(); w < nw; w += kWarps) {
    const int e = w * kWarp + lane;
    int key = -1;
    if (e < G) key = valid_part(part_s[e], E) ? part_s[e] : E;
    const unsigned peers = match_peers(key, nbits);
    if (e < G) {
      pos[e] = __popc(peers & lt);  // rank among the chunk's experts of its key
      if (lane == __ffs(peers) - 1) wcnt[key * nw + w] = __popc(peers);
    }
  }
  __syncthreads();
  if (warp_id() == 0) (void)warp_exclusive_scan(wcnt, (E + 1) * nw);
  __syncthreads();
  for (int e = threadIdx.x; e < G; e += kThreads) {
    const int key = valid_part(part_s[e], E) ? part_s[e] : E;
    pos[e] += wcnt[key * nw + e / kWarp];
  }
  __syncthreads();
}

// ---------------------------------------------------------------------------
// grouped-GEMM tile metadata emitted by the layout kernels themselves
// (DeepSpeed PR #8180, "Key points": per-tile -> group map from the offsets,
// on the device): tiles of block_m rows that never straddle two experts,
// numbered in row order.
// ---------------------------------------------------------------------------
struct TileOut {
  int block_m;       // 0: no tiles requested
  int* tile_first;   // [G + 1]
  int* tile_expert;  // [cap]
  int* tile_row;
  int* tile_rows;
};

// One warp: tiles per expert in row order (pos[e] = the expert's position in
// it, rows(e) = its rows) scanned into tscan[pos] = first tile, with
// order[pos] = the expert; returns the number of tiles.  A layout's counts
// sum to at most M * topk, so the total fits an int.
template <class Rows>
__device__ __forceinline__ int tiles_scan_warp(const int* pos, int G, int block_m, Rows rows,
                                               int* tscan, int* order) {
  for (int e = lane_id(); e < G; e += kWarp) {
    const int c = rows(e);
    tscan[pos[e]] = c > 0 ? (c - 1) / block_m + 1 : 0;
    order[pos[e]] = e;
  }
  __syncwarp();
  return warp_exclusive_scan(tscan, G);
}

// Tiles [i0, i1) (this block's share), all threads of the block: each finds
// its expert by binary search in tscan (largest q with tscan[q] <= i) and
// writes expert, first row (row_off(e) + j * block_m) and rows.
template <class RowOff, class Rows>
__device__ __forceinline__ void tiles_write(const TileOut& t, const int* tscan, const int* order,
                                            int G, int i0, int i1, RowOff row_off, Rows rows) {
  for (int i = i0 + (int)threadIdx.x; i < i1; i += (int)blockDim.x) {
    int lo = 0, hi = G - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (tscan[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int e = order[lo];
    const int j = i - tscan[lo];
    t.tile_expert[i] = e;
    t.tile_row[i] = row_off(e) + j * t.block_m;
    t.tile_rows[i] = min(t.block_m, rows(e) - j * t.block_m);
  }
}

// This block's share [i0, i1) of n tiles split over nb blocks.
__device__ __forceinline__ void tiles_share(int n, int b, int nb, int& i0, int& i1) {
  const int per = (n + nb - 1) / nb;
  i0 = min(n, b * per);
  i1 = min(n, i0 + per);
}

}  // namespace moe
