// Routing layout and dispatch permute of a small batch (decode) in ONE
// kernel.  At a few hundred tokens the tiled layout and the dispatch are
// bound by latency, not bandwidth (Triton-distributed issue #117, "Results
// (Latency in us)": M = 2..512 at N = 7168, G = 256, topk = 8), so this
// schedule removes a launch and every inter-block step: each block recomputes
// the whole (small) layout in shared memory from all routing ids, derives the
// rows of its own chunk of T consecutive tokens and copies their rows there.
// No block waits for another.  T = ceil(M / 148) keeps the grid at about one
// block per SM.
//
// Block (b, y) of 512 threads, chunk tokens [t0, t0 + nt), t0 = b * T:
//   1. issues the loads of its slice of x[t0 .. t0 + nt) -- the chunk's rows
//      are contiguous, so thread i holds flat vectors i, i + 512, ... --
//      while the layout is computed;
//   2. stages every routing id and the placement map in shared memory;
//      warp 0 orders the experts by (partition, id) meanwhile;
//   3. counts, per expert, the valid pairs before t0 and from t0 on (with
//      dedup also, per partition, the tokens before t0 and from t0 on);
//   4. scans the expert totals in that order (warp 0) and the partition
//      sizes (warp 1);
//   5. warp 0 walks the chunk's tokens in order with running counters:
//        exp_row[t,k]  = expert_offset[e] + (pairs of e before t)
//                        + (slots k' < k of t with the same expert)
//        disp_row[t,p] = part_offset[p] + (tokens before t holding p)
//   6. copies (bf16) or quantises and copies (fp8) its vectors to the rows;
//   7. if asked, writes its share of the grouped-GEMM tile metadata (warp 1
//      scanned the tiles per expert during step 5).
// Every index is the one the tiled layout gives (stable (partition, expert,
// token, slot) order, dedup rows in (partition, token) order), so results are
// bit-identical to moe_layout followed by moe_dispatch.  Block (0, 0) writes
// the counts, offsets and status word; blocks with y = 0 write their chunk's
// index entries.  Work per block grows with M * topk, so the schedule is
// taken only up to MOE_FUSED_ITEMS routed pairs.
#include <algorithm>

#include "fp8_device.cuh"
#include "layout_device.cuh"
#include "moe_device.cuh"
#include "moe_internal.h"

// Compile-time tuning constant: batches of at most this many routed pairs
// (M * topk) take the one-kernel schedule.
#ifndef MOE_FUSED_ITEMS
#define MOE_FUSED_ITEMS 4096
#endif

namespace moe {
namespace {

constexpr int kFThreads = 512;
constexpr int kMaxFusedItems = 8192;  // the shared-memory plan holds at most this many ids
constexpr int kMaxChunk = 16;         // tokens per block
constexpr int kSMs = 148;
static_assert(MOE_FUSED_ITEMS >= 1 && MOE_FUSED_ITEMS <= kMaxFusedItems, "fused batch limit");
constexpr int kMaxDest = MOE_MAX_E_PART > MOE_MAX_TOPK ? MOE_MAX_E_PART : MOE_MAX_TOPK;

__host__ __device__ constexpr int up4(int x) { return (x + 3) & ~3; }

struct FusedArgs {
  int M, G, topk, E, dedup;
  int N8;   // 16-byte chunks per bf16 row (N / 8)
  int T;    // tokens per block
  const int* __restrict__ idx;      // [M][topk]
  const int* __restrict__ part_of;  // [G]
  const uint4* __restrict__ x;      // [M][N8]
  void* recv;                       // [M*topk][N] bf16 or u8
  float* recv_scale;                // [M*topk][N / 128], fp8 only
  int* expert_count;
  int* expert_offset;
  int* part_count;
  int* part_offset;
  int* exp_row;
  int* disp_token;
  int* disp_row;
  int* exp_to_disp;
  int* status;
  TileOut tiles;  // grouped-GEMM tile metadata (tiles.block_m = 0: none)
};

// shared-memory plan in ints, every array 16-byte aligned
struct FusedSmem {
  int ids, part_s, hb, ha, pos, scan, tscan, order, kcnt, pb, pa, poff, prow, dst, nd, misc, total;
  __host__ __device__ FusedSmem(int n_items, int G, int E) {
    int o = 0;
    ids = o; o += up4(n_items);   // every routing id
    part_s = o; o += up4(G);      // placement map
    hb = o; o += up4(G);          // per expert: valid pairs before the current token
    ha = o; o += up4(G);          // ... from t0 on, then the expert's total
    pos = o; o += up4(G);         // expert -> position in (partition, id) order
    scan = o; o += up4(G);        // expert totals in that order -> exclusive scan
    tscan = o; o += up4(G);       // tiles: first tile per expert in that order
    order = o; o += up4(G);       // tiles: expert at each position of that order
    kcnt = o; o += up4(E + 1);    // scratch of the expert order
    pb = o; o += up4(E);          // dedup: tokens before the current token holding p
    pa = o; o += up4(E);          // ... from t0 on (without dedup: rows); then the total
    poff = o; o += up4(E + 1);    // partition offsets
    prow = o; o += up4(E);        // dedup: the current token's row per partition (-1: none)
    dst = o; o += kMaxChunk * kMaxDest;  // destination rows of each chunk token
    nd = o; o += kMaxChunk;              // ... and their number
    misc = o; o += 4;             // [bad expert, bad placement, R_exp, number of tiles]
    total = o;
  }
};

// Units: bf16 16-byte chunks, or fp8 16-column groups (two chunks, one lane
// of an 8-lane scale block).  Block (b, y) owns flat units
// [y * 512 * U, (y + 1) * 512 * U) of its chunk's nt * units.
template <bool FP8, int U>
__global__ void __launch_bounds__(kFThreads, 1) layout_dispatch_kernel(FusedArgs a) {
  extern __shared__ __align__(16) int sm[];
  const int n_items = a.M * a.topk;
  const FusedSmem P(n_items, a.G, a.E);
  int* ids = sm + P.ids;
  int* part_s = sm + P.part_s;
  int* hb = sm + P.hb;
  int* ha = sm + P.ha;
  int* pos = sm + P.pos;
  int* scan = sm + P.scan;
  int* pb = sm + P.pb;
  int* pa = sm + P.pa;
  int* poff = sm + P.poff;
  int* misc = sm + P.misc;
  const int tid = threadIdx.x;
  const int G = a.G, E = a.E, topk = a.topk;
  const int t0 = blockIdx.x * a.T;
  const int nt = min(a.T, a.M - t0);
  const int i0 = t0 * topk;  // first routed pair of the chunk
  const bool writer = blockIdx.y == 0;
  pdl_wait();
  pdl_trigger();

  // 1. this block's units of the chunk, in flight while the layout is computed
  const int units = FP8 ? (a.N8 >> 1) : a.N8;
  const int V = nt * units;
  const uint4* src = a.x + (size_t)t0 * a.N8;
  const int v0 = blockIdx.y * (kFThreads * U) + tid;
  uint4 lo[U], hi[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int v = v0 + u * kFThreads;
    lo[u] = make_uint4(0, 0, 0, 0);
    hi[u] = lo[u];
    if (v < V) {
      if (FP8) {
        lo[u] = ld_nc_v4(src + 2 * (size_t)v);
        hi[u] = ld_nc_v4(src + 2 * (size_t)v + 1);
      } else {
        lo[u] = ld_nc_v4(src + v);
      }
    }
  }

  // 2. warp 0: the placement map and the expert order (which needs nothing
  // else); warps 1..: the routing ids and the zeroed counters
  if (warp_id() == 0) {
    for (int e = lane_id(); e < G; e += kWarp) part_s[e] = __ldg(a.part_of + e);
    __syncwarp();
    expert_order_warp(part_s, G, E, pos, sm + P.kcnt);
  } else {
    constexpr int kRest = kFThreads - kWarp;
    const int r = tid - kWarp;
    if ((reinterpret_cast<uintptr_t>(a.idx) & 15) == 0) {
      const int n4 = n_items >> 2;
      const int4* s4 = reinterpret_cast<const int4*>(a.idx);
      int4* k4 = reinterpret_cast<int4*>(ids);
      for (int i = r; i < n4; i += kRest) k4[i] = __ldg(s4 + i);
      for (int i = (n4 << 2) + r; i < n_items; i += kRest) ids[i] = __ldg(a.idx + i);
    } else {
      for (int i = r; i < n_items; i += kRest) ids[i] = __ldg(a.idx + i);
    }
    for (int e = r; e < G; e += kRest) {
      hb[e] = 0;
      ha[e] = 0;
    }
    for (int p = r; p < E; p += kRest) {
      pb[p] = 0;
      pa[p] = 0;
    }
    if (r < 4) misc[r] = 0;
  }
  __syncthreads();

  // 3. counts before / from t0; invalid input
  bool bad = false;
  for (int i = tid; i < n_items; i += kFThreads) {
    const int e = ids[i];
    if (e >= 0 && e < G) {
      if (valid_part(part_s[e], E)) atomicAdd(i < i0 ? &hb[e] : &ha[e], 1);
    } else {
      bad = true;
    }
  }
  if (bad) atomicOr(&misc[0], 1);
  bool badp = false;
  for (int e = tid; e < G; e += kFThreads) badp |= !valid_part(part_s[e], E);
  if (badp) atomicOr(&misc[1], 1);
  if (a.dedup) {
    const int lane = lane_id();
    for (int base = 0; base < a.M; base += kFThreads) {
      const int tt = base + tid;
      unsigned long long mask = 0ull;
      if (tt < a.M) {
        for (int k = 0; k < topk; ++k) {
          const int e = ids[tt * topk + k];
          if (e >= 0 && e < G && valid_part(part_s[e], E)) mask |= 1ull << part_s[e];
        }
      }
      const bool before = tt < t0;
      for (int p = 0; p < E; ++p) {
        const bool has = (mask >> p) & 1ull;
        const unsigned bb = __ballot_sync(kFull, has && before);
        const unsigned ba = __ballot_sync(kFull, has && !before);
        if (lane == 0) {
          if (bb) atomicAdd(&pb[p], __popc(bb));
          if (ba) atomicAdd(&pa[p], __popc(ba));
        }
      }
    }
  }
  __syncthreads();

  // 4. expert totals (into ha) in (partition, id) order; rows per partition
  for (int e = tid; e < G; e += kFThreads) {
    const int tot = hb[e] + ha[e];
    ha[e] = tot;
    scan[pos[e]] = tot;
    if (!a.dedup && tot && valid_part(part_s[e], E)) atomicAdd(&pa[part_s[e]], tot);
  }
  __syncthreads();
  if (warp_id() == 0) {
    const int R_exp = warp_exclusive_scan(scan, G);
    if (lane_id() == 0) misc[2] = R_exp;
  } else if (warp_id() == 1) {  // partition totals (into pa) and offsets
    for (int p = lane_id(); p < E; p += kWarp) {
      const int tot = pb[p] + pa[p];
      pa[p] = tot;
      poff[p] = tot;
    }
    __syncwarp();
    const int R_disp = warp_exclusive_scan(poff, E);
    if (lane_id() == 0) poff[E] = R_disp;
  }
  __syncthreads();

  // 5. the chunk's rows, token by token (warp 0; hb and pb become running
  // counters); the tiles per expert (warp 1); the batch's counts and offsets
  // (block (0, 0))
  if (warp_id() == 1 && a.tiles.block_m > 0) {
    const int n = tiles_scan_warp(pos, G, a.tiles.block_m, [&](int e) { return ha[e]; },
                                  sm + P.tscan, sm + P.order);
    if (lane_id() == 0) misc[3] = n;
  }
  if (warp_id() == 0) {
    int* prow = sm + P.prow;
    const int lane = lane_id();
    const unsigned lt = lanemask_lt();
    for (int j = 0; j < nt; ++j) {
      const int t = t0 + j;
      const int* tid_ids = ids + t * topk;
      int* dst = sm + P.dst + j * kMaxDest;
      int nd = 0;
      if (a.dedup) {  // one row per partition holding any of t's experts, in partition order
        for (int base = 0; base < E; base += kWarp) {
          const int p = base + lane;
          bool has = false;
          if (p < E) {
            for (int k = 0; k < topk; ++k) {
              const int e = tid_ids[k];
              has |= e >= 0 && e < G && part_s[e] == p;
            }
            const int row = has ? poff[p] + pb[p] : -1;
            prow[p] = row;
            pb[p] += has;
            if (writer) {
              a.disp_row[(size_t)t * E + p] = row;
              if (has) a.disp_token[row] = t;
            }
          }
          const unsigned bal = __ballot_sync(kFull, has);
          if (has) dst[nd + __popc(bal & lt)] = prow[p];
          nd += __popc(bal);
        }
        __syncwarp();
      }
      for (int base = 0; base < topk; base += kWarp) {  // one row per valid slot
        const int k = base + lane;
        int row = -1, e = -1;
        if (k < topk) {
          e = tid_ids[k];
          if (e >= 0 && e < G && valid_part(part_s[e], E)) {
            int dup = 0;
            for (int q = 0; q < k; ++q) dup += tid_ids[q] == e;
            row = scan[pos[e]] + hb[e] + dup;
          }
          if (writer) {
            a.exp_row[(size_t)t * topk + k] = row;
            if (row >= 0) {
              if (a.dedup)
                a.exp_to_disp[row] = prow[part_s[e]];
              else
                a.disp_token[row] = t;
            }
          }
        }
        if (!a.dedup) {
          const unsigned bal = __ballot_sync(kFull, row >= 0);
          if (row >= 0) dst[nd + __popc(bal & lt)] = row;
          nd += __popc(bal);
        }
        __syncwarp();
        if (row >= 0) atomicAdd(&hb[e], 1);  // after every lane of this pass has read hb
        __syncwarp();
      }
      if (lane == 0) sm[P.nd + j] = nd;
      __syncwarp();
    }
  }
  if (blockIdx.x == 0 && writer) {
    for (int e = tid; e < G; e += kFThreads) {
      a.expert_count[e] = ha[e];
      a.expert_offset[e] = scan[pos[e]];
    }
    for (int p = tid; p < E; p += kFThreads) {
      a.part_count[p] = pa[p];
      a.part_offset[p] = poff[p];
    }
    if (tid == 0) {
      a.expert_offset[G] = misc[2];
      a.part_offset[E] = poff[E];
      *a.status = (misc[0] ? MOE_STATUS_BAD_EXPERT : 0) | (misc[1] ? MOE_STATUS_BAD_PART : 0);
    }
  }
  __syncthreads();

  // 6. copy (bf16) or quantise once and copy (fp8) each unit to its token's rows
  const int* dst_all = sm + P.dst;
  const int* nd_all = sm + P.nd;
  uint4* recv = static_cast<uint4*>(a.recv);  // rows of `units` 16-byte chunks
  if (!FP8) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * kFThreads;
      if (v < V) {
        const int j = v / units, c = v - j * units;
        const int* dst = dst_all + j * kMaxDest;
        for (int d = 0; d < nd_all[j]; ++d) st_v4(recv + (size_t)dst[d] * units + c, lo[u]);
      }
    }
  } else {
    const int N128 = units >> 3;
    const bool scale_lane = (tid & 7) == 0;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float s;
      const uint4 q = quantize_lane(lo[u], hi[u], s);  // every lane: the amax uses shuffles
      const int v = v0 + u * kFThreads;
      if (v < V) {
        const int j = v / units, c = v - j * units;
        const int* dst = dst_all + j * kMaxDest;
        for (int d = 0; d < nd_all[j]; ++d) {
          const size_t r = (size_t)dst[d];
          st_v4(recv + r * units + c, q);
          if (scale_lane) a.recv_scale[r * N128 + (c >> 3)] = s;
        }
      }
    }
  }
  // 7. this block's share of the tiles; block (0, 0): each expert's first tile
  if (a.tiles.block_m > 0 && writer) {
    const int* tscan = sm + P.tscan;
    const int n = misc[3];
    if (blockIdx.x == 0) {
      for (int e = tid; e < G; e += kFThreads) a.tiles.tile_first[e] = tscan[pos[e]];
      if (tid == 0) a.tiles.tile_first[G] = n;
    }
    int k0, k1;
    tiles_share(n, blockIdx.x, gridDim.x, k0, k1);
    tiles_write(a.tiles, tscan, sm + P.order, G, k0, k1, [&](int e) { return scan[pos[e]]; },
                [&](int e) { return ha[e]; });
  }
}

template <bool FP8, int U>
cudaError_t launch_u(const FusedArgs& a, dim3 grid, size_t smem, cudaStream_t stream) {
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(layout_dispatch_kernel<FP8, U>), smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(layout_dispatch_kernel<FP8, U>, grid, dim3(kFThreads), smem, stream, a);
}

}  // namespace

bool layout_dispatch_fused(const moe_problem_t& p) {
  return p.M >= 1 && (int64_t)p.M * p.topk <= MOE_FUSED_ITEMS;
}

cudaError_t launch_layout_dispatch(const moe_problem_t& p, const int32_t* topk_idx,
                                   const int32_t* part_of, const moe_layout_t& lay,
                                   const void* x, void* recv_x, float* recv_scale,
                                   const TileOut& tiles, cudaStream_t stream) {
  FusedArgs a;
  a.M = p.M;
  a.G = p.G;
  a.topk = p.topk;
  a.E = p.E_part;
  a.dedup = p.dedup;
  a.N8 = p.N / 8;
  a.idx = topk_idx;
  a.part_of = part_of;
  a.x = static_cast<const uint4*>(x);
  a.recv = recv_x;
  a.recv_scale = recv_scale;
  a.expert_count = lay.expert_count;
  a.expert_offset = lay.expert_offset;
  a.part_count = lay.part_count;
  a.part_offset = lay.part_offset;
  a.exp_row = lay.exp_row;
  a.disp_token = lay.disp_token;
  a.disp_row = lay.disp_row;
  a.exp_to_disp = lay.exp_to_disp;
  a.status = lay.status;
  a.tiles = tiles;

  a.T = std::min(kMaxChunk, (p.M + kSMs - 1) / kSMs);
  const int blocks = (p.M + a.T - 1) / a.T;
  const size_t smem = sizeof(int) * (size_t)FusedSmem(p.M * p.topk, p.G, p.E_part).total;
  const int units = p.fp8 ? a.N8 / 2 : a.N8;
  const int V = a.T * units;  // units of a full chunk
  const int Umax = p.fp8 ? 4 : 8;
  const int U = std::min(Umax, (V + kFThreads - 1) / kFThreads);
  const int per_block = kFThreads * U;
  const dim3 grid(blocks, (V + per_block - 1) / per_block);
  cudaError_t e;
  if (!p.fp8) {
    switch (U) {
      case 1: e = launch_u<false, 1>(a, grid, smem, stream); break;
      case 2: e = launch_u<false, 2>(a, grid, smem, stream); break;
      case 3: e = launch_u<false, 3>(a, grid, smem, stream); break;
      case 4: e = launch_u<false, 4>(a, grid, smem, stream); break;
      case 5: e = launch_u<false, 5>(a, grid, smem, stream); break;
      case 6: e = launch_u<false, 6>(a, grid, smem, stream); break;
      case 7: e = launch_u<false, 7>(a, grid, smem, stream); break;
      default: e = launch_u<false, 8>(a, grid, smem, stream); break;
    }
  } else {
    switch (U) {
      case 1: e = launch_u<true, 1>(a, grid, smem, stream); break;
      case 2: e = launch_u<true, 2>(a, grid, smem, stream); break;
      case 3: e = launch_u<true, 3>(a, grid, smem, stream); break;
      default: e = launch_u<true, 4>(a, grid, smem, stream); break;
    }
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
