// Routing layout on the device: per-expert / per-partition counts, their
// prefix sums and the stable row index of every routed (token, slot) pair.
//
// Split counts and their cumulative sum are what an all-to-all dispatch
// consumes (Triton-distributed issue #117, test snippet: split_send_buf,
// send_split_cumsum); the receive side is a scattered-V buffer, contiguous
// variable-sized partitions indexed by destination (Purlin, section 3.1
// "Layouts").  With dedup a token owns one dispatch row per partition that
// holds any of its experts (Zyphra news item, correlated expert placement).
//
// The routed pairs are cut into tiles of consecutive tokens.  A tile's rows
// of expert e start at  expert_offset[e] + (rows of e in earlier tiles), and
// inside the tile they are ranked stably in (token, slot) order: each warp
// counts its contiguous segment into a warp-private histogram, an exclusive
// scan across warps gives each warp's base, and a ballot match (one vote per key
// bit) ranks the lanes of a 32-pair chunk.  Everything is fixed by the data, so the result is
// bitwise reproducible.
//
// Two schedules, no host round trip in either:
//   * up to kClusterItems routed pairs (decode-sized batches): ONE launch of
//     a cluster of kClusterCTAs blocks.  Each block counts its tile into shared memory,
//     the blocks exchange their tile histograms through distributed shared
//     memory between two hardware cluster barriers, and every block finishes
//     its own tile.  No workspace is touched.
//   * larger batches: one tile per SM in two launches -- layout_count_kernel
//     writes per-tile histograms to the workspace, layout_rank_kernel reduces
//     them (batched 16-byte loads from L2) and ranks its tile.
// In both, the tile's expert ids are cached in shared memory when they fit.
#include <cooperative_groups.h>

#include <algorithm>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace cg = cooperative_groups;

namespace moe {
namespace {

constexpr int kLThreads = 512;
constexpr int kLWarps = kLThreads / kWarp;
constexpr int kClusterCTAs = 8;
constexpr int kMaxTileItems = 16384;  // tile ids cached in shared memory (64 KB)
// Compile-time tuning constants: batches of at most MOE_CLUSTER_ITEMS routed
// pairs take the one-cluster schedule; tiles of the two-launch schedule hold
// at least MOE_TILE_MIN_TOKENS tokens.
#ifndef MOE_CLUSTER_ITEMS
#define MOE_CLUSTER_ITEMS 8192  // measured on B200: one cluster wins only for small batches
#endif
#ifndef MOE_TILE_MIN_TOKENS
#define MOE_TILE_MIN_TOKENS 64
#endif
constexpr int kClusterItems = MOE_CLUSTER_ITEMS;
static_assert(kClusterItems <= kClusterCTAs * kMaxTileItems, "cluster tiles must fit the id cache");
// width of each half of the column-sum reduction buffer: one slot per thread
// and 4 columns per slot (>= MOE_MAX_G, the widest matrix reduced)
constexpr int kRedW = 4 * kLThreads;
static_assert(kRedW >= MOE_MAX_G, "reduction buffer narrower than the expert count");

struct LayoutArgs {
  int M, G, topk, E, dedup;
  int T;        // tokens per tile
  int n_tiles;  // tiles (= blocks)
  int key_cap;  // ids the shared-memory cache holds (0: read from global)
  const int* __restrict__ idx;
  const int* __restrict__ part_of;
  int* tile_hist;   // [n_tiles][G]   (two-launch schedule)
  int* tile_phist;  // [n_tiles][E]   (two-launch schedule, dedup)
  int* tile_flags;  // [n_tiles]      (two-launch schedule)
  int* expert_count;
  int* expert_offset;
  int* part_count;
  int* part_offset;
  int* exp_row;
  int* disp_token;
  int* disp_row;
  int* exp_to_disp;
  int* status;
};

__device__ __forceinline__ bool valid_part(int p, int E) { return p >= 0 && p < E; }

struct Tile {
  int t0, ntok, n_items;
};

__device__ __forceinline__ Tile tile_of(const LayoutArgs& a, int b) {
  Tile t;
  t.t0 = b * a.T;
  t.ntok = max(0, min(a.M - t.t0, a.T));
  t.n_items = t.ntok * a.topk;
  return t;
}

// ---------------------------------------------------------------------------
// shared-memory plan (ints, every array 16-byte aligned)
// ---------------------------------------------------------------------------
struct LayoutSmem {
  int part_s, tot, pre, eoff, pos, scanbuf, cta_hist, red, whist, ewhist, keycnt, keystart, pc,
      poff, ptot, ppre, pbase, cta_phist, wp, warp_tot, misc, keys, total;
  __host__ __device__ static int up4(int x) { return (x + 3) & ~3; }
  __host__ __device__ LayoutSmem(int G, int E, int key_cap) {
    const int RW = kRedW;
    int o = 0;
    part_s = o; o += up4(G);
    tot = o; o += up4(G);
    pre = o; o += up4(G);
    eoff = o; o += up4(G);
    pos = o; o += up4(G);
    scanbuf = o; o += up4(G);
    cta_hist = o; o += up4(G);
    red = o; o += up4(2 * RW);
    whist = o; o += up4(kLWarps * G);
    ewhist = o; o += up4(kLWarps * (E + 1));
    keycnt = o; o += up4(E + 1);
    keystart = o; o += up4(E + 1);
    pc = o; o += up4(E);
    poff = o; o += up4(E + 1);
    ptot = o; o += up4(E);
    ppre = o; o += up4(E);
    pbase = o; o += up4(E);
    cta_phist = o; o += up4(E);
    wp = o; o += up4(kLWarps * E);
    warp_tot = o; o += up4(kLWarps);
    misc = o; o += 4;
    keys = o; o += up4(key_cap);
    total = o;
  }
};

struct Smem {
  int *part_s, *tot, *pre, *eoff, *pos, *scanbuf, *cta_hist, *red, *whist, *ewhist, *keycnt,
      *keystart, *pc, *poff, *ptot, *ppre, *pbase, *cta_phist, *wp, *warp_tot, *misc, *keys;
  __device__ Smem(int* sm, const LayoutSmem& P)
      : part_s(sm + P.part_s), tot(sm + P.tot), pre(sm + P.pre), eoff(sm + P.eoff),
        pos(sm + P.pos), scanbuf(sm + P.scanbuf), cta_hist(sm + P.cta_hist), red(sm + P.red),
        whist(sm + P.whist), ewhist(sm + P.ewhist), keycnt(sm + P.keycnt),
        keystart(sm + P.keystart), pc(sm + P.pc), poff(sm + P.poff), ptot(sm + P.ptot),
        ppre(sm + P.ppre), pbase(sm + P.pbase), cta_phist(sm + P.cta_phist), wp(sm + P.wp),
        warp_tot(sm + P.warp_tot), misc(sm + P.misc), keys(sm + P.keys) {}
};

// ---------------------------------------------------------------------------
// block-wide building blocks
// ---------------------------------------------------------------------------

// Expert id of tile pair i (shared-memory cache or global).
struct RawIds {
  const int* g;  // tile base in global memory
  const int* s;  // shared-memory cache or nullptr
  __device__ __forceinline__ int operator()(int i) const { return s ? s[i] : __ldg(g + i); }
};

// Fill the shared-memory cache of the tile's ids (16-byte loads when aligned),
// zero the block's scratch and load the placement map.  Ends with a barrier.
__device__ void stage_tile(const LayoutArgs& a, const Tile& tl, const Smem& S, RawIds& ids) {
  const int tid = threadIdx.x;
  const int* src = a.idx + (size_t)tl.t0 * a.topk;
  ids.g = src;
  ids.s = nullptr;
  if (tl.n_items <= a.key_cap) {
    ids.s = S.keys;
    const int n = tl.n_items;
    if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
      const int n4 = n >> 2;
      const int4* s4 = reinterpret_cast<const int4*>(src);
      int4* k4 = reinterpret_cast<int4*>(S.keys);
#pragma unroll 4
      for (int i = tid; i < n4; i += kLThreads) k4[i] = __ldg(s4 + i);
      for (int i = (n4 << 2) + tid; i < n; i += kLThreads) S.keys[i] = __ldg(src + i);
    } else {
#pragma unroll 4
      for (int i = tid; i < n; i += kLThreads) S.keys[i] = __ldg(src + i);
    }
  }
  for (int e = tid; e < a.G; e += kLThreads) S.part_s[e] = __ldg(a.part_of + e);
  for (int i = tid; i < kLWarps * a.G; i += kLThreads) S.whist[i] = 0;
  for (int i = tid; i < kLWarps * (a.E + 1); i += kLThreads) S.ewhist[i] = 0;
  for (int p = tid; p < a.E; p += kLThreads) {
    S.pc[p] = 0;
    S.pbase[p] = 0;
    S.cta_phist[p] = 0;
  }
  if (tid < 4) S.misc[tid] = 0;
  __syncthreads();
}

// Status bits of the tile (bad expert ids; block `first` also checks the map).
__device__ int scan_flags(const LayoutArgs& a, const Tile& tl, const Smem& S, const RawIds& ids,
                          bool first) {
  int f = 0;
  for (int i = threadIdx.x; i < tl.n_items; i += kLThreads) {
    const int e = ids(i);
    if (e < 0 || e >= a.G) f |= MOE_STATUS_BAD_EXPERT;
  }
  if (first)
    for (int e = threadIdx.x; e < a.G; e += kLThreads)
      if (!valid_part(S.part_s[e], a.E)) f |= MOE_STATUS_BAD_PART;
  return f;
}

// Per-warp counts of the keys of [0, n) (warp w owns the w-th contiguous
// segment), then an exclusive scan across warps: on return whist[w*K + k]
// is the number of elements with key k in segments before w, and
// key_count[k] (if given) the total.  whist must be zero on entry.
template <class KeyOf>
__device__ void rank_count(int n, int K, int* whist, int* key_count, KeyOf key_of) {
  const int lane = lane_id(), warp = warp_id();
  const int seg = (n + kLWarps - 1) / kLWarps;
  const int beg = min(n, warp * seg), end = min(n, beg + seg);
  const int nbits = key_bits(K);
  int* wh = whist + warp * K;
  for (int c = beg; c < end; c += kWarp) {
    const int i = c + lane;
    const int key = i < end ? key_of(i) : -1;
    const unsigned peers = match_peers(key, nbits);
    if (key >= 0 && lane == __ffs(peers) - 1) wh[key] += __popc(peers);
    __syncwarp();
  }
  __syncthreads();
  for (int key = threadIdx.x; key < K; key += kLThreads) {
    int v[kLWarps];
#pragma unroll
    for (int w = 0; w < kLWarps; ++w) v[w] = whist[w * K + key];
    int run = 0;
#pragma unroll
    for (int w = 0; w < kLWarps; ++w) {
      whist[w * K + key] = run;
      run += v[w];
    }
    if (key_count) key_count[key] = run;
  }
  __syncthreads();
}

// Second pass of the stable rank: on_rank(i, key, rank) with rank = number of
// elements j < i with the same key; on_skip(i) for keys < 0.
template <class KeyOf, class OnRank, class OnSkip>
__device__ void rank_assign(int n, int K, int* whist, KeyOf key_of, OnRank on_rank,
                            OnSkip on_skip) {
  const int lane = lane_id(), warp = warp_id();
  const int seg = (n + kLWarps - 1) / kLWarps;
  const int beg = min(n, warp * seg), end = min(n, beg + seg);
  int* wh = whist + warp * K;
  const unsigned lt = lanemask_lt();
  const int nbits = key_bits(K);
  for (int c = beg; c < end; c += kWarp) {
    const int i = c + lane;
    const int key = i < end ? key_of(i) : -1;
    const unsigned peers = match_peers(key, nbits);
    const int base = key >= 0 ? wh[key] : 0;
    __syncwarp();
    if (key >= 0) {
      on_rank(i, key, base + __popc(peers & lt));
      if (lane == __ffs(peers) - 1) wh[key] = base + __popc(peers);
    } else if (i < end) {
      on_skip(i);
    }
    __syncwarp();
  }
  __syncthreads();
}

// In-place exclusive scan of data[0..n) in shared memory; returns the total.
__device__ int block_exclusive_scan(int* data, int n, int* warp_tot) {
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  const int ipt = (n + kLThreads - 1) / kLThreads;
  const int beg = min(n, tid * ipt), end = min(n, beg + ipt);
  int s = 0;
  for (int i = beg; i < end; ++i) s += data[i];
  int x = s;
#pragma unroll
  for (int o = 1; o < kWarp; o <<= 1) {
    const int y = __shfl_up_sync(kFull, x, o);
    if (lane >= o) x += y;
  }
  if (lane == kWarp - 1) warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int v = lane < kLWarps ? warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < kWarp; o <<= 1) {
      const int y = __shfl_up_sync(kFull, v, o);
      if (lane >= o) v += y;
    }
    if (lane < kLWarps) warp_tot[lane] = v;
  }
  __syncthreads();
  int run = x - s + (warp > 0 ? warp_tot[warp - 1] : 0);
  for (int i = beg; i < end; ++i) {
    const int v = data[i];
    data[i] = run;
    run += v;
  }
  const int total = warp_tot[kLWarps - 1];
  __syncthreads();
  return total;
}

// Partition bit mask of token tl of the tile (valid pairs only).
__device__ __forceinline__ unsigned long long token_mask(const LayoutArgs& a, const RawIds& ids,
                                                        const int* part_s, int tl) {
  unsigned long long mask = 0ull;
  for (int k = 0; k < a.topk; ++k) {
    const int e = ids(tl * a.topk + k);
    if (e >= 0 && e < a.G) {
      const int p = part_s[e];
      if (valid_part(p, a.E)) mask |= 1ull << p;
    }
  }
  return mask;
}

// dedup: tokens of the tile holding partition p, into cta_phist[p]
__device__ void count_tile_parts(const LayoutArgs& a, const Tile& tl, const Smem& S,
                                 const RawIds& ids) {
  const int lane = lane_id();
  for (int r0 = 0; r0 < tl.ntok; r0 += kLThreads) {
    const int t = r0 + threadIdx.x;
    const unsigned long long mask = t < tl.ntok ? token_mask(a, ids, S.part_s, t) : 0ull;
    for (int p = 0; p < a.E; ++p) {
      const unsigned bal = __ballot_sync(kFull, (mask >> p) & 1ull);
      if (lane == 0 && bal) atomicAdd(&S.cta_phist[p], __popc(bal));
    }
  }
  __syncthreads();
}

// expert order (partition, id) -> pos[e]; offsets eoff[e], partition counts
// and offsets.  Needs tot[] (and ptot[] with dedup).  Returns R_exp.
__device__ int finish_offsets(const LayoutArgs& a, const Smem& S) {
  const int G = a.G, E = a.E, tid = threadIdx.x;
  auto ekey = [&](int e) {
    const int p = S.part_s[e];
    return valid_part(p, E) ? p : E;
  };
  rank_count(G, E + 1, S.ewhist, S.keycnt, ekey);
  if (tid == 0) {
    int run = 0;
    for (int k = 0; k <= E; ++k) {
      S.keystart[k] = run;
      run += S.keycnt[k];
    }
  }
  __syncthreads();
  rank_assign(
      G, E + 1, S.ewhist, ekey, [&](int e, int k, int r) { S.pos[e] = S.keystart[k] + r; },
      [](int) {});
  for (int e = tid; e < G; e += kLThreads) S.scanbuf[S.pos[e]] = S.tot[e];
  __syncthreads();
  const int R_exp = block_exclusive_scan(S.scanbuf, G, S.warp_tot);
  for (int e = tid; e < G; e += kLThreads) {
    S.eoff[e] = S.scanbuf[S.pos[e]];
    if (!a.dedup && valid_part(S.part_s[e], E) && S.tot[e]) atomicAdd(&S.pc[S.part_s[e]], S.tot[e]);
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int p = 0; p < E; ++p) {
      if (a.dedup) S.pc[p] = S.ptot[p];
      S.poff[p] = run;
      run += S.pc[p];
    }
    S.poff[E] = run;
  }
  __syncthreads();
  return R_exp;
}

__device__ void write_globals(const LayoutArgs& a, const Smem& S, int R_exp, int flags) {
  for (int e = threadIdx.x; e < a.G; e += kLThreads) {
    a.expert_count[e] = S.tot[e];
    a.expert_offset[e] = S.eoff[e];
  }
  for (int p = threadIdx.x; p < a.E; p += kLThreads) {
    a.part_count[p] = S.pc[p];
    a.part_offset[p] = S.poff[p];
  }
  if (threadIdx.x == 0) {
    a.expert_offset[a.G] = R_exp;
    a.part_offset[a.E] = S.poff[a.E];
    *a.status = flags;
  }
}

// dedup: dispatch row of each distinct (token, partition) of the tile
__device__ void rank_tile_parts(const LayoutArgs& a, const Tile& tl, const Smem& S,
                                const RawIds& ids) {
  const int E = a.E, lane = lane_id(), warp = warp_id(), tid = threadIdx.x;
  const unsigned lt = lanemask_lt();
  for (int r0 = 0; r0 < tl.ntok; r0 += kLThreads) {
    const int t = r0 + tid;
    const unsigned long long mask = t < tl.ntok ? token_mask(a, ids, S.part_s, t) : 0ull;
    for (int p = 0; p < E; ++p) {
      const unsigned bal = __ballot_sync(kFull, (mask >> p) & 1ull);
      if (lane == 0) S.wp[warp * E + p] = __popc(bal);
    }
    __syncthreads();
    for (int p = tid; p < E; p += kLThreads) {
      int run = S.pbase[p];
      for (int w = 0; w < kLWarps; ++w) {
        const int v = S.wp[w * E + p];
        S.wp[w * E + p] = run;
        run += v;
      }
      S.pbase[p] = run;
    }
    __syncthreads();
    const int tg = tl.t0 + t;
    for (int p = 0; p < E; ++p) {
      const bool has = (mask >> p) & 1ull;
      const unsigned bal = __ballot_sync(kFull, has);
      if (t < tl.ntok) {
        int row = -1;
        if (has) {
          row = S.poff[p] + S.ppre[p] + S.wp[warp * E + p] + __popc(bal & lt);
          a.disp_token[row] = tg;
        }
        a.disp_row[(size_t)tg * E + p] = row;
      }
    }
    __syncthreads();
  }
}

// expert row of every pair of the tile (second pass of the stable rank)
__device__ void rank_tile_items(const LayoutArgs& a, const Tile& tl, const Smem& S,
                                const RawIds& ids) {
  const int G = a.G, E = a.E;
  int* exp_row = a.exp_row + (size_t)tl.t0 * a.topk;
  auto ikey = [&](int i) {
    const int e = ids(i);
    return (e >= 0 && e < G && valid_part(S.part_s[e], E)) ? e : -1;
  };
  rank_assign(
      tl.n_items, G, S.whist, ikey,
      [&](int i, int e, int r) {
        const int row = S.eoff[e] + S.pre[e] + r;
        exp_row[i] = row;
        const int t = tl.t0 + i / a.topk;
        if (!a.dedup) {
          a.disp_token[row] = t;
        } else {
          a.exp_to_disp[row] = a.disp_row[(size_t)t * E + S.part_s[e]];
        }
      },
      [&](int i) { exp_row[i] = -1; });
}

__device__ __forceinline__ int item_key(const LayoutArgs& a, const Smem& S, const RawIds& ids,
                                        int i) {
  const int e = ids(i);
  return (e >= 0 && e < a.G && valid_part(S.part_s[e], a.E)) ? e : -1;
}

// ---------------------------------------------------------------------------
// schedule 1: one cluster
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLThreads) layout_cluster_kernel(LayoutArgs a) {
  extern __shared__ __align__(16) int sm[];
  cg::cluster_group cluster = cg::this_cluster();
  const LayoutSmem P(a.G, a.E, a.key_cap);
  const Smem S(sm, P);
  const int r = (int)cluster.block_rank();
  const int tid = threadIdx.x;
  const Tile tl = tile_of(a, r);
  pdl_wait();
  pdl_trigger();
  RawIds ids;
  stage_tile(a, tl, S, ids);

  // count the tile; the per-warp bases stay in whist for the ranks below
  const int f = scan_flags(a, tl, S, ids, r == 0);
  if (f) atomicOr(&S.misc[0], f);
  rank_count(tl.n_items, a.G, S.whist, S.cta_hist, [&](int i) { return item_key(a, S, ids, i); });
  if (a.dedup) count_tile_parts(a, tl, S, ids);
  cluster.sync();

  // exchange: totals over the cluster and the prefix of the tiles before r
  for (int e = tid; e < a.G; e += kLThreads) {
    int v[kClusterCTAs];
#pragma unroll
    for (int q = 0; q < kClusterCTAs; ++q) v[q] = cluster.map_shared_rank(S.cta_hist, q)[e];
    int all = 0, bef = 0;
#pragma unroll
    for (int q = 0; q < kClusterCTAs; ++q) {
      all += v[q];
      bef += q < r ? v[q] : 0;
    }
    S.tot[e] = all;
    S.pre[e] = bef;
  }
  if (a.dedup) {
    for (int p = tid; p < a.E; p += kLThreads) {
      int all = 0, bef = 0;
      for (int q = 0; q < kClusterCTAs; ++q) {
        const int v = cluster.map_shared_rank(S.cta_phist, q)[p];
        all += v;
        bef += q < r ? v : 0;
      }
      S.ptot[p] = all;
      S.ppre[p] = bef;
    }
  }
  int flags = 0;
  if (r == 0 && tid < kClusterCTAs) flags = cluster.map_shared_rank(S.misc, tid)[0];
  __syncthreads();
  if (r == 0 && flags) atomicOr(&S.misc[1], flags);

  const int R_exp = finish_offsets(a, S);
  if (r == 0) write_globals(a, S, R_exp, S.misc[1]);
  if (a.dedup) rank_tile_parts(a, tl, S, ids);
  rank_tile_items(a, tl, S, ids);
  cluster.sync();  // no block leaves while another may still read its histograms
}

// ---------------------------------------------------------------------------
// schedule 2: one tile per SM, two launches
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLThreads) layout_count_kernel(LayoutArgs a) {
  extern __shared__ __align__(16) int sm[];
  const LayoutSmem P(a.G, a.E, a.key_cap);
  const Smem S(sm, P);
  const int b = blockIdx.x;
  const Tile tl = tile_of(a, b);
  pdl_wait();
  pdl_trigger();
  RawIds ids;
  stage_tile(a, tl, S, ids);
  const int f = scan_flags(a, tl, S, ids, b == 0);
  if (f) atomicOr(&S.misc[0], f);
  rank_count(tl.n_items, a.G, S.whist, S.cta_hist, [&](int i) { return item_key(a, S, ids, i); });
  if (a.dedup) count_tile_parts(a, tl, S, ids);
  int* th = a.tile_hist + (size_t)b * a.G;
  for (int i = threadIdx.x; i < a.G; i += kLThreads) th[i] = S.cta_hist[i];
  if (a.dedup)
    for (int i = threadIdx.x; i < a.E; i += kLThreads)
      a.tile_phist[(size_t)b * a.E + i] = S.cta_phist[i];
  if (threadIdx.x == 0) a.tile_flags[b] = S.misc[0];
}

// Column sums of a [rows][cols] int matrix in global memory (L2): total over
// all rows and over rows < b.  Each thread keeps up to 8 16-byte loads in
// flight.  `red` holds 2 * kRedW ints (cols <= MOE_MAX_G <= kRedW).
__device__ void column_sums(const int* src, int rows, int cols, int b, int* red, int* total,
                            int* before) {
  const int tid = threadIdx.x;
  const int RW = kRedW;
  const bool vec = (cols & 3) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
  if (vec) {
    const int C4 = cols >> 2;
    const int S = C4 <= kLThreads ? kLThreads / C4 : 1;
    for (int slot = tid; slot < C4 * S; slot += kLThreads) {
      const int c4 = slot % C4, s = slot / C4;
      int4 all = make_int4(0, 0, 0, 0), bef = all;
#pragma unroll 8
      for (int r = s; r < rows; r += S) {
        const int4 v = __ldcg(reinterpret_cast<const int4*>(src + (size_t)r * cols) + c4);
        all.x += v.x; all.y += v.y; all.z += v.z; all.w += v.w;
        if (r < b) {
          bef.x += v.x; bef.y += v.y; bef.z += v.z; bef.w += v.w;
        }
      }
      const int base = s * cols + 4 * c4;
      red[base] = all.x; red[base + 1] = all.y; red[base + 2] = all.z; red[base + 3] = all.w;
      red[RW + base] = bef.x; red[RW + base + 1] = bef.y;
      red[RW + base + 2] = bef.z; red[RW + base + 3] = bef.w;
    }
    __syncthreads();
    for (int c = tid; c < cols; c += kLThreads) {
      int all = 0, bef = 0;
      for (int s = 0; s < S; ++s) {
        all += red[s * cols + c];
        bef += red[RW + s * cols + c];
      }
      total[c] = all;
      before[c] = bef;
    }
  } else {
    const int S = cols <= kLThreads ? kLThreads / cols : 1;
    for (int slot = tid; slot < cols * S; slot += kLThreads) {
      const int c = slot % cols, s = slot / cols;
      int all = 0, bef = 0;
#pragma unroll 8
      for (int r = s; r < rows; r += S) {
        const int v = __ldcg(src + (size_t)r * cols + c);
        all += v;
        bef += (r < b) ? v : 0;
      }
      red[slot] = all;
      red[RW + slot] = bef;
    }
    __syncthreads();
    for (int c = tid; c < cols; c += kLThreads) {
      int all = 0, bef = 0;
      for (int s = 0; s < S; ++s) {
        all += red[s * cols + c];
        bef += red[RW + s * cols + c];
      }
      total[c] = all;
      before[c] = bef;
    }
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kLThreads) layout_rank_kernel(LayoutArgs a) {
  extern __shared__ __align__(16) int sm[];
  const LayoutSmem P(a.G, a.E, a.key_cap);
  const Smem S(sm, P);
  const int b = blockIdx.x;
  const Tile tl = tile_of(a, b);
  // the caller's inputs were complete before layout_count_kernel started,
  // so they are staged before waiting for its histograms
  RawIds ids;
  stage_tile(a, tl, S, ids);
  pdl_wait();
  pdl_trigger();

  column_sums(a.tile_hist, a.n_tiles, a.G, b, S.red, S.tot, S.pre);
  if (a.dedup) column_sums(a.tile_phist, a.n_tiles, a.E, b, S.red, S.ptot, S.ppre);
  rank_count(tl.n_items, a.G, S.whist, nullptr, [&](int i) { return item_key(a, S, ids, i); });

  const int R_exp = finish_offsets(a, S);
  if (b == 0) {
    int f = 0;
    for (int q = threadIdx.x; q < a.n_tiles; q += kLThreads) f |= __ldcg(a.tile_flags + q);
    if (f) atomicOr(&S.misc[1], f);
    __syncthreads();
    write_globals(a, S, R_exp, S.misc[1]);
  }
  if (a.dedup) rank_tile_parts(a, tl, S, ids);
  rank_tile_items(a, tl, S, ids);
}

bool use_cluster(const moe_problem_t& p) { return (int64_t)p.M * p.topk <= kClusterItems; }

size_t smem_bytes(const moe_problem_t& p, int key_cap) {
  return sizeof(int) * (size_t)LayoutSmem(p.G, p.E_part, key_cap).total;
}

}  // namespace

int layout_tile_tokens(int M) {
  int t = (M + 147) / 148;
  t = (t + 31) / 32 * 32;
  return std::max(MOE_TILE_MIN_TOKENS, t);
}

int layout_num_tiles(int M) {
  const int T = layout_tile_tokens(M);
  return std::max(1, (M + T - 1) / T);
}

size_t layout_workspace_bytes(const moe_problem_t& p) {
  const size_t nt = (size_t)layout_num_tiles(p.M);
  const size_t ints = nt * ((size_t)p.G + (p.dedup ? (size_t)p.E_part : 0) + 1);
  return (ints * sizeof(int) + 255) / 256 * 256;
}

cudaError_t launch_layout(const moe_problem_t& p, const int32_t* topk_idx,
                          const int32_t* part_of, const moe_layout_t& lay,
                          void* workspace, cudaStream_t stream) {
  LayoutArgs a;
  a.M = p.M;
  a.G = p.G;
  a.topk = p.topk;
  a.E = p.E_part;
  a.dedup = p.dedup;
  a.idx = topk_idx;
  a.part_of = part_of;
  a.expert_count = lay.expert_count;
  a.expert_offset = lay.expert_offset;
  a.part_count = lay.part_count;
  a.part_offset = lay.part_offset;
  a.exp_row = lay.exp_row;
  a.disp_token = lay.disp_token;
  a.disp_row = lay.disp_row;
  a.exp_to_disp = lay.exp_to_disp;
  a.status = lay.status;

  if (use_cluster(p)) {
    // tiles of a multiple of 4 tokens keep every tile's ids 16-byte aligned
    a.T = std::max(4, ((p.M + kClusterCTAs - 1) / kClusterCTAs + 3) / 4 * 4);
    a.n_tiles = kClusterCTAs;
    a.key_cap = a.T * p.topk;
    a.tile_hist = a.tile_phist = a.tile_flags = nullptr;
    const size_t smem = smem_bytes(p, a.key_cap);
    cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(layout_cluster_kernel), smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kClusterCTAs);
    cfg.blockDim = dim3(kLThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kClusterCTAs;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = MOE_USE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, layout_cluster_kernel, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }

  a.T = layout_tile_tokens(p.M);
  a.n_tiles = layout_num_tiles(p.M);
  a.key_cap = a.T * p.topk <= kMaxTileItems ? a.T * p.topk : 0;
  int* ws = static_cast<int*>(workspace);
  a.tile_hist = ws;
  a.tile_phist = ws + (size_t)a.n_tiles * p.G;
  a.tile_flags = a.tile_phist + (p.dedup ? (size_t)a.n_tiles * p.E_part : 0);
  const size_t smem = smem_bytes(p, a.key_cap);
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(layout_count_kernel), smem);
  if (e != cudaSuccess) return e;
  e = allow_dynamic_smem(reinterpret_cast<const void*>(layout_rank_kernel), smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(layout_count_kernel, dim3(a.n_tiles), dim3(kLThreads), smem, stream, a);
  if (e != cudaSuccess) return e;
  e = launch_pdl(layout_rank_kernel, dim3(a.n_tiles), dim3(kLThreads), smem, stream, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
