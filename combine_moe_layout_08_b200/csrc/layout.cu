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
// scan across warps gives each warp's base, and a ballot match (one vote per
// key bit) ranks the lanes of a 32-pair chunk.  Everything is fixed by the
// data, so the result is bitwise reproducible.
//
// Each tile summarises itself in one row of W ints: its count per expert,
// with dedup its distinct (token, partition) count per partition, and two
// counters of invalid input (expert ids outside [0, G); placement entries
// outside [0, E_part), first tile only).  One column reduction over the rows
// then gives every total, every tile prefix and the status word.
//
// Two schedules, no host round trip in either:
//   * small batches (<= kClusterItems routed pairs): ONE launch of a cluster
//     of C <= 8 blocks (one per MOE_CLUSTER_BLOCK_ITEMS pairs); the blocks
//     exchange their rows through distributed shared memory between two
//     hardware cluster barriers.  No workspace is touched.
//   * larger batches: about one tile per SM in two launches.
//     layout_count_kernel writes the rows to the workspace;
//     layout_rank_kernel stages its tile, orders the experts by (partition,
//     id) with every warp at once and counts its tile per warp -- all from the
//     caller's inputs, before it waits for layout_count_kernel (programmatic
//     dependent launch) -- then reduces the rows with batched 16-byte loads
//     from L2 and ranks its tile.
// In both, the tile's expert ids are cached in shared memory when they fit.
// Asked for it, both also emit the grouped-GEMM tile metadata: one warp
// scans the tiles per expert while the others rank, and every block writes
// its share of the tiles at the end.
#include <cooperative_groups.h>

#include <algorithm>

#include "layout_device.cuh"
#include "moe_device.cuh"
#include "moe_internal.h"

namespace cg = cooperative_groups;

namespace moe {
namespace {

constexpr int kLThreads = 512;
constexpr int kLWarps = kLThreads / kWarp;
// Register budget of the layout kernels: two blocks per SM, so that a rank
// block that launches early (programmatic launch) fits beside a count block.
constexpr int kLMinBlocks = 2;
constexpr int kMaxCluster = 8;
constexpr int kMaxTileItems = 16384;  // tile ids cached in shared memory (64 KB)
// Compile-time tuning constants: batches of at most MOE_CLUSTER_ITEMS routed
// pairs take the one-cluster schedule, with one block per
// MOE_CLUSTER_BLOCK_ITEMS pairs; tiles of the two-launch schedule hold at
// least MOE_TILE_MIN_TOKENS tokens.
#ifndef MOE_CLUSTER_ITEMS
#define MOE_CLUSTER_ITEMS 8192  // measured on B200: one cluster wins only for small batches
#endif
#ifndef MOE_CLUSTER_BLOCK_ITEMS
#define MOE_CLUSTER_BLOCK_ITEMS 256  // measured on B200 (decode batch: 4 blocks beat 1)
#endif
#ifndef MOE_TILE_MIN_TOKENS
#define MOE_TILE_MIN_TOKENS 128  // measured on B200 (64..256 within noise; 128 best for fp8)
#endif
constexpr int kClusterItems = MOE_CLUSTER_ITEMS;
static_assert(kClusterItems <= kMaxCluster * kMaxTileItems, "cluster tiles must fit the id cache");
// width of each half of the column-sum reduction buffer: one slot per thread,
// 4 columns per slot, and at least the widest tile row (MOE_MAX_G +
// MOE_MAX_E_PART + 2, padded)
constexpr int kRedW = 4 * kLThreads;
static_assert(kRedW >= MOE_MAX_G + MOE_MAX_E_PART + 4, "reduction buffer narrower than a tile row");
static_assert(2 * kRedW >= (MOE_MAX_E_PART + 1) * ((MOE_MAX_G + 31) / 32),
              "reduction buffer smaller than the expert order's counts");

__host__ __device__ constexpr int up4(int x) { return (x + 3) & ~3; }

// ints per tile row: [G expert counts | E partition counts (dedup) | 2 flag counts], padded
__host__ __device__ constexpr int row_width(int G, int E, int dedup) {
  return up4(G + (dedup ? E : 0) + 2);
}

struct LayoutArgs {
  int M, G, topk, E, dedup;
  int T;        // tokens per tile
  int n_tiles;  // tiles (= blocks)
  int key_cap;  // ids the shared-memory cache holds (0: read from global)
  int W;        // ints per tile row
  unsigned topk_magic;  // floor((2^32 - 1) / topk): i / topk without a divide
  const int* __restrict__ idx;
  const int* __restrict__ part_of;
  int* tile_rows;  // [n_tiles][W]   (two-launch schedule)
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
  int part_s, eoff, pos, scanbuf, row, ctot, cpre, red, whist, pc, poff, pbase, wp, misc,
      keys, total;
  __host__ __device__ LayoutSmem(int G, int E, int W, int key_cap) {
    int o = 0;
    part_s = o; o += up4(G);
    eoff = o; o += up4(G);
    pos = o; o += up4(G);
    scanbuf = o; o += up4(G);
    row = o; o += up4(W);
    ctot = o; o += up4(W);
    cpre = o; o += up4(W);
    red = o; o += 2 * kRedW;
    whist = o; o += up4(kLWarps * G);
    pc = o; o += up4(E);
    poff = o; o += up4(E + 1);
    pbase = o; o += up4(E);
    wp = o; o += up4(kLWarps * E);
    misc = o; o += 4;
    keys = o; o += up4(key_cap);
    total = o;
  }
};

struct Smem {
  int *part_s, *eoff, *pos, *scanbuf, *row, *ctot, *cpre, *red, *whist, *pc, *poff, *pbase,
      *wp, *misc, *keys;
  // views: totals / tile prefixes per expert and per partition
  int *tot, *pre, *ptot, *ppre;
  __device__ Smem(int* sm, const LayoutSmem& P, int G)
      : part_s(sm + P.part_s), eoff(sm + P.eoff), pos(sm + P.pos), scanbuf(sm + P.scanbuf),
        row(sm + P.row), ctot(sm + P.ctot), cpre(sm + P.cpre), red(sm + P.red),
        whist(sm + P.whist), pc(sm + P.pc), poff(sm + P.poff),
        pbase(sm + P.pbase), wp(sm + P.wp), misc(sm + P.misc), keys(sm + P.keys) {
    tot = ctot;
    pre = cpre;
    ptot = ctot + G;
    ppre = cpre + G;
  }
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
// zero the block's scratch and load the placement map; with `order`, then
// order the experts by (partition, id) (all warps, expert_order_block, which
// needs only the placement map).  Reads only the caller's inputs.  Ends with
// a barrier.
__device__ void stage_tile(const LayoutArgs& a, const Tile& tl, const Smem& S, RawIds& ids,
                           bool order) {
  const int* src = a.idx + (size_t)tl.t0 * a.topk;
  ids.g = src;
  ids.s = nullptr;
  const bool cache = tl.n_items <= a.key_cap;
  if (cache) ids.s = S.keys;
  const int r = threadIdx.x;
  // the first placement entry of this thread, in flight with the ids
  const int part0 = r < a.G ? __ldg(a.part_of + r) : 0;
  if (cache) {
    const int n = tl.n_items;
    // batches of 4 predicated loads per thread, all in flight before the
    // first shared-memory store
    constexpr int B = 4;
    if ((reinterpret_cast<uintptr_t>(src) & 15) == 0) {
      const int n4 = n >> 2;
      const int4* s4 = reinterpret_cast<const int4*>(src);
      int4* k4 = reinterpret_cast<int4*>(S.keys);
      for (int i0 = r; i0 < n4; i0 += B * kLThreads) {
        int4 v[B];
#pragma unroll
        for (int j = 0; j < B; ++j)
          if (i0 + j * kLThreads < n4) v[j] = __ldg(s4 + i0 + j * kLThreads);
#pragma unroll
        for (int j = 0; j < B; ++j)
          if (i0 + j * kLThreads < n4) k4[i0 + j * kLThreads] = v[j];
      }
      for (int i = (n4 << 2) + r; i < n; i += kLThreads) S.keys[i] = __ldg(src + i);
    } else {
      for (int i0 = r; i0 < n; i0 += B * kLThreads) {
        int v[B];
#pragma unroll
        for (int j = 0; j < B; ++j)
          if (i0 + j * kLThreads < n) v[j] = __ldg(src + i0 + j * kLThreads);
#pragma unroll
        for (int j = 0; j < B; ++j)
          if (i0 + j * kLThreads < n) S.keys[i0 + j * kLThreads] = v[j];
      }
    }
  }
  if (r < a.G) S.part_s[r] = part0;
  for (int e = r + kLThreads; e < a.G; e += kLThreads) S.part_s[e] = __ldg(a.part_of + e);
  for (int i = r; i < kLWarps * a.G; i += kLThreads) S.whist[i] = 0;
  for (int i = r; i < a.W; i += kLThreads) S.row[i] = 0;
  for (int p = r; p < a.E; p += kLThreads) {
    S.pc[p] = 0;
    S.pbase[p] = 0;
  }
  if (r < 4) S.misc[r] = 0;
  // the expert order's per-(key, chunk) counts live in red (free until the
  // column sums)
  if (order)
    for (int i = r; i < (a.E + 1) * ((a.G + kWarp - 1) / kWarp); i += kLThreads) S.red[i] = 0;
  __syncthreads();
  if (order) expert_order_block<kLThreads>(S.part_s, a.G, a.E, S.pos, S.red);
}

__device__ __forceinline__ int item_key(const LayoutArgs& a, const Smem& S, const RawIds& ids,
                                        int i) {
  const int e = ids(i);
  return (e >= 0 && e < a.G && valid_part(S.part_s[e], a.E)) ? e : -1;
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
  int* wh = whist + warp * K;
  // per-warp counts only (the order inside a segment does not matter
  // here): shared-memory atomics on the warp's own histogram
  for (int i = beg + lane; i < end; i += kWarp) {
    const int key = key_of(i);
    if (key >= 0) atomicAdd(&wh[key], 1);
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

// Where the tile's dedup rows [token][partition] are kept in shared memory
// for the inverse map: the reduction buffer (free once the column sums are
// done), past the G ints that the tile metadata's expert list may occupy
// there; nullptr when ntok * E_part does not fit.
__device__ __forceinline__ int* tile_drows(const LayoutArgs& a, const Tile& tl, const Smem& S) {
  const int off = up4(a.G);
  return (long long)tl.ntok * a.E <= 2 * kRedW - off ? S.red + off : nullptr;
}

// The tile's own row: expert counts (and per-warp bases in whist), with
// dedup its distinct (token, partition) counts, and the invalid-input
// counters.  Ends with a barrier.
// per_warp: also leave the per-warp bases of the stable rank in whist (the
// one-cluster schedule ranks its tile with them); otherwise only the totals
// are needed, counted with shared-memory atomics.
__device__ void count_tile(const LayoutArgs& a, const Tile& tl, const Smem& S, const RawIds& ids,
                           bool first, bool per_warp) {
  const int G = a.G, E = a.E, lane = lane_id();
  const int fcol = G + (a.dedup ? E : 0);
  int bad = 0;
  if (per_warp) {
    rank_count(tl.n_items, G, S.whist, S.row, [&](int i) {
      const int e = ids(i);
      bad += (e < 0 || e >= G);
      return (e >= 0 && e < G && valid_part(S.part_s[e], E)) ? e : -1;
    });
  } else {
    for (int i = threadIdx.x; i < tl.n_items; i += kLThreads) {
      const int e = ids(i);
      if (e < 0 || e >= G)
        ++bad;
      else if (valid_part(S.part_s[e], E))
        atomicAdd(&S.row[e], 1);
    }
  }
  int badp = 0;
  if (first)
    for (int e = threadIdx.x; e < G; e += kLThreads) badp += !valid_part(S.part_s[e], E);
  if (bad) atomicAdd(&S.row[fcol], bad);
  if (badp) atomicAdd(&S.row[fcol + 1], badp);
  if (a.dedup) {
    for (int r0 = 0; r0 < tl.ntok; r0 += kLThreads) {
      const int t = r0 + threadIdx.x;
      const unsigned long long mask = t < tl.ntok ? token_mask(a, ids, S.part_s, t) : 0ull;
      for (int p = 0; p < E; ++p) {
        const unsigned bal = __ballot_sync(kFull, (mask >> p) & 1ull);
        if (lane == 0 && bal) atomicAdd(&S.row[G + p], __popc(bal));
      }
    }
  }
  __syncthreads();
}

// expert offsets (needs pos[], tot[]), partition counts and offsets (needs
// ptot[] with dedup).  Returns R_exp.  Ends with a barrier.
__device__ int finish_offsets(const LayoutArgs& a, const Smem& S) {
  const int G = a.G, E = a.E, tid = threadIdx.x;
  for (int e = tid; e < G; e += kLThreads) {
    S.scanbuf[S.pos[e]] = S.tot[e];
    if (!a.dedup && valid_part(S.part_s[e], E) && S.tot[e]) atomicAdd(&S.pc[S.part_s[e]], S.tot[e]);
  }
  __syncthreads();
  if (warp_id() == 0) {
    const int R_exp = warp_exclusive_scan(S.scanbuf, G);
    if (a.dedup)
      for (int p = lane_id(); p < E; p += kWarp) S.pc[p] = S.ptot[p];
    __syncwarp();
    for (int p = lane_id(); p < E; p += kWarp) S.poff[p] = S.pc[p];
    __syncwarp();
    const int R_disp = warp_exclusive_scan(S.poff, E);
    if (lane_id() == 0) {
      S.poff[E] = R_disp;
      S.misc[2] = R_exp;
    }
  }
  __syncthreads();
  for (int e = tid; e < G; e += kLThreads) S.eoff[e] = S.scanbuf[S.pos[e]];
  __syncthreads();
  return S.misc[2];
}

__device__ void write_globals(const LayoutArgs& a, const Smem& S, int R_exp) {
  const int fcol = a.G + (a.dedup ? a.E : 0);
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
    *a.status = (S.ctot[fcol] > 0 ? MOE_STATUS_BAD_EXPERT : 0) |
                (S.ctot[fcol + 1] > 0 ? MOE_STATUS_BAD_PART : 0);
  }
}

// dedup: dispatch row of each distinct (token, partition) of the tile
__device__ void rank_tile_parts(const LayoutArgs& a, const Tile& tl, const Smem& S,
                                const RawIds& ids) {
  const int E = a.E, lane = lane_id(), warp = warp_id(), tid = threadIdx.x;
  const unsigned lt = lanemask_lt();
  int* drs = tile_drows(a, tl, S);
  const bool vec8 = E == 8 && (reinterpret_cast<uintptr_t>(a.disp_row) & 15) == 0;
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
    auto row_of = [&](int p, bool has, unsigned bal) {
      int row = -1;
      if (has) {
        row = S.poff[p] + S.ppre[p] + S.wp[warp * E + p] + __popc(bal & lt);
        a.disp_token[row] = tg;
      }
      if (drs) drs[t * E + p] = row;
      return row;
    };
    if (vec8) {
      // eight partitions: the token's rows leave as two 16-byte stores
      int rr[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) {
        const bool has = (mask >> p) & 1ull;
        const unsigned bal = __ballot_sync(kFull, has);
        rr[p] = t < tl.ntok ? row_of(p, has, bal) : -1;
      }
      if (t < tl.ntok) {
        int4* d = reinterpret_cast<int4*>(a.disp_row + (size_t)tg * 8);
        d[0] = make_int4(rr[0], rr[1], rr[2], rr[3]);
        d[1] = make_int4(rr[4], rr[5], rr[6], rr[7]);
      }
    } else {
      for (int p = 0; p < E; ++p) {
        const bool has = (mask >> p) & 1ull;
        const unsigned bal = __ballot_sync(kFull, has);
        if (t < tl.ntok) a.disp_row[(size_t)tg * E + p] = row_of(p, has, bal);
      }
    }
    __syncthreads();
  }
}

// i / topk for 0 <= i < 2^31: the high product with floor((2^32 - 1) / topk)
// is at most one below the quotient (its error is below 2i / 2^32 < 1), and
// one correction step makes it exact.
__device__ __forceinline__ int div_topk(const LayoutArgs& a, int i) {
  unsigned q = __umulhi((unsigned)i, a.topk_magic);
  if ((unsigned)i - q * (unsigned)a.topk >= (unsigned)a.topk) ++q;
  return (int)q;
}

// expert row of every pair of the tile (second pass of the stable rank)
__device__ void rank_tile_items(const LayoutArgs& a, const Tile& tl, const Smem& S,
                                const RawIds& ids) {
  const int G = a.G, E = a.E;
  int* exp_row = a.exp_row + (size_t)tl.t0 * a.topk;
  const int* drs = a.dedup ? tile_drows(a, tl, S) : nullptr;
  rank_assign(
      tl.n_items, G, S.whist, [&](int i) { return item_key(a, S, ids, i); },
      [&](int i, int e, int r) {
        const int row = S.eoff[e] + S.pre[e] + r;
        exp_row[i] = row;
        const int tk = div_topk(a, i);
        const int t = tl.t0 + tk;
        if (!a.dedup) {
          a.disp_token[row] = t;
        } else {
          a.exp_to_disp[row] = drs ? drs[tk * E + S.part_s[e]]
                                   : a.disp_row[(size_t)t * E + S.part_s[e]];
        }
      },
      [&](int i) { exp_row[i] = -1; });
}

// Tile metadata: one warp scans the tiles per expert in row order into
// scanbuf (free once the offsets are final) with the experts in red (free
// after the column sums) and the count in misc[3] ...
__device__ void scan_tiles(const LayoutArgs& a, const Smem& S) {
  const int n = tiles_scan_warp(S.pos, a.G, a.tiles.block_m, [&](int e) { return S.tot[e]; },
                                S.scanbuf, S.red);
  if (lane_id() == 0) S.misc[3] = n;
}

// ... and, after a block barrier, block b of nb writes its share of the tiles
// (block 0 also each expert's first tile).
__device__ void write_tiles(const LayoutArgs& a, const Smem& S, int b, int nb) {
  const int n = S.misc[3];
  if (b == 0) {
    for (int e = threadIdx.x; e < a.G; e += kLThreads) a.tiles.tile_first[e] = S.scanbuf[S.pos[e]];
    if (threadIdx.x == 0) a.tiles.tile_first[a.G] = n;
  }
  int i0, i1;
  tiles_share(n, b, nb, i0, i1);
  tiles_write(a.tiles, S.scanbuf, S.red, a.G, i0, i1, [&](int e) { return S.eoff[e]; },
              [&](int e) { return S.tot[e]; });
}

// ---------------------------------------------------------------------------
// schedule 1: one cluster of gridDim.x blocks
// ---------------------------------------------------------------------------
// The layout kernels are instantiated per mode (bit 0: dedup, bit 1:
// tile metadata), fixed in a local copy of the arguments, so that each
// instantiation holds only the code its mode runs.  Measured on B200: the
// denser code (an SM fetches a kernel's instructions afresh at every
// launch) takes 1.6 us off the M = 4096 layout and 0.7 us off the dedup ones.
template <int kMode>
__device__ __forceinline__ LayoutArgs with_mode(const LayoutArgs& in) {
  LayoutArgs a = in;
  a.dedup = kMode & 1;
  if (!(kMode & 2)) a.tiles.block_m = 0;
  return a;
}

template <int kMode>
__global__ void __launch_bounds__(kLThreads, kLMinBlocks) layout_cluster_kernel(LayoutArgs a_in) {
  const LayoutArgs a = with_mode<kMode>(a_in);
  extern __shared__ __align__(16) int sm[];
  cg::cluster_group cluster = cg::this_cluster();
  const LayoutSmem P(a.G, a.E, a.W, a.key_cap);
  const Smem S(sm, P, a.G);
  const int C = (int)cluster.num_blocks();
  const int r = (int)cluster.block_rank();
  const int tid = threadIdx.x;
  const Tile tl = tile_of(a, r);
  pdl_wait();
  pdl_trigger();
  RawIds ids;
  stage_tile(a, tl, S, ids, true);
  count_tile(a, tl, S, ids, r == 0, true);
  cluster.sync();

  // exchange: totals over the cluster and the prefix of the tiles before r
  for (int c = tid; c < a.W; c += kLThreads) {
    int v[kMaxCluster];
#pragma unroll
    for (int q = 0; q < kMaxCluster; ++q) v[q] = q < C ? cluster.map_shared_rank(S.row, q)[c] : 0;
    int all = 0, bef = 0;
#pragma unroll
    for (int q = 0; q < kMaxCluster; ++q) {
      all += v[q];
      bef += q < r ? v[q] : 0;
    }
    S.ctot[c] = all;
    S.cpre[c] = bef;
  }
  __syncthreads();

  const int R_exp = finish_offsets(a, S);
  if (r == 0) write_globals(a, S, R_exp);
  if (a.tiles.block_m > 0 && warp_id() == 0) scan_tiles(a, S);
  if (a.dedup) rank_tile_parts(a, tl, S, ids);
  rank_tile_items(a, tl, S, ids);  // ends with a block barrier
  if (a.tiles.block_m > 0) write_tiles(a, S, r, C);
  cluster.sync();  // no block leaves while another may still read its row
}

// ---------------------------------------------------------------------------
// schedule 2: one tile per SM, two launches
// ---------------------------------------------------------------------------
template <int kMode>
__global__ void __launch_bounds__(kLThreads, kLMinBlocks) layout_count_kernel(LayoutArgs a_in) {
  const LayoutArgs a = with_mode<kMode>(a_in);
  extern __shared__ __align__(16) int sm[];
  const LayoutSmem P(a.G, a.E, a.W, a.key_cap);
  const Smem S(sm, P, a.G);
  const int b = blockIdx.x;
  const Tile tl = tile_of(a, b);
  pdl_wait();
  pdl_trigger();
  RawIds ids;
  stage_tile(a, tl, S, ids, false);
  count_tile(a, tl, S, ids, b == 0, false);
  int4* dst = reinterpret_cast<int4*>(a.tile_rows + (size_t)b * a.W);
  const int4* src = reinterpret_cast<const int4*>(S.row);
  for (int i = threadIdx.x; i < (a.W >> 2); i += kLThreads) dst[i] = src[i];
}

// Column sums of the [rows][W] tile rows in global memory (L2): total over
// all rows and over rows < b.  Thread slot (c4, s) sums columns 4*c4 .. +3
// over rows s, s + S, ... with 16-byte loads in batches of 8 rows, all
// issued (predicated) before any is used -- a rolled loop would wait out one
// L2 round trip per row; the S partial sums of each column are then added in
// shared memory.  W is a multiple of 4 and at most kRedW.
__device__ void column_sums(const int* src, int rows, int W, int b, int* red, int* total,
                            int* before) {
  constexpr int B = 8;
  const int tid = threadIdx.x;
  const int C4 = W >> 2;
  const int S = C4 <= kLThreads ? kLThreads / C4 : 1;
  for (int slot = tid; slot < C4 * S; slot += kLThreads) {
    const int c4 = slot % C4, s = slot / C4;
    int4 all = make_int4(0, 0, 0, 0), bef = all;
    for (int r0 = s; r0 < rows; r0 += B * S) {
      int4 v[B];
#pragma unroll
      for (int j = 0; j < B; ++j) {
        const int r = r0 + j * S;
        v[j] = r < rows ? __ldcg(reinterpret_cast<const int4*>(src + (size_t)r * W) + c4)
                        : make_int4(0, 0, 0, 0);
      }
#pragma unroll
      for (int j = 0; j < B; ++j) {
        all.x += v[j].x; all.y += v[j].y; all.z += v[j].z; all.w += v[j].w;
        if (r0 + j * S < b) {
          bef.x += v[j].x; bef.y += v[j].y; bef.z += v[j].z; bef.w += v[j].w;
        }
      }
    }
    const int base = s * W + 4 * c4;
    red[base] = all.x; red[base + 1] = all.y; red[base + 2] = all.z; red[base + 3] = all.w;
    red[kRedW + base] = bef.x; red[kRedW + base + 1] = bef.y;
    red[kRedW + base + 2] = bef.z; red[kRedW + base + 3] = bef.w;
  }
  __syncthreads();
  for (int c = tid; c < W; c += kLThreads) {
    int all = 0, bef = 0;
    for (int s = 0; s < S; ++s) {
      all += red[s * W + c];
      bef += red[kRedW + s * W + c];
    }
    total[c] = all;
    before[c] = bef;
  }
  __syncthreads();
}

template <int kMode>
__global__ void __launch_bounds__(kLThreads, kLMinBlocks) layout_rank_kernel(LayoutArgs a_in) {
  const LayoutArgs a = with_mode<kMode>(a_in);
  extern __shared__ __align__(16) int sm[];
  const LayoutSmem P(a.G, a.E, a.W, a.key_cap);
  const Smem S(sm, P, a.G);
  const int b = blockIdx.x;
  const Tile tl = tile_of(a, b);
  // Everything that depends only on the caller's inputs -- which were
  // complete before layout_count_kernel started -- runs before the wait:
  // the tile's ids, the expert order (every warp) and the tile's
  // per-warp counts.
  RawIds ids;
  stage_tile(a, tl, S, ids, true);
  rank_count(tl.n_items, a.G, S.whist, nullptr, [&](int i) { return item_key(a, S, ids, i); });
  pdl_wait();
  pdl_trigger();

  column_sums(a.tile_rows, a.n_tiles, a.W, b, S.red, S.ctot, S.cpre);
  const int R_exp = finish_offsets(a, S);
  if (b == 0) write_globals(a, S, R_exp);
  if (a.tiles.block_m > 0 && warp_id() == 0) scan_tiles(a, S);
  if (a.dedup) rank_tile_parts(a, tl, S, ids);
  rank_tile_items(a, tl, S, ids);  // ends with a block barrier
  if (a.tiles.block_m > 0) write_tiles(a, S, b, a.n_tiles);
}

// the count kernel, then the rank kernel as its programmatic dependent
cudaError_t launch_two(void (*count)(LayoutArgs), void (*rank)(LayoutArgs), const LayoutArgs& a,
                       size_t smem, cudaStream_t stream) {
  cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(count), smem);
  if (e != cudaSuccess) return e;
  e = allow_dynamic_smem(reinterpret_cast<const void*>(rank), smem);
  if (e != cudaSuccess) return e;
  e = launch_pdl(count, dim3(a.n_tiles), dim3(kLThreads), smem, stream, a);
  if (e != cudaSuccess) return e;
  e = launch_pdl(rank, dim3(a.n_tiles), dim3(kLThreads), smem, stream, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

bool use_cluster(const moe_problem_t& p) { return (int64_t)p.M * p.topk <= kClusterItems; }

size_t smem_bytes(const moe_problem_t& p, int key_cap) {
  const int W = row_width(p.G, p.E_part, p.dedup);
  return sizeof(int) * (size_t)LayoutSmem(p.G, p.E_part, W, key_cap).total;
}

}  // namespace

// In 64 bits: M may be as large as 2^31 - 1 (topk = E_part = 1), where
// M + 147 no longer fits an int.  The results do (T <= 2^31 / 148 + 32,
// at most 148 tiles).
int layout_tile_tokens(int M) {
  int64_t t = ((int64_t)M + 147) / 148;
  t = (t + 31) / 32 * 32;
  return (int)std::max<int64_t>(MOE_TILE_MIN_TOKENS, t);
}

int layout_num_tiles(int M) {
  const int64_t T = layout_tile_tokens(M);
  return (int)std::max<int64_t>(1, ((int64_t)M + T - 1) / T);
}

size_t layout_workspace_bytes(const moe_problem_t& p) {
  const size_t ints = (size_t)layout_num_tiles(p.M) * row_width(p.G, p.E_part, p.dedup);
  return (ints * sizeof(int) + 255) / 256 * 256;
}

cudaError_t launch_layout(const moe_problem_t& p, const int32_t* topk_idx,
                          const int32_t* part_of, const moe_layout_t& lay,
                          void* workspace, cudaStream_t stream, const TileOut& tiles) {
  LayoutArgs a;
  a.M = p.M;
  a.G = p.G;
  a.topk = p.topk;
  a.E = p.E_part;
  a.dedup = p.dedup;
  a.W = row_width(p.G, p.E_part, p.dedup);
  a.topk_magic = 0xffffffffu / (unsigned)p.topk;
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
  a.tiles = tiles;

  if (use_cluster(p)) {
    const int items = p.M * p.topk;
    const int C = std::min(kMaxCluster, std::max(1, (items + MOE_CLUSTER_BLOCK_ITEMS - 1) /
                                                        MOE_CLUSTER_BLOCK_ITEMS));
    // tiles of a multiple of 4 tokens keep every tile's ids 16-byte aligned
    a.T = std::max(4, ((p.M + C - 1) / C + 3) / 4 * 4);
    a.n_tiles = C;
    a.key_cap = a.T * p.topk;
    a.tile_rows = nullptr;
    const size_t smem = smem_bytes(p, a.key_cap);
    const int mode = (p.dedup ? 1 : 0) | (tiles.block_m > 0 ? 2 : 0);
    void (*kernel)(LayoutArgs) = mode == 0 ? layout_cluster_kernel<0> : mode == 1 ? layout_cluster_kernel<1>
                                 : mode == 2 ? layout_cluster_kernel<2> : layout_cluster_kernel<3>;
    cudaError_t e = allow_dynamic_smem(reinterpret_cast<const void*>(kernel), smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C);
    cfg.blockDim = dim3(kLThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = MOE_USE_PDL;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kernel, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }

  a.T = layout_tile_tokens(p.M);
  a.n_tiles = layout_num_tiles(p.M);
  a.key_cap = a.T * p.topk <= kMaxTileItems ? a.T * p.topk : 0;
  a.tile_rows = static_cast<int*>(workspace);
  const size_t smem = smem_bytes(p, a.key_cap);
  const int mode = (p.dedup ? 1 : 0) | (tiles.block_m > 0 ? 2 : 0);
  switch (mode) {
    case 0: return launch_two(layout_count_kernel<0>, layout_rank_kernel<0>, a, smem, stream);
    case 1: return launch_two(layout_count_kernel<1>, layout_rank_kernel<1>, a, smem, stream);
    case 2: return launch_two(layout_count_kernel<2>, layout_rank_kernel<2>, a, smem, stream);
    default: return launch_two(layout_count_kernel<3>, layout_rank_kernel<3>, a, smem, stream);
  }
}

}  // namespace moe
