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
// Two launches, no host round trip:
//   1. layout_count_kernel: one block per tile of T tokens.  Warp-aggregated
//      (match.any) shared-memory histogram of the tile's experts, ballot
//      counts of the tile's (token, partition) pairs, and status flags.
//   2. layout_rank_kernel: one block per tile.  Every block reduces the
//      per-tile histograms (a few hundred KB from L2) into totals and its own
//      tile prefix, orders experts by (partition, id), scans, and ranks its
//      pairs stably: warp-private counts, an exclusive scan across warps,
//      then match.any ranks in (token, slot) order.  Block 0 writes the
//      global counts / offsets / status.
// The order of every row is fixed by the data, so results are bitwise
// reproducible.
#include <algorithm>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kLThreads = 512;
constexpr int kLWarps = kLThreads / kWarp;

struct LayoutArgs {
  int M, G, topk, E, dedup, T, n_tiles;
  const int* __restrict__ idx;
  const int* __restrict__ part_of;
  int* tile_hist;   // [n_tiles][G]
  int* tile_phist;  // [n_tiles][E], dedup only
  int* tile_flags;  // [n_tiles]
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

// ---------------------------------------------------------------------------
// kernel 1: per-tile histograms
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLThreads) layout_count_kernel(LayoutArgs a) {
  extern __shared__ int sm[];
  int* hist = sm;              // [G]
  int* part_s = hist + a.G;    // [G]
  int* phist = part_s + a.G;   // [E]
  __shared__ int flags;

  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  const int b = blockIdx.x;
  for (int i = tid; i < a.G; i += kLThreads) {
    hist[i] = 0;
    part_s[i] = __ldg(a.part_of + i);
  }
  for (int i = tid; i < a.E; i += kLThreads) phist[i] = 0;
  if (tid == 0) flags = 0;
  __syncthreads();

  int my_flags = 0;
  if (b == 0) {
    for (int e = tid; e < a.G; e += kLThreads)
      if (!valid_part(part_s[e], a.E)) my_flags |= MOE_STATUS_BAD_PART;
  }

  const int t0 = b * a.T;
  const int ntok = max(0, min(a.M - t0, a.T));
  const int n_items = ntok * a.topk;
  const int* idx = a.idx + (size_t)t0 * a.topk;

  // expert histogram; lanes holding the same expert add once
  for (int i0 = warp * kWarp; i0 < n_items; i0 += kLThreads) {
    const int i = i0 + lane;
    int key = -1;
    if (i < n_items) {
      const int e = __ldg(idx + i);
      if (e < 0 || e >= a.G) {
        my_flags |= MOE_STATUS_BAD_EXPERT;
      } else if (valid_part(part_s[e], a.E)) {
        key = e;
      }
    }
    const unsigned peers = __match_any_sync(kFull, key);
    if (key >= 0 && lane == __ffs(peers) - 1) atomicAdd(&hist[key], __popc(peers));
  }

  // distinct (token, partition) pairs of the tile
  if (a.dedup) {
    for (int j0 = warp * kWarp; j0 < ntok; j0 += kLThreads) {
      const int tl = j0 + lane;
      unsigned long long mask = 0ull;
      if (tl < ntok) {
        for (int k = 0; k < a.topk; ++k) {
          const int e = __ldg(idx + (size_t)tl * a.topk + k);
          if (e >= 0 && e < a.G) {
            const int p = part_s[e];
            if (valid_part(p, a.E)) mask |= 1ull << p;
          }
        }
      }
      for (int p = 0; p < a.E; ++p) {
        const unsigned bal = __ballot_sync(kFull, (mask >> p) & 1ull);
        if (lane == 0 && bal) atomicAdd(&phist[p], __popc(bal));
      }
    }
  }
  if (my_flags) atomicOr(&flags, my_flags);
  __syncthreads();

  int* th = a.tile_hist + (size_t)b * a.G;
  for (int i = tid; i < a.G; i += kLThreads) th[i] = hist[i];
  if (a.dedup)
    for (int i = tid; i < a.E; i += kLThreads) a.tile_phist[(size_t)b * a.E + i] = phist[i];
  if (tid == 0) a.tile_flags[b] = flags;
}

// ---------------------------------------------------------------------------
// block-wide building blocks of kernel 2
// ---------------------------------------------------------------------------

// Column sums of a [rows][cols] int matrix in global memory: total over all
// rows and partial over rows < b.  `red` holds 2 * max(kLThreads, cols) ints.
__device__ void column_sums(const int* src, int rows, int cols, int b, int* red,
                            int* total, int* before) {
  const int tid = threadIdx.x;
  const int S = cols <= kLThreads ? kLThreads / cols : 1;
  const int RW = max(kLThreads, cols);
  for (int slot = tid; slot < cols * S; slot += kLThreads) {
    const int c = slot % cols, s = slot / cols;
    int all = 0, bef = 0;
#pragma unroll 4
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

// Stable counting rank of n elements: rank(i) = number of j < i with the same
// key.  The elements are cut into kLWarps contiguous segments, one per warp.
//   key_of(i) -> key in [0, K) or -1 (element skipped: on_skip(i))
//   on_rank(i, key, rank)
//   whist: kLWarps * K ints, zero on entry
//   key_count: [K] totals per key, or nullptr
template <class KeyOf, class OnRank, class OnSkip>
__device__ void block_stable_rank(int n, int K, int* whist, int* key_count,
                                  KeyOf key_of, OnRank on_rank, OnSkip on_skip) {
  const int lane = lane_id(), warp = warp_id();
  const int seg = (n + kLWarps - 1) / kLWarps;
  const int beg = min(n, warp * seg), end = min(n, beg + seg);
  int* wh = whist + warp * K;
  for (int c = beg; c < end; c += kWarp) {
    const int i = c + lane;
    const int key = i < end ? key_of(i) : -1;
    const unsigned peers = __match_any_sync(kFull, key);
    if (key >= 0 && lane == __ffs(peers) - 1) wh[key] += __popc(peers);
  }
  __syncthreads();
  for (int key = threadIdx.x; key < K; key += kLThreads) {
    int run = 0;
    for (int w = 0; w < kLWarps; ++w) {
      const int v = whist[w * K + key];
      whist[w * K + key] = run;
      run += v;
    }
    if (key_count) key_count[key] = run;
  }
  __syncthreads();
  const unsigned lt = lanemask_lt();
  for (int c = beg; c < end; c += kWarp) {
    const int i = c + lane;
    const int key = i < end ? key_of(i) : -1;
    const unsigned peers = __match_any_sync(kFull, key);
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

// shared-memory plan of kernel 2 (ints)
struct RankSmem {
  int part_s, tot, pre, eoff, erank, scanbuf, red, whist, keycnt, keystart, pc, poff, ptot,
      ppre, pbase, wp, warp_tot, misc, total;
  __host__ __device__ RankSmem(int G, int E) {
    const int RW = G > kLThreads ? G : kLThreads;
    const int KW = G > E + 1 ? G : E + 1;
    int o = 0;
    part_s = o; o += G;
    tot = o; o += G;
    pre = o; o += G;
    eoff = o; o += G;
    erank = o; o += G;
    scanbuf = o; o += G;
    red = o; o += 2 * RW;
    whist = o; o += kLWarps * KW;
    keycnt = o; o += E + 1;
    keystart = o; o += E + 1;
    pc = o; o += E;
    poff = o; o += E + 1;
    ptot = o; o += E;
    ppre = o; o += E;
    pbase = o; o += E;
    wp = o; o += kLWarps * E;
    warp_tot = o; o += kLWarps;
    misc = o; o += 4;
    total = o;
  }
};

// ---------------------------------------------------------------------------
// kernel 2: totals, offsets and stable ranks
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(kLThreads) layout_rank_kernel(LayoutArgs a) {
  extern __shared__ int sm[];
  const int G = a.G, E = a.E, b = blockIdx.x, nt = a.n_tiles;
  const RankSmem P(G, E);
  int* part_s = sm + P.part_s;
  int* tot = sm + P.tot;
  int* pre = sm + P.pre;
  int* eoff = sm + P.eoff;
  int* erank = sm + P.erank;
  int* scanbuf = sm + P.scanbuf;
  int* red = sm + P.red;
  int* whist = sm + P.whist;
  int* keycnt = sm + P.keycnt;
  int* keystart = sm + P.keystart;
  int* pc = sm + P.pc;
  int* poff = sm + P.poff;
  int* ptot = sm + P.ptot;
  int* ppre = sm + P.ppre;
  int* pbase = sm + P.pbase;
  int* wp = sm + P.wp;
  int* warp_tot = sm + P.warp_tot;
  int* misc = sm + P.misc;
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  const int KW = G > E + 1 ? G : E + 1;

  for (int e = tid; e < G; e += kLThreads) part_s[e] = __ldg(a.part_of + e);
  for (int i = tid; i < kLWarps * KW; i += kLThreads) whist[i] = 0;
  for (int p = tid; p < E; p += kLThreads) {
    pc[p] = 0;
    pbase[p] = 0;
  }
  if (tid == 0) misc[0] = 0;
  __syncthreads();

  // 1. totals over all tiles and the prefix of the tiles before this one
  column_sums(a.tile_hist, nt, G, b, red, tot, pre);
  if (a.dedup) column_sums(a.tile_phist, nt, E, b, red, ptot, ppre);

  // 2. expert order (partition, id); experts of invalid partitions last
  auto ekey = [&](int e) {
    const int p = part_s[e];
    return valid_part(p, E) ? p : E;
  };
  block_stable_rank(
      G, E + 1, whist, keycnt, ekey, [&](int e, int, int r) { erank[e] = r; }, [](int) {});
  if (tid == 0) {
    int run = 0;
    for (int k = 0; k <= E; ++k) {
      keystart[k] = run;
      run += keycnt[k];
    }
  }
  __syncthreads();
  for (int e = tid; e < G; e += kLThreads) {
    const int pos = keystart[ekey(e)] + erank[e];
    erank[e] = pos;
    scanbuf[pos] = tot[e];
  }
  __syncthreads();
  const int R_exp = block_exclusive_scan(scanbuf, G, warp_tot);
  for (int e = tid; e < G; e += kLThreads) {
    eoff[e] = scanbuf[erank[e]];
    if (!a.dedup && valid_part(part_s[e], E) && tot[e]) atomicAdd(&pc[part_s[e]], tot[e]);
  }
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int p = 0; p < E; ++p) {
      if (a.dedup) pc[p] = ptot[p];
      poff[p] = run;
      run += pc[p];
    }
    poff[E] = run;
  }
  __syncthreads();

  // 3. global counts and offsets (block 0)
  if (b == 0) {
    for (int e = tid; e < G; e += kLThreads) {
      a.expert_count[e] = tot[e];
      a.expert_offset[e] = eoff[e];
    }
    for (int p = tid; p < E; p += kLThreads) {
      a.part_count[p] = pc[p];
      a.part_offset[p] = poff[p];
    }
    int f = 0;
    for (int r = tid; r < nt; r += kLThreads) f |= __ldcg(a.tile_flags + r);
    if (f) atomicOr(&misc[0], f);
    __syncthreads();
    if (tid == 0) {
      a.expert_offset[G] = R_exp;
      a.part_offset[E] = poff[E];
      *a.status = misc[0];
    }
  }

  const int t0 = b * a.T;
  const int ntok = max(0, min(a.M - t0, a.T));
  const int n_items = ntok * a.topk;
  const int* idx = a.idx + (size_t)t0 * a.topk;

  // 4. dedup: dispatch row of each distinct (token, partition) of the tile
  if (a.dedup) {
    const unsigned lt = lanemask_lt();
    for (int r0 = 0; r0 < ntok; r0 += kLThreads) {
      const int tl = r0 + tid;
      unsigned long long mask = 0ull;
      if (tl < ntok) {
        for (int k = 0; k < a.topk; ++k) {
          const int e = __ldg(idx + (size_t)tl * a.topk + k);
          if (e >= 0 && e < G) {
            const int p = part_s[e];
            if (valid_part(p, E)) mask |= 1ull << p;
          }
        }
      }
      for (int p = 0; p < E; ++p) {
        const unsigned bal = __ballot_sync(kFull, (mask >> p) & 1ull);
        if (lane == 0) wp[warp * E + p] = __popc(bal);
      }
      __syncthreads();
      for (int p = tid; p < E; p += kLThreads) {
        int run = pbase[p];
        for (int w = 0; w < kLWarps; ++w) {
          const int v = wp[w * E + p];
          wp[w * E + p] = run;
          run += v;
        }
        pbase[p] = run;
      }
      __syncthreads();
      const int t = t0 + tl;
      for (int p = 0; p < E; ++p) {
        const bool has = (mask >> p) & 1ull;
        const unsigned bal = __ballot_sync(kFull, has);
        if (tl < ntok) {
          int row = -1;
          if (has) {
            row = poff[p] + ppre[p] + wp[warp * E + p] + __popc(bal & lt);
            a.disp_token[row] = t;
          }
          a.disp_row[(size_t)t * E + p] = row;
        }
      }
      __syncthreads();
    }
  }

  // 5. expert row of every pair of the tile, stable in (token, slot) order
  for (int i = tid; i < kLWarps * G; i += kLThreads) whist[i] = 0;
  __syncthreads();
  auto ikey = [&](int i) {
    const int e = __ldg(idx + i);
    return (e >= 0 && e < G && valid_part(part_s[e], E)) ? e : -1;
  };
  int* exp_row = a.exp_row + (size_t)t0 * a.topk;
  block_stable_rank(
      n_items, G, whist, nullptr, ikey,
      [&](int i, int e, int r) {
        const int row = eoff[e] + pre[e] + r;
        exp_row[i] = row;
        const int t = t0 + i / a.topk;
        if (!a.dedup) {
          a.disp_token[row] = t;
        } else {
          a.exp_to_disp[row] = a.disp_row[(size_t)t * E + part_s[e]];
        }
      },
      [&](int i) { exp_row[i] = -1; });
}

}  // namespace

int layout_tile_tokens(int M) {
  int t = (M + 147) / 148;
  t = (t + 31) / 32 * 32;
  return std::max(64, t);
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
  a.T = layout_tile_tokens(p.M);
  a.n_tiles = layout_num_tiles(p.M);
  a.idx = topk_idx;
  a.part_of = part_of;
  int* ws = static_cast<int*>(workspace);
  a.tile_hist = ws;
  a.tile_phist = ws + (size_t)a.n_tiles * p.G;
  a.tile_flags = a.tile_phist + (p.dedup ? (size_t)a.n_tiles * p.E_part : 0);
  a.expert_count = lay.expert_count;
  a.expert_offset = lay.expert_offset;
  a.part_count = lay.part_count;
  a.part_offset = lay.part_offset;
  a.exp_row = lay.exp_row;
  a.disp_token = lay.disp_token;
  a.disp_row = lay.disp_row;
  a.exp_to_disp = lay.exp_to_disp;
  a.status = lay.status;

  const size_t smem1 = sizeof(int) * (2 * (size_t)p.G + p.E_part);
  const size_t smem2 = sizeof(int) * (size_t)RankSmem(p.G, p.E_part).total;
  if (smem2 > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(layout_rank_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem2);
    if (e != cudaSuccess) return e;
  }
  layout_count_kernel<<<a.n_tiles, kLThreads, smem1, stream>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  layout_rank_kernel<<<a.n_tiles, kLThreads, smem2, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
