// Routing layout and dispatch permute of a small batch (decode) in ONE
// kernel.  At a few hundred tokens the tiled layout and the dispatch are
// bound by latency, not bandwidth (Triton-distributed issue #117, "Results
// (Latency in us)": M = 2..512 at N = 7168, G = 256, topk = 8), so this
// schedule has no inter-block step at all and as few block-wide phases as
// the layout allows.
//
// Every index of the layout is a rank.  Give each routed pair i = t * topk + k
// whose expert e is valid (e in [0, G), placed on a partition p in
// [0, E_part)) the sort key  K_i = (p * G + e) << 13 | i,  and every other
// pair no key.  The expert rows order the pairs by (partition, expert, token,
// slot), i.e. by K, so
//   exp_row[t, k]     = #{ valid i : K_i < K_(t,k) }
//   expert_offset[e]  = #{ valid i : K_i < (p(e) * G + e) << 13 }
//                     = sum of the counts of the experts before e in
//                       (partition, id) order (experts placed nowhere last)
//   part_offset[p]    = sum of the counts of the experts on partitions < p
// and with dedup, token masks m_t (bit p: t holds an expert on p) give
//   disp_row[t, p]    = sum over t' of popc(m_t' & (2^p - 1))
//                       + #{ t' < t : bit p of m_t' }     (bit p of m_t set)
//   part_offset[p]    = sum over t' of popc(m_t' & (2^p - 1)).
// A block therefore needs no scan and no expert order for its own rows: it
// counts.
//
// Block (b, y) of 512 threads owns tokens [t0, t0 + nt), t0 = b * T, T =
// ceil(M / 148) (about one block per SM), and slice y of their flat 16-byte
// units:
//   1. issues the loads of its units of x[t0 .. t0 + nt) (contiguous rows)
//      so they are in flight while the layout is computed;
//   2. stages every routing id and the placement map in shared memory;
//   3. computes every pair's key, the expert histogram of the valid pairs,
//      the invalid-input flags and, with dedup, every token's mask;
//   4. answers rank queries, one warp per query: the rows of its own pairs
//      (and dedup rows of its own tokens), and -- blocks with y = 0 -- its
//      share of the per-expert and per-partition outputs (expert e and
//      partition p go to block e mod gridDim.x and p mod gridDim.x), from the
//      histogram; block (0, 0) also the totals and the status word.  With
//      tile metadata requested, the owner of an expert also counts the tiles
//      of the experts before it (tile_first[e]) and writes the expert's
//      tiles;
//   5. (y = 0) writes its pairs' index entries.  The rows themselves: bf16
//      slices are staged in shared memory at step 2 and each query warp's
//      lane 0 stores its token's slice to the row it has just found with one
//      bulk copy (cp.async.bulk, shared -> global), so the stores overlap the
//      remaining queries; fp8 is quantised once and stored from registers to
//      every row after the queries.
// Three block barriers in all.  Every index equals the one the tiled layout
// gives (the same stable order, the same dedup rows), so results are
// bit-identical to moe_layout followed by moe_dispatch.  Work per block grows
// with M * topk (every block reads every id once per query), so the schedule
// is taken only up to MOE_FUSED_ITEMS routed pairs.
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
// Compile-time switch: bf16 rows go from shared memory to their destination
// rows with bulk copies issued by the query warps (1), or from registers
// after the queries (0).  Measured on B200 (decode recipe, flush-to-flush
// step): 8.71 vs 9.30 us at M = 2, 12.53 vs 13.21 at M = 128, 30.29 vs 32.97
// at M = 512.
#ifndef MOE_FUSED_BULK_STORE
#define MOE_FUSED_BULK_STORE 1
#endif

namespace moe {
namespace {

constexpr int kFThreads = 512;
constexpr int kFWarps = kFThreads / kWarp;
constexpr int kIdxBits = 13;                   // pair index field of the sort key
constexpr int kMaxFusedItems = 1 << kIdxBits;  // so at most this many pairs
static_assert(MOE_FUSED_ITEMS >= 1 && MOE_FUSED_ITEMS <= kMaxFusedItems, "fused batch limit");
// (partition * G + expert) for partitions 0..E_part (E_part: placed nowhere)
static_assert(((long long)(MOE_MAX_E_PART + 1) * MOE_MAX_G << kIdxBits) <= 0xffffffffLL,
              "sort key width");
constexpr unsigned kNoKey = 0xffffffffu;  // pair left out: above every key
constexpr int kMaxChunk = 16;             // tokens per block
constexpr int kSMs = 148;
constexpr int kExpertsPerBlock = 16;      // blocks added so that none owns more experts

__host__ __device__ constexpr int up4(int x) { return (x + 3) & ~3; }

struct FusedArgs {
  int M, G, topk, E, dedup;
  int N8;   // 16-byte chunks per bf16 row (N / 8)
  int T;    // tokens per block
  int nb;   // blocks with tokens (blocks [nb, gridDim.x) only write per-expert outputs)
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
  int ids, keys, part_s, hist, masks, rows, drows, misc, xs, total;
  __host__ __device__ FusedSmem(int n_items, int M, int G, int E, int T, int topk, int dedup,
                                int x_ints) {
    int o = 0;
    ids = o; o += up4(n_items);                 // every routing id
    keys = o; o += up4(n_items);                // every pair's sort key
    part_s = o; o += up4(G);                    // placement map
    hist = o; o += up4(G);                      // valid pairs per expert
    masks = o; o += dedup ? 2 * up4(M) : 0;     // dedup: partition mask of every token (u64)
    rows = o; o += up4(T * topk);               // expert row of each pair of the chunk
    drows = o; o += dedup ? up4(T * E) : 0;     // dedup: row of each (chunk token, partition)
    misc = o; o += 4;                           // [invalid-input flags]
    xs = o; o += x_ints;                        // bulk stores: the block's slice of x
    total = o;
  }
};

// Bulk copy of `bytes` (a multiple of 16) from this block's shared memory to
// global memory by the copy engine, as one bulk group; both addresses
// 16-byte aligned.  The issuing thread waits for its groups (bulk_wait_all)
// before it exits.
__device__ __forceinline__ void bulk_store(void* dst, const void* src_smem, uint32_t bytes) {
  const uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(src_smem));
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst), "r"(s),
               "r"(bytes)
               : "memory");
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

// Warp-wide sum (every lane gets it).
__device__ __forceinline__ int warp_sum(int v) { return __reduce_add_sync(kFull, v); }

// (partition * G + e): the expert's place in (partition, id) order, experts
// placed nowhere last.
__device__ __forceinline__ int expert_rank_key(const int* part_s, int G, int E, int e) {
  const int p = part_s[e];
  return (valid_part(p, E) ? p : E) * G + e;
}

// Units: bf16 16-byte chunks, or fp8 16-column groups (two chunks, one lane
// of an 8-lane scale block).  Block (b, y) owns flat units
// [y * 512 * U, (y + 1) * 512 * U) of its chunk's nt * units.
// Instantiated per mode as well (bit 0: dedup, bit 1: tile metadata), fixed
// in a local copy of the arguments, so each instantiation keeps only the code
// its mode runs (an SM fetches a kernel's instructions afresh at every
// launch).  Measured on B200 at M = 128: 0.85 us off the event-timed step.
template <bool FP8, int U, int kMode>
__global__ void __launch_bounds__(kFThreads, 1) layout_dispatch_kernel(FusedArgs a_in) {
  FusedArgs a = a_in;
  a.dedup = kMode & 1;
  if (!(kMode & 2)) a.tiles.block_m = 0;
  extern __shared__ __align__(16) int sm[];
  const int n_items = a.M * a.topk;
  constexpr bool kBulk = MOE_FUSED_BULK_STORE && !FP8;
  const FusedSmem P(n_items, a.M, a.G, a.E, a.T, a.topk, a.dedup, kBulk ? kFThreads * U * 4 : 0);
  int* ids = sm + P.ids;
  unsigned* keys = reinterpret_cast<unsigned*>(sm + P.keys);
  int* part_s = sm + P.part_s;
  int* hist = sm + P.hist;
  unsigned long long* masks = reinterpret_cast<unsigned long long*>(sm + P.masks);
  int* rows = sm + P.rows;
  int* drows = sm + P.drows;
  int* misc = sm + P.misc;
  const int tid = threadIdx.x, lane = lane_id(), warp = warp_id();
  const int G = a.G, E = a.E, topk = a.topk, M = a.M;
  const int bx = blockIdx.x, nbx = gridDim.x;
  const bool writer = blockIdx.y == 0;
  const int t0 = bx * a.T;
  const int nt = bx < a.nb ? min(a.T, M - t0) : 0;
  const int i0 = t0 * topk;  // first routed pair of the chunk
  pdl_wait();
  pdl_trigger();
  if (nt == 0 && !writer) return;  // an expert-only column past the first slice: no work

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

  // 2. every routing id and the placement map (each thread's first entry
  // in flight with its ids); zeroed histogram and flags
  const int part0 = tid < G ? __ldg(a.part_of + tid) : 0;
  if ((reinterpret_cast<uintptr_t>(a.idx) & 15) == 0) {
    const int n4 = n_items >> 2;
    const int4* s4 = reinterpret_cast<const int4*>(a.idx);
    int4* k4 = reinterpret_cast<int4*>(ids);
    // two predicated loads per thread in flight together (n4 <= 1024 here)
    for (int i0 = tid; i0 < n4; i0 += 2 * kFThreads) {
      const int i1 = i0 + kFThreads;
      const int4 v0 = __ldg(s4 + i0);
      int4 v1 = make_int4(0, 0, 0, 0);
      if (i1 < n4) v1 = __ldg(s4 + i1);
      k4[i0] = v0;
      if (i1 < n4) k4[i1] = v1;
    }
    for (int i = (n4 << 2) + tid; i < n_items; i += kFThreads) ids[i] = __ldg(a.idx + i);
  } else {
    for (int i = tid; i < n_items; i += kFThreads) ids[i] = __ldg(a.idx + i);
  }
  for (int e = tid; e < G; e += kFThreads) {
    part_s[e] = e == tid ? part0 : __ldg(a.part_of + e);
    hist[e] = 0;
  }
  if (tid < 4) misc[tid] = 0;
  // bulk stores: the slice into shared memory, made visible to the copy
  // engine (the async proxy) before the block barrier
  uint4* xs = reinterpret_cast<uint4*>(sm + P.xs);
  const int vbeg = blockIdx.y * (kFThreads * U);
  if (kBulk) {
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (v0 + u * kFThreads < V) xs[tid + u * kFThreads] = lo[u];
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  uint4* recv = static_cast<uint4*>(a.recv);  // rows of `units` 16-byte chunks
  // the part of chunk token j's row in this block's slice, to row r
  auto store_token_slice = [&](int j, int r) {
    const int lo_u = max(j * units, vbeg), hi_u = min(min((j + 1) * units, V), vbeg + kFThreads * U);
    if (lo_u < hi_u)
      bulk_store(recv + (size_t)r * units + (lo_u - j * units), xs + (lo_u - vbeg),
                 (uint32_t)(hi_u - lo_u) * 16u);
  };
  __syncthreads();

  // 3. sort keys, histogram of the valid pairs, invalid input, token masks
  int bad = 0;
  for (int i = tid; i < n_items; i += kFThreads) {
    const int e = ids[i];
    unsigned key = kNoKey;
    if (e >= 0 && e < G) {
      const int p = part_s[e];
      if (valid_part(p, E)) {
        key = ((unsigned)(p * G + e) << kIdxBits) | (unsigned)i;
        atomicAdd(&hist[e], 1);
      }
    } else {
      bad |= MOE_STATUS_BAD_EXPERT;
    }
    keys[i] = key;
  }
  for (int e = tid; e < G; e += kFThreads)
    if (!valid_part(part_s[e], E)) bad |= MOE_STATUS_BAD_PART;
  if (bad) atomicOr(&misc[0], bad);
  if (a.dedup) {
    for (int t = tid; t < M; t += kFThreads) {
      unsigned long long m = 0ull;
      for (int k = 0; k < topk; ++k) {
        const int e = ids[t * topk + k];
        if (e >= 0 && e < G && valid_part(part_s[e], E)) m |= 1ull << part_s[e];
      }
      masks[t] = m;
    }
  }
  __syncthreads();

  // 4. rank queries, one warp each: [own pairs | own dedup (token, partition)
  // | owned experts | owned partitions | totals (block (0, 0))]
  const int n_pair = nt * topk;
  const int n_dd = a.dedup ? nt * E : 0;
  const int n_exp = writer && bx < G ? (G - bx + nbx - 1) / nbx : 0;
  const int n_prt = writer && bx < E ? (E - bx + nbx - 1) / nbx : 0;
  const int n_tot = writer && bx == 0 ? 1 : 0;
  const int q_dd = n_pair, q_exp = q_dd + n_dd, q_prt = q_exp + n_exp, q_tot = q_prt + n_prt;
  const int nq = q_tot + n_tot;
  const int bm = a.tiles.block_m;
  for (int q = warp; q < nq; q += kFWarps) {
    if (q < q_dd) {  // expert row of pair i0 + q
      const unsigned kj = keys[i0 + q];
      int r = -1;
      if (kj != kNoKey) {
        int c = 0;
        for (int i = lane; i < n_items; i += kWarp) c += keys[i] < kj;
        r = warp_sum(c);
      }
      if (lane == 0) {
        rows[q] = r;
        // without dedup the pair's expert row is a dispatch row; with dedup the
        // dispatch rows are the (token, partition) rows, stored below
        if (kBulk && !a.dedup && r >= 0) store_token_slice(q / topk, r);
      }
    } else if (q < q_exp) {  // dedup row of (token t0 + j, partition p)
      const int j = (q - q_dd) / E, p = (q - q_dd) - j * E;
      const int t = t0 + j;
      int r = -1;
      if ((masks[t] >> p) & 1ull) {
        const unsigned long long below = (1ull << p) - 1ull;  // p <= 63
        int c = 0;
        for (int u = lane; u < M; u += kWarp) {
          const unsigned long long m = masks[u];
          c += __popcll(m & below) + (u < t ? (int)((m >> p) & 1ull) : 0);
        }
        r = warp_sum(c);
      }
      if (lane == 0) {
        drows[j * E + p] = r;
        if (kBulk && r >= 0) store_token_slice(j, r);
      }
    } else if (q < q_prt) {  // expert e: count, first row, and its tiles
      const int e = bx + (q - q_exp) * nbx;
      const int ke = expert_rank_key(part_s, G, E, e);
      int off = 0, tf = 0;
      for (int f = lane; f < G; f += kWarp) {
        if (expert_rank_key(part_s, G, E, f) < ke) {
          const int c = hist[f];
          off += c;
          if (bm > 0) tf += c > 0 ? (c - 1) / bm + 1 : 0;
        }
      }
      off = warp_sum(off);
      const int cnt = hist[e];
      if (lane == 0) {
        a.expert_count[e] = cnt;
        a.expert_offset[e] = off;
      }
      if (bm > 0) {
        tf = warp_sum(tf);
        if (lane == 0) a.tiles.tile_first[e] = tf;
        const int nt_e = cnt > 0 ? (cnt - 1) / bm + 1 : 0;
        for (int j = lane; j < nt_e; j += kWarp) {
          a.tiles.tile_expert[tf + j] = e;
          a.tiles.tile_row[tf + j] = off + j * bm;
          a.tiles.tile_rows[tf + j] = min(bm, cnt - j * bm);
        }
      }
    } else if (q < q_tot) {  // partition p: rows and first row
      const int p = bx + (q - q_prt) * nbx;
      int off = 0, cnt = 0;
      if (a.dedup) {
        const unsigned long long below = (1ull << p) - 1ull;
        for (int u = lane; u < M; u += kWarp) {
          const unsigned long long m = masks[u];
          off += __popcll(m & below);
          cnt += (int)((m >> p) & 1ull);
        }
      } else {
        for (int f = lane; f < G; f += kWarp) {
          const int pf = part_s[f];
          if (valid_part(pf, E)) {
            off += pf < p ? hist[f] : 0;
            cnt += pf == p ? hist[f] : 0;
          }
        }
      }
      off = warp_sum(off);
      cnt = warp_sum(cnt);
      if (lane == 0) {
        a.part_count[p] = cnt;
        a.part_offset[p] = off;
      }
    } else {  // totals: R_exp, R_disp, number of tiles; the status word
      int r_exp = 0, n_tiles = 0, r_disp = 0;
      for (int f = lane; f < G; f += kWarp) {
        const int c = hist[f];
        r_exp += c;
        if (bm > 0) n_tiles += c > 0 ? (c - 1) / bm + 1 : 0;
      }
      if (a.dedup)
        for (int u = lane; u < M; u += kWarp) r_disp += __popcll(masks[u]);
      r_exp = warp_sum(r_exp);
      n_tiles = warp_sum(n_tiles);
      r_disp = a.dedup ? warp_sum(r_disp) : r_exp;
      if (lane == 0) {
        a.expert_offset[G] = r_exp;
        a.part_offset[E] = r_disp;
        if (bm > 0) a.tiles.tile_first[G] = n_tiles;
        *a.status = misc[0];
      }
    }
  }
  __syncthreads();

  // 5. the chunk's index entries (y = 0), then the copy to every row
  if (writer) {
    for (int q = tid; q < n_pair; q += kFThreads) {
      const int r = rows[q];
      a.exp_row[(size_t)i0 + q] = r;
      if (r >= 0) {
        const int j = q / topk;
        if (a.dedup)
          a.exp_to_disp[r] = drows[j * E + part_s[ids[i0 + q]]];
        else
          a.disp_token[r] = t0 + j;
      }
    }
    for (int q = tid; q < n_dd; q += kFThreads) {
      const int j = q / E, t = t0 + j;
      const int r = drows[q];
      a.disp_row[(size_t)t * E + (q - j * E)] = r;
      if (r >= 0) a.disp_token[r] = t;
    }
  }
  // destinations of chunk token j: its pairs' rows in slot order, or with
  // dedup its rows in partition order (-1 entries skipped)
  const int nd = a.dedup ? E : topk;
  const int* dtab = a.dedup ? drows : rows;
  if (kBulk) {  // the rows went out with the queries: wait for this thread's copies
    bulk_wait_all();
  } else if (!FP8) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int v = v0 + u * kFThreads;
      if (v < V) {
        const int j = v / units, c = v - j * units;
        const int* dst = dtab + j * nd;
        for (int d = 0; d < nd; ++d) {
          const int r = dst[d];
          if (r >= 0) st_v4(recv + (size_t)r * units + c, lo[u]);
        }
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
        const int* dst = dtab + j * nd;
        for (int d = 0; d < nd; ++d) {
          const int r = dst[d];
          if (r < 0) continue;
          st_v4(recv + (size_t)r * units + c, q);
          if (scale_lane) a.recv_scale[(size_t)r * N128 + (c >> 3)] = s;
        }
      }
    }
  }
}

template <bool FP8, int U, int kMode>
cudaError_t launch_m(const FusedArgs& a, dim3 grid, size_t smem, cudaStream_t stream) {
  const void* k = reinterpret_cast<const void*>(layout_dispatch_kernel<FP8, U, kMode>);
  cudaError_t e = allow_dynamic_smem(k, smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(layout_dispatch_kernel<FP8, U, kMode>, grid, dim3(kFThreads), smem, stream, a);
}

template <bool FP8, int U>
cudaError_t launch_u(const FusedArgs& a, dim3 grid, size_t smem, cudaStream_t stream) {
  switch ((a.dedup ? 1 : 0) | (a.tiles.block_m > 0 ? 2 : 0)) {
    case 0: return launch_m<FP8, U, 0>(a, grid, smem, stream);
    case 1: return launch_m<FP8, U, 1>(a, grid, smem, stream);
    case 2: return launch_m<FP8, U, 2>(a, grid, smem, stream);
    default: return launch_m<FP8, U, 3>(a, grid, smem, stream);
  }
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
  a.nb = (p.M + a.T - 1) / a.T;
  // enough blocks that none owns more than kExpertsPerBlock experts
  const int nbx = std::max(a.nb, (p.G + kExpertsPerBlock - 1) / kExpertsPerBlock);
  const int units = p.fp8 ? a.N8 / 2 : a.N8;
  const int V = a.T * units;  // units of a full chunk
  const int Umax = p.fp8 ? 4 : 8;
  const int U = std::min(Umax, (V + kFThreads - 1) / kFThreads);
  const int x_ints = (MOE_FUSED_BULK_STORE && !p.fp8) ? kFThreads * U * 4 : 0;
  const size_t smem = sizeof(int) *
      (size_t)FusedSmem(p.M * p.topk, p.M, p.G, p.E_part, a.T, p.topk, p.dedup, x_ints).total;
  const int per_block = kFThreads * U;
  const dim3 grid(nbx, (V + per_block - 1) / per_block);
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
