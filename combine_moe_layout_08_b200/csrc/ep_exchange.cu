// Expert-parallel data plane: the dispatch and the combine with the E_part
// partitions on E_part ranks.  Partition p's buffers live on rank p; this
// GPU addresses them through a device array of pointers (peer mappings over
// NVLink, symmetric memory, or plain local buffers when every rank is
// emulated on one GPU).
//
// The exchange is laid out by moe_ep_plan: rank r's dispatch rows of
// partition p, [part_offset[p], part_offset[p+1]) in its layout, occupy rows
// [send_offset[p], send_offset[p] + count) of rank p's receive buffer, in
// the same order -- Purlin's transposed-V layout (section 3.1: each
// destination holds every source's partition in source-rank order).  So
// dispatch row r of partition p lives at row  send_offset[p] + r -
// part_offset[p]  of rank p's buffers, and the expert outputs (y, or the
// two-level partial rows z) that rank p computes in its receive order come
// back from the same row.
//
//   ep_dispatch  push: every token row is read once and stored straight
//                into each destination rank's receive buffer (P2P stores; FP8
//                quantised once per token, scales stored beside).  Purlin
//                (section 3.2) pushes in its latency path; stores also need
//                no notification round trip before the data moves.
//   ep_combine   pull: each token gathers its expert-output rows from the
//                ranks that computed them (P2P loads) and sums them in slot
//                order in fp32 (the SCORE contract of Purlin section 3.3),
//                one rounding to bf16.  No dedup.
//   ep_reduce    pull, dedup: each token sums its partition rows z (one per
//                partition holding any of its experts) in partition order.
//
// The kernels never wait on another rank: the caller orders the exchange
// (the destinations' receive buffers are complete once every rank's dispatch
// has finished -- a barrier or an NCCL collective between the steps).
// Rows outside a buffer's capacity are skipped and raise MOE_STATUS_BAD_ROW.
#include <algorithm>

#include "fp8_device.cuh"
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kEThreads = 128;
constexpr int kMaxDest = MOE_MAX_E_PART > MOE_MAX_TOPK ? MOE_MAX_E_PART : MOE_MAX_TOPK;

struct EpArgs {
  int M, N8, topk, E, dedup, cap;  // cap: local row capacity (M * topk)
  int peer_cap;                    // rows each rank's buffer holds
  const uint4* __restrict__ x;     // dispatch: [M][N8]
  const float* __restrict__ w;     // combine: [M][topk]
  const int* exp_row;              // [M][topk]
  const int* disp_row;             // [M][E], dedup
  const int* part_offset;          // [E + 1], this rank's layout
  const int* send_offset;          // [E], this rank's plan
  void* const* peer_rows;          // [E] device pointers
  float* const* peer_scales;       // [E] device pointers (fp8 dispatch)
  uint4* out;                      // combine / reduce: [M][N8]
  int* status;
};

// Per-block copy of the partition offsets, send offsets and peer pointers.
struct EpTable {
  int po[MOE_MAX_E_PART + 1];
  int so[MOE_MAX_E_PART];
  char* rows[MOE_MAX_E_PART];
  float* scales[MOE_MAX_E_PART];
};

// A pointer the table cannot use (null, or a row buffer not 16-byte aligned,
// a scale buffer not 4-byte aligned) becomes null: that rank's rows are
// skipped and raise MOE_STATUS_BAD_ROW instead of a misaligned access.
__device__ __forceinline__ void load_table(const EpArgs& a, EpTable& tb, bool scales) {
  for (int p = threadIdx.x; p <= a.E; p += blockDim.x) {
    tb.po[p] = a.part_offset[p];
    if (p < a.E) {
      tb.so[p] = a.send_offset[p];
      char* r = static_cast<char*>(a.peer_rows[p]);
      tb.rows[p] = (reinterpret_cast<uintptr_t>(r) & 15) == 0 ? r : nullptr;
      float* f = scales ? a.peer_scales[p] : nullptr;
      tb.scales[p] = (reinterpret_cast<uintptr_t>(f) & 3) == 0 ? f : nullptr;
    }
  }
}

// Partition of expert row r: the largest p with po[p] <= r (po ascending;
// empty partitions share their offset with the next one).
__device__ __forceinline__ int part_of_row(const EpTable& tb, int E, int r) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tb.po[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Row of rank p's buffer holding this rank's dispatch row r (-1: outside the
// buffer, outside partition p, or no usable buffer).
__device__ __forceinline__ int peer_row(const EpArgs& a, const EpTable& tb, int p, int r,
                                        bool need_scales) {
  const long long d = (long long)tb.so[p] + r - tb.po[p];
  const bool usable = tb.rows[p] != nullptr && (!need_scales || tb.scales[p] != nullptr);
  return (usable && d >= 0 && d < a.peer_cap && r >= tb.po[p] && r < tb.po[p + 1]) ? (int)d : -1;
}

// Warp 0: the token's destinations (rank, row in that rank's buffer), in slot
// order, or with dedup in partition order.
__device__ __forceinline__ int ep_destinations(const EpArgs& a, const EpTable& tb, int t, int* dp,
                                               int* dr, int* nd, bool need_scales) {
  if (warp_id() == 0) {
    const int lane = lane_id();
    const int n_ent = a.dedup ? a.E : a.topk;
    const int* ent = a.dedup ? a.disp_row + (size_t)t * a.E : a.exp_row + (size_t)t * a.topk;
    int count = 0;
    bool bad = false;
    for (int base = 0; base < n_ent; base += kWarp) {
      const int i = base + lane;
      const int r = i < n_ent ? ld_nc_i32(ent + i) : -1;
      int p = -1, d = -1;
      if (r >= 0 && r < a.cap) {
        p = a.dedup ? i : part_of_row(tb, a.E, r);
        d = peer_row(a, tb, p, r, need_scales);
      }
      bad |= (r < -1) || (r >= a.cap) || (r >= 0 && r < a.cap && d < 0);
      const bool ok = d >= 0;
      const unsigned bal = __ballot_sync(kFull, ok);
      if (ok) {
        const int slot = count + __popc(bal & lanemask_lt());
        dp[slot] = p;
        dr[slot] = d;
      }
      count += __popc(bal);
    }
    if (lane == 0) *nd = count;
    if (bad) raise_status(a.status, MOE_STATUS_BAD_ROW);
  }
  __syncthreads();
  return *nd;
}

template <bool FP8, int U>
__global__ void __launch_bounds__(kEThreads) ep_dispatch_kernel(EpArgs a) {
  __shared__ EpTable tb;
  __shared__ int dp[kMaxDest], dr[kMaxDest];
  __shared__ int nd;
  const int t = blockIdx.x;
  const int units = FP8 ? (a.N8 >> 1) : a.N8;
  const int g0 = blockIdx.y * (kEThreads * U) + threadIdx.x;
  const uint4* src = a.x + (size_t)t * a.N8;
  pdl_wait();
  pdl_trigger();
  uint4 lo[U], hi[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int g = g0 + u * kEThreads;
    lo[u] = make_uint4(0, 0, 0, 0);
    hi[u] = lo[u];
    if (g < units) {
      if (FP8) {
        lo[u] = ld_nc_v4(src + 2 * g);
        hi[u] = ld_nc_v4(src + 2 * g + 1);
      } else {
        lo[u] = ld_nc_v4(src + g);
      }
    }
  }
  load_table(a, tb, FP8);
  __syncthreads();
  const int n = ep_destinations(a, tb, t, dp, dr, &nd, FP8);
  if (!FP8) {
    for (int d = 0; d < n; ++d) {
      uint4* o = reinterpret_cast<uint4*>(tb.rows[dp[d]]) + (size_t)dr[d] * a.N8;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int g = g0 + u * kEThreads;
        if (g < units) st_v4(o + g, lo[u]);
      }
    }
  } else {
    uint4 q[U];
    float s[U];
#pragma unroll
    for (int u = 0; u < U; ++u) q[u] = quantize_lane(lo[u], hi[u], s[u]);
    const int N128 = units >> 3;
    const bool scale_lane = (threadIdx.x & 7) == 0;
    for (int d = 0; d < n; ++d) {
      uint4* o = reinterpret_cast<uint4*>(tb.rows[dp[d]]) + (size_t)dr[d] * units;
      float* os = tb.scales[dp[d]] + (size_t)dr[d] * N128;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int g = g0 + u * kEThreads;
        if (g < units) {
          st_v4(o + g, q[u]);
          if (scale_lane) os[g >> 3] = s[u];
        }
      }
    }
  }
}

__device__ __forceinline__ void fma8(float* acc, float w, const uint4& v) {
  acc[0] = fmaf(w, bf16_lo(v.x), acc[0]);
  acc[1] = fmaf(w, bf16_hi(v.x), acc[1]);
  acc[2] = fmaf(w, bf16_lo(v.y), acc[2]);
  acc[3] = fmaf(w, bf16_hi(v.y), acc[3]);
  acc[4] = fmaf(w, bf16_lo(v.z), acc[4]);
  acc[5] = fmaf(w, bf16_hi(v.z), acc[5]);
  acc[6] = fmaf(w, bf16_lo(v.w), acc[6]);
  acc[7] = fmaf(w, bf16_hi(v.w), acc[7]);
}

__device__ __forceinline__ uint4 pack8(const float* acc) {
  return make_uint4(pack_bf16x2_rn(acc[0], acc[1]), pack_bf16x2_rn(acc[2], acc[3]),
                    pack_bf16x2_rn(acc[4], acc[5]), pack_bf16x2_rn(acc[6], acc[7]));
}

// out[t] = bf16( sum_k w[t,k] * y_rank(k)[row(k)] ), fp32 fma in slot order
// from +0 (pairs left out, or whose row falls outside the peer's buffer,
// contribute nothing).  KG slots gathered per batch.
template <int KG>
__global__ void __launch_bounds__(kEThreads) ep_combine_kernel(EpArgs a) {
  __shared__ EpTable tb;
  __shared__ const uint4* srow[MOE_MAX_TOPK];
  __shared__ float wts[MOE_MAX_TOPK];
  const int t = blockIdx.x, tid = threadIdx.x;
  if (tid == 0) {  // the gates are the router's output: warm L2 before the wait
    prefetch_line_l2(a.w + (size_t)t * a.topk);
    prefetch_line_l2(a.w + (size_t)t * a.topk + a.topk - 1);
  }
  pdl_wait();
  pdl_trigger();
  load_table(a, tb, false);
  __syncthreads();
  if (tid < a.topk) {
    const int r = ld_nc_i32(a.exp_row + (size_t)t * a.topk + tid);
    const uint4* p_ = nullptr;
    bool bad = r < -1 || r >= a.cap;
    if (r >= 0 && r < a.cap) {
      const int p = part_of_row(tb, a.E, r);
      const int d = peer_row(a, tb, p, r, false);
      if (d >= 0)
        p_ = reinterpret_cast<const uint4*>(tb.rows[p]) + (size_t)d * a.N8;
      else
        bad = true;
    }
    if (bad) raise_status(a.status, MOE_STATUS_BAD_ROW);
    srow[tid] = p_;
    wts[tid] = __ldg(a.w + (size_t)t * a.topk + tid);
  }
  __syncthreads();
  const int c = blockIdx.y * kEThreads + tid;
  if (c >= a.N8) return;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
  for (int k0 = 0; k0 < a.topk; k0 += KG) {
    uint4 v[KG];
#pragma unroll
    for (int j = 0; j < KG; ++j)
      if (k0 + j < a.topk && srow[k0 + j]) v[j] = ld_nc_v4(srow[k0 + j] + c);
#pragma unroll
    for (int j = 0; j < KG; ++j)
      if (k0 + j < a.topk && srow[k0 + j]) fma8(acc, wts[k0 + j], v[j]);
  }
  st_v4(a.out + (size_t)t * a.N8 + c, pack8(acc));
}

// out[t] = bf16( sum over the token's partitions p, in order, of
// z_rank(p)[row(p)] ), fp32 additions from +0.
__global__ void __launch_bounds__(kEThreads) ep_reduce_kernel(EpArgs a) {
  __shared__ EpTable tb;
  __shared__ int dp[kMaxDest], dr[kMaxDest];
  __shared__ int nd;
  const int t = blockIdx.x, tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  load_table(a, tb, false);
  __syncthreads();
  const int n = ep_destinations(a, tb, t, dp, dr, &nd, false);
  const int c = blockIdx.y * kEThreads + tid;
  if (c >= a.N8) return;
  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
  constexpr int B = 8;  // rows in flight per thread
  for (int q0 = 0; q0 < n; q0 += B) {
    uint4 v[B];
#pragma unroll
    for (int j = 0; j < B; ++j)
      if (q0 + j < n)
        v[j] = ld_nc_v4(reinterpret_cast<const uint4*>(tb.rows[dp[q0 + j]]) +
                        (size_t)dr[q0 + j] * a.N8 + c);
#pragma unroll
    for (int j = 0; j < B; ++j)
      if (q0 + j < n) {
        acc[0] = acc[0] + bf16_lo(v[j].x);
        acc[1] = acc[1] + bf16_hi(v[j].x);
        acc[2] = acc[2] + bf16_lo(v[j].y);
        acc[3] = acc[3] + bf16_hi(v[j].y);
        acc[4] = acc[4] + bf16_lo(v[j].z);
        acc[5] = acc[5] + bf16_hi(v[j].z);
        acc[6] = acc[6] + bf16_lo(v[j].w);
        acc[7] = acc[7] + bf16_hi(v[j].w);
      }
  }
  st_v4(a.out + (size_t)t * a.N8 + c, pack8(acc));
}

EpArgs ep_args(const moe_problem_t& p, const moe_layout_t& lay, const int32_t* send_offset,
               const moe_ep_peers_t& peers) {
  EpArgs a{};
  a.M = p.M;
  a.N8 = p.N / 8;
  a.topk = p.topk;
  a.E = p.E_part;
  a.dedup = p.dedup;
  a.cap = p.M * p.topk;
  a.peer_cap = peers.capacity;
  a.exp_row = lay.exp_row;
  a.disp_row = lay.disp_row;
  a.part_offset = lay.part_offset;
  a.send_offset = send_offset;
  a.peer_rows = peers.rows;
  a.peer_scales = peers.scales;
  a.status = lay.status;
  return a;
}

template <bool FP8, int U>
cudaError_t launch_dispatch_u(const EpArgs& a, cudaStream_t s) {
  const int units = FP8 ? a.N8 / 2 : a.N8;
  const dim3 grid(a.M, (units + kEThreads * U - 1) / (kEThreads * U));
  return launch_pdl(ep_dispatch_kernel<FP8, U>, grid, dim3(kEThreads), 0, s, a);
}

}  // namespace

cudaError_t launch_ep_dispatch(const moe_problem_t& p, const void* x, const moe_layout_t& lay,
                               const int32_t* send_offset, const moe_ep_peers_t& peers,
                               cudaStream_t stream) {
  if (p.M == 0) return cudaSuccess;
  EpArgs a = ep_args(p, lay, send_offset, peers);
  a.x = static_cast<const uint4*>(x);
  // fan-out (no dedup, topk >= 4): one vector per thread in narrow blocks;
  // otherwise up to 4 (fp8: 2 chunk pairs) per thread
  const bool fan_out = !p.dedup && p.topk >= 4;
  const int units = p.fp8 ? a.N8 / 2 : a.N8;
  const int U = fan_out ? 1 : std::min(4, (units + kEThreads - 1) / kEThreads);
  cudaError_t e;
  if (!p.fp8) {
    e = U == 1 ? launch_dispatch_u<false, 1>(a, stream)
        : U == 2 ? launch_dispatch_u<false, 2>(a, stream)
        : U == 3 ? launch_dispatch_u<false, 3>(a, stream)
                 : launch_dispatch_u<false, 4>(a, stream);
  } else {
    e = U == 1 ? launch_dispatch_u<true, 1>(a, stream)
        : U == 2 ? launch_dispatch_u<true, 2>(a, stream)
        : U == 3 ? launch_dispatch_u<true, 3>(a, stream)
                 : launch_dispatch_u<true, 4>(a, stream);
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_ep_combine(const moe_problem_t& p, const moe_ep_peers_t& y, const float* w,
                              const moe_layout_t& lay, const int32_t* send_offset, void* out,
                              cudaStream_t stream) {
  if (p.M == 0) return cudaSuccess;
  EpArgs a = ep_args(p, lay, send_offset, y);
  a.w = w;
  a.out = static_cast<uint4*>(out);
  const dim3 grid(p.M, (a.N8 + kEThreads - 1) / kEThreads);
  cudaError_t e = p.topk >= 4 ? launch_pdl(ep_combine_kernel<4>, grid, dim3(kEThreads), 0, stream, a)
                              : launch_pdl(ep_combine_kernel<2>, grid, dim3(kEThreads), 0, stream, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_ep_reduce(const moe_problem_t& p, const moe_ep_peers_t& z,
                             const moe_layout_t& lay, const int32_t* send_offset, void* out,
                             cudaStream_t stream) {
  if (p.M == 0) return cudaSuccess;
  EpArgs a = ep_args(p, lay, send_offset, z);
  a.out = static_cast<uint4*>(out);
  const dim3 grid(p.M, (a.N8 + kEThreads - 1) / kEThreads);
  cudaError_t e = launch_pdl(ep_reduce_kernel, grid, dim3(kEThreads), 0, stream, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
