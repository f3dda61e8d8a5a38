// Expert-parallel exchange plan: the counts exchange of an all-to-all over W
// ranks, turned into every offset a rank needs to move its dispatch rows.
//
// The Triton-distributed issue #117 all-to-all exchanges split counts before
// the data (test snippet: split_send_buf -> split_recv_buf, with the
// send side's cumulative sum send_split_cumsum).  After that exchange every
// rank holds the matrix P[s][d] of the rows each source s sends to each
// destination d (the part_count of every rank's layout, partition d = rank
// d).  The receive side is Purlin's transposed-V layout (section 3.1):
// destination r holds partition r of every source, in source-rank order.
// For rank r this kernel writes
//   send_offset[d] = sum_{s<r} P[s][d]    where r's rows start in d's buffer (push)
//   src_offset[s]  = sum_{d<r} P[s][d]    where the rows for r start in s's buffer (pull)
//   recv_count[s]  = P[s][r]
//   recv_offset[s] = sum_{s'<s} P[s'][r]  where s's rows land in r's buffer ([W] = total)
// and, given every rank's expert counts X[s][e] (no dedup: a source's rows for
// r are its expert rows of partition r, in expert-id order),
//   recv_expert_count[e]    = sum_s X[s][e] for the experts on r, else 0
//   recv_block_offset[s][e] = recv_offset[s] + sum of X[s][f] over the experts
//                             f < e on r (the (source, expert) blocks a grouped
//                             GEMM over r's receive buffer consumes), else -1.
// Sums are 64-bit; an entry past INT32_MAX is written as -1.  Negative counts,
// such entries and a source whose expert counts on r do not add up to
// P[s][r] set MOE_STATUS_BAD_COUNT in the status word.
//
// One block of 1024 threads: the per-partition sums by thread, the expert
// blocks by one warp per source (an exclusive scan over the experts in 64
// bits).  The whole matrix is a few KB, so the kernel is bound by launch
// latency; it reads nothing another rank writes while it runs.
#include <climits>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kPThreads = 1024;
constexpr int kPWarps = kPThreads / kWarp;

struct PlanArgs {
  int W, r, G;
  const int* __restrict__ P;  // [W][W]
  const int* __restrict__ X;  // [W][G] or nullptr
  const int* __restrict__ part_of;
  moe_ep_plan_t out;
};

__device__ __forceinline__ int fit(long long v, int& bad) {
  if (v < 0 || v > INT_MAX) {
    bad |= MOE_STATUS_BAD_COUNT;
    return -1;
  }
  return (int)v;
}

__global__ void __launch_bounds__(kPThreads) ep_plan_kernel(PlanArgs a) {
  __shared__ long long recv_off[MOE_MAX_E_PART + 1];
  __shared__ int status;
  const int W = a.W, r = a.r, tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (tid == 0) status = 0;
  int bad = 0;
  for (int i = tid; i < W * W; i += kPThreads) bad |= a.P[i] < 0 ? MOE_STATUS_BAD_COUNT : 0;
  if (tid < W) {
    const int d = tid, s = tid;
    long long snd = 0, src = 0;
    for (int q = 0; q < r; ++q) {
      snd += a.P[q * W + d];
      src += a.P[s * W + q];
    }
    a.out.send_offset[d] = fit(snd, bad);
    a.out.src_offset[s] = fit(src, bad);
    a.out.recv_count[s] = a.P[s * W + r];
  }
  if (tid <= W) {
    long long off = 0;
    for (int q = 0; q < tid; ++q) off += a.P[q * W + r];
    recv_off[tid] = off;
    a.out.recv_offset[tid] = fit(off, bad);
  }
  __syncthreads();
  if (a.X) {
    const int G = a.G;
    for (int e = tid; e < G; e += kPThreads) {
      long long c = 0;
      if (a.part_of[e] == r)
        for (int s = 0; s < W; ++s) c += a.X[s * G + e];
      a.out.recv_expert_count[e] = fit(c, bad);
    }
    // one warp per source: exclusive scan over the experts on r, in id order
    const int lane = lane_id();
    for (int s = warp_id(); s < W; s += kPWarps) {
      const int* xs = a.X + (size_t)s * G;
      int* blk = a.out.recv_block_offset + (size_t)s * G;
      long long base = recv_off[s];
      for (int e0 = 0; e0 < G; e0 += kWarp) {
        const int e = e0 + lane;
        const bool on_r = e < G && a.part_of[e] == r;
        const int c = e < G ? xs[e] : 0;
        if (c < 0) bad |= MOE_STATUS_BAD_COUNT;
        const long long v = on_r ? c : 0;
        long long inc = v;
#pragma unroll
        for (int o = 1; o < kWarp; o <<= 1) {
          const long long y = __shfl_up_sync(kFull, inc, o);
          if (lane >= o) inc += y;
        }
        if (e < G) blk[e] = on_r ? fit(base + inc - v, bad) : -1;
        base += __shfl_sync(kFull, inc, kWarp - 1);
      }
      // the source's expert counts on r must add up to its partition count
      if (lane == 0 && base - recv_off[s] != a.P[s * W + r]) bad |= MOE_STATUS_BAD_COUNT;
    }
  }
  if (bad) atomicOr(&status, bad);
  __syncthreads();
  if (tid == 0) *a.out.status = status;
}

}  // namespace

cudaError_t launch_ep_plan(int world, int rank, int G, const int32_t* part_counts,
                           const int32_t* expert_counts, const int32_t* part_of,
                           const moe_ep_plan_t& plan, cudaStream_t stream) {
  PlanArgs a;
  a.W = world;
  a.r = rank;
  a.G = G;
  a.P = part_counts;
  a.X = expert_counts;
  a.part_of = part_of;
  a.out = plan;
  cudaError_t e = launch_pdl(ep_plan_kernel, dim3(1), dim3(kPThreads), 0, stream, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
