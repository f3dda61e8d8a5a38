// Two-level combine of a deduplicated dispatch: the return path of
// per-partition dedup (Zyphra news item: each token reaches a partition once;
// on the way back the partition first reduces the outputs of the token's
// experts it holds).  Deterministic like the one-level combine (Purlin
// section 3.3, SCORE: one owner per output element, accumulation in source
// order).
//
//   partition side  z[disp_row[t,p], :] = bf16( sum over the token's slots k
//                   held by partition p, in slot order, of w[t,k] *
//                   y[exp_row[t,k], :] )      fp32 fma from +0
//   token side      out[t, :] = bf16( sum over p in partition order of
//                   z[disp_row[t,p], :] )     fp32 additions from +0
//
// Both kernels: one block of 128 threads per (token, column slice), U 16-byte
// vectors (8 columns each) per thread, U chosen from topk so that about eight
// loads are in flight per thread.  A slot's partition is identified by
// the dispatch row it shares with the token's other slots in that partition
// (exp_to_disp of its expert row), so the kernels need only the layout.
#include <algorithm>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kTThreads = 128;
constexpr int kRegSlots = 8;  // slots kept in registers (larger topk: reloaded per group)

struct PartialArgs {
  const uint4* __restrict__ y;  // [cap][N8] expert-row space
  const float* __restrict__ w;  // [M][topk]
  const int* exp_row;           // [M][topk]
  const int* exp_to_disp;       // [cap]
  uint4* z;                     // [cap][N8] dispatch-row space
  int N8, topk, cap;
  int* status;
};

struct ReduceArgs {
  const uint4* __restrict__ z;  // [cap][N8]
  const int* disp_row;          // [M][E]
  uint4* out;                   // [M][N8]
  int N8, E, cap;
  int* status;
};

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

__device__ __forceinline__ void add8(float* acc, const uint4& v) {
  acc[0] = acc[0] + bf16_lo(v.x);
  acc[1] = acc[1] + bf16_hi(v.x);
  acc[2] = acc[2] + bf16_lo(v.y);
  acc[3] = acc[3] + bf16_hi(v.y);
  acc[4] = acc[4] + bf16_lo(v.z);
  acc[5] = acc[5] + bf16_hi(v.z);
  acc[6] = acc[6] + bf16_lo(v.w);
  acc[7] = acc[7] + bf16_hi(v.w);
}

__device__ __forceinline__ uint4 pack8(const float* acc) {
  uint4 o;
  o.x = pack_bf16x2_rn(acc[0], acc[1]);
  o.y = pack_bf16x2_rn(acc[2], acc[3]);
  o.z = pack_bf16x2_rn(acc[4], acc[5]);
  o.w = pack_bf16x2_rn(acc[6], acc[7]);
  return o;
}

// Slot k of the token: expert row rows[k] (-1: left out), gate wts[k], and
// group grp[k] = the dispatch row of its partition (-1: left out); lead[k]
// marks the first slot of each group.  Returns after the shared arrays are
// ready; the caller reads them after the block barrier.
__device__ __forceinline__ void load_slots(const PartialArgs& a, int t, int* rows, int* grp,
                                           float* wts, int* lead) {
  const int tid = threadIdx.x;
  if (tid < a.topk) {
    const int r = ld_nc_i32(a.exp_row + (size_t)t * a.topk + tid);
    bool ok = r >= 0 && r < a.cap;
    int g = -1;
    if (ok) {
      g = ld_nc_i32(a.exp_to_disp + r);
      if (g < 0 || g >= a.cap) {
        raise_status(a.status, MOE_STATUS_BAD_ROW);
        ok = false;
      }
    } else if (r < -1 || r >= a.cap) {
      raise_status(a.status, MOE_STATUS_BAD_ROW);
    }
    rows[tid] = ok ? r : -1;
    grp[tid] = ok ? g : -1;
    wts[tid] = __ldg(a.w + (size_t)t * a.topk + tid);
  }
  __syncthreads();
  if (tid < a.topk) {
    bool first = grp[tid] >= 0;
    for (int j = 0; j < tid && first; ++j) first = grp[j] != grp[tid];
    lead[tid] = first;
  }
  __syncthreads();
}

// S slots held in registers (topk <= S), U column vectors per thread spaced
// kTThreads apart, so that S*U 16-byte loads are in flight per thread.
template <int S, int U>
__global__ void __launch_bounds__(kTThreads) combine_partial_kernel(PartialArgs a) {
  __shared__ int rows[MOE_MAX_TOPK];
  __shared__ int grp[MOE_MAX_TOPK];
  __shared__ float wts[MOE_MAX_TOPK];
  __shared__ int lead[MOE_MAX_TOPK];
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  load_slots(a, t, rows, grp, wts, lead);
  const int c0 = blockIdx.y * (kTThreads * U) + threadIdx.x;
  if (c0 >= a.N8) return;
  uint4 v[S][U];
#pragma unroll
  for (int j = 0; j < S; ++j)
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (j < a.topk && rows[j] >= 0 && c0 + u * kTThreads < a.N8)
        v[j][u] = ld_nc_v4(a.y + (size_t)rows[j] * a.N8 + c0 + u * kTThreads);
#pragma unroll
  for (int k = 0; k < S; ++k) {
    if (k >= a.topk || !lead[k]) continue;
    const int g = grp[k];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (c0 + u * kTThreads >= a.N8) break;
      float acc[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
#pragma unroll
      for (int j = 0; j < S; ++j)
        if (j >= k && j < a.topk && grp[j] == g) fma8(acc, wts[j], v[j][u]);
      st_v4(a.z + (size_t)g * a.N8 + c0 + u * kTThreads, pack8(acc));
    }
  }
}

// topk > 8: each group's slots reloaded from HBM/L2 group by group
__global__ void __launch_bounds__(kTThreads) combine_partial_wide_kernel(PartialArgs a) {
  __shared__ int rows[MOE_MAX_TOPK];
  __shared__ int grp[MOE_MAX_TOPK];
  __shared__ float wts[MOE_MAX_TOPK];
  __shared__ int lead[MOE_MAX_TOPK];
  const int t = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  load_slots(a, t, rows, grp, wts, lead);
  const int c = blockIdx.y * kTThreads + threadIdx.x;
  if (c >= a.N8) return;
  for (int k = 0; k < a.topk; ++k) {
    if (!lead[k]) continue;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j = k; j < a.topk; ++j)
      if (grp[j] == grp[k]) fma8(acc, wts[j], ld_nc_v4(a.y + (size_t)rows[j] * a.N8 + c));
    st_v4(a.z + (size_t)grp[k] * a.N8 + c, pack8(acc));
  }
}

// out[t] = sum of the token's partition rows in partition order; B rows of
// U column vectors gathered per batch (B*U = 8 loads in flight per thread)
template <int U>
__global__ void __launch_bounds__(kTThreads) combine_reduce_kernel(ReduceArgs a) {
  constexpr int B = 8 / U;
  __shared__ int prow[MOE_MAX_E_PART];
  __shared__ int nprow;
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  if (tid < kWarp) {  // compact the token's partition rows, in partition order
    int count = 0;
    bool bad = false;
    for (int base = 0; base < a.E; base += kWarp) {
      const int p = base + tid;
      const int r = p < a.E ? ld_nc_i32(a.disp_row + (size_t)t * a.E + p) : -1;
      const bool ok = r >= 0 && r < a.cap;
      bad |= (r < -1) || (r >= a.cap);
      const unsigned bal = __ballot_sync(kFull, ok);
      if (ok) prow[count + __popc(bal & lanemask_lt())] = r;
      count += __popc(bal);
    }
    if (tid == 0) nprow = count;
    if (bad) raise_status(a.status, MOE_STATUS_BAD_ROW);
  }
  __syncthreads();
  const int c0 = blockIdx.y * (kTThreads * U) + tid;
  if (c0 >= a.N8) return;
  const int n = nprow;
  float acc[U][8];
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[u][i] = 0.0f;
  for (int q0 = 0; q0 < n; q0 += B) {
    uint4 v[B][U];
#pragma unroll
    for (int j = 0; j < B; ++j)
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (q0 + j < n && c0 + u * kTThreads < a.N8)
          v[j][u] = ld_nc_v4(a.z + (size_t)prow[q0 + j] * a.N8 + c0 + u * kTThreads);
#pragma unroll
    for (int j = 0; j < B; ++j)
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (q0 + j < n) add8(acc[u], v[j][u]);
  }
#pragma unroll
  for (int u = 0; u < U; ++u)
    if (c0 + u * kTThreads < a.N8) st_v4(a.out + (size_t)t * a.N8 + c0 + u * kTThreads, pack8(acc[u]));
}

}  // namespace

cudaError_t launch_combine_partial(const moe_problem_t& p, const void* y, const float* w,
                                   const moe_layout_t& lay, void* z, cudaStream_t stream) {
  if (p.M == 0) return cudaSuccess;
  PartialArgs a;
  a.y = static_cast<const uint4*>(y);
  a.w = w;
  a.exp_row = lay.exp_row;
  a.exp_to_disp = lay.exp_to_disp;
  a.z = static_cast<uint4*>(z);
  a.N8 = p.N / 8;
  a.topk = p.topk;
  a.cap = p.M * p.topk;
  a.status = lay.status;
  auto grid = [&](int U) { return dim3(p.M, (a.N8 + kTThreads * U - 1) / (kTThreads * U)); };
  const dim3 blk(kTThreads);
  cudaError_t e;
  if (p.topk == 1)
    e = launch_pdl(combine_partial_kernel<1, 8>, grid(8), blk, 0, stream, a);
  else if (p.topk == 2)
    e = launch_pdl(combine_partial_kernel<2, 4>, grid(4), blk, 0, stream, a);
  else if (p.topk <= 4)
    e = launch_pdl(combine_partial_kernel<4, 2>, grid(2), blk, 0, stream, a);
  else if (p.topk <= 8)
    e = launch_pdl(combine_partial_kernel<8, 1>, grid(1), blk, 0, stream, a);
  else
    e = launch_pdl(combine_partial_wide_kernel, grid(1), blk, 0, stream, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_combine_reduce(const moe_problem_t& p, const void* z, const moe_layout_t& lay,
                                  void* out, cudaStream_t stream) {
  if (p.M == 0) return cudaSuccess;
  ReduceArgs a;
  a.z = static_cast<const uint4*>(z);
  a.disp_row = lay.disp_row;
  a.out = static_cast<uint4*>(out);
  a.N8 = p.N / 8;
  a.E = p.E_part;
  a.cap = p.M * p.topk;
  a.status = lay.status;
  // a token has at most min(topk, E_part) partition rows
  const int rmax = std::min(p.topk, p.E_part);
  auto grid = [&](int U) { return dim3(p.M, (a.N8 + kTThreads * U - 1) / (kTThreads * U)); };
  const dim3 blk(kTThreads);
  cudaError_t e;
  if (rmax <= 2)
    e = launch_pdl(combine_reduce_kernel<4>, grid(4), blk, 0, stream, a);
  else if (rmax <= 4)
    e = launch_pdl(combine_reduce_kernel<2>, grid(2), blk, 0, stream, a);
  else
    e = launch_pdl(combine_reduce_kernel<1>, grid(1), blk, 0, stream, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
