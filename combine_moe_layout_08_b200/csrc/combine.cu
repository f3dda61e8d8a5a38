// Combine: out[t, :] = bf16( sum_k w[t,k] * y[exp_row[t,k], :] ).
//
// Deterministic by construction, as in the SCORE reduction of Purlin
// (section 3.3, "The Atom"): exclusive ownership -- one thread owns 8
// consecutive output columns of one token per vector -- and ordered
// accumulation -- the fp32 fused multiply-adds run in slot order
// k = 0..topk-1 from +0, one rounding to bf16 at the end.
//
// One block of 128 threads per (token, column slice).  The token's slot rows
// and gates are read once into shared memory.  A thread owns U 16-byte
// vectors and gathers KG slots of all of them before accumulating them in
// order (KG * U = 4 to 8 loads in flight per thread: few slots -> more
// columns per thread), so the fixed order costs no memory parallelism.
#include <algorithm>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kCThreads = 128;
// Compile-time tuning constant: topk 5..8 batches of at most this many routed
// pairs gather all their slots in one round (0: never).
#ifndef MOE_COMBINE_ONE_ROUND_ITEMS
#define MOE_COMBINE_ONE_ROUND_ITEMS 1024  // measured on B200: decode batches up to M = 128 at topk 8
#endif

struct CombineArgs {
  const uint4* __restrict__ y;  // [cap][N8]
  const float* __restrict__ w;  // [M][topk]
  const int* exp_row;           // [M][topk]
  uint4* out;                   // [M][N8]
  int N8, topk, cap;
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

template <int KG, int U>
__global__ void __launch_bounds__(kCThreads) combine_kernel(CombineArgs a) {
  __shared__ int rows[MOE_MAX_TOPK];
  __shared__ float wts[MOE_MAX_TOPK];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  // The gates are the router's output, not the previous kernel's: warm L2
  // with the token's row while that kernel may still run (a prefetch is
  // safe before the wait, see prefetch_line_l2).
  if (tid == 0) {
    const float* g = a.w + (size_t)t * a.topk;
    prefetch_line_l2(g);
    prefetch_line_l2(g + a.topk - 1);
  }
  pdl_wait();
  pdl_trigger();
  if (tid < a.topk) {
    const int r = ld_nc_i32(a.exp_row + (size_t)t * a.topk + tid);
    const bool ok = r >= 0 && r < a.cap;
    if (r < -1 || r >= a.cap) raise_status(a.status, MOE_STATUS_BAD_ROW);
    rows[tid] = ok ? r : -1;
    wts[tid] = __ldg(a.w + (size_t)t * a.topk + tid);
  }
  __syncthreads();
  const int c0 = blockIdx.y * (kCThreads * U) + tid;

  float acc[U][8];
#pragma unroll
  for (int u = 0; u < U; ++u)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[u][j] = 0.0f;
  for (int k0 = 0; k0 < a.topk; k0 += KG) {
    uint4 v[U][KG];
#pragma unroll
    for (int j = 0; j < KG; ++j) {
      const int k = k0 + j;
      if (k >= a.topk || rows[k] < 0) continue;
      const uint4* src = a.y + (size_t)rows[k] * a.N8;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * kCThreads;
        if (c < a.N8) v[u][j] = ld_nc_v4(src + c);
      }
    }
#pragma unroll
    for (int j = 0; j < KG; ++j) {
      const int k = k0 + j;
      if (k >= a.topk || rows[k] < 0) continue;
#pragma unroll
      for (int u = 0; u < U; ++u) {
        const int c = c0 + u * kCThreads;
        if (c < a.N8) fma8(acc[u], wts[k], v[u][j]);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = c0 + u * kCThreads;
    if (c < a.N8) {
      uint4 o;
      o.x = pack_bf16x2_rn(acc[u][0], acc[u][1]);
      o.y = pack_bf16x2_rn(acc[u][2], acc[u][3]);
      o.z = pack_bf16x2_rn(acc[u][4], acc[u][5]);
      o.w = pack_bf16x2_rn(acc[u][6], acc[u][7]);
      st_v4(a.out + (size_t)t * a.N8 + c, o);
    }
  }
}

template <int KG, int U>
cudaError_t launch(const CombineArgs& a, int M, cudaStream_t stream) {
  const dim3 grid(M, (a.N8 + kCThreads * U - 1) / (kCThreads * U));
  const cudaError_t e = launch_pdl(combine_kernel<KG, U>, grid, dim3(kCThreads), 0, stream, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const moe_problem_t& p, const void* y, const float* w,
                           const moe_layout_t& lay, void* out, cudaStream_t stream) {
  if (p.M == 0) return cudaSuccess;
  CombineArgs a;
  a.y = static_cast<const uint4*>(y);
  a.w = w;
  a.exp_row = lay.exp_row;
  a.out = static_cast<uint4*>(out);
  a.N8 = p.N / 8;
  a.topk = p.topk;
  a.cap = p.M * p.topk;
  a.status = lay.status;
  // KG slots gathered per batch x U vectors per thread.  Measured on B200
  // (combine us at topk 8, M4096 / M8192 / M65536): KG = 4 beats 8, 2 and 1
  // (90.2 / 170.3 / 1290 against 90.6 / 172.5 / 1307 for 8, 91.3 / 174.0 /
  // 1316 for 2); at topk 2, U = 4 beats 2 and 1.
  // Small batches are bound by latency, not bandwidth: all slots (up to 8)
  // in one round trip to memory instead of two.
  if (p.topk >= 5 && p.topk <= 8 && (int64_t)p.M * p.topk <= MOE_COMBINE_ONE_ROUND_ITEMS)
    return launch<8, 1>(a, p.M, stream);
  if (p.topk >= 5) return launch<4, 1>(a, p.M, stream);
  if (p.topk >= 3) return launch<4, 2>(a, p.M, stream);
  if (p.topk == 2) return launch<2, 4>(a, p.M, stream);
  return launch<1, 8>(a, p.M, stream);
}

}  // namespace moe
