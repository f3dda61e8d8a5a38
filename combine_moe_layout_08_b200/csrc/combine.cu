// Combine: out[t, :] = bf16( sum_k w[t,k] * y[exp_row[t,k], :] ).
//
// Deterministic by construction, as in the SCORE reduction of Purlin
// (section 3.3, "The Atom"): exclusive ownership -- one thread owns 8
// consecutive output columns of one token -- and ordered accumulation -- the
// fp32 fused multiply-adds run in slot order k = 0..topk-1 from +0.  The
// gathers of all slots are issued before the first accumulation (up to kKG
// 16-byte loads in flight per thread), so the ordering costs no memory
// parallelism; one rounding to bf16 at the end.
#include <algorithm>

#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kCThreads = 128;
constexpr int kKG = 8;  // slots gathered per batch

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

__global__ void __launch_bounds__(kCThreads) combine_kernel(CombineArgs a) {
  __shared__ int rows[MOE_MAX_TOPK];
  __shared__ float wts[MOE_MAX_TOPK];
  const int t = blockIdx.x;
  const int tid = threadIdx.x;
  if (tid < a.topk) {
    const int r = ld_nc_i32(a.exp_row + (size_t)t * a.topk + tid);
    const bool ok = r >= 0 && r < a.cap;
    if (r < -1 || r >= a.cap) raise_status(a.status, MOE_STATUS_BAD_ROW);
    rows[tid] = ok ? r : -1;
    wts[tid] = __ldg(a.w + (size_t)t * a.topk + tid);
  }
  __syncthreads();
  const int c = blockIdx.y * kCThreads + tid;
  if (c >= a.N8) return;

  float acc[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) acc[j] = 0.0f;
  for (int k0 = 0; k0 < a.topk; k0 += kKG) {
    uint4 v[kKG];
#pragma unroll
    for (int j = 0; j < kKG; ++j) {
      const int k = k0 + j;
      if (k < a.topk && rows[k] >= 0) v[j] = ld_nc_v4(a.y + (size_t)rows[k] * a.N8 + c);
    }
#pragma unroll
    for (int j = 0; j < kKG; ++j) {
      const int k = k0 + j;
      if (k < a.topk && rows[k] >= 0) fma8(acc, wts[k], v[j]);
    }
  }
  uint4 o;
  o.x = pack_bf16x2_rn(acc[0], acc[1]);
  o.y = pack_bf16x2_rn(acc[2], acc[3]);
  o.z = pack_bf16x2_rn(acc[4], acc[5]);
  o.w = pack_bf16x2_rn(acc[6], acc[7]);
  st_v4(a.out + (size_t)t * a.N8 + c, o);
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
  dim3 grid(p.M, (a.N8 + kCThreads - 1) / kCThreads);
  combine_kernel<<<grid, kCThreads, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace moe
