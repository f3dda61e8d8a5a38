// Dispatch permute: every token row is read from HBM once and written to each
// dispatch row that holds it -- topk rows without dedup, one row per
// partition with dedup.  The all_to_all_kernel of the Triton-distributed
// issue #117 moves data_src rows into data_dst with optional per-row scales
// (WITH_SCALE); here the destinations are partitions of one receive buffer
// in this GPU's HBM.
//
// One block of 128 threads per (token, column slice): a fan-out dispatch (no
// dedup, topk >= 4) cuts each row into slices of one 16-byte vector per
// thread; otherwise a block takes the whole row (up to 8 vectors per thread).
//
// bf16: 16-byte vector loads (non-coherent, no L1 allocation) of the block's
// row slice into registers, then 16-byte stores to each destination.
//
// fp8: the same read, then per 128-column block amax (8 lanes, 16 columns
// each, reduced with shuffles), scale = amax / 448 (IEEE division), each
// value divided by the scale (IEEE division) and cast to e4m3 with the
// saturating round-to-nearest-even conversion; the 16 bytes of a lane are
// stored to every destination and one lane of the 8 writes the block's
// scale.  The quantisation is done once per token, not once per copy.
#include <algorithm>

#include "fp8_device.cuh"
#include "moe_device.cuh"
#include "moe_internal.h"

namespace moe {
namespace {

constexpr int kDThreads = 128;
constexpr int kMaxDest = MOE_MAX_E_PART > MOE_MAX_TOPK ? MOE_MAX_E_PART : MOE_MAX_TOPK;

struct DispatchArgs {
  const uint4* __restrict__ x;  // [M][N8]
  int N8;                       // 16-byte chunks per bf16 row (N / 8)
  int topk, E, dedup;
  int cap;                      // receive capacity in rows (M * topk)
  int M;
  int prefetch_stride;          // blocks [0, stride) warm L2 with rows b, b + stride, ...
  int prefetch_rows;            // ... below this row (the first rows processed)
  const int* exp_row;           // [M][topk]
  const int* disp_row;          // [M][E], dedup only
  void* recv;                   // [cap][N] bf16 or u8
  float* recv_scale;            // [cap][N / 128], fp8 only
  int* status;
};

// While the previous kernel (the routing layout) still runs, the blocks that
// are already resident warm L2 with the first token rows: block b < stride
// prefetches rows b, b + stride, ... (stride = resident blocks) up to
// kPrefetchBytes in all -- a third of L2, so the prefetched rows are still
// there when their blocks run -- and those rows come from L2 once the
// destinations are known.
#ifndef MOE_DISPATCH_PREFETCH
#define MOE_DISPATCH_PREFETCH 1
#endif
constexpr size_t kPrefetchBytes = 40u << 20;

__device__ __forceinline__ void prefetch_rows(const DispatchArgs& a) {
  if (!MOE_DISPATCH_PREFETCH) return;
  if (threadIdx.x != 0 || blockIdx.y != 0 || (int)blockIdx.x >= a.prefetch_stride) return;
  const uint32_t row_bytes = (uint32_t)a.N8 * 16u;
  for (int t = blockIdx.x; t < a.prefetch_rows; t += a.prefetch_stride)
    prefetch_l2(a.x + (size_t)t * a.N8, row_bytes);
}

// Destination rows of token t, in slot (or partition) order, into smem.
__device__ __forceinline__ int destinations(const DispatchArgs& a, int t, int* dst, int* nd) {
  if (warp_id() == 0) {
    const int lane = lane_id();
    const int n_ent = a.dedup ? a.E : a.topk;
    const int* ent = a.dedup ? a.disp_row + (size_t)t * a.E : a.exp_row + (size_t)t * a.topk;
    int count = 0;
    bool bad = false;
    for (int base = 0; base < n_ent; base += kWarp) {
      const int i = base + lane;
      const int r = i < n_ent ? ld_nc_i32(ent + i) : -1;
      const bool ok = r >= 0 && r < a.cap;
      bad |= (r < -1) || (r >= a.cap);
      const unsigned bal = __ballot_sync(kFull, ok);
      if (ok) dst[count + __popc(bal & lanemask_lt())] = r;
      count += __popc(bal);
    }
    if (lane == 0) *nd = count;
    if (bad) raise_status(a.status, MOE_STATUS_BAD_ROW);
  }
  __syncthreads();
  return *nd;
}

template <int U>
__global__ void __launch_bounds__(kDThreads, 8) dispatch_bf16_kernel(DispatchArgs a) {
  __shared__ int dst[kMaxDest];
  __shared__ int nd;
  const int t = blockIdx.x;
  const int c0 = blockIdx.y * (kDThreads * U) + threadIdx.x;
  const uint4* src = a.x + (size_t)t * a.N8;
  prefetch_rows(a);
  pdl_wait();
  pdl_trigger();
  uint4 v[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int c = c0 + u * kDThreads;
    if (c < a.N8) v[u] = ld_nc_v4(src + c);
  }
  const int n = destinations(a, t, dst, &nd);
  uint4* recv = static_cast<uint4*>(a.recv);
  for (int d = 0; d < n; ++d) {
    uint4* o = recv + (size_t)dst[d] * a.N8;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * kDThreads;
      if (c < a.N8) st_v4(o + c, v[u]);
    }
  }
}

// Each thread owns a 16-column group g; 8 consecutive lanes form one
// 128-column scale block.  N is a multiple of 128 and kDThreads of 8, so a
// lane group is either entirely inside the row or entirely past its end.
template <int U>
__global__ void __launch_bounds__(kDThreads, 8) dispatch_fp8_kernel(DispatchArgs a) {
  __shared__ int dst[kMaxDest];
  __shared__ int nd;
  const int t = blockIdx.x;
  const int N16 = a.N8 >> 1;
  const int g0 = blockIdx.y * (kDThreads * U) + threadIdx.x;
  const uint4* src = a.x + (size_t)t * a.N8;
  prefetch_rows(a);
  pdl_wait();
  pdl_trigger();
  uint4 lo[U], hi[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    const int g = g0 + u * kDThreads;
    if (g < N16) {
      lo[u] = ld_nc_v4(src + 2 * g);
      hi[u] = ld_nc_v4(src + 2 * g + 1);
    } else {
      lo[u] = make_uint4(0, 0, 0, 0);
      hi[u] = lo[u];
    }
  }
  const int n = destinations(a, t, dst, &nd);
  uint4 q[U];
  float s[U];
#pragma unroll
  for (int u = 0; u < U; ++u) q[u] = quantize_lane(lo[u], hi[u], s[u]);
  uint4* recv = static_cast<uint4*>(a.recv);  // a row is N bytes = N16 chunks
  const int N128 = N16 >> 3;
  const bool scale_lane = (threadIdx.x & 7) == 0;
  for (int d = 0; d < n; ++d) {
    const size_t r = (size_t)dst[d];
    uint4* o = recv + r * N16;
    float* os = a.recv_scale + r * N128;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int g = g0 + u * kDThreads;
      if (g < N16) {
        st_v4(o + g, q[u]);
        if (scale_lane) os[g >> 3] = s[u];
      }
    }
  }
}

}  // namespace

cudaError_t launch_dispatch(const moe_problem_t& p, const void* x, const moe_layout_t& lay,
                            void* recv_x, float* recv_scale, cudaStream_t stream) {
  if (p.M == 0) return cudaSuccess;
  DispatchArgs a;
  a.x = static_cast<const uint4*>(x);
  a.N8 = p.N / 8;
  a.topk = p.topk;
  a.E = p.E_part;
  a.dedup = p.dedup;
  a.cap = p.M * p.topk;
  a.M = p.M;
  a.exp_row = lay.exp_row;
  a.disp_row = lay.disp_row;
  a.recv = recv_x;
  a.recv_scale = recv_scale;
  a.status = lay.status;

  // Fan-out dispatch: every row read is written to topk >= 4 rows (no dedup).
  const bool fan_out = !p.dedup && p.topk >= 4;
  // U vectors per thread, the row cut into slices of U * 128 units.
  // Measured on B200: with fan-out one vector per thread in more, narrower
  // blocks is fastest (M4096 topk 8: 79.9 us vs 85.0 for the whole row per
  // block; the long per-thread store sequences queue up otherwise); with
  // dedup (fewer copies per row read) the whole row per block is (hot-pairs
  // topk 2: 51.3 us vs 73.7 at U = 1).
  const int units = p.fp8 ? a.N8 / 2 : a.N8;
  const int Umax = fan_out ? 1 : (p.fp8 ? 4 : 8);
  const int U = std::min(Umax, (units + kDThreads - 1) / kDThreads);
  const int per_block = kDThreads * U;
  dim3 grid(p.M, (units + per_block - 1) / per_block);
  // blocks resident at once on this device (an estimate from the register
  // budget of the widest variant; only the L2 prefetch uses it)
  a.prefetch_stride = std::max(1, std::min(p.M, device_block_slots(
      reinterpret_cast<const void*>(dispatch_bf16_kernel<8>), kDThreads) / (int)grid.y));
  // measured on B200: the prefetch pays when every row fans out to many
  // copies (HBM busy writing); with dedup or small topk it only adds L2
  // pressure
  a.prefetch_rows = fan_out ? (int)std::min<size_t>((size_t)p.M, kPrefetchBytes / (2 * (size_t)p.N)) : 0;
  cudaError_t e = cudaSuccess;
  if (!p.fp8) {
    switch (U) {
      case 1: e = launch_pdl(dispatch_bf16_kernel<1>, grid, dim3(kDThreads), 0, stream, a); break;
      case 2: e = launch_pdl(dispatch_bf16_kernel<2>, grid, dim3(kDThreads), 0, stream, a); break;
      case 3: e = launch_pdl(dispatch_bf16_kernel<3>, grid, dim3(kDThreads), 0, stream, a); break;
      case 4: e = launch_pdl(dispatch_bf16_kernel<4>, grid, dim3(kDThreads), 0, stream, a); break;
      case 5: e = launch_pdl(dispatch_bf16_kernel<5>, grid, dim3(kDThreads), 0, stream, a); break;
      case 6: e = launch_pdl(dispatch_bf16_kernel<6>, grid, dim3(kDThreads), 0, stream, a); break;
      case 7: e = launch_pdl(dispatch_bf16_kernel<7>, grid, dim3(kDThreads), 0, stream, a); break;
      default: e = launch_pdl(dispatch_bf16_kernel<8>, grid, dim3(kDThreads), 0, stream, a); break;
    }
  } else {
    switch (U) {
      case 1: e = launch_pdl(dispatch_fp8_kernel<1>, grid, dim3(kDThreads), 0, stream, a); break;
      case 2: e = launch_pdl(dispatch_fp8_kernel<2>, grid, dim3(kDThreads), 0, stream, a); break;
      case 3: e = launch_pdl(dispatch_fp8_kernel<3>, grid, dim3(kDThreads), 0, stream, a); break;
      default: e = launch_pdl(dispatch_fp8_kernel<4>, grid, dim3(kDThreads), 0, stream, a); break;
    }
  }
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace moe
