// FP8 e4m3 quantisation of bf16 rows with one fp32 scale per 128 columns,
// shared by the dispatch kernels.  A lane owns 16 consecutive columns (two
// 16-byte chunks); 8 consecutive lanes form one 128-column scale block.
//   scale = amax / 448 (IEEE division), q = e4m3_rne_satfinite(x / scale)
//   (IEEE division); an all-zero block gives scale 0 and bytes 0.
#pragma once

#include <cuda_fp8.h>

#include "moe_device.cuh"

namespace moe {

// 16 bf16 values (two 16-byte chunks) -> 16 e4m3 bytes, given the block scale
__device__ __forceinline__ uint4 quantize16(const uint4& lo, const uint4& hi, float scale) {
  const uint32_t w[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t q[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f0 = make_float2(__fdiv_rn(bf16_lo(w[2 * i]), scale), __fdiv_rn(bf16_hi(w[2 * i]), scale));
    const float2 f1 =
        make_float2(__fdiv_rn(bf16_lo(w[2 * i + 1]), scale), __fdiv_rn(bf16_hi(w[2 * i + 1]), scale));
    const uint32_t b0 = __nv_cvt_float2_to_fp8x2(f0, __NV_SATFINITE, __NV_E4M3);
    const uint32_t b1 = __nv_cvt_float2_to_fp8x2(f1, __NV_SATFINITE, __NV_E4M3);
    q[i] = (b0 & 0xffffu) | (b1 << 16);
  }
  return make_uint4(q[0], q[1], q[2], q[3]);
}

__device__ __forceinline__ float absmax8(const uint4& v) {
  float m = fabsf(bf16_lo(v.x));
  m = fmaxf(m, fabsf(bf16_hi(v.x)));
  m = fmaxf(m, fabsf(bf16_lo(v.y)));
  m = fmaxf(m, fabsf(bf16_hi(v.y)));
  m = fmaxf(m, fabsf(bf16_lo(v.z)));
  m = fmaxf(m, fabsf(bf16_hi(v.z)));
  m = fmaxf(m, fabsf(bf16_lo(v.w)));
  m = fmaxf(m, fabsf(bf16_hi(v.w)));
  return m;
}

// The lane's 16 columns -> 16 bytes and the block scale s.  Every lane of
// the 8-lane group must call it (the amax is reduced with shuffles); lanes
// past the row end pass zeros.
__device__ __forceinline__ uint4 quantize_lane(const uint4& lo, const uint4& hi, float& s) {
  float m = fmaxf(absmax8(lo), absmax8(hi));
  m = fmaxf(m, __shfl_xor_sync(kFull, m, 1));
  m = fmaxf(m, __shfl_xor_sync(kFull, m, 2));
  m = fmaxf(m, __shfl_xor_sync(kFull, m, 4));
  if (m == 0.0f) {
    s = 0.0f;
    return make_uint4(0, 0, 0, 0);
  }
  s = __fdiv_rn(m, 448.0f);
  return quantize16(lo, hi, s);
}

}  // namespace moe
