// Device-side helpers shared by the layout, dispatch and combine kernels.
// sm_100a only: plain 16-byte vector memory operations with explicit cache
// hints, warp-synchronous primitives and status bits.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "moe_layout.h"

namespace moe {

constexpr int kWarp = 32;
constexpr unsigned kFull = 0xffffffffu;

// ---------------------------------------------------------------------------
// 16-byte global memory operations
// ---------------------------------------------------------------------------

// Read-only, streaming: the line is not kept in L1 (each token row is read
// once per kernel).
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
      : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
      : "l"(p));
  return v;
}

// Store that does not allocate in L1.
__device__ __forceinline__ void st_v4(void* p, const uint4& v) {
  asm volatile("st.global.L1::no_allocate.v4.u32 [%0], {%1, %2, %3, %4};"
               :
               : "l"(p), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// Bulk prefetch of [p, p + bytes) into L2 (no registers, no shared memory;
// 16-byte aligned, bytes a multiple of 16).  Always safe to issue early: L2
// is the GPU's point of coherence, so a line prefetched before its last
// writer finishes is simply updated in place.
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Prefetch the line holding p into L2 (a hint: it loads nothing into the SM,
// and L2 is the point of coherence, so it may be issued before the data's
// last writer has finished).
__device__ __forceinline__ void prefetch_line_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

__device__ __forceinline__ int ld_nc_i32(const int* p) {
  int v;
  asm("ld.global.nc.L1::no_allocate.b32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}

// ---------------------------------------------------------------------------
// warp helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned lanemask_lt() {
  unsigned m;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
  return m;
}

__device__ __forceinline__ int lane_id() { return threadIdx.x & (kWarp - 1); }

// Lanes of the warp holding the same key as this lane (all lanes active).
// Keys are in [-1, 2^nbits - 1): -1 (all ones in the low nbits bits) is a key
// of its own.  One ballot per key bit, intersected: on sm_100a this runs at
// the vote rate on every sub-partition, several times the throughput of
// match.any.
__device__ __forceinline__ unsigned match_peers(int key, int nbits) {
  unsigned m = kFull;
  for (int b = 0; b < nbits; ++b) {
    const bool bit = (key >> b) & 1;
    const unsigned bal = __ballot_sync(kFull, bit);
    m &= bit ? bal : ~bal;
  }
  return m;
}

// Key bits for keys in [-1, K): enough that K - 1 < 2^nbits - 1.
__device__ __forceinline__ int key_bits(int K) { return 32 - __clz(K); }
__device__ __forceinline__ int warp_id() { return threadIdx.x >> 5; }

// ---------------------------------------------------------------------------
// bf16 <-> fp32 (bf16 = upper half of binary32)
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// two fp32 -> packed bf16x2, each rounded to nearest-even; `lo` in bits 0..15
__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// ---------------------------------------------------------------------------
// programmatic dependent launch (sm_90+).  A kernel launched with the
// programmatic-serialisation attribute may start while the previous kernel
// in the stream is still running; pdl_wait() blocks (in hardware) until that
// kernel has completed and its memory is visible, and pdl_trigger() lets the
// next such kernel start once every block of this one has passed it.  In a
// kernel launched without the attribute both are no-ops.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// status word
// ---------------------------------------------------------------------------
__device__ __forceinline__ void raise_status(int* status, int bits) {
  if (bits && status) atomicOr(status, bits);
}

}  // namespace moe
