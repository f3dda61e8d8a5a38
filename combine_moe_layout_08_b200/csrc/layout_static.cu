// moe_layout_static: the routing layout without a caller-supplied workspace.
//
// Some callers cannot allocate device memory at the point where they route
// tokens: code running inside a CUDA-graph capture that must not call
// cudaMalloc, inference runtimes whose memory planner owns every byte and
// hands out no scratch, or plain C hosts without an allocator of their own.
// For them the layout's per-tile histograms live in a fixed device array
// compiled into this library.  Every GPU that loads the library holds the
// array (kMoeStaticScratchBytes) until the process exits.
//
// The array's name in host code is only a host-side stand-in, not a device
// address, so the device address is looked up with cudaGetSymbolAddress, with
// the device current, and then passed to the kernels like any other
// workspace.  The address belongs to the module loaded in one CUDA context:
// it is looked up on the first call in each context (the process's first
// call on a device, and the first call after that device's context was
// destroyed and re-created, e.g. by cudaDeviceReset) and remembered under the
// context's id, which is never reused within a process, so a stale address is
// never handed to a kernel.  Such a first call should come before any stream
// capture.
//
// All calls share the one array and it keeps the last call's contents.  The
// layout kernels need nothing in it to start at zero (the count kernel writes
// every histogram entry and flag the rank kernel reads), so nothing is
// cleared.  Calls whose execution overlaps on the GPU -- on different
// streams, or from different threads -- race on the array; serialise them.
#include <cuda_runtime.h>

#include <mutex>
#include <unordered_map>

#include "moe_internal.h"
#include "moe_layout.h"

namespace {

constexpr size_t kMoeStaticScratchBytes = MOE_STATIC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_layout_scratch[kMoeStaticScratchBytes];

std::mutex g_setup_mutex;
std::unordered_map<unsigned long long, void*> g_scratch_addr;  // context id -> address

// Device address of g_layout_scratch in the current context.
cudaError_t scratch_address(void** out) {
  unsigned long long ctx = 0;
  cudaError_t e = moe::current_context_id(&ctx);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_setup_mutex);
  auto it = g_scratch_addr.find(ctx);
  if (it == g_scratch_addr.end()) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_layout_scratch);
    if (e != cudaSuccess) return e;
    it = g_scratch_addr.emplace(ctx, p).first;
  }
  *out = it->second;
  return cudaSuccess;
}

}  // namespace

extern "C" int moe_layout_static(const moe_problem_t* prob, const int32_t* topk_idx,
                                 const int32_t* part_of, const moe_layout_t* lay,
                                 moe_stream_t stream) {
  const size_t need = moe_layout_workspace_size(prob);
  if (need == 0) return MOE_ERR_ARG;
  if (need > kMoeStaticScratchBytes) return MOE_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (scratch_address(&scratch) != cudaSuccess) return MOE_ERR_CUDA;
  return moe_layout(prob, topk_idx, part_of, lay, scratch, kMoeStaticScratchBytes, stream);
}
