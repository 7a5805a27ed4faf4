// Allocation-free routing entry point.
//
// Some callers cannot allocate device memory at the point where they need the
// routing decision: code that runs while another component owns the CUDA
// allocator (a serving loop with a fixed, pre-carved memory pool), hooks that
// are not allowed to call back into an allocator, or runtimes that only hand
// out raw stream and buffer pointers.  moe_route_noalloc serves them: it
// computes the same top-k ids and gates as moe_debug_routing, with the same
// kernels, but keeps its intermediate arrays (router logits, per-copy ranks,
// per-group counts) in a fixed scratch array that lives in the library's own
// device memory instead of a caller-provided workspace.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "../../include/moe_b200.h"
#include "kernels.h"

namespace {

constexpr size_t kScratchBytes = MOE_ROUTE_NOALLOC_SCRATCH_BYTES;

// Every device that loads the library holds this array until the process exits.
static __device__ __align__(256) unsigned char g_route_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mutex;

size_t round_up(size_t v) { return (v + 255) & ~size_t(255); }

// Device address of the scratch array on the current device.  The host-side
// name g_route_scratch is only a stand-in for the symbol, so the address is
// looked up once per device (with that device current) and cached for the
// life of the process; a reset of the device (cudaDeviceReset) unloads the
// module that holds the array and leaves the cached address stale.
int scratch_on_current_device(unsigned char** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MOE_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_route_scratch) != cudaSuccess || p == nullptr) return MOE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_scratch_addr[dev]);
  return MOE_OK;
}

bool aligned(const void* p, uintptr_t a) { return p != nullptr && (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// True when p is device (or managed) memory that the device `dev` owns.  The kernels run on the
// current device, so a buffer of another device would be read through a foreign address.
// cudaPointerGetAttributes allocates nothing.
bool on_device(const void* p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();                // clear the (non-sticky) error so later calls do not see it
    return false;
  }
  return (a.type == cudaMemoryTypeDevice || a.type == cudaMemoryTypeManaged) && a.device == dev;
}

}  // namespace

extern "C" int moe_route_noalloc(int T, int H, int E, int k, const void* x_bf16, const float* W_router,
                                 const float* bias, int32_t* topk_ids, float* gates, void* stream) {
  if (T < 1 || H < 128 || H % 128 || E < 1 || E > 1024 || k < 1 || k > 16 || k > E) return MOE_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x_bf16, 16) || !aligned(W_router, 16) || !aligned(bias, 4) || !aligned(topk_ids, 4) ||
      !aligned(gates, 4))
    return MOE_ERR_INVALID_ARG;
  const size_t G = ((size_t)T + 31) / 32;
  const size_t logits_bytes = round_up((size_t)T * E * 4);
  const size_t rank_bytes = round_up((size_t)T * k * 4);
  const size_t counts_bytes = round_up(G * E * 4);
  const size_t status_bytes = 256;
  if (logits_bytes + rank_bytes + counts_bytes + status_bytes > kScratchBytes) return MOE_ERR_WORKSPACE;

  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return MOE_ERR_CUDA;
  if (!on_device(x_bf16, dev) || !on_device(W_router, dev) || !on_device(bias, dev) || !on_device(topk_ids, dev) ||
      !on_device(gates, dev))
    return MOE_ERR_INVALID_ARG;
  unsigned char* scratch = nullptr;
  int rc = scratch_on_current_device(&scratch);
  if (rc != MOE_OK) return rc;
  float* logits = reinterpret_cast<float*>(scratch);
  int32_t* local_rank = reinterpret_cast<int32_t*>(scratch + logits_bytes);
  int32_t* group_counts = reinterpret_cast<int32_t*>(scratch + logits_bytes + rank_bytes);
  uint32_t* status = reinterpret_cast<uint32_t*>(scratch + logits_bytes + rank_bytes + counts_bytes);
  // Everything the kernels read from the scratch is written earlier in the same
  // call (logits, ranks and group counts are overwritten in full), so nothing
  // has to be cleared; the status words are only written by the id-validating
  // mode, which this entry point does not use.
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (moe::launch_router_logits(static_cast<const uint16_t*>(x_bf16), W_router, logits, T, H, E, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (moe::launch_topk_rank(0, logits, 1, bias, topk_ids, gates, local_rank, group_counts, status, T, E, k, s) !=
      cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}
