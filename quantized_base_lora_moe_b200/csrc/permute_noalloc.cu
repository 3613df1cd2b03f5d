// moe_permute_noalloc: the stable token-to-expert permutation for callers that
// cannot allocate device memory.
//
// Some callers may not call cudaMalloc at all: runtimes that hand out device
// memory only through their own pre-partitioned pool and forbid allocations
// from libraries, processes that must not block in the driver's allocator
// while serving requests, and code that has no place to keep a workspace
// between calls. For them this entry point keeps the permutation's scratch in
// a fixed array that is part of this library's device image (every GPU that
// loads the library holds it until the process exits) instead of a
// caller-provided workspace.
//
// Host code cannot use the array's name as a device address: on the host it
// names a stand-in, not the GPU copy. The address of the GPU copy is looked up
// once per device with cudaGetSymbolAddress, with that device current, during
// the first call on the device.
#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/tqp_moe.h"
#include "tqp_launch.h"

namespace {

// Largest supported problem: T <= 16384 tokens and E <= 512 experts need
// ceil(T/32)*E*4 bytes of per-chunk counts plus E*4 bytes of totals.
constexpr int kMaxTokens = 16384;
constexpr int kMaxExperts = 512;
constexpr size_t kScratchBytes = (size_t(1) << 20) + 4096;

static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::atomic<void*> g_scratch_ptr[kMaxDevices];

// Device address of the scratch array on the current device (looked up once).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQP_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return TQP_ERR_UNSUPPORTED;
  void* p = g_scratch_ptr[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return TQP_ERR_CUDA;
    g_scratch_ptr[dev].store(p, std::memory_order_release);
  }
  *out = p;
  return TQP_OK;
}

}  // namespace

extern "C" size_t moe_permute_noalloc_max_bytes(void) { return kScratchBytes; }

extern "C" int moe_permute_noalloc(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* perm_token,
                                   int32_t* inv, int32_t* dev_status, void* stream) {
  if (T < 0 || E < 1 || k < 1 || k > E || !offsets) return TQP_ERR_INVALID_ARG;
  if (T > 0 && (!ids || !perm_token || !inv)) return TQP_ERR_INVALID_ARG;
  if (T > kMaxTokens || E > kMaxExperts || tqp::permute_ws_bytes(T, E) > kScratchBytes) return TQP_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int rc = scratch_address(&scratch);
  if (rc != TQP_OK) return rc;
  // The kernels write every scratch word before reading it, so the previous
  // call's contents need no clearing.
  return tqp::launch_permute(ids, T, E, k, offsets, perm_token, inv, scratch, dev_status,
                             static_cast<cudaStream_t>(stream));
}
