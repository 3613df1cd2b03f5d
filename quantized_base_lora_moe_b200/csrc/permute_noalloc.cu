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
// with cudaGetSymbolAddress, with the device current, on the first call made
// under a given CUDA context, and cached per context: a context created after
// a device reset, or another (non-primary) context, gets a fresh lookup instead
// of a stale address.
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>
#include <mutex>

#include "../../include/tqp_moe.h"
#include "tqp_launch.h"

namespace {

// Largest supported problem: T <= 16384 tokens and E <= 512 experts need
// ceil(T/32)*E*4 bytes of per-chunk counts plus E*4 bytes of totals.
constexpr int kMaxTokens = 16384;
constexpr int kMaxExperts = 512;
constexpr size_t kScratchBytes = (size_t(1) << 20) + 4096;

static __device__ __align__(256) unsigned char g_permute_scratch[kScratchBytes];

// Cached device addresses of the array, one per (device, context) seen. A
// context is identified by its process-unique id (cuCtxGetId), so that a
// context created after a device reset never reuses the address looked up in
// the one it replaced, even if the driver hands out the same handle again.
constexpr int kCacheSlots = 64;
struct Slot {
  int dev;
  unsigned long long ctx_id;
  void* ptr;
};
std::mutex g_mu;
Slot g_slots[kCacheSlots];
int g_nslots = 0;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename F>
F driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(p);
}

// Process-unique id of the current context; false when none is current.
bool current_context_id(unsigned long long* id) {
  static CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return false;
  CUcontext c = nullptr;
  if (get_current(&c) != CUDA_SUCCESS || c == nullptr) return false;
  return get_id(c, id) == CUDA_SUCCESS;
}

// Device address of the scratch array in the current context (looked up with
// cudaGetSymbolAddress on the first call under each context).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return TQP_ERR_CUDA;
  unsigned long long id = 0;
  void* p = nullptr;
  if (!current_context_id(&id)) {
    // no context yet: the lookup makes the runtime create the device's primary one
    if (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr) return TQP_ERR_CUDA;
    if (!current_context_id(&id)) return TQP_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  for (int i = 0; i < g_nslots; ++i)
    if (g_slots[i].dev == dev && g_slots[i].ctx_id == id) {
      *out = g_slots[i].ptr;
      return TQP_OK;
    }
  if (p == nullptr && (cudaGetSymbolAddress(&p, g_permute_scratch) != cudaSuccess || p == nullptr))
    return TQP_ERR_CUDA;
  if (g_nslots == kCacheSlots) g_nslots = 0;   // start over rather than grow
  g_slots[g_nslots++] = Slot{dev, id, p};
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
