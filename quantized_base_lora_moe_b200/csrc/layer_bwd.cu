// Backward of the TQP MoE layer (adapters only; base and router frozen).
#include <cstdint>
#include <cuda_runtime.h>

#include "tqp_device.cuh"
#include "tqp_launch.h"

namespace tqp {

__global__ void add_f32_kernel(const float* __restrict__ a, const float* __restrict__ b, float* __restrict__ out,
                               size_t n) {
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i < n) out[i] = a[i] + b[i];
}

int launch_add_f32(const float* a, const float* b, float* out, size_t n, cudaStream_t s) {
  if (n == 0) return TQP_OK;
  add_f32_kernel<<<unsigned((n + 255) / 256), 256, 0, s>>>(a, b, out, n);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

size_t layer_bwd_ws_bytes(int T, const tqp_moe_weights* w) { (void)T; (void)w; return 256; }

int launch_layer_bwd(const uint16_t*, const float*, int, const tqp_moe_weights*, float*, const tqp_adapter_grads*,
                     void*, int32_t*, cudaStream_t) {
  return TQP_ERR_UNSUPPORTED;
}

}  // namespace tqp
