// Fused AdamW step over the adapter parameters of the TQP layer (sm_100a).
//
// Only the adapters train and only they carry optimizer state ("Reversible
// Sparse MoE Single Node", Principle 3 and Pattern 3: optimizer state on the
// adapters alone, the quantised base frozen). The pages do not name the
// optimizer; this is AdamW with decoupled weight decay (Loshchilov & Hutter):
//   g  = grad * grad_scale
//   m  = beta1 m + (1 - beta1) g
//   v  = beta2 v + (1 - beta2) g^2
//   p  = p - lr ( (m / (1 - beta1^t)) / (sqrt(v / (1 - beta2^t)) + eps) + weight_decay p )
// and the bf16 copy of p that the layer reads is rewritten in the same pass.
//
// The step is HBM-bound: 16 bytes read and 14 written per parameter (fp32 p,
// m, v, grad in; p, m, v and the bf16 copy out). One thread handles 4
// consecutive parameters with 16-byte loads and stores; a grid of a few
// blocks per SM strides over the buffer; the ragged tail (n % 4) is done
// element by element.
#include <cmath>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/tqp_moe.h"
#include "tqp_device.cuh"
#include "tqp_launch.h"

namespace tqp {
namespace {

struct AdamArgs {
  float lr, beta1, beta2, eps, wd, grad_scale;
  float bc1, bc2;   // 1 / (1 - beta^t), computed on the host in double
};

__device__ __forceinline__ float adam_one(float& p, float& m, float& v, float g, const AdamArgs& a, bool& bad) {
  g *= a.grad_scale;
  bad |= !isfinite(g);
  m = fmaf(a.beta1, m, (1.0f - a.beta1) * g);
  v = fmaf(a.beta2, v, (1.0f - a.beta2) * (g * g));
  const float mh = m * a.bc1;
  const float vh = v * a.bc2;
  p = p - a.lr * (mh / (sqrtf(vh) + a.eps) + a.wd * p);
  return p;
}

__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, float* __restrict__ m,
                                                    float* __restrict__ v, const float* __restrict__ g,
                                                    uint16_t* __restrict__ pb, size_t n, AdamArgs a,
                                                    int32_t* status) {
  bool bad = false;
  const size_t n4 = n / 4;
  const size_t stride = size_t(gridDim.x) * blockDim.x;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += stride) {
    float4 P = reinterpret_cast<float4*>(p)[i];
    float4 M = reinterpret_cast<float4*>(m)[i];
    float4 V = reinterpret_cast<float4*>(v)[i];
    const float4 G = __ldg(reinterpret_cast<const float4*>(g) + i);
    adam_one(P.x, M.x, V.x, G.x, a, bad);
    adam_one(P.y, M.y, V.y, G.y, a, bad);
    adam_one(P.z, M.z, V.z, G.z, a, bad);
    adam_one(P.w, M.w, V.w, G.w, a, bad);
    reinterpret_cast<float4*>(p)[i] = P;
    reinterpret_cast<float4*>(m)[i] = M;
    reinterpret_cast<float4*>(v)[i] = V;
    if (pb) reinterpret_cast<uint2*>(pb)[i] = make_uint2(pack_bf16x2(P.x, P.y), pack_bf16x2(P.z, P.w));
  }
  // ragged tail: the first threads of block 0
  if (blockIdx.x == 0 && threadIdx.x < n - n4 * 4) {
    const size_t j = n4 * 4 + threadIdx.x;
    float P = p[j], M = m[j], V = v[j];
    adam_one(P, M, V, g[j], a, bad);
    p[j] = P;
    m[j] = M;
    v[j] = V;
    if (pb) pb[j] = f32_to_bf16(P);
  }
  if (__any_sync(0xFFFFFFFFu, bad) && (threadIdx.x & 31) == 0) raise_status(status, TQP_STATUS_NONFINITE);
}

}  // namespace
}  // namespace tqp

extern "C" int tqp_adamw_step(float* param, float* exp_avg, float* exp_avg_sq, const float* grad,
                              uint16_t* param_bf16, size_t n, float lr, float beta1, float beta2, float eps,
                              float weight_decay, int step, float grad_scale, int32_t* dev_status, void* stream) {
  if (n == 0) return TQP_OK;
  if (!param || !exp_avg || !exp_avg_sq || !grad) return TQP_ERR_INVALID_ARG;
  auto al = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; };
  if (!al(param) || !al(exp_avg) || !al(exp_avg_sq) || !al(grad) ||
      (param_bf16 && (reinterpret_cast<uintptr_t>(param_bf16) & 7u)))
    return TQP_ERR_INVALID_ARG;
  if (step < 1 || !(beta1 >= 0.0f && beta1 < 1.0f) || !(beta2 >= 0.0f && beta2 < 1.0f) || !(eps > 0.0f) ||
      !(lr >= 0.0f) || !(weight_decay >= 0.0f))
    return TQP_ERR_INVALID_ARG;
  tqp::AdamArgs a;
  a.lr = lr;
  a.beta1 = beta1;
  a.beta2 = beta2;
  a.eps = eps;
  a.wd = weight_decay;
  a.grad_scale = grad_scale;
  a.bc1 = float(1.0 / (1.0 - std::pow(double(beta1), step)));
  a.bc2 = float(1.0 / (1.0 - std::pow(double(beta2), step)));
  const size_t n4 = n / 4;
  const size_t want = (n4 + 255) / 256;
  const size_t cap = size_t(4) * tqp::num_sms();
  const unsigned grid = unsigned(want == 0 ? 1 : (want < cap ? want : cap));
  tqp::adamw_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(param, exp_avg, exp_avg_sq, grad,
                                                                           param_bf16, n, a, dev_status);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}
