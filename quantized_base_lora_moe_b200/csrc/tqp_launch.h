// Internal launcher declarations shared by the kernel files and the C ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/tqp_moe.h"

namespace tqp {

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// route / permute / combine
int launch_route(const float* logits, int T, int E, int k, int32_t* ids, float* gates, int32_t* status,
                 cudaStream_t s);
size_t permute_ws_bytes(int T, int E);
int launch_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* perm_token, int32_t* inv,
                   void* ws, int32_t* status, cudaStream_t s);
int launch_combine(const uint16_t* out_perm, const int32_t* inv, const float* gates, int T, int k, int d,
                   const void* residual, int residual_f32, float sign, void* y, int y_f32, uint16_t* y_bf16,
                   cudaStream_t s);

// grouped tensor-core GEMMs
size_t router_ws_bytes(int T, const tqp_moe_weights* w);
int launch_router_gemm(const uint16_t* x, int T, const tqp_moe_weights* w, float* logits, void* ws,
                       int32_t* status, cudaStream_t s);
size_t ffn_ws_bytes(int T, const tqp_moe_weights* w);
int launch_grouped_ffn(const uint16_t* x, int T, const int32_t* offsets, const int32_t* perm_token,
                       const tqp_moe_weights* w, uint16_t* h, uint16_t* out_perm, void* ws, int32_t* status,
                       cudaStream_t s);

// backward
size_t layer_bwd_ws_bytes(int T, const tqp_moe_weights* w);
int launch_layer_bwd(const uint16_t* x, const float* dy, int T, const tqp_moe_weights* w, float* dx,
                     const tqp_adapter_grads* grads, void* ws, int32_t* status, cudaStream_t s);

int num_sms();

}  // namespace tqp

namespace tqp {
int launch_add_f32(const float* a, const float* b, float* out, size_t n, cudaStream_t s);
}  // namespace tqp
