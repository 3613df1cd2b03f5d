// Internal launcher declarations shared by the kernel files and the C ABI.
#pragma once

#include <atomic>
#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/tqp_moe.h"

namespace tqp {

inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

// Per-device "done" bits of a one-time setting of a kernel (its dynamic
// shared-memory limit): the attribute belongs to the kernel on the current
// device, so a process that drives several GPUs sets it once on each.
struct DeviceFlags {
  std::atomic<unsigned long long> bits{0};
  // Sets the kernel's dynamic shared-memory limit on the current device unless
  // already done there; false if the runtime refused.
  template <typename K>
  bool test_and_set_device(K kernel, int smem_bytes) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const unsigned long long bit = dev < 64 ? (1ull << dev) : 0ull;
    if (bit && (bits.load(std::memory_order_acquire) & bit)) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_bytes) != cudaSuccess)
      return false;
    bits.fetch_or(bit, std::memory_order_acq_rel);
    return true;
  }
};

// Limit of one device-side barrier wait for the next launches, in ns (0 = the
// kernels' default). Set only through tqp_debug_set_wait_limit_ns.
unsigned long long wait_limit_ns();

// route / permute / combine
int launch_route(const float* logits, int T, int E, int k, int32_t* ids, float* gates, int32_t* status,
                 cudaStream_t s);
size_t permute_ws_bytes(int T, int E);
int launch_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* perm_token, int32_t* inv,
                   void* ws, int32_t* status, cudaStream_t s);
// grid: round the residual and the branch to the coupling's stream grid (exact
// adds; a result of magnitude >= 256 raises TQP_STATUS_RANGE into status)
int launch_combine(const uint16_t* out_perm, const int32_t* inv, const float* gates, int T, int k, int d,
                   const void* residual, int residual_f32, float sign, void* y, int y_f32, uint16_t* y_bf16,
                   cudaStream_t s, bool grid = false, int32_t* status = nullptr);

// grouped tensor-core GEMMs
size_t router_ws_bytes(int T, const tqp_moe_weights* w);
int launch_router_gemm(const uint16_t* x, int T, const tqp_moe_weights* w, float* logits, void* ws,
                       int32_t* status, cudaStream_t s);
size_t ffn_ws_bytes(int T, const tqp_moe_weights* w);
// Buffers inside the grouped-FFN workspace (valid after launch_grouped_ffn):
// per-expert m-block prefix, x in fp16, s*X[Ag|Au] [A][2r] and s*H*Ad [A][r] (fp16),
// and Ad^T in fp16.
struct FfnBufs {
  int32_t* mb_prefix;      // per-expert prefix of 128-row blocks
  int32_t* mb_prefix256;   // per-expert prefix of 256-row blocks (the down projection)
  uint16_t* x16;     // x in fp16 [T][d] (the shared-memory engine's gate/up fallback)
  uint16_t* xperm;   // expert-sorted token rows in fp16 [A][d] (same region as x16)
  uint16_t* xa;
  uint16_t* ha;
  uint16_t* adT16;   // Ad^T converted to fp16 [E][r][f]
  int4* unit_tab;    // decoded work units of the current expert-kernel launch
};
FfnBufs ffn_carve(void* ws, int T, const tqp_moe_weights* w);
int launch_grouped_ffn(const uint16_t* x, int T, const int32_t* offsets, const int32_t* perm_token,
                       const tqp_moe_weights* w, uint16_t* h, uint16_t* out_perm, void* ws, int32_t* status,
                       cudaStream_t s, uint16_t* aux_gu = nullptr);
int launch_grouped_ffn_part(int part, const uint16_t* x, int T, const int32_t* offsets, const int32_t* perm_token,
                            const tqp_moe_weights* w, uint16_t* h, uint16_t* out_perm, void* ws, int32_t* status,
                            cudaStream_t s, uint16_t* aux_gu = nullptr);
// dgrads: which 0 dH (+ SwiGLU backward into dG|dU), 1 dX. mb_prefix256 and
// unit_tab (the FFN workspace's 256-row schedule and unit table) select the
// tensor-memory dX kernel; null keeps the shared-memory engine.
int launch_dgrad(int which, const uint16_t* a_src, const uint16_t* a_lora, const int32_t* offsets,
                 const int32_t* mb_prefix, const tqp_moe_weights* w, int T, const uint16_t* aux_gu, uint16_t* out,
                 int32_t* status, cudaStream_t s, const int32_t* mb_prefix256 = nullptr, int4* unit_tab = nullptr,
                 const uint16_t* a_rows = nullptr);
// Row copy of the adapter A factors for the dgrads' rank-space stage (grouped_gemm.cu):
// which 0: Ad as [E][f][r] (dH), which 1: [Ag | Au] as [E][d][2r] (dX), fp16.
int launch_lora_a_rows(int which, const tqp_moe_weights* w, uint16_t* out, int32_t* status, cudaStream_t s);
// rank-space products of the backward on the tensor cores (grouped_gemm.cu):
//   which 0: dha = s dO Bd      (P = dO [A][d]      -> C [A][r])
//   which 1: dxa = s [dG|dU] blockdiag(Bg, Bu)   (P = dgu [A][2f] -> C [A][2r])
// bk16: scratch for the K-major fp16 B operand, E * max(r d, 4 r f) values.
int launch_rank_bwd(int which, const uint16_t* P, const int32_t* offsets, const int32_t* mb_prefix,
                    const tqp_moe_weights* w, int T, uint16_t* bk16, uint16_t* C, int32_t* status, cudaStream_t s);

// backward pieces (layer_bwd.cu). dmax holds max|dy| (launch_grad_absmax): the
// fp16 intermediates are computed for dy * 2^P, and dx and the adapter
// gradients are scaled back by 2^-P.
int launch_grad_absmax(const float* dy, size_t n, uint32_t* dmax, cudaStream_t s);
int launch_bwd_combine(const uint16_t* O, const int32_t* inv, const float* gates, const int32_t* ids,
                       const float* router_w, const float* dy, int T, int k, int d, const uint32_t* dmax, uint16_t* dO,
                       const float* addend, float* dx, int32_t* status, cudaStream_t s);   // dx = addend (or 0) + router term
int launch_gather_add(const uint16_t* dX, const int32_t* inv, int T, int k, int d, const uint32_t* dmax, float* dx,
                      cudaStream_t s);
// adapter gradients on the tensor cores (wgrad.cu); TQP_ERR_UNSUPPORTED for ranks above 32
// A: the routed rows of the expert-sorted operands (T * top_k)
int launch_wgrad(const tqp_moe_weights* w, size_t A, const int32_t* offsets, const int32_t* perm, const uint16_t* dO,
                 const uint16_t* h, const uint16_t* dgu, const uint16_t* x16, const uint16_t* ha, const uint16_t* dha,
                 const uint16_t* xa, const uint16_t* dxa, const tqp_adapter_grads* g, const uint32_t* dmax,
                 int32_t* status, cudaStream_t s);
int launch_outer(int E, int M, int N, const int32_t* offsets, const int32_t* perm, const uint16_t* P, int ldp,
                 int offp, const uint16_t* Q, int ldq, int offq, float* C, const uint32_t* dmax, cudaStream_t s);

int num_sms();

}  // namespace tqp
