// C ABI of the TQP MoE library: argument validation, workspace layout and the
// composition of the per-step kernels into the layer, the reversible coupling
// and its backward. Declarations and contracts: include/tqp_moe.h.
#include <atomic>
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "../../include/tqp_moe.h"
#include "tqp_device.cuh"
#include "tqp_launch.h"

using namespace tqp;

namespace {
std::atomic<unsigned long long> g_wait_limit_ns{0};
}  // namespace

unsigned long long tqp::wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

namespace {

constexpr int kMaxE = 4096;
constexpr int kMaxTopK = 32;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_weights(const tqp_moe_weights* w) {
  if (!w) return TQP_ERR_INVALID_ARG;
  if (w->E < 1 || w->E > kMaxE || w->top_k < 1 || w->top_k > w->E || w->top_k > kMaxTopK)
    return TQP_ERR_INVALID_ARG;
  if (w->d < 128 || w->d > 16384 || w->d % 128 != 0) return TQP_ERR_INVALID_ARG;
  if (w->ffn < 64 || w->ffn > 16384 || w->ffn % 64 != 0) return TQP_ERR_INVALID_ARG;
  if (!(w->group == 32 || w->group == 64 || w->group == 128 || w->group == 256)) return TQP_ERR_UNSUPPORTED;
  if (w->d % w->group != 0 || w->ffn % w->group != 0) return TQP_ERR_INVALID_ARG;
  if (w->rank < 0 || w->rank > 64 || w->rank % 8 != 0) return TQP_ERR_UNSUPPORTED;
  if (!(w->bits == 0 || w->bits == 4 || w->bits == 8)) return TQP_ERR_INVALID_ARG;
  if (w->bits == 8 && w->ffn % 128 != 0) return TQP_ERR_UNSUPPORTED;   // int8 runs on the tensor-memory kernels only
  if (!w->router_w || !aligned16(w->router_w)) return TQP_ERR_INVALID_ARG;
  if (w->router_bias && !aligned16(w->router_bias)) return TQP_ERR_INVALID_ARG;
  for (int p = 0; p < 3; ++p) {
    if (!w->wq[p] || !w->wscale[p] || !aligned16(w->wq[p]) || !aligned16(w->wscale[p])) return TQP_ERR_INVALID_ARG;
    if (w->rank > 0 && (!w->lora_a[p] || !w->lora_b[p] || !aligned16(w->lora_a[p]) || !aligned16(w->lora_b[p])))
      return TQP_ERR_INVALID_ARG;
  }
  return TQP_OK;
}

inline bool ptr_ok(const void* p, bool need) { return need ? (p && aligned16(p)) : true; }

// Workspace of one full layer forward (kept for the backward's recompute too).
struct LayerWs {
  float* logits;
  int32_t* ids;
  float* gates;
  int32_t* offsets;
  int32_t* perm;
  int32_t* inv;
  uint16_t* h;
  uint16_t* out_perm;
  void* router_ws;
  void* permute_ws;
  void* ffn_ws;
};

size_t layer_ws_size(int T, const tqp_moe_weights* w) {
  const size_t A = size_t(T) * w->top_k;
  size_t b = 0;
  b += align_up(size_t(T) * w->E * 4, 256);
  b += align_up(A * 4, 256) * 2;                 // ids, gates
  b += align_up(size_t(w->E + 1) * 4, 256);
  b += align_up(A * 4, 256) * 2;                 // perm, inv
  b += align_up(A * w->ffn * 2, 256);            // h
  b += align_up(A * w->d * 2, 256);              // out_perm
  b += align_up(router_ws_bytes(T, w), 256);
  b += align_up(permute_ws_bytes(T, w->E), 256);
  b += align_up(ffn_ws_bytes(T, w), 256);
  return b + 256;
}

LayerWs carve_layer_ws(void* ws, int T, const tqp_moe_weights* w) {
  const size_t A = size_t(T) * w->top_k;
  char* p = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
  LayerWs L;
  auto take = [&](size_t bytes) {
    char* q = p;
    p += align_up(bytes, 256);
    return static_cast<void*>(q);
  };
  L.logits = static_cast<float*>(take(size_t(T) * w->E * 4));
  L.ids = static_cast<int32_t*>(take(A * 4));
  L.gates = static_cast<float*>(take(A * 4));
  L.offsets = static_cast<int32_t*>(take(size_t(w->E + 1) * 4));
  L.perm = static_cast<int32_t*>(take(A * 4));
  L.inv = static_cast<int32_t*>(take(A * 4));
  L.h = static_cast<uint16_t*>(take(A * w->ffn * 2));
  L.out_perm = static_cast<uint16_t*>(take(A * w->d * 2));
  L.router_ws = take(router_ws_bytes(T, w));
  L.permute_ws = take(permute_ws_bytes(T, w->E));
  L.ffn_ws = take(ffn_ws_bytes(T, w));
  return L;
}

// router -> route -> permute -> experts (leaves everything in the workspace)
int layer_experts(const uint16_t* x, int T, const tqp_moe_weights* w, const LayerWs& L, int32_t* status,
                  cudaStream_t s, uint16_t* aux_gu = nullptr) {
  int rc;
  if ((rc = launch_router_gemm(x, T, w, L.logits, L.router_ws, status, s)) != TQP_OK) return rc;
  if ((rc = launch_route(L.logits, T, w->E, w->top_k, L.ids, L.gates, status, s)) != TQP_OK) return rc;
  if ((rc = launch_permute(L.ids, T, w->E, w->top_k, L.offsets, L.perm, L.inv, L.permute_ws, status, s)) != TQP_OK)
    return rc;
  return launch_grouped_ffn(x, T, L.offsets, L.perm, w, L.h, L.out_perm, L.ffn_ws, status, s, aux_gu);
}

// Extra workspace of the layer backward, after the forward recompute's.
struct BwdWs {
  uint16_t* gu;     // G | U pre-activations [A][2f] fp16
  uint16_t* dO;     // gamma * dy [A][d] fp16 (reused for dX rows)
  uint16_t* dha;    // s dO Bd^T [A][r] fp16
  uint16_t* dgu;    // dG | dU [A][2f] fp16
  uint16_t* dxa;    // s [dG|dU] [Bg|Bu]^T [A][2r] fp16
  uint16_t* bk16;   // K-major fp16 B operand of dha / dxa, E * max(r d, 4 r f) values
  uint16_t* arow;   // row copy of Ad ([E][f][r]) or [Ag | Au] ([E][d][2r]) in fp16 for the dgrads
  uint32_t* dmax;   // max |dy| (sets the power-of-two scale of the fp16 intermediates)
};

// Adapter-gradient buffers: present and 16-byte aligned when the rank is nonzero.
bool grads_ok(const tqp_moe_weights* w, const tqp_adapter_grads* g) {
  if (!g) return false;
  if (w->rank > 0)
    for (int p = 0; p < 3; ++p)
      if (!g->dA[p] || !g->dB[p] || !aligned16(g->dA[p]) || !aligned16(g->dB[p])) return false;
  return true;
}

size_t rank_b_values(const tqp_moe_weights* w) {
  const size_t rd = size_t(w->rank) * w->d, rf4 = size_t(4) * w->rank * w->ffn;
  return size_t(w->E) * (rd > rf4 ? rd : rf4);
}

size_t arow_values(const tqp_moe_weights* w) {
  const size_t fr = size_t(w->ffn) * w->rank, d2r = size_t(2) * w->d * w->rank;
  return size_t(w->E) * (fr > d2r ? fr : d2r);
}

size_t bwd_extra_bytes(int T, const tqp_moe_weights* w) {
  const size_t A = size_t(T) * w->top_k;
  return align_up(A * 2 * w->ffn * 2, 256) * 2 + align_up(A * w->d * 2, 256) + align_up(A * w->rank * 2, 256) +
         align_up(A * 2 * w->rank * 2, 256) + align_up(rank_b_values(w) * 2, 256) + align_up(arow_values(w) * 2, 256) +
         256 + 256;
}

BwdWs carve_bwd(void* p0, int T, const tqp_moe_weights* w) {
  const size_t A = size_t(T) * w->top_k;
  char* p = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(p0), 256));
  BwdWs b;
  auto take = [&](size_t bytes) {
    char* q = p;
    p += align_up(bytes, 256);
    return static_cast<void*>(q);
  };
  b.gu = static_cast<uint16_t*>(take(A * 2 * w->ffn * 2));
  b.dO = static_cast<uint16_t*>(take(A * w->d * 2));
  b.dha = static_cast<uint16_t*>(take(A * w->rank * 2));
  b.dgu = static_cast<uint16_t*>(take(A * 2 * w->ffn * 2));
  b.dxa = static_cast<uint16_t*>(take(A * 2 * w->rank * 2));
  b.bk16 = static_cast<uint16_t*>(take(rank_b_values(w) * 2));
  b.arow = static_cast<uint16_t*>(take(arow_values(w) * 2));
  b.dmax = static_cast<uint32_t*>(take(sizeof(uint32_t)));
  return b;
}

// Backward of one layer: recompute the forward (keeping G, U), then
// combine/gate/router backward, dH (+SwiGLU backward) and dX on the tensor
// cores, rank-space products and adapter gradients, and the token gather.
// recompute = false: the forward of this x has just run on the same workspace
// with the G|U pre-activations kept (layer_forward with aux_gu = the backward
// scratch's gu), so its routing and intermediates are still in place.
int layer_backward(const uint16_t* x, const float* dy, int T, const tqp_moe_weights* w, float* dx,
                   const tqp_adapter_grads* g, void* ws, int32_t* status, cudaStream_t s, bool recompute = true,
                   const float* dx_addend = nullptr) {
  const LayerWs L = carve_layer_ws(ws, T, w);
  const BwdWs B = carve_bwd(static_cast<char*>(ws) + layer_ws_size(T, w), T, w);
  const int k = w->top_k, d = w->d, f = w->ffn, r = w->rank, E = w->E;
  int rc;
  if (recompute && (rc = layer_experts(x, T, w, L, status, s, B.gu)) != TQP_OK) return rc;
  const FfnBufs fb = ffn_carve(L.ffn_ws, T, w);
  if ((rc = launch_grad_absmax(dy, size_t(T) * d, B.dmax, s)) != TQP_OK) return rc;
  if ((rc = launch_bwd_combine(L.out_perm, L.inv, L.gates, L.ids, w->router_w, dy, T, k, d, B.dmax, B.dO, dx_addend,
                               dx, status, s)) != TQP_OK)
    return rc;
  if (r > 0 && (rc = launch_rank_bwd(0, B.dO, L.offsets, fb.mb_prefix, w, T, B.bk16, B.dha, status, s)) != TQP_OK)
    return rc;
  if (r > 0 && (rc = launch_lora_a_rows(0, w, B.arow, status, s)) != TQP_OK) return rc;
  if ((rc = launch_dgrad(0, B.dO, B.dha, L.offsets, fb.mb_prefix, w, T, B.gu, B.dgu, status, s, fb.mb_prefix256,
                         fb.unit_tab, B.arow)) != TQP_OK)
    return rc;
  if (r > 0) {
    if ((rc = launch_rank_bwd(1, B.dgu, L.offsets, fb.mb_prefix, w, T, B.bk16, B.dxa, status, s)) != TQP_OK)
      return rc;
    // adapter gradients, in the storage layouts A^T [r][in], B^T [out][r]: on the
    // tensor cores for ranks up to 32, else as outer products on the CUDA cores
    rc = launch_wgrad(w, size_t(T) * k, L.offsets, nullptr, B.dO, L.h, B.dgu, fb.xperm, fb.ha, B.dha, fb.xa, B.dxa, g, B.dmax, status, s);
    if (rc != TQP_OK && rc != TQP_ERR_UNSUPPORTED) return rc;
  }
  if (r > 0 && rc == TQP_ERR_UNSUPPORTED) {
    if ((rc = launch_outer(E, d, r, L.offsets, nullptr, B.dO, d, 0, fb.ha, r, 0, g->dB[2], B.dmax, s)) != TQP_OK) return rc;
    if ((rc = launch_outer(E, r, f, L.offsets, nullptr, B.dha, r, 0, L.h, f, 0, g->dA[2], B.dmax, s)) != TQP_OK) return rc;
    if ((rc = launch_outer(E, f, r, L.offsets, nullptr, B.dgu, 2 * f, 0, fb.xa, 2 * r, 0, g->dB[0], B.dmax, s)) != TQP_OK)
      return rc;
    if ((rc = launch_outer(E, f, r, L.offsets, nullptr, B.dgu, 2 * f, f, fb.xa, 2 * r, r, g->dB[1], B.dmax, s)) != TQP_OK)
      return rc;
    if ((rc = launch_outer(E, r, d, L.offsets, nullptr, B.dxa, 2 * r, 0, fb.xperm, d, 0, g->dA[0], B.dmax, s)) != TQP_OK)
      return rc;
    if ((rc = launch_outer(E, r, d, L.offsets, nullptr, B.dxa, 2 * r, r, fb.xperm, d, 0, g->dA[1], B.dmax, s)) != TQP_OK)
      return rc;
  }
  uint16_t* dX = B.dO;  // dO is no longer needed
  if (r > 0 && (rc = launch_lora_a_rows(1, w, B.arow, status, s)) != TQP_OK) return rc;
  if ((rc = launch_dgrad(1, B.dgu, B.dxa, L.offsets, fb.mb_prefix, w, T, nullptr, dX, status, s, fb.mb_prefix256,
                         fb.unit_tab, B.arow)) != TQP_OK)
    return rc;
  return launch_gather_add(dX, L.inv, T, k, d, B.dmax, dx, s);
}

// grid: the residual add is the coupling's, on the stream grid (exact adds)
int layer_forward(const uint16_t* x, int T, const tqp_moe_weights* w, const void* residual, int res_f32,
                  float sign, void* y, int y_f32, uint16_t* y_bf16, void* ws, int32_t* status, cudaStream_t s,
                  uint16_t* aux_gu = nullptr, bool grid = false) {
  const LayerWs L = carve_layer_ws(ws, T, w);
  int rc = layer_experts(x, T, w, L, status, s, aux_gu);
  if (rc != TQP_OK) return rc;
  return launch_combine(L.out_perm, L.inv, L.gates, T, w->top_k, w->d, residual, res_f32, sign, y, y_f32, y_bf16, s,
                        grid, status);
}

// bf16(x) of a bf16 stream input put on the coupling's stream grid: the input
// a coupling's first layer reads, so that its inverse, which can only return
// the grid value, feeds that layer the same bits
__global__ void stream_grid_bf16_kernel(const uint16_t* __restrict__ in, uint16_t* __restrict__ out, size_t n) {
  const size_t i = (size_t(blockIdx.x) * blockDim.x + threadIdx.x) * 8;
  if (i + 7 < n) {
    const uint4 v = *reinterpret_cast<const uint4*>(in + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      o[q] = pack_bf16x2(to_stream_grid(__uint_as_float(w[q] << 16)), to_stream_grid(__uint_as_float(w[q] & 0xFFFF0000u)));
    *reinterpret_cast<uint4*>(out + i) = make_uint4(o[0], o[1], o[2], o[3]);
  } else {
    for (size_t j = i; j < n; ++j) out[j] = f32_to_bf16(to_stream_grid(bf16_to_f32(in[j])));
  }
}

int to_stream_grid_bf16(const uint16_t* in, uint16_t* out, size_t n, cudaStream_t s) {
  if (n == 0) return TQP_OK;
  const size_t threads = (n + 7) / 8;
  stream_grid_bf16_kernel<<<unsigned((threads + 255) / 256), 256, 0, s>>>(in, out, n);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

__global__ void f32_to_bf16_kernel(const float* __restrict__ in, uint16_t* __restrict__ out, size_t n) {
  const size_t i = (size_t(blockIdx.x) * blockDim.x + threadIdx.x) * 4;
  if (i + 3 < n) {
    const float4 v = *reinterpret_cast<const float4*>(in + i);
    uint2 o;
    o.x = pack_bf16x2(v.x, v.y);
    o.y = pack_bf16x2(v.z, v.w);
    *reinterpret_cast<uint2*>(out + i) = o;
  } else {
    for (size_t j = i; j < n; ++j) out[j] = f32_to_bf16(in[j]);
  }
}

int to_bf16(const float* in, uint16_t* out, size_t n, cudaStream_t s) {
  if (n == 0) return TQP_OK;
  const size_t threads = (n + 3) / 4;
  f32_to_bf16_kernel<<<unsigned((threads + 255) / 256), 256, 0, s>>>(in, out, n);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

// ----------------------------------------------------------------------------
// reversible stack of L coupling blocks
// ----------------------------------------------------------------------------
// Block l maps fp32 streams (a1, a2) to (b1, b2):  b1 = a1 + F_l(bf16(a2)),
// b2 = a2 + G_l(bf16(b1)). The streams stay fp32 on the stream grid between
// blocks, so every add and subtract is exact; every layer reads the bf16
// rounding of its stream. Block 0 puts its bf16 inputs x1, x2 on the grid as
// rev_couple_fwd does, so one block is exactly rev_couple_fwd. The
// workspace holds two sets of stream buffers that the blocks alternate
// between, two bf16 layer inputs, one fp32 input gradient and one layer's
// workspace: activation memory does not grow with L.

constexpr int kMaxStack = 4096;

int check_stack(int T, int L, const tqp_moe_weights* const* F, const tqp_moe_weights* const* G, bool bwd) {
  if (T < 0 || L < 1 || L > kMaxStack || !F || !G) return TQP_ERR_INVALID_ARG;
  int rc;
  for (int l = 0; l < L; ++l) {
    if ((rc = check_weights(F[l])) != TQP_OK || (rc = check_weights(G[l])) != TQP_OK) return rc;
    if (F[l]->d != F[0]->d || G[l]->d != F[0]->d) return TQP_ERR_INVALID_ARG;
    if (bwd && (F[l]->ffn % 128 != 0 || G[l]->ffn % 128 != 0)) return TQP_ERR_UNSUPPORTED;
  }
  return TQP_OK;
}

size_t stack_layer_ws(int T, int L, const tqp_moe_weights* const* F, const tqp_moe_weights* const* G) {
  size_t m = 0;
  for (int l = 0; l < L; ++l) {
    const size_t a = layer_ws_size(T, F[l]) + bwd_extra_bytes(T, F[l]);
    const size_t b = layer_ws_size(T, G[l]) + bwd_extra_bytes(T, G[l]);
    m = a > m ? a : m;
    m = b > m ? b : m;
  }
  return m;
}

struct StackWs {
  float* s[2][4];     // two sets of (stream 1, stream 2, cotangent 1, cotangent 2), fp32 [T][d]
  uint16_t* zb;       // bf16 layer input
  uint16_t* ab;       // bf16 layer input
  void* lws;          // one layer's forward + backward workspace
};

StackWs carve_stack(void* ws, int T, int d) {
  const size_t Td = size_t(T) * d;
  char* p = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
  StackWs w;
  for (int i = 0; i < 2; ++i)
    for (int j = 0; j < 4; ++j) {
      w.s[i][j] = reinterpret_cast<float*>(p);
      p += align_up(Td * 4, 256);
    }
  w.zb = reinterpret_cast<uint16_t*>(p);
  p += align_up(Td * 2, 256);
  w.ab = reinterpret_cast<uint16_t*>(p);
  p += align_up(Td * 2, 256);
  w.lws = p;
  return w;
}

size_t stack_ws_size(int T, int L, const tqp_moe_weights* const* F, const tqp_moe_weights* const* G) {
  const size_t Td = size_t(T) * F[0]->d;
  return 8 * align_up(Td * 4, 256) + 2 * align_up(Td * 2, 256) + stack_layer_ws(T, L, F, G) + 512;
}

// Block backward on fp32 streams: from the block outputs (y1, y2) and their
// cotangents, the block inputs (a1, a2) and their cotangents (da1, da2) plus
// both layers' adapter gradients. Each layer's backward follows the inverse
// step that ran its forward on the same workspace. a2b receives bf16(a2).
int block_backward_f32(const float* y1, const float* y2, const float* dy1, const float* dy2, int T,
                       const tqp_moe_weights* F, const tqp_moe_weights* G, float* a1, float* a2, float* da1,
                       float* da2, const tqp_adapter_grads* gF, const tqp_adapter_grads* gG, const StackWs& w,
                       int32_t* status, cudaStream_t s) {
  const size_t Td = size_t(T) * F->d;
  int rc;
  if ((rc = to_bf16(y1, w.zb, Td, s)) != TQP_OK) return rc;
  uint16_t* gu = carve_bwd(static_cast<char*>(w.lws) + layer_ws_size(T, G), T, G).gu;
  if ((rc = layer_forward(w.zb, T, G, y2, 1, -1.0f, a2, 1, w.ab, w.lws, status, s, gu, true)) != TQP_OK) return rc;
  // da1 = dy1 + J_G^T dy2, the sum taken inside G's backward
  if ((rc = layer_backward(w.zb, dy2, T, G, da1, gG, w.lws, status, s, false, dy1)) != TQP_OK) return rc;
  gu = carve_bwd(static_cast<char*>(w.lws) + layer_ws_size(T, F), T, F).gu;
  if ((rc = layer_forward(w.ab, T, F, y1, 1, -1.0f, a1, 1, nullptr, w.lws, status, s, gu, true)) != TQP_OK) return rc;
  // da2 = dy2 + J_F^T da1
  return layer_backward(w.ab, da1, T, F, da2, gF, w.lws, status, s, false, dy2);
}

}  // namespace

extern "C" {

int tqp_version(void) { return 200; }

const char* tqp_error_string(int code) {
  switch (code) {
    case TQP_OK: return "ok";
    case TQP_ERR_INVALID_ARG: return "invalid argument";
    case TQP_ERR_UNSUPPORTED: return "unsupported configuration";
    case TQP_ERR_WORKSPACE: return "workspace too small";
    case TQP_ERR_CUDA: return "CUDA launch or runtime error";
    default: return "unknown error";
  }
}

size_t moe_router_gemm_workspace_size(int T, const tqp_moe_weights* w) {
  if (check_weights(w) != TQP_OK || T < 0) return 0;
  return router_ws_bytes(T, w);
}

int moe_router_gemm(const uint16_t* x, int T, const tqp_moe_weights* w, float* logits, void* ws, size_t ws_bytes,
                    int32_t* dev_status, void* stream) {
  int rc = check_weights(w);
  if (rc != TQP_OK) return rc;
  if (T < 0 || !ptr_ok(x, T > 0) || !ptr_ok(logits, T > 0) || !ptr_ok(ws, T > 0)) return TQP_ERR_INVALID_ARG;
  if (T > 0 && ws_bytes < router_ws_bytes(T, w)) return TQP_ERR_WORKSPACE;
  return launch_router_gemm(x, T, w, logits, ws, dev_status, static_cast<cudaStream_t>(stream));
}

int moe_route(const float* logits, int T, int E, int k, int32_t* ids, float* gates, int32_t* dev_status,
              void* stream) {
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > E || k > kMaxTopK) return TQP_ERR_INVALID_ARG;
  if (T > 0 && (!logits || !ids || !gates)) return TQP_ERR_INVALID_ARG;
  return launch_route(logits, T, E, k, ids, gates, dev_status, static_cast<cudaStream_t>(stream));
}

size_t moe_permute_workspace_size(int T, int E, int k) {
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > E) return 0;
  return permute_ws_bytes(T, E);
}

int moe_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* perm_token, int32_t* inv,
                void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  if (T < 0 || E < 1 || E > kMaxE || k < 1 || k > E || !offsets) return TQP_ERR_INVALID_ARG;
  if (T > 0 && (!ids || !perm_token || !inv || !ws)) return TQP_ERR_INVALID_ARG;
  if (T > 0 && ws_bytes < permute_ws_bytes(T, E)) return TQP_ERR_WORKSPACE;
  return launch_permute(ids, T, E, k, offsets, perm_token, inv, ws, dev_status, static_cast<cudaStream_t>(stream));
}

size_t tqp_grouped_ffn_workspace_size(int T, const tqp_moe_weights* w) {
  if (check_weights(w) != TQP_OK || T < 0) return 0;
  return ffn_ws_bytes(T, w);
}

int tqp_grouped_ffn(const uint16_t* x, int T, const int32_t* offsets, const int32_t* perm_token,
                    const tqp_moe_weights* w, uint16_t* h, uint16_t* out_perm, void* ws, size_t ws_bytes,
                    int32_t* dev_status, void* stream) {
  int rc = check_weights(w);
  if (rc != TQP_OK) return rc;
  const bool n = T > 0;
  if (T < 0 || !ptr_ok(x, n) || !ptr_ok(offsets, n) || !ptr_ok(perm_token, n) || !ptr_ok(h, n) ||
      !ptr_ok(out_perm, n) || !ptr_ok(ws, n))
    return TQP_ERR_INVALID_ARG;
  if (n && ws_bytes < ffn_ws_bytes(T, w)) return TQP_ERR_WORKSPACE;
  return launch_grouped_ffn(x, T, offsets, perm_token, w, h, out_perm, ws, dev_status,
                            static_cast<cudaStream_t>(stream));
}

int tqp_grouped_ffn_part(int part, const uint16_t* x, int T, const int32_t* offsets, const int32_t* perm_token,
                         const tqp_moe_weights* w, uint16_t* h, uint16_t* out_perm, void* ws, size_t ws_bytes,
                         int32_t* dev_status, void* stream) {
  if (part < TQP_FFN_PREPARE || part > TQP_FFN_DOWN) return TQP_ERR_INVALID_ARG;
  int rc = check_weights(w);
  if (rc != TQP_OK) return rc;
  const bool n = T > 0;
  if (T < 0 || !ptr_ok(x, n) || !ptr_ok(offsets, n) || !ptr_ok(perm_token, n) || !ptr_ok(h, n) ||
      !ptr_ok(out_perm, n) || !ptr_ok(ws, n))
    return TQP_ERR_INVALID_ARG;
  if (n && ws_bytes < ffn_ws_bytes(T, w)) return TQP_ERR_WORKSPACE;
  return launch_grouped_ffn_part(part, x, T, offsets, perm_token, w, h, out_perm, ws, dev_status,
                                 static_cast<cudaStream_t>(stream));
}

int moe_combine(const uint16_t* out_perm, const int32_t* inv, const float* gates, int T, int k, int d,
                const void* residual, int residual_dtype, float sign, void* y, int y_dtype, uint16_t* y_bf16,
                void* stream) {
  if (T < 0 || k < 1 || k > kMaxTopK || d < 8 || d % 8 != 0) return TQP_ERR_INVALID_ARG;
  if ((residual_dtype != TQP_DTYPE_BF16 && residual_dtype != TQP_DTYPE_F32) ||
      (y_dtype != TQP_DTYPE_BF16 && y_dtype != TQP_DTYPE_F32))
    return TQP_ERR_INVALID_ARG;
  const bool n = T > 0;
  if (!ptr_ok(out_perm, n) || !ptr_ok(inv, n) || !ptr_ok(gates, n) || !ptr_ok(y, n) || !ptr_ok(residual, false) ||
      (residual && !aligned16(residual)) || (y_bf16 && !aligned16(y_bf16)))
    return TQP_ERR_INVALID_ARG;
  return launch_combine(out_perm, inv, gates, T, k, d, residual, residual_dtype == TQP_DTYPE_F32, sign, y,
                        y_dtype == TQP_DTYPE_F32, y_bf16, static_cast<cudaStream_t>(stream));
}

size_t tqp_moe_layer_workspace_size(int T, const tqp_moe_weights* w) {
  if (check_weights(w) != TQP_OK || T < 0) return 0;
  return layer_ws_size(T, w);
}

int tqp_moe_layer_fwd(const uint16_t* x, int T, const tqp_moe_weights* w, uint16_t* y, void* ws, size_t ws_bytes,
                      int32_t* dev_status, void* stream) {
  int rc = check_weights(w);
  if (rc != TQP_OK) return rc;
  const bool n = T > 0;
  if (T < 0 || !ptr_ok(x, n) || !ptr_ok(y, n) || !ptr_ok(ws, n)) return TQP_ERR_INVALID_ARG;
  if (!n) return TQP_OK;
  if (ws_bytes < layer_ws_size(T, w)) return TQP_ERR_WORKSPACE;
  return layer_forward(x, T, w, nullptr, 0, 1.0f, y, 0, nullptr, ws, dev_status, static_cast<cudaStream_t>(stream));
}

size_t rev_couple_workspace_size(int T, const tqp_moe_weights* F, const tqp_moe_weights* G) {
  if (check_weights(F) != TQP_OK || check_weights(G) != TQP_OK || T < 0 || F->d != G->d) return 0;
  const size_t a = layer_ws_size(T, F), b = layer_ws_size(T, G);
  return (a > b ? a : b) + 2 * align_up(size_t(T) * F->d * 2, 256) + 256;
}

int rev_couple_fwd(const uint16_t* x1, const uint16_t* x2, int T, const tqp_moe_weights* F, const tqp_moe_weights* G,
                   float* y1, float* y2, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  int rc;
  if ((rc = check_weights(F)) != TQP_OK || (rc = check_weights(G)) != TQP_OK) return rc;
  if (F->d != G->d || T < 0) return TQP_ERR_INVALID_ARG;
  const bool n = T > 0;
  if (!ptr_ok(x1, n) || !ptr_ok(x2, n) || !ptr_ok(y1, n) || !ptr_ok(y2, n) || !ptr_ok(ws, n))
    return TQP_ERR_INVALID_ARG;
  if (!n) return TQP_OK;
  if (ws_bytes < rev_couple_workspace_size(T, F, G)) return TQP_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
  const size_t Td = size_t(T) * F->d;
  uint16_t* y1b = reinterpret_cast<uint16_t*>(base);
  uint16_t* x2g = reinterpret_cast<uint16_t*>(base + align_up(Td * 2, 256));
  void* lws = base + 2 * align_up(Td * 2, 256);
  // the streams on the stream grid: F reads x2 on the grid, the value its inverse returns
  if ((rc = to_stream_grid_bf16(x2, x2g, Td, s)) != TQP_OK) return rc;
  // y1 = x1 + F(x2) (fp32), plus its bf16 copy as G's input
  if ((rc = layer_forward(x2g, T, F, x1, 0, 1.0f, y1, 1, y1b, lws, dev_status, s, nullptr, true)) != TQP_OK) return rc;
  // y2 = x2 + G(bf16(y1))
  return layer_forward(y1b, T, G, x2, 0, 1.0f, y2, 1, nullptr, lws, dev_status, s, nullptr, true);
}

int rev_couple_inv(const float* y1, const float* y2, int T, const tqp_moe_weights* F, const tqp_moe_weights* G,
                   uint16_t* x1, uint16_t* x2, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  int rc;
  if ((rc = check_weights(F)) != TQP_OK || (rc = check_weights(G)) != TQP_OK) return rc;
  if (F->d != G->d || T < 0) return TQP_ERR_INVALID_ARG;
  const bool n = T > 0;
  if (!ptr_ok(x1, n) || !ptr_ok(x2, n) || !ptr_ok(y1, n) || !ptr_ok(y2, n) || !ptr_ok(ws, n))
    return TQP_ERR_INVALID_ARG;
  if (!n) return TQP_OK;
  if (ws_bytes < rev_couple_workspace_size(T, F, G)) return TQP_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
  uint16_t* y1b = reinterpret_cast<uint16_t*>(base);
  void* lws = base + 2 * align_up(size_t(T) * F->d * 2, 256);
  if ((rc = to_bf16(y1, y1b, size_t(T) * F->d, s)) != TQP_OK) return rc;
  // x2 = y2 - G(bf16(y1)), exact on the stream grid, then rounded to bf16 (a no-op there)
  if ((rc = layer_forward(y1b, T, G, y2, 1, -1.0f, x2, 0, nullptr, lws, dev_status, s, nullptr, true)) != TQP_OK)
    return rc;
  // x1 = y1 - F(x2)
  return layer_forward(x2, T, F, y1, 1, -1.0f, x1, 0, nullptr, lws, dev_status, s, nullptr, true);
}

size_t tqp_moe_layer_bwd_workspace_size(int T, const tqp_moe_weights* w) {
  if (check_weights(w) != TQP_OK || T < 0) return 0;
  return layer_ws_size(T, w) + bwd_extra_bytes(T, w);
}

int tqp_moe_layer_bwd(const uint16_t* x, const float* dy, int T, const tqp_moe_weights* w, float* dx,
                      const tqp_adapter_grads* grads, void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  int rc = check_weights(w);
  if (rc != TQP_OK) return rc;
  const bool n = T > 0;
  if (T < 0 || !ptr_ok(x, n) || !ptr_ok(dy, n) || !ptr_ok(dx, n) || !grads) return TQP_ERR_INVALID_ARG;
  if (w->ffn % 128 != 0) return TQP_ERR_UNSUPPORTED;   // the dH tiles are 128 columns of ffn
  if (!grads_ok(w, grads)) return TQP_ERR_INVALID_ARG;
  if (n && (!ws || ws_bytes < tqp_moe_layer_bwd_workspace_size(T, w))) return TQP_ERR_WORKSPACE;
  if (!n) return TQP_OK;
  return layer_backward(x, dy, T, w, dx, grads, ws, dev_status, static_cast<cudaStream_t>(stream));
}

size_t tqp_adapter_bwd_workspace_size(int T, const tqp_moe_weights* F, const tqp_moe_weights* G) {
  if (check_weights(F) != TQP_OK || check_weights(G) != TQP_OK || T < 0 || F->d != G->d) return 0;
  const size_t a = tqp_moe_layer_bwd_workspace_size(T, F), b = tqp_moe_layer_bwd_workspace_size(T, G);
  const size_t fw = rev_couple_workspace_size(T, F, G);
  size_t m = a > b ? a : b;
  m = m > fw ? m : fw;
  return m + align_up(size_t(T) * F->d * 2, 256) + 512;
}

int tqp_adapter_bwd(const float* y1, const float* y2, const float* dy1, const float* dy2, int T,
                    const tqp_moe_weights* F, const tqp_moe_weights* G, uint16_t* x1, uint16_t* x2, float* dx1,
                    float* dx2, const tqp_adapter_grads* gF, const tqp_adapter_grads* gG, void* ws, size_t ws_bytes,
                    int32_t* dev_status, void* stream) {
  int rc;
  if ((rc = check_weights(F)) != TQP_OK || (rc = check_weights(G)) != TQP_OK) return rc;
  if (F->d != G->d || T < 0 || !grads_ok(F, gF) || !grads_ok(G, gG)) return TQP_ERR_INVALID_ARG;
  if (F->ffn % 128 != 0 || G->ffn % 128 != 0) return TQP_ERR_UNSUPPORTED;
  const bool n = T > 0;
  if (!ptr_ok(y1, n) || !ptr_ok(y2, n) || !ptr_ok(dy1, n) || !ptr_ok(dy2, n) || !ptr_ok(x1, n) || !ptr_ok(x2, n) ||
      !ptr_ok(dx1, n) || !ptr_ok(dx2, n))
    return TQP_ERR_INVALID_ARG;
  if (!n) return TQP_OK;
  if (ws_bytes < tqp_adapter_bwd_workspace_size(T, F, G)) return TQP_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t Td = size_t(T) * F->d;
  char* base = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), 256));
  uint16_t* zb = reinterpret_cast<uint16_t*>(base);                     // bf16(y1)
  void* lws = base + align_up(Td * 2, 256);
  // Each layer's backward follows the inverse step that ran that layer's forward
  // on the same workspace (keeping G|U), so it does not recompute the forward.
  // G-step: reconstruct x2 = y2 - G(bf16(y1)); G's grads for cotangent dy2
  if ((rc = to_bf16(y1, zb, Td, s)) != TQP_OK) return rc;
  uint16_t* gu = carve_bwd(static_cast<char*>(lws) + layer_ws_size(T, G), T, G).gu;
  if ((rc = layer_forward(zb, T, G, y2, 1, -1.0f, x2, 0, nullptr, lws, dev_status, s, gu, true)) != TQP_OK) return rc;
  // dz1 = dy1 + J_G^T dy2 -> dx1 (dx1 = dz1), the sum taken inside G's backward
  if ((rc = layer_backward(zb, dy2, T, G, dx1, gG, lws, dev_status, s, false, dy1)) != TQP_OK) return rc;
  // F-step: x1 = y1 - F(x2); F's grads for cotangent dz1; dx2 = dy2 + J_F^T dz1
  gu = carve_bwd(static_cast<char*>(lws) + layer_ws_size(T, F), T, F).gu;
  if ((rc = layer_forward(x2, T, F, y1, 1, -1.0f, x1, 0, nullptr, lws, dev_status, s, gu, true)) != TQP_OK) return rc;
  return layer_backward(x2, dx1, T, F, dx2, gF, lws, dev_status, s, false, dy2);
}

size_t rev_stack_workspace_size(int T, int L, const tqp_moe_weights* const* F, const tqp_moe_weights* const* G) {
  if (check_stack(T, L, F, G, false) != TQP_OK) return 0;
  return stack_ws_size(T, L, F, G);
}

int rev_stack_fwd(const uint16_t* x1, const uint16_t* x2, int T, int L, const tqp_moe_weights* const* F,
                  const tqp_moe_weights* const* G, float* y1, float* y2, void* ws, size_t ws_bytes,
                  int32_t* dev_status, void* stream) {
  int rc;
  if ((rc = check_stack(T, L, F, G, false)) != TQP_OK) return rc;
  const bool n = T > 0;
  if (!ptr_ok(x1, n) || !ptr_ok(x2, n) || !ptr_ok(y1, n) || !ptr_ok(y2, n) || !ptr_ok(ws, n))
    return TQP_ERR_INVALID_ARG;
  if (!n) return TQP_OK;
  if (ws_bytes < stack_ws_size(T, L, F, G)) return TQP_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const StackWs w = carve_stack(ws, T, F[0]->d);
  const size_t Td = size_t(T) * F[0]->d;
  for (int l = 0; l < L; ++l) {
    float* b1 = (l == L - 1) ? y1 : w.s[l & 1][0];
    float* b2 = (l == L - 1) ? y2 : w.s[l & 1][1];
    if (l == 0) {
      // b1 = x1 + F(x2), with bf16(b1) for G; b2 = x2 + G(bf16(b1)) (x1, x2 and F's
      // input put on the stream grid)
      if ((rc = to_stream_grid_bf16(x2, w.ab, Td, s)) != TQP_OK) return rc;
      if ((rc = layer_forward(w.ab, T, F[0], x1, 0, 1.0f, b1, 1, w.zb, w.lws, dev_status, s, nullptr, true)) != TQP_OK)
        return rc;
      if ((rc = layer_forward(w.zb, T, G[0], x2, 0, 1.0f, b2, 1, nullptr, w.lws, dev_status, s, nullptr, true)) !=
          TQP_OK)
        return rc;
    } else {
      const float* a1 = w.s[(l - 1) & 1][0];
      const float* a2 = w.s[(l - 1) & 1][1];
      if ((rc = to_bf16(a2, w.ab, Td, s)) != TQP_OK) return rc;
      if ((rc = layer_forward(w.ab, T, F[l], a1, 1, 1.0f, b1, 1, w.zb, w.lws, dev_status, s, nullptr, true)) !=
          TQP_OK)
        return rc;
      if ((rc = layer_forward(w.zb, T, G[l], a2, 1, 1.0f, b2, 1, nullptr, w.lws, dev_status, s, nullptr, true)) !=
          TQP_OK)
        return rc;
    }
  }
  return TQP_OK;
}

int rev_stack_inv(const float* y1, const float* y2, int T, int L, const tqp_moe_weights* const* F,
                  const tqp_moe_weights* const* G, uint16_t* x1, uint16_t* x2, void* ws, size_t ws_bytes,
                  int32_t* dev_status, void* stream) {
  int rc;
  if ((rc = check_stack(T, L, F, G, false)) != TQP_OK) return rc;
  const bool n = T > 0;
  if (!ptr_ok(x1, n) || !ptr_ok(x2, n) || !ptr_ok(y1, n) || !ptr_ok(y2, n) || !ptr_ok(ws, n))
    return TQP_ERR_INVALID_ARG;
  if (!n) return TQP_OK;
  if (ws_bytes < stack_ws_size(T, L, F, G)) return TQP_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const StackWs w = carve_stack(ws, T, F[0]->d);
  const size_t Td = size_t(T) * F[0]->d;
  const float* c1 = y1;
  const float* c2 = y2;
  for (int l = L - 1; l >= 0; --l) {
    if ((rc = to_bf16(c1, w.zb, Td, s)) != TQP_OK) return rc;
    if (l == 0) {
      // the block inputs are bf16: x2 = y2 - G(bf16(y1)), x1 = y1 - F(x2)
      if ((rc = layer_forward(w.zb, T, G[0], c2, 1, -1.0f, x2, 0, nullptr, w.lws, dev_status, s, nullptr, true)) !=
          TQP_OK)
        return rc;
      return layer_forward(x2, T, F[0], c1, 1, -1.0f, x1, 0, nullptr, w.lws, dev_status, s, nullptr, true);
    }
    float* a1 = w.s[l & 1][0];
    float* a2 = w.s[l & 1][1];
    if ((rc = layer_forward(w.zb, T, G[l], c2, 1, -1.0f, a2, 1, w.ab, w.lws, dev_status, s, nullptr, true)) != TQP_OK)
      return rc;
    if ((rc = layer_forward(w.ab, T, F[l], c1, 1, -1.0f, a1, 1, nullptr, w.lws, dev_status, s, nullptr, true)) !=
        TQP_OK)
      return rc;
    c1 = a1;
    c2 = a2;
  }
  return TQP_OK;
}

int rev_stack_bwd(const float* y1, const float* y2, const float* dy1, const float* dy2, int T, int L,
                  const tqp_moe_weights* const* F, const tqp_moe_weights* const* G, uint16_t* x1, uint16_t* x2,
                  float* dx1, float* dx2, const tqp_adapter_grads* const* gF, const tqp_adapter_grads* const* gG,
                  void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
  int rc;
  if ((rc = check_stack(T, L, F, G, true)) != TQP_OK) return rc;
  if (!gF || !gG) return TQP_ERR_INVALID_ARG;
  for (int l = 0; l < L; ++l)
    if (!grads_ok(F[l], gF[l]) || !grads_ok(G[l], gG[l])) return TQP_ERR_INVALID_ARG;
  const bool n = T > 0;
  if (!ptr_ok(y1, n) || !ptr_ok(y2, n) || !ptr_ok(dy1, n) || !ptr_ok(dy2, n) || !ptr_ok(x1, n) || !ptr_ok(x2, n) ||
      !ptr_ok(dx1, n) || !ptr_ok(dx2, n) || !ptr_ok(ws, n))
    return TQP_ERR_INVALID_ARG;
  if (!n) return TQP_OK;
  if (ws_bytes < stack_ws_size(T, L, F, G)) return TQP_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const StackWs w = carve_stack(ws, T, F[0]->d);
  const size_t Td = size_t(T) * F[0]->d;
  const float *c1 = y1, *c2 = y2, *c3 = dy1, *c4 = dy2;
  for (int l = L - 1; l >= 0; --l) {
    float* const* o = w.s[l & 1];
    // block 0's cotangents are the call's outputs; its inputs are rounded to bf16 below
    float* da1 = (l == 0) ? dx1 : o[2];
    float* da2 = (l == 0) ? dx2 : o[3];
    if ((rc = block_backward_f32(c1, c2, c3, c4, T, F[l], G[l], o[0], o[1], da1, da2, gF[l], gG[l], w, dev_status,
                                 s)) != TQP_OK)
      return rc;
    c1 = o[0];
    c2 = o[1];
    c3 = da1;
    c4 = da2;
  }
  if ((rc = to_bf16(c1, x1, Td, s)) != TQP_OK) return rc;
  return to_bf16(c2, x2, Td, s);
}

int tqp_debug_set_wait_limit_ns(unsigned long long ns) {
  g_wait_limit_ns.store(ns, std::memory_order_relaxed);
  return TQP_OK;
}

}  // extern "C"
