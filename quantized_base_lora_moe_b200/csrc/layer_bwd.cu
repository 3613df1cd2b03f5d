// Backward of the TQP MoE layer: adapters only, with the quantised base weights
// and the router frozen (TQP Quantization; Principle 3 / Pattern 3 of
// "Reversible Sparse MoE Single Node" keep optimizer state on the adapters).
//
// The dense dgrad contractions and the rank-space products dhA = s dO Bd^T and
// dxa = s [dG|dU] [Bg|Bu]^T run on the tensor cores (launch_dgrad and
// launch_rank_bwd in grouped_gemm.cu). This file holds the rest:
//   absmax       : max|dy|, from which every fp16 intermediate is computed for
//                  dy * 2^P (P chosen so that dO peaks near 2^8) and the fp32
//                  gradients are scaled back by 2^-P, so that the fp16 path
//                  neither underflows nor overflows whatever the size of dy
//   bwd_combine  : dO = gamma * dy * 2^P (fp16, permuted rows), dgamma = <dy, O>, the
//                  softmax-over-chosen backward dl = gamma (dgamma - sum gamma dgamma)
//                  and the frozen router's input gradient sum_j dl_j W_r[id_j]
//   outer        : per-expert adapter gradients, sums over the expert's routed rows
//                  of outer products (dA^T, dB^T in the storage layouts)
//   gather_add   : dx[t] += sum_j dX[row(t, j)]
#include <cstdint>
#include <cuda_runtime.h>

#include "tqp_device.cuh"
#include "tqp_launch.h"

namespace tqp {

// ----------------------------------------------------------------------------
// cotangent scale
// ----------------------------------------------------------------------------

// dmax = max |dy| as the bits of a non-negative float (ordered like unsigned
// integers), by atomicMax; dmax must be zeroed first.
__global__ void __launch_bounds__(256) absmax_kernel(const float* __restrict__ x, size_t n4, uint32_t* dmax) {
  uint32_t m = 0;
  for (size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n4; i += size_t(gridDim.x) * blockDim.x) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(x) + i);
    m = max(m, max(max(__float_as_uint(fabsf(v.x)), __float_as_uint(fabsf(v.y))),
                   max(__float_as_uint(fabsf(v.z)), __float_as_uint(fabsf(v.w)))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m) atomicMax(dmax, m);
}

// 2^P with max|dy| * 2^P in [2^7, 2^8); 1 when dy is all zeros or not finite.
__device__ __forceinline__ float grad_scale(const uint32_t* dmax) {
  const float m = __uint_as_float(*dmax);
  if (!(m > 0.0f) || !isfinite(m)) return 1.0f;
  int e;
  frexpf(m, &e);   // m = f * 2^e, 0.5 <= f < 1
  return ldexpf(1.0f, max(-120, min(120, 8 - e)));
}

// ----------------------------------------------------------------------------
// combine backward + softmax-gate backward + router input gradient
// ----------------------------------------------------------------------------

constexpr int kMaxK = 32;

// One block per token. The token's slots (row, gate, expert) go to shared memory
// first; the O and router rows are then loaded four slots at a time, so that
// their latencies overlap, and each slot's dot product <dy, O> is reduced per
// warp straight into shared memory.
__global__ void __launch_bounds__(256) bwd_combine_kernel(const uint16_t* __restrict__ O, const int32_t* __restrict__ inv,
                                                          const float* __restrict__ gates,
                                                          const int32_t* __restrict__ ids,
                                                          const float* __restrict__ router_w,
                                                          const float* __restrict__ dy, int T, int k, int d,
                                                          const uint32_t* __restrict__ dmax, uint16_t* __restrict__ dO,
                                                          const float* __restrict__ addend, float* __restrict__ dx,
                                                          int32_t* status) {
  __shared__ float red[8][kMaxK];
  __shared__ float dl_s[kMaxK];
  __shared__ int row_s[kMaxK], id_s[kMaxK];
  __shared__ float g_s[kMaxK];
  const int t = blockIdx.x;
  const float gsc = grad_scale(dmax);
  uint32_t bad = 0;
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  if (threadIdx.x < k) {
    row_s[threadIdx.x] = inv[size_t(t) * k + threadIdx.x];
    id_s[threadIdx.x] = ids[size_t(t) * k + threadIdx.x];
    g_s[threadIdx.x] = gates[size_t(t) * k + threadIdx.x];
  }
  for (int i = threadIdx.x; i < 8 * kMaxK; i += blockDim.x) (&red[0][0])[i] = 0.0f;
  __syncthreads();
  // the column loop runs whole warps (lanes past d idle inside it), so the
  // full-mask shuffles below always see all 32 lanes
  for (int cw = (threadIdx.x & ~31) * 8; cw < d; cw += blockDim.x * 8) {
    const int c = cw + lane * 8;
    const bool act = c < d;
    float4 a0 = make_float4(0.0f, 0.0f, 0.0f, 0.0f), a1 = a0;
    if (act) {
      const float4* dp = reinterpret_cast<const float4*>(dy + size_t(t) * d + c);
      a0 = __ldg(dp);
      a1 = __ldg(dp + 1);
    }
    const float dv[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
    for (int j0 = 0; j0 < k; j0 += 4) {
      uint4 ov[4];
#pragma unroll
      for (int b = 0; b < 4; ++b)
        ov[b] = (act && j0 + b < k) ? __ldg(reinterpret_cast<const uint4*>(O + size_t(row_s[j0 + b]) * d + c))
                                    : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = j0 + b;
        if (j >= k) break;
        const float g = g_s[j] * gsc;
        const uint32_t ow[4] = {ov[b].x, ov[b].y, ov[b].z, ov[b].w};
        float acc = 0.0f;
        uint32_t pk[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc = fmaf(dv[2 * q], f16_to_f32(uint16_t(ow[q] & 0xFFFFu)), acc);
          acc = fmaf(dv[2 * q + 1], f16_to_f32(uint16_t(ow[q] >> 16)), acc);
          pk[q] = pack_f16x2(g * dv[2 * q], g * dv[2 * q + 1]);
          bad |= f16x2_nonfinite(pk[q]);
        }
        if (act) *reinterpret_cast<uint4*>(dO + size_t(row_s[j]) * d + c) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        // dgamma_j partial of this warp's columns
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, o);
        if (lane == 0) red[wid][j] += acc;
      }
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad != 0) && lane == 0) raise_status(status, TQP_STATUS_NONFINITE);
  __syncthreads();
  if (wid == 0) {
    // lane j < k: dgamma_j over the warps' partials, then the softmax backward over
    // the chosen logits, dl_j = gamma_j (dgamma_j - sum_i gamma_i dgamma_i)
    float v = 0.0f;
    if (lane < k)
      for (int w = 0; w < nwarps; ++w) v += red[w][lane];
    const float gj = lane < k ? g_s[lane] : 0.0f;
    float sum = gj * v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
    if (lane < k) dl_s[lane] = gj * (v - sum);
  }
  __syncthreads();
  // dx[t] = addend[t] + sum_j dl_j W_r[id_j]  (through the frozen full-precision router)
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8) {
    float acc[8];
    if (addend) {
      const float4* ap = reinterpret_cast<const float4*>(addend + size_t(t) * d + c);
      const float4 b0 = __ldg(ap), b1 = __ldg(ap + 1);
      acc[0] = b0.x; acc[1] = b0.y; acc[2] = b0.z; acc[3] = b0.w;
      acc[4] = b1.x; acc[5] = b1.y; acc[6] = b1.z; acc[7] = b1.w;
    } else {
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    }
    for (int j0 = 0; j0 < k; j0 += 4) {
      float4 w[4][2];
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (j0 + b < k) {
          const float4* wp = reinterpret_cast<const float4*>(router_w + size_t(id_s[j0 + b]) * d + c);
          w[b][0] = __ldg(wp);
          w[b][1] = __ldg(wp + 1);
        } else {
          w[b][0] = w[b][1] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
        }
      }
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float l = (j0 + b < k) ? dl_s[j0 + b] : 0.0f;
        const float wv[8] = {w[b][0].x, w[b][0].y, w[b][0].z, w[b][0].w, w[b][1].x, w[b][1].y, w[b][1].z, w[b][1].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = fmaf(l, wv[i], acc[i]);
      }
    }
    float4* xp = reinterpret_cast<float4*>(dx + size_t(t) * d + c);
    xp[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    xp[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
}

// dx[t] += 2^-P sum_j dX[inv[t*k + j]]  (fp16 rows computed for dy * 2^P, fp32
// accumulation, fixed j order)
__global__ void __launch_bounds__(256) gather_add_kernel(const uint16_t* __restrict__ dX, const int32_t* __restrict__ inv,
                                                         int T, int k, int d, const uint32_t* __restrict__ dmax,
                                                         float* __restrict__ dx) {
  const int t = blockIdx.x;
  const float inv_sc = 1.0f / grad_scale(dmax);   // a power of two: exact
  for (int c = threadIdx.x * 8; c < d; c += blockDim.x * 8) {
    float4* xp = reinterpret_cast<float4*>(dx + size_t(t) * d + c);
    const float4 b0 = xp[0], b1 = xp[1];
    float acc[8] = {0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f, 0.0f};
    // four slots' rows in flight at a time; the sum keeps the fixed j order
    for (int j0 = 0; j0 < k; j0 += 4) {
      uint4 v[4];
#pragma unroll
      for (int b = 0; b < 4; ++b)
        v[b] = (j0 + b < k) ? __ldg(reinterpret_cast<const uint4*>(dX + size_t(__ldg(inv + size_t(t) * k + j0 + b)) * d + c))
                            : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (j0 + b >= k) break;
        const uint32_t w[4] = {v[b].x, v[b].y, v[b].z, v[b].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[2 * q] += f16_to_f32(uint16_t(w[q] & 0xFFFFu));
          acc[2 * q + 1] += f16_to_f32(uint16_t(w[q] >> 16));
        }
      }
    }
    xp[0] = make_float4(fmaf(acc[0], inv_sc, b0.x), fmaf(acc[1], inv_sc, b0.y), fmaf(acc[2], inv_sc, b0.z),
                        fmaf(acc[3], inv_sc, b0.w));
    xp[1] = make_float4(fmaf(acc[4], inv_sc, b1.x), fmaf(acc[5], inv_sc, b1.y), fmaf(acc[6], inv_sc, b1.z),
                        fmaf(acc[7], inv_sc, b1.w));
  }
}

// ----------------------------------------------------------------------------
// adapter gradients: C[e][m][n] = sum_{rows of e} P(row, m) * Q(row, n)
// ----------------------------------------------------------------------------

struct OuterArgs {
  int E, M, N;
  const int32_t* offsets;
  const int32_t* perm;       // row gather for Q (token rows of x), or null
  const uint16_t* P;         // fp16, row stride ldp, column offset offp
  int ldp, offp;
  const uint16_t* Q;
  int ldq, offq;
  float* C;                  // fp32 [E][M][N]
  const uint32_t* dmax;      // the cotangent's max |dy|: C is scaled back by 2^-P
};

// One block computes a TM x TN tile of C[e] (TM x TN = 4096, 4 x 4 per thread)
// over all routed rows of expert e, 32 rows at a time. Rows are read as 16-byte
// pieces (8 fp16 values; M, N, the strides and the column offsets are multiples
// of 8). The tile shape follows the operand widths: one of M, N is the rank r,
// so a 64 x 64 tile would leave half its FMAs on zero padding when r = 32.
template <int TM, int TN>
__global__ void __launch_bounds__(256) outer_kernel(const OuterArgs a) {
  static_assert(TM * TN == 4096, "4 x 4 outputs per thread");
  __shared__ __align__(16) float Ps[32][TM + 4];
  __shared__ __align__(16) float Qs[32][TN + 4];
  const int e = blockIdx.x;
  const int m0 = blockIdx.y * TM, n0 = blockIdx.z * TN;
  const int tx = threadIdx.x % (TN / 4), ty = threadIdx.x / (TN / 4);
  const int r0 = a.offsets[e], r1 = a.offsets[e + 1];
  float acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0f;
  auto stage8 = [](float* dst, uint4 v) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      f[2 * t] = f16_to_f32(uint16_t(w[t] & 0xFFFFu));
      f[2 * t + 1] = f16_to_f32(uint16_t(w[t] >> 16));
    }
    *reinterpret_cast<float4*>(dst) = make_float4(f[0], f[1], f[2], f[3]);
    *reinterpret_cast<float4*>(dst + 4) = make_float4(f[4], f[5], f[6], f[7]);
  };
  for (int rb = r0; rb < r1; rb += 32) {
    __syncthreads();
    for (int i = threadIdx.x; i < 32 * (TM / 8); i += blockDim.x) {
      const int rr = i / (TM / 8), c = (i % (TM / 8)) * 8;
      const int row = rb + rr;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < r1 && m0 + c < a.M)
        v = __ldg(reinterpret_cast<const uint4*>(a.P + size_t(row) * a.ldp + a.offp + m0 + c));
      stage8(&Ps[rr][c], v);
    }
    for (int i = threadIdx.x; i < 32 * (TN / 8); i += blockDim.x) {
      const int rr = i / (TN / 8), c = (i % (TN / 8)) * 8;
      const int row = rb + rr;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < r1 && n0 + c < a.N) {
        const int qrow = a.perm ? __ldg(a.perm + row) : row;
        v = __ldg(reinterpret_cast<const uint4*>(a.Q + size_t(qrow) * a.ldq + a.offq + n0 + c));
      }
      stage8(&Qs[rr][c], v);
    }
    __syncthreads();
#pragma unroll 8
    for (int rr = 0; rr < 32; ++rr) {
      const float4 pv = *reinterpret_cast<const float4*>(&Ps[rr][ty * 4]);
      const float4 qv = *reinterpret_cast<const float4*>(&Qs[rr][tx * 4]);
      const float p4[4] = {pv.x, pv.y, pv.z, pv.w}, q4[4] = {qv.x, qv.y, qv.z, qv.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(p4[i], q4[j], acc[i][j]);
    }
  }
  const float inv_sc = 1.0f / grad_scale(a.dmax);   // a power of two: exact
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < a.N) a.C[(size_t(e) * a.M + m) * a.N + n] = acc[i][j] * inv_sc;
    }
  }
}

// ----------------------------------------------------------------------------
// host launchers
// ----------------------------------------------------------------------------

int launch_grad_absmax(const float* dy, size_t n, uint32_t* dmax, cudaStream_t s) {
  if (cudaMemsetAsync(dmax, 0, sizeof(uint32_t), s) != cudaSuccess) return TQP_ERR_CUDA;
  const size_t n4 = n / 4;
  if (n4 == 0) return TQP_OK;
  const size_t blocks = (n4 + 255) / 256;
  const int grid = int(blocks < size_t(4 * num_sms()) ? blocks : size_t(4 * num_sms()));
  absmax_kernel<<<grid, 256, 0, s>>>(dy, n4, dmax);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

int launch_bwd_combine(const uint16_t* O, const int32_t* inv, const float* gates, const int32_t* ids,
                       const float* router_w, const float* dy, int T, int k, int d, const uint32_t* dmax, uint16_t* dO,
                       const float* addend, float* dx, int32_t* status, cudaStream_t s) {
  if (T == 0) return TQP_OK;
  // whole warps only: the row reductions use full-mask warp shuffles
  const int threads = d / 8 >= 256 ? 256 : ((d / 8 + 31) / 32) * 32;
  bwd_combine_kernel<<<T, threads, 0, s>>>(O, inv, gates, ids, router_w, dy, T, k, d, dmax, dO, addend, dx, status);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

int launch_gather_add(const uint16_t* dX, const int32_t* inv, int T, int k, int d, const uint32_t* dmax, float* dx,
                      cudaStream_t s) {
  if (T == 0) return TQP_OK;
  const int threads = d / 8 < 256 ? d / 8 : 256;
  gather_add_kernel<<<T, threads, 0, s>>>(dX, inv, T, k, d, dmax, dx);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

int launch_outer(int E, int M, int N, const int32_t* offsets, const int32_t* perm, const uint16_t* P, int ldp,
                 int offp, const uint16_t* Q, int ldq, int offq, float* C, const uint32_t* dmax, cudaStream_t s) {
  OuterArgs a{};
  a.dmax = dmax;
  a.E = E;
  a.M = M;
  a.N = N;
  a.offsets = offsets;
  a.perm = perm;
  a.P = P;
  a.ldp = ldp;
  a.offp = offp;
  a.Q = Q;
  a.ldq = ldq;
  a.offq = offq;
  a.C = C;
  if (N <= 32) {
    outer_kernel<128, 32><<<dim3(E, (M + 127) / 128, (N + 31) / 32), 256, 0, s>>>(a);
  } else if (M <= 32) {
    outer_kernel<32, 128><<<dim3(E, (M + 31) / 32, (N + 127) / 128), 256, 0, s>>>(a);
  } else {
    outer_kernel<64, 64><<<dim3(E, (M + 63) / 64, (N + 63) / 64), 256, 0, s>>>(a);
  }
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

}  // namespace tqp
