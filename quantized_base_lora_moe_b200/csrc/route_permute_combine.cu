// Routing, permutation and combine kernels of the TQP MoE layer (sm_100a).
//
//  moe_route    : one warp per token; top-k by k rounds of warp arg-max over an
//                 orderable 32-bit logit key, exact ties broken by the lower
//                 expert id; renormalised softmax over the chosen logits ("Top-12 routing",
//                 Architecture Details; stateless routing, Reversibility
//                 Implementation).
//  moe_permute  : stable counting sort by expert in three passes: per 32-token
//                 chunk expert bitmaps -> per-expert column prefix over chunks
//                 (block-parallel) -> scatter with rank = popcount of earlier
//                 tokens' bits.
//  moe_combine  : gate-weighted gather back to token order (fixed j order, fp32,
//                 no atomics) with the additive coupling fused in ("Pattern 1":
//                 addition/subtraction are invertible).
#include <cstdint>
#include <cuda_runtime.h>

#include "tqp_device.cuh"
#include "tqp_launch.h"

namespace tqp {

// ----------------------------------------------------------------------------
// moe_route
// ----------------------------------------------------------------------------

// Orderable key: larger key = larger logit; +0.0 == -0.0; NaN lowest.
__device__ __forceinline__ uint32_t logit_key(float v) {
  if (v != v) return 0u;
  if (v == 0.0f) v = 0.0f;
  const uint32_t b = __float_as_uint(v);
  return (b & 0x80000000u) ? (~b) : (b | 0x80000000u);
}

// (one warp-wide reduction instruction each)
__device__ __forceinline__ uint32_t warp_max_u32(uint32_t v) { return __reduce_max_sync(0xFFFFFFFFu, v); }

__device__ __forceinline__ uint32_t warp_min_u32(uint32_t v) { return __reduce_min_sync(0xFFFFFFFFu, v); }

// One warp per token. Lane l holds the orderable keys of experts l, l+32, ...
// Each of the k rounds takes every lane's best key not yet chosen (lowest
// expert id among equal keys: the lane's elements are visited in increasing
// id order), the warp maximum of those, and among the lanes that hold it the
// lowest expert id (one ballot; a min-reduction only when several lanes tie).
// The winner lane marks its element as chosen.
// Up to 16 logits per lane (E <= 512) the kernel is held to 32 registers, so that
// 8 blocks fit an SM and the 1024 blocks of an 8192-token batch run in one wave.
template <int EPL>  // logits per lane kept in registers (E <= 32 * EPL)
__global__ void __launch_bounds__(256, EPL <= 16 ? 8 : 1) route_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                    int32_t* __restrict__ ids, float* __restrict__ gates,
                                                    int32_t* status) {
  constexpr int NW = (EPL + 31) / 32;   // exclusion mask words
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  const float* row = logits + size_t(t) * E;
  uint32_t key[EPL];
  bool nonfinite = false;
  uint32_t excl[NW];   // bit i: element lane + 32 i chosen already, or past E
#pragma unroll
  for (int w = 0; w < NW; ++w) excl[w] = 0u;
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < E) {
      const float v = __ldg(row + e);
      nonfinite |= !isfinite(v);
      key[i] = logit_key(v);
    } else {
      key[i] = 0u;
      excl[i >> 5] |= 1u << (i & 31);
    }
  }
  if (__any_sync(0xFFFFFFFFu, nonfinite) && lane == 0) raise_status(status, TQP_STATUS_NONFINITE);

  int my_id = 0;
  float my_val = 0.0f;
  for (int j = 0; j < k; ++j) {
    uint32_t best = 0u;
    int bi = -1;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const bool take = !((excl[i >> 5] >> (i & 31)) & 1u) && (bi < 0 || key[i] > best);
      best = take ? key[i] : best;
      bi = take ? i : bi;
    }
    const uint32_t m = warp_max_u32(bi >= 0 ? best : 0u);
    const uint32_t cand = __ballot_sync(0xFFFFFFFFu, bi >= 0 && best == m);
    int winner = __ffs(cand) - 1;                  // lowest lane; its id is lowest unless elements differ in i
    const uint32_t my = (bi >= 0 && ((cand >> lane) & 1u)) ? uint32_t(lane + 32 * bi) : 0xFFFFFFFFu;
    uint32_t wid;
    if (__popc(cand) == 1) {
      wid = __shfl_sync(0xFFFFFFFFu, my, winner);
    } else {
      wid = warp_min_u32(my);                      // exact tie between lanes: the lowest expert id
      winner = int(wid & 31u);
    }
    if (lane == winner) {
#pragma unroll
      for (int w = 0; w < NW; ++w)
        if (w == (bi >> 5)) excl[w] |= 1u << (bi & 31);
    }
    if (lane == j) {
      my_id = int(wid);
      my_val = __ldg(row + my_id);
    }
  }
  const float mx = __shfl_sync(0xFFFFFFFFu, my_val, 0);
  float ex = (lane < k) ? expf(my_val - mx) : 0.0f;
  float sum = ex;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  if (lane < k) {
    ids[size_t(t) * k + lane] = my_id;
    gates[size_t(t) * k + lane] = ex / sum;
  }
}

int launch_route(const float* logits, int T, int E, int k, int32_t* ids, float* gates, int32_t* status,
                 cudaStream_t s) {
  if (T == 0) return TQP_OK;
  const dim3 block(256);
  const dim3 grid((T + 7) / 8);
  const int epl = (E + 31) / 32;
#define TQP_ROUTE(N) route_kernel<N><<<grid, block, 0, s>>>(logits, T, E, k, ids, gates, status)
  if (epl <= 1) TQP_ROUTE(1);
  else if (epl <= 2) TQP_ROUTE(2);
  else if (epl <= 4) TQP_ROUTE(4);
  else if (epl <= 8) TQP_ROUTE(8);
  else if (epl <= 16) TQP_ROUTE(16);
  else if (epl <= 32) TQP_ROUTE(32);
  else if (epl <= 64) TQP_ROUTE(64);
  else TQP_ROUTE(128);
#undef TQP_ROUTE
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

// ----------------------------------------------------------------------------
// moe_permute
// ----------------------------------------------------------------------------

// Pass 1: per 32-token chunk w, count[w][e] = #tokens of the chunk routed to e.
// An id outside [0, E), or a token that lists one expert twice (its bit is
// already set when the second slot is recorded), raises TQP_STATUS_BAD_ID.
__global__ void permute_count_kernel(const int32_t* __restrict__ ids, int T, int E, int k,
                                     int32_t* __restrict__ count, int32_t* status) {
  extern __shared__ uint32_t bits_all[];
  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int w = blockIdx.x * (blockDim.x >> 5) + wib;
  const int W = (T + 31) / 32;
  if (w >= W) return;
  uint32_t* bits = bits_all + size_t(wib) * E;
  for (int e = lane; e < E; e += 32) bits[e] = 0u;
  __syncwarp();
  const int t = w * 32 + lane;
  bool bad = false;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[size_t(t) * k + j];
      if (e >= 0 && e < E) bad |= (atomicOr(&bits[e], 1u << lane) & (1u << lane)) != 0u;
      else bad = true;
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad) && lane == 0) raise_status(status, TQP_STATUS_BAD_ID);
  __syncwarp();
  for (int e = lane; e < E; e += 32) count[size_t(w) * E + e] = __popc(bits[e]);
}

// Pass 2: exclusive prefix of count[.][e] over the chunks (in place) and the
// expert totals. A block takes 32 experts (lane = expert, so every row access
// is one coalesced 128-byte piece); its warps split the chunks into slices,
// sum their slices, take the prefix over the earlier slices from shared
// memory, and rewrite their slices with the running prefix.
__global__ void __launch_bounds__(1024) permute_colscan_kernel(int32_t* __restrict__ count, int W, int E,
                                                               int32_t* __restrict__ total) {
  __shared__ int32_t part[32][33];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int e = blockIdx.x * 32 + lane;
  const int per = (W + nw - 1) / nw;
  const int w0 = min(W, wid * per), w1 = min(W, w0 + per);
  int sum = 0;
  if (e < E)
    for (int w = w0; w < w1; ++w) sum += count[size_t(w) * E + e];
  part[wid][lane] = sum;
  __syncthreads();
  int run = 0;
  for (int i = 0; i < wid; ++i) run += part[i][lane];
  if (e < E) {
    for (int w = w0; w < w1; ++w) {
      const size_t i = size_t(w) * E + e;
      const int c = count[i];
      count[i] = run;
      run += c;
    }
    if (wid == nw - 1) total[e] = run;
  }
}

// Block-wide exclusive scan of total[0..E) into off[0..E] (shared memory).
__device__ void block_exclusive_scan(const int32_t* __restrict__ total, int E, int32_t* off, int32_t* warp_sums) {
  const int nt = blockDim.x;
  const int per = (E + nt - 1) / nt;
  const int lo = threadIdx.x * per;
  const int hi = min(E, lo + per);
  int local = 0;
  for (int e = lo; e < hi; ++e) local += total[e];
  // inclusive warp scan of the per-thread sums
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xFFFFFFFFu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) warp_sums[wid] = v;
  __syncthreads();
  if (wid == 0) {
    int s = (lane < (nt >> 5)) ? warp_sums[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xFFFFFFFFu, s, o);
      if (lane >= o) s += u;
    }
    if (lane < (nt >> 5)) warp_sums[lane] = s;  // inclusive
  }
  __syncthreads();
  int run = v - local + (wid > 0 ? warp_sums[wid - 1] : 0);
  for (int e = lo; e < hi; ++e) {
    off[e] = run;
    run += total[e];
  }
  if (threadIdx.x == nt - 1) off[E] = run;
  __syncthreads();
}

// Pass 3: scatter. Row of (t, j) with expert e = offsets[e] + prefix[w][e] +
// #earlier tokens of the chunk routed to e.
__global__ void permute_scatter_kernel(const int32_t* __restrict__ ids, int T, int E, int k,
                                       const int32_t* __restrict__ prefix, const int32_t* __restrict__ total,
                                       int32_t* __restrict__ offsets, int32_t* __restrict__ perm_token,
                                       int32_t* __restrict__ inv, int warps_per_block) {
  extern __shared__ int32_t smem_i[];
  int32_t* off = smem_i;                       // E + 1
  int32_t* warp_sums = smem_i + E + 1;         // 32
  uint32_t* bits_all = reinterpret_cast<uint32_t*>(smem_i + E + 1 + 32);
  block_exclusive_scan(total, E, off, warp_sums);
  if (blockIdx.x == 0)
    for (int e = threadIdx.x; e <= E; e += blockDim.x) offsets[e] = off[e];

  const int lane = threadIdx.x & 31;
  const int wib = threadIdx.x >> 5;
  const int w = blockIdx.x * warps_per_block + wib;
  const int W = (T + 31) / 32;
  if (w >= W) return;
  uint32_t* bits = bits_all + size_t(wib) * E;
  for (int e = lane; e < E; e += 32) bits[e] = 0u;
  __syncwarp();
  const int t = w * 32 + lane;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = ids[size_t(t) * k + j];
      if (e >= 0 && e < E) atomicOr(&bits[e], 1u << lane);
    }
  }
  __syncwarp();
  if (t < T) {
    const uint32_t lt = (1u << lane) - 1u;
    for (int j = 0; j < k; ++j) {
      const int e = ids[size_t(t) * k + j];
      if (e < 0 || e >= E) continue;
      const int row = off[e] + prefix[size_t(w) * E + e] + __popc(bits[e] & lt);
      perm_token[row] = t;
      inv[size_t(t) * k + j] = row;
    }
  }
}

size_t permute_ws_bytes(int T, int E) {
  const size_t W = (size_t(T) + 31) / 32;
  return align_up(W * E * 4, 256) + align_up(size_t(E) * 4, 256);
}

int launch_permute(const int32_t* ids, int T, int E, int k, int32_t* offsets, int32_t* perm_token, int32_t* inv,
                   void* ws, int32_t* status, cudaStream_t s) {
  if (T == 0) {
    return cudaMemsetAsync(offsets, 0, sizeof(int32_t) * (E + 1), s) == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
  }
  const int W = (T + 31) / 32;
  int32_t* count = static_cast<int32_t*>(ws);
  int32_t* total = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + align_up(size_t(W) * E * 4, 256));
  // pass 1
  int wpb = 8;
  while (wpb > 1 && size_t(wpb) * E * 4 > 64 * 1024) wpb >>= 1;
  const size_t smem1 = size_t(wpb) * E * 4;
  // the largest dynamic shared memory either pass can ask for (E <= 4096), set
  // once per device
  static DeviceFlags count_attr, scatter_attr;
  if (smem1 > 48 * 1024 && !count_attr.test_and_set_device(permute_count_kernel, 64 * 1024)) return TQP_ERR_CUDA;
  permute_count_kernel<<<(W + wpb - 1) / wpb, wpb * 32, smem1, s>>>(ids, T, E, k, count, status);
  // pass 2
  // 32 warps per block whatever W: each warp's serial run over its chunks stays short
  permute_colscan_kernel<<<(E + 31) / 32, 1024, 0, s>>>(count, W, E, total);
  // pass 3
  const size_t smem3 = size_t(E + 1 + 32) * 4 + size_t(wpb) * E * 4;
  if (smem3 > 48 * 1024 && !scatter_attr.test_and_set_device(permute_scatter_kernel, (4096 + 1 + 32) * 4 + 64 * 1024))
    return TQP_ERR_CUDA;
  permute_scatter_kernel<<<(W + wpb - 1) / wpb, wpb * 32, smem3, s>>>(ids, T, E, k, count, total, offsets,
                                                                      perm_token, inv, wpb);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

// ----------------------------------------------------------------------------
// moe_combine
// ----------------------------------------------------------------------------

constexpr int kCombMaxK = 32;   // top-k limit of the C ABI

// One block per token row; each thread owns 8 consecutive columns (16 B of bf16).
// grid (with a residual): the coupling's stream format. The residual and the
// branch m are rounded to multiples of 2^-kStreamGridBits, so that
// residual +- m is exact in fp32 while |y| < kStreamMax (24-bit significand);
// a y outside that range raises TQP_STATUS_RANGE.
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ out_perm,
                                                      const int32_t* __restrict__ inv,
                                                      const float* __restrict__ gates, int T, int k, int d,
                                                      const void* __restrict__ residual, int residual_f32,
                                                      float sign, void* __restrict__ y, int y_f32,
                                                      uint16_t* __restrict__ y_bf16, int grid,
                                                      int32_t* __restrict__ status) {
  // the token's slots (row, gate) in shared memory; the rows' pieces are then
  // loaded four slots at a time so that their latencies overlap (the sum keeps
  // the fixed j order)
  __shared__ int32_t row_s[kCombMaxK];
  __shared__ float g_s[kCombMaxK];
  const int t = blockIdx.x;
  for (int i = threadIdx.x; i < k; i += blockDim.x) {
    row_s[i] = __ldg(inv + size_t(t) * k + i);
    g_s[i] = __ldg(gates + size_t(t) * k + i);
  }
  __syncthreads();
  const int c0 = threadIdx.x * 8;
  for (int c = c0; c < d; c += blockDim.x * 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.0f;
    for (int j0 = 0; j0 < k; j0 += 4) {
      uint4 ov[4];
#pragma unroll
      for (int b = 0; b < 4; ++b)
        ov[b] = (j0 + b < k) ? __ldg(reinterpret_cast<const uint4*>(out_perm + size_t(row_s[j0 + b]) * d + c))
                             : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        if (j0 + b >= k) break;
        const float gmm = g_s[j0 + b];
        const uint32_t w[4] = {ov[b].x, ov[b].y, ov[b].z, ov[b].w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          acc[2 * i] = fmaf(gmm, f16_to_f32(uint16_t(w[i] & 0xFFFFu)), acc[2 * i]);
          acc[2 * i + 1] = fmaf(gmm, f16_to_f32(uint16_t(w[i] >> 16)), acc[2 * i + 1]);
        }
      }
    }
    float out[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) out[i] = bf16_to_f32(f32_to_bf16(acc[i]));   // m = bf16(sum)
    if (residual) {
      float res[8];
      if (residual_f32) {
        const float4* rp = reinterpret_cast<const float4*>(static_cast<const float*>(residual) + size_t(t) * d + c);
        const float4 a = __ldg(rp), b = __ldg(rp + 1);
        res[0] = a.x; res[1] = a.y; res[2] = a.z; res[3] = a.w;
        res[4] = b.x; res[5] = b.y; res[6] = b.z; res[7] = b.w;
      } else {
        const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(residual) + size_t(t) * d + c));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          res[2 * i] = __uint_as_float(w[i] << 16);
          res[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
        }
      }
      if (grid) {
        bool in_range = true;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          out[i] = to_stream_grid(res[i]) + sign * to_stream_grid(out[i]);
          in_range &= fabsf(out[i]) < kStreamMax;
        }
        if (!in_range && status) atomicOr(status, TQP_STATUS_RANGE);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) out[i] = res[i] + sign * out[i];
      }
    }
    uint4 ob;
    ob.x = pack_bf16x2(out[0], out[1]);
    ob.y = pack_bf16x2(out[2], out[3]);
    ob.z = pack_bf16x2(out[4], out[5]);
    ob.w = pack_bf16x2(out[6], out[7]);
    if (y_f32) {
      float4* yp = reinterpret_cast<float4*>(static_cast<float*>(y) + size_t(t) * d + c);
      yp[0] = make_float4(out[0], out[1], out[2], out[3]);
      yp[1] = make_float4(out[4], out[5], out[6], out[7]);
    } else {
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(y) + size_t(t) * d + c) = ob;
    }
    if (y_bf16) *reinterpret_cast<uint4*>(y_bf16 + size_t(t) * d + c) = ob;
  }
}

int launch_combine(const uint16_t* out_perm, const int32_t* inv, const float* gates, int T, int k, int d,
                   const void* residual, int residual_f32, float sign, void* y, int y_f32, uint16_t* y_bf16,
                   cudaStream_t s, bool grid, int32_t* status) {
  if (T == 0) return TQP_OK;
  const int threads = d / 8 < 256 ? d / 8 : 256;
  combine_kernel<<<T, threads, 0, s>>>(out_perm, inv, gates, T, k, d, residual, residual_f32, sign, y, y_f32,
                                       y_bf16, grid ? 1 : 0, status);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

}  // namespace tqp
