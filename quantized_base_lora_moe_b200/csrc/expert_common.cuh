// Epilogue helpers shared by the expert kernels (expert_gateup.cu, expert_down.cu).
#pragma once

#include <cstdint>
#include <cuda_fp16.h>

#include "tqp_device.cuh"

namespace tqp {

constexpr int kTRow = 272;   // staging row: one token's 128 features in fp16, +16 B against bank conflicts

// Barrier among the 4 warps of one epilogue group only, on an mbarrier so
// that the wait is bounded: false once the CTA has aborted or the limit expired.
// The barrier expects one arrival per warp when kPerWarp (else one per thread).
template <bool kPerWarp = false>
struct EpiSyncT {
  uint64_t* bar;
  uint32_t phase = 0;
  // The result is warp-uniform (the callers go on to warp-collective tcgen05 loads).
  __device__ __forceinline__ bool sync(Abort* abort_flag, int32_t* status) {
    bool ok;
    if (kPerWarp) {
      mbar_arrive_warp(bar);
      ok = mbar_wait_warp<32>(bar, phase, abort_flag, status);
    } else {
      mbar_arrive(bar);
      ok = __all_sync(0xFFFFFFFFu, mbar_wait<32>(bar, phase, abort_flag, status));
    }
    phase ^= 1u;
    return ok;
  }
};
using EpiSync = EpiSyncT<false>;

// 2*NW tokens x this lane's feature (NW words of fp16 pairs, word j = tokens
// t0+2j, t0+2j+1) into a [token][feature] tile: lane pairs trade halves so that
// each lane writes two adjacent features of one token as one 32-bit word.
template <int NW>
__device__ __forceinline__ void stage_tokens(uint8_t* tile, int t0, int row, const uint32_t* w) {
  const bool odd = (threadIdx.x & 1) != 0;
  uint8_t* colp = tile + (row & ~1) * 2;
#pragma unroll
  for (int j = 0; j < NW; ++j) {
    const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, w[j], 1);
    const uint32_t v = odd ? __byte_perm(other, w[j], 0x7632) : __byte_perm(w[j], other, 0x5410);
    *reinterpret_cast<uint32_t*>(colp + (t0 + 2 * j + (odd ? 1 : 0)) * kTRow) = v;
  }
}

__device__ __forceinline__ uint32_t f32x2_to_f16x2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// silu(g) * u for a pair of fp16 values each, as an fp16 pair
__device__ __forceinline__ uint32_t swiglu_pair(uint32_t g2, uint32_t u2) {
  const float2 g = __half22float2(*reinterpret_cast<const __half2*>(&g2));
  const float2 u = __half22float2(*reinterpret_cast<const __half2*>(&u2));
  const float h0 = __fdividef(g.x * u.x, 1.0f + __expf(-g.x));
  const float h1 = __fdividef(g.y * u.y, 1.0f + __expf(-g.y));
  return f32x2_to_f16x2(h0, h1);
}

}  // namespace tqp
