// Device-side pieces shared by the grouped GEMM kernels: work-unit arguments and
// decoding, pipeline ring counters, and the exact int4 -> fp16 dequantisation.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "tqp_device.cuh"

namespace tqp {

enum Mode : int { GATEUP = 0, LORA_XA = 2, LORA_HA = 3, ROUTER = 4, DH = 5, DX = 6 };

constexpr int kMBlock = 128;

struct GemmArgs {
  int E;
  int nkb_main;        // main K-blocks (64 wide)
  int kb_per_piece;    // ROUTER: K-blocks per bf16 part (the A columns repeat)
  int nkb_lora;        // rank-space K-blocks, issued first in each unit
  int lora_k;          // rank-space contraction extent (2r gate/up and dX, r down and dH)
  int n_tiles;         // n-tiles per m-block
  int ntile;           // MMA N (16..256)
  int g;               // quantisation group
  int r;               // LoRA rank
  int in_dim;          // input dim of the int4 projection (scale rows)
  int out_dim;         // output dim of the int4 projection (code rows)
  float lora_scale;
  const int32_t* offsets;
  const int32_t* mb_prefix;
  const int32_t* perm_token;
  const uint16_t* a_src;   // gathered A rows (GATEUP, LORA_XA)
  int a_ld;
  const uint16_t* a_lora;  // rank-space A rows [A][lora_ld]
  int lora_ld;
  const uint16_t* b0;      // rank-space B^T sources (GATEUP: Bg^T, DOWN: Bd^T)
  const uint16_t* b1;      // GATEUP: Bu^T
  void* out;
  int out_ld;
  int n_valid;             // valid output columns
  const float* bias;
  int32_t* status;
  uint16_t* aux;           // GATEUP: optional G|U pre-activations out [A][2f]; DH: G|U in
  int f_dim;
  int half_kb;             // DX: K-blocks of the gate part
  const uint16_t* lb0;     // DH / DX rank-space step: A^T sources read transposed (Ad^T | Ag^T)
  const uint16_t* lb1;     // DX: Au^T
  int lb_ld;
  const uint16_t* lt;      // DH / DX rank-space step, if set: the same A values row by row in fp16,
                           // [E][in][lt_w] (lt_w = lora_k), read as whole rows instead of lb0 / lb1
  int lt_w;
  const int4* unit_tab;    // expert kernels: decoded units {e, n-tile, rows, base}, one per unit
  int bits;                // base-weight code width: 4 (packed int4) or 8 (int8)
  unsigned long long wait_ns;   // limit of one barrier wait (0: the default kWaitLimitNs)
};

struct Unit {
  int e, nt, mb, rows, base;
};

// Expert schedule (m-block prefix and row offsets) as the kernels read it: a
// copy in shared memory when E <= kSchedSmemE (a unit then decodes in a few
// shared-memory loads instead of a chain of dependent global loads), else the
// global arrays.
constexpr int kSchedSmemE = 512;
struct Sched {
  const int32_t* mbp;
  const int32_t* off;
};

// Called by every thread before the kernel's first __syncthreads().
__device__ __forceinline__ Sched load_sched(const GemmArgs& a, int32_t* smem_sched) {
  if (a.E > kSchedSmemE) return Sched{a.mb_prefix, a.offsets};
  for (int i = threadIdx.x; i <= a.E; i += blockDim.x) {
    smem_sched[i] = __ldg(a.mb_prefix + i);
    smem_sched[kSchedSmemE + 1 + i] = __ldg(a.offsets + i);
  }
  return Sched{smem_sched, smem_sched + kSchedSmemE + 1};
}

__device__ __forceinline__ int total_units(const GemmArgs& a, const Sched& sc) { return sc.mbp[a.E] * a.n_tiles; }

// Units are ordered (expert, n-tile, m-block): m-blocks of one n-tile share a B
// tile, n-tiles of one m-block share the A rows; neighbours run concurrently.
__device__ __forceinline__ Unit decode_unit(const GemmArgs& a, const Sched& sc, int u) {
  int lo = 0, hi = a.E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (sc.mbp[mid] * a.n_tiles <= u) lo = mid;
    else hi = mid;
  }
  Unit un;
  un.e = lo;
  const int p0 = sc.mbp[lo];
  const int nmb = sc.mbp[lo + 1] - p0;
  const int idx = u - p0 * a.n_tiles;
  un.nt = idx / nmb;
  un.mb = idx - un.nt * nmb;
  const int o0 = sc.off[lo];
  const int cnt = sc.off[lo + 1] - o0;
  un.rows = min(kMBlock, cnt - un.mb * kMBlock);
  un.base = o0 + un.mb * kMBlock;
  return un;
}

// Units read from a table decoded beforehand (unit_table_kernel): one 16-byte
// load per unit, issued one unit ahead so that its latency stays off the
// consumer's critical path.
struct UnitStream {
  const int4* tab;
  int total, stride;
  int4 nxt;
  __device__ __forceinline__ void start(int u0) { nxt = u0 < total ? __ldg(tab + u0) : make_int4(0, 0, 0, 0); }
  // unit u (the one loaded last), and the load of unit u + stride
  __device__ __forceinline__ Unit take(int u) {
    const int4 c = nxt;
    if (u + stride < total) nxt = __ldg(tab + u + stride);
    Unit un;
    un.e = c.x;
    un.nt = c.y;
    un.mb = 0;
    un.rows = c.z;
    un.base = c.w;
    return un;
  }
  // the unit after the one last taken (valid when u + stride < total)
  __device__ __forceinline__ Unit peek() const {
    Unit un;
    un.e = nxt.x;
    un.nt = nxt.y;
    un.mb = 0;
    un.rows = nxt.z;
    un.base = nxt.w;
    return un;
  }
};

struct Ring {
  int stage = 0;
  uint32_t phase = 0;
  template <int N>
  __device__ __forceinline__ void next() {
    if (++stage == N) { stage = 0; phase ^= 1u; }
  }
};

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t f16x2_sub(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("sub.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

__device__ __forceinline__ uint32_t f16x2_mul(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// 8 int4 codes (one storage word) -> 8 fp16 values q * s as a 16-byte chunk.
// (n & 0xF) ^ 8 = q + 8 for a two's-complement nibble n, and 0x6400 | m is the
// fp16 value 1024 + m, so one AND/XOR gives the pair (1032 + q); subtracting
// 1032 is exact and q * s (3-bit code times 8-bit scale) is exact in fp16.
__device__ __forceinline__ uint4 dequant_word(uint32_t w, uint32_t s2) {
  const uint32_t k1032 = 0x64086408u;  // fp16 pair (1032, 1032)
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t v = ((w >> (4 * i)) & 0x000F000Fu) ^ 0x64086408u;  // fp16 pair 1032 + q
    o[i] = f16x2_mul(f16x2_sub(v, k1032), s2);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// 4 int8 codes (one storage word, code j in byte j) -> 4 fp16 values q * s as
// two pairs (codes 0,1 | codes 2,3). (b ^ 0x80) = q + 128 for a two's-complement
// byte b, and 0x6400 | m is the fp16 value 1024 + m, so one byte permute gives
// 1152 + q exactly; subtracting 1152 is exact, and q * s (7-bit code times 8-bit
// scale) is rounded once to fp16.
__device__ __forceinline__ uint2 dequant_word8(uint32_t w, uint32_t s2) {
  const uint32_t k1152 = 0x64806480u;   // fp16 pair (1152, 1152)
  const uint32_t b = w ^ 0x80808080u;
  const uint32_t lo = __byte_perm(b, 0x64646464u, 0x4140);
  const uint32_t hi = __byte_perm(b, 0x64646464u, 0x4342);
  return make_uint2(f16x2_mul(f16x2_sub(lo, k1152), s2), f16x2_mul(f16x2_sub(hi, k1152), s2));
}

__device__ __forceinline__ uint32_t scale_pair(uint16_t sbits) {
  const uint32_t sh = bf16_to_f16_bits(sbits);
  return sh | (sh << 16);
}

// As scale_pair, setting `inexact` when q * s is not exact in fp16 for every
// int4 code q: a scale whose bf16 exponent is below -17 (bits under fp16's
// subnormal spacing) or whose magnitude reaches 8192 (8 * s overflows), or inf/nan.
__device__ __forceinline__ uint32_t scale_pair_chk(uint16_t sbits, bool& inexact) {
  const uint32_t mag = sbits & 0x7FFFu;
  inexact |= (mag != 0u) && ((mag >> 7) < 127u - 17u || mag >= 0x4600u);   // 0x4600 = 8192 in bf16
  const uint32_t sh = bf16_to_f16_bits(sbits);
  return sh | (sh << 16);
}

// Host side: the tensor maps handed to a grouped GEMM launch.
// 128B-swizzled tile map of a row-major 16-bit matrix [rows][cols]: box {64, box_rows}
// (grouped_gemm.cu).
bool make_tile_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows);

struct Maps {
  CUtensorMap m[7];
};
enum { TQ0 = 0, TQ1 = 1, TS0 = 2, TS1 = 3, TA = 4, TB0 = 5, TB1 = 6 };

// Gate/up expert projection with the dequantised weights held in tensor memory,
// 64 gate + 64 up features per unit over blocks of up to 256 expert-sorted rows
// (expert_gateup.cu): TA = X_perm [A][d], TB0 = s X [Ag|Au] [A][2r] (box {64, 128}
// each); a.bits selects int4 or int8 codes.
int run_expert_gateup_wide(const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s);
// Input gradients with W^T in TMEM (expert_dgrad.cu), mode DX: dX = [dG|dU][Wg;Wu]
// + dxa [Ag;Au]^T (TA = [dG|dU] rows [A][2f], TB0 = dxa [A][2r]); mode DH: dH = dO Wd
// + dha Ad^T and the SwiGLU backward into [dG|dU] (TA = dO [A][d], TB0 = dha [A][r]).
int run_expert_dgrad(int mode, const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s);
// The wide gate/up kernel runs on CTA pairs (cta_group::2, M = 256 per MMA): a
// unit then covers 128 features of gate and of up (64 per CTA), else 64.
constexpr bool kGateUpPair = false;
constexpr int kGateUpUnitFeatures = kGateUpPair ? 128 : 64;

// Down projection with blocks of up to 256 routed rows (expert_down.cu).
int run_expert_down_wide(const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s);

}  // namespace tqp
