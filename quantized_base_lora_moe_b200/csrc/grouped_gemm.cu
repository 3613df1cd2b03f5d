// Grouped tensor-core GEMM engine for the TQP MoE layer (sm_100a, tcgen05).
//
// One persistent, warp-specialised kernel template serves the contractions of
// the layer that do not run on the tensor-memory expert kernels (low-rank
// adapters per expert over frozen quantised base weights: "Reversible Sparse
// MoE Single Node", Pattern 3; full-precision router: TQP Quantization):
//   GATEUP  : [G|U] = X_e [Wg|Wu]^T + s (X [Ag|Au]) [Bg|Bu],  H = silu(G) * U   (fp16;
//             for hidden widths that are not a multiple of 128)
//   LORA_XA : xa = s * X_e [Ag | Au]            (bf16 operands, fp16 out)
//   LORA_HA : ha = s * H_e Ad                   (fp16)
//   ROUTER  : logits = x W_r^T (+ bias), W_r split exactly into 3 bf16 parts
//   DX      : dX = [dG|dU] [Wg;Wu] + dxa [Ag;Au]^T, for model widths that are not
//             a multiple of 128 (else expert_dgrad.cu); the weight tile is an
//             MN-major B operand: W is stored with the contraction index as its
//             row, so the int4 rows are dequantised straight into the tile)
//
// Work unit = (expert e, n-tile of up to 256 columns, m-block of up to 128
// routed rows); one 128 x N x 64 tcgen05.mma step per K-block. Per CTA (1 per
// SM, 576 threads):
//   warps 0-3   epilogue: tcgen05.ld from TMEM, activation, stores
//   warp  4     TMEM allocation + one thread issuing tcgen05.mma
//   warp  5     TMA producer of the int4 code / bf16 scale ring
//   warps 6-9   A producer: TMA 128B-swizzled tiles for contiguous rows, or
//               cp.async 16-byte row gathers (rows picked by perm_token); the
//               rank-space (LoRA) A tiles; TMA B tiles of the rank-space GEMMs
//   warps 10-17 B producer: int4 -> fp16 dequantisation into 128B-swizzled
//               tiles (K-major for the forward, MN-major for the dgrads), the
//               adapter factors of the rank-space stage (idle where B comes by
//               TMA); one arrival per warp
// Accumulators are double-buffered in TMEM (2 x 256 fp32 columns), so the
// epilogue of one unit overlaps the main loop of the next. The operand rings
// (16 KB A tiles, B tiles, 9 KB code stages) share one 216 KB region whose
// split depends on the mode (Layout below). No TMA multicast is used.
#include <cstdint>
#include <cstring>
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "gemm_common.cuh"
#include "tqp_device.cuh"
#include "tqp_launch.h"

namespace tqp {

constexpr int kThreads = 576;
constexpr int kAStages = 5;           // A tiles (TMA / cp.async from L2): deep, to cover L2 latency
constexpr int kBStages = 2;           // dequantised B tiles, produced just ahead of the MMA
constexpr int kQStages = 8;           // int4 codes + scales from DRAM: deepest prefetch
constexpr int kAStageBytes = 16384;   // 128 rows x 64 K x 2 B
constexpr int kBStageBytes = 32768;   // up to 256 rows x 64 K x 2 B
constexpr int kQStageBytes = 9216;    // up to 8192 B of codes + 1024 B of scales
constexpr int kBStagesMax = 8;

constexpr size_t kOperandBytes = size_t(kAStages) * kAStageBytes + size_t(kBStages) * kBStageBytes +
                                 size_t(kQStages) * kQStageBytes;

// Split of the operand region for one mode.
// - Dequantising forward modes: 5 A, 2 B and 8 code stages.
// - Modes whose B tile comes by TMA (rank-space GEMMs, router) read no codes, so
//   their B ring also takes the code region and runs deeper: two TMA fills in
//   flight cannot cover the L2/DRAM latency of a 4-MMA stage, and the A
//   producer's TMA issuer waits on the same ring.
// - Dequantisation for the dgrads (MN-major B tiles): two producer groups of 128
//   threads take alternate stages (one stage's chain of code reads, dequant and
//   stores is latency-bound), which needs a third B slot: 4 A, 3 B, 6 code stages.
template <int MODE>
struct Layout {
  static constexpr bool kTma = (MODE == LORA_XA || MODE == LORA_HA || MODE == ROUTER);
  static constexpr bool kTrans = (MODE == DX);
  static constexpr int kA = kTrans ? 4 : kAStages;
  static constexpr int kB = kTma ? (MODE == ROUTER ? 4 : 8) : (kTrans ? 3 : kBStages);
  // LORA_XA: 2r rows (r <= 64), LORA_HA: r rows, ROUTER: up to 256 rows, x 128 B
  static constexpr int kBBytes = (kTma && MODE != ROUTER) ? 16384 : kBStageBytes;
  static constexpr int kQ = kTma ? 0 : (kTrans ? 6 : kQStages);
  static constexpr int kBGroups = kTrans ? 2 : 1;
  static_assert(kB <= kBStagesMax && kQ <= kQStages && kA <= kAStages, "ring barriers");
  static_assert(size_t(kA) * kAStageBytes + size_t(kB) * kBBytes + size_t(kQ) * kQStageBytes <= kOperandBytes,
                "operand region");
};

struct SmemCtl {
  uint64_t a_full[kAStages];
  uint64_t a_empty[kAStages];
  uint64_t b_full[kBStagesMax];
  uint64_t b_empty[kBStagesMax];
  uint64_t q_full[kQStages];
  uint64_t q_empty[kQStages];
  uint64_t acc_full[2];
  uint64_t acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  Abort ab;
};

constexpr size_t kSmemBytes = 1024 /*align slack*/ + kOperandBytes + sizeof(SmemCtl);
static_assert(kSmemBytes <= 232448, "shared memory budget");

// MN-major B tiles of the dgrads: 64 K rows x up to 256 features, as 64-feature
// (128-byte) columns of 8-row, 1024-byte swizzle atoms; the columns are
// kMnAtomBytes apart.
constexpr uint32_t kMnAtomBytes = 64 * 128;

// Byte offset of the 16-byte chunk of features [8J, 8J+8) of K row k.
__device__ __forceinline__ uint32_t mn_tile_offset(int k, int J) {
  return uint32_t((J >> 3) * kMnAtomBytes + (k >> 3) * 1024 + (k & 7) * 128 + (((J & 7) ^ (k & 7)) << 4));
}


// s_lo / s_hi: fp16 scale pairs of the first / second 32-wide group (equal when g >= 64).
template <int NW>
__device__ __forceinline__ void dequant_row(const uint8_t* qs, uint8_t* bst, int brow, int part, uint32_t s_lo,
                                            uint32_t s_hi) {
  uint32_t w[NW];
#pragma unroll
  for (int i = 0; i < NW; i += 4) {
    const uint4 v = *reinterpret_cast<const uint4*>(qs + brow * 32 + part * NW * 4 + i * 4);
    w[i] = v.x; w[i + 1] = v.y; w[i + 2] = v.z; w[i + 3] = v.w;
  }
  uint8_t* rowp = bst + (brow >> 3) * 1024 + (brow & 7) * 128;
  const int x = brow & 7;
#pragma unroll
  for (int i = 0; i < NW; ++i) {
    const int c = part * NW + i;
    *reinterpret_cast<uint4*>(rowp + ((c ^ x) << 4)) = dequant_word(w[i], c < 4 ? s_lo : s_hi);
  }
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tq0,
                        const __grid_constant__ CUtensorMap tq1, const __grid_constant__ CUtensorMap ts0,
                        const __grid_constant__ CUtensorMap ts1, const __grid_constant__ CUtensorMap ta,
                        const __grid_constant__ CUtensorMap tb0, const __grid_constant__ CUtensorMap tb1) {
  constexpr bool kTrans = (MODE == DX);      // dgrad: B = the weight tile, MN-major
  constexpr bool kDequant = (MODE == GATEUP || kTrans);
  constexpr bool kATma = (MODE == LORA_HA || MODE == ROUTER || kTrans);
  constexpr bool kBTma = (MODE == LORA_XA || MODE == LORA_HA || MODE == ROUTER);
  constexpr bool kBf16 = (MODE == LORA_XA || MODE == ROUTER);
  constexpr int kASt = Layout<MODE>::kA;
  constexpr int kBSt = Layout<MODE>::kB;
  constexpr int kBStride = Layout<MODE>::kBBytes;
  constexpr int kQSt = Layout<MODE>::kQ > 0 ? Layout<MODE>::kQ : 1;
  constexpr int kBGroups = Layout<MODE>::kBGroups;
  static_assert(Layout<MODE>::kTma == kBTma && Layout<MODE>::kTrans == kTrans, "layout mode");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_base = smem;
  uint8_t* b_base = a_base + size_t(kASt) * kAStageBytes;
  uint8_t* q_base = b_base + size_t(kBSt) * kBStride;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(smem + kOperandBytes);
  Abort* abort_flag = &ctl->ab;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  __shared__ int32_t s_sched[2 * (kSchedSmemE + 1)];
  const Sched sc = load_sched(a, s_sched);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kASt; ++i) {
      mbar_init(&ctl->a_full[i], 128);
      mbar_init(&ctl->a_empty[i], 1);
    }
    for (int i = 0; i < kBSt; ++i) {
      // one arrival per warp of a dequantising group, or the TMA issuer alone
      mbar_init(&ctl->b_full[i], kBTma ? 1 : 8 / kBGroups);
      mbar_init(&ctl->b_empty[i], 1);
    }
    for (int i = 0; i < kQSt; ++i) {
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_empty[i], 8 / kBGroups);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->acc_full[i], 1);
      mbar_init(&ctl->acc_empty[i], 4);   // one arrival per epilogue warp
    }
    mbar_init(&ctl->drain, 1);
    abort_init(&ctl->ab, a.wait_ns);
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 5 * 32 && kDequant) {
    prefetch_tmap(&tq0);
    prefetch_tmap(&ts0);
    if (MODE == GATEUP || MODE == DX) {
      prefetch_tmap(&tq1);
      prefetch_tmap(&ts1);
    }
  }
  if (threadIdx.x == 6 * 32) {
    if (kATma) prefetch_tmap(&ta);
    if (kBTma) prefetch_tmap(&tb0);
    if (MODE == LORA_XA) prefetch_tmap(&tb1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  const int nunits = total_units(a, sc);
  const int nkb = a.nkb_main + a.nkb_lora;

  if (warp < 4) {
    // ------------------------------------------------------------ epilogue
    const int row = warp * 32 + lane;
    uint32_t bad = 0;   // nonzero once an fp16 output of a valid row overflowed
    int it = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
      const Unit un = decode_unit(a, sc, u);
      const int ab = it & 1;
      const uint32_t aph = uint32_t(it >> 1) & 1u;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait<128>(&ctl->acc_full[ab], aph, abort_flag, a.status))) break;
      tc_fence_after();
      const bool valid = row < un.rows;
      const size_t grow = size_t(un.base) + row;
      const uint32_t tacc = tmem_base + (uint32_t(warp * 32) << 16) + uint32_t(ab * 256);
      if (MODE == GATEUP) {
        const int half = a.ntile >> 1;
        uint16_t* hrow = static_cast<uint16_t*>(a.out) + grow * a.out_ld + un.nt * half;
#pragma unroll 1
        for (int c = 0; c < half; c += 32) {
          float gv[32], uv[32];
          tmem_ld32(tacc + c, gv);
          tmem_ld32(tacc + half + c, uv);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float g0 = gv[2 * i], g1 = gv[2 * i + 1];
            const float h0 = g0 / (1.0f + __expf(-g0)) * uv[2 * i];
            const float h1 = g1 / (1.0f + __expf(-g1)) * uv[2 * i + 1];
            pk[i] = pack_f16x2(h0, h1);
            if (valid) bad |= f16x2_nonfinite(pk[i]);
          }
          if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(hrow + c);
#pragma unroll
            for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            if (a.aux) {  // keep the pre-activations for the backward
              uint16_t* gr = a.aux + grow * (2 * size_t(a.f_dim)) + un.nt * half + c;
              uint4* ga = reinterpret_cast<uint4*>(gr);
              uint4* ua = reinterpret_cast<uint4*>(gr + a.f_dim);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint4 gq = make_uint4(pack_f16x2(gv[8 * i], gv[8 * i + 1]), pack_f16x2(gv[8 * i + 2], gv[8 * i + 3]),
                                            pack_f16x2(gv[8 * i + 4], gv[8 * i + 5]),
                                            pack_f16x2(gv[8 * i + 6], gv[8 * i + 7]));
                const uint4 uq = make_uint4(pack_f16x2(uv[8 * i], uv[8 * i + 1]), pack_f16x2(uv[8 * i + 2], uv[8 * i + 3]),
                                            pack_f16x2(uv[8 * i + 4], uv[8 * i + 5]),
                                            pack_f16x2(uv[8 * i + 6], uv[8 * i + 7]));
                bad |= f16x2_nonfinite(gq.x) | f16x2_nonfinite(gq.y) | f16x2_nonfinite(gq.z) | f16x2_nonfinite(gq.w) |
                       f16x2_nonfinite(uq.x) | f16x2_nonfinite(uq.y) | f16x2_nonfinite(uq.z) | f16x2_nonfinite(uq.w);
                ga[i] = gq;
                ua[i] = uq;
              }
            }
          }
        }
      } else if (MODE == ROUTER) {
        float* lrow = static_cast<float*>(a.out) + grow * a.out_ld;
#pragma unroll 1
        for (int c = 0; c < a.ntile; c += 32) {
          float v[32];
          tmem_ld32(tacc + c, v);
          const int n0 = un.nt * a.ntile + c;
          if (valid) {
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int n = n0 + i;
              if (n < a.n_valid) lrow[n] = v[i] + (a.bias ? __ldg(a.bias + n) : 0.0f);
            }
          }
        }
      } else {
        // DX / LORA_XA / LORA_HA: fp16 output, optional scale
        const float sc = (MODE == DX) ? 1.0f : a.lora_scale;
        uint16_t* orow = static_cast<uint16_t*>(a.out) + grow * a.out_ld + un.nt * a.ntile;
#pragma unroll 1
        for (int c = 0; c < a.ntile; c += 32) {
          float v[32];
          tmem_ld32(tacc + c, v);
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = pack_f16x2(sc * v[2 * i], sc * v[2 * i + 1]);
          if (valid) {
            const int ncol = min(32, a.n_valid - (un.nt * a.ntile + c));
            for (int i = 0; i < 16 && 2 * i < ncol; ++i) bad |= f16x2_nonfinite(pk[i]);
            uint4* dst = reinterpret_cast<uint4*>(orow + c);
            if (ncol >= 32) {
#pragma unroll
              for (int i = 0; i < 4; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            } else {
              for (int i = 0; i < ncol / 8; ++i) dst[i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive_warp(&ctl->acc_empty[ab]);
    }
    if (__any_sync(0xFFFFFFFFu, bad != 0) && lane == 0) raise_status(a.status, TQP_STATUS_NONFINITE);
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      Ring ra, rb;
      int it = 0;
      bool ok = true;
      // dgrads: B (the weight tile) is MN-major, features contiguous
      const uint32_t idesc = kBf16 ? idesc_bf16(128, a.ntile) : (kTrans ? idesc_f16_bmn(128, a.ntile) : idesc_f16(128, a.ntile));
      // descriptors of ring stage 0; a stage's are these plus a fixed offset
      const uint64_t adesc0 = sdesc_k_sw128(smem_u32(a_base));
      const uint64_t bdesc0 = kTrans ? sdesc_mn_sw128(smem_u32(b_base), kMnAtomBytes) : sdesc_k_sw128(smem_u32(b_base));
      // a K step of 16 advances a K-major tile by 32 B and an MN-major one by two 1024-byte atoms
      constexpr uint64_t kBStep = kTrans ? uint64_t(2048 >> 4) : uint64_t(2);
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++it) {
        const int ab = it & 1;
        const uint32_t aph = uint32_t(it >> 1) & 1u;
        if (!mbar_wait(&ctl->acc_empty[ab], aph ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dt = tmem_base + uint32_t(ab * 256);
        uint32_t accf = 0u;   // the unit's first MMA overwrites the accumulator
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&ctl->a_full[ra.stage], ra.phase, abort_flag, a.status) ||
              !mbar_wait(&ctl->b_full[rb.stage], rb.phase, abort_flag, a.status)) {
            ok = false;
            break;
          }
          // no proxy fence here: TMA fills are async-proxy writes, the dequantising
          // threads fence their own generic stores before arriving, and cp.async
          // completion is tracked by the barrier itself
          tc_fence_after();
          const uint64_t adesc = adesc0 + uint64_t(ra.stage) * uint64_t(kAStageBytes >> 4);
          const uint64_t bdesc = bdesc0 + uint64_t(rb.stage) * uint64_t(kBStride >> 4);
          if (kb >= a.nkb_lora) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              umma_bf16(dt, adesc + uint64_t(2 * kk), bdesc + kBStep * uint64_t(kk), idesc, accf);
              accf = 1u;
            }
          } else {
            const int ksteps = (min(64, a.lora_k - kb * 64) + 15) / 16;
            for (int kk = 0; kk < ksteps; ++kk) {
              umma_bf16(dt, adesc + uint64_t(2 * kk), bdesc + kBStep * uint64_t(kk), idesc, accf);
              accf = 1u;
            }
          }
          umma_commit(&ctl->a_empty[ra.stage]);
          umma_commit(&ctl->b_empty[rb.stage]);
          ra.next<kASt>();
          rb.next<kBSt>();
        }
        if (!ok) break;
        umma_commit(&ctl->acc_full[ab]);
      }
      // no MMA may still read or write TMEM when it is freed: wait for all of
      // them (they run to completion whether or not the CTA aborted)
      umma_commit(&ctl->drain);
      mbar_drain(&ctl->drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ TMA producer (int4 + scales)
    if (kDequant && lane == 0) {
      Ring q;
      // forward: per n-tile rows of W [rows][64 K]: codes rows*32 B, scales [ngrp][rows] bf16
      // dgrad:   tile [64 K rows][ntile N]: codes 64*ntile/2 B, scales [ngn][64] bf16
      const int ngrp = kTrans ? (a.g >= a.ntile ? 1 : a.ntile / a.g) : (a.g >= 64 ? 1 : 64 / a.g);
      // dgrad code rows: ntile features at bits/8 bytes each (int4 or int8)
      const int code_bytes = kTrans ? 64 * (a.ntile * a.bits / 8) : a.ntile * 32;
      const uint32_t bytes = uint32_t(code_bytes) + uint32_t(kTrans ? 128 * ngrp : a.ntile * ngrp * 2);
      const int rows_box = (MODE == GATEUP) ? (a.ntile >> 1) : a.ntile;
      const int gpe = a.in_dim / a.g;  // scale rows per expert
      PendingFills pend;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit un = decode_unit(a, sc, u);
        bool ok = true;
        for (int km = 0; km < a.nkb_main; ++km) {
          if (!mbar_wait<64>(&ctl->q_empty[q.stage], q.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
          uint8_t* qs = q_base + size_t(q.stage) * kQStageBytes;
          uint64_t* bar = &ctl->q_full[q.stage];
          mbar_arrive_expect_tx(bar, bytes);
          if (kTrans) {
            const bool up = (MODE == DX) && km >= a.half_kb;
            const int kl = up ? km - a.half_kb : km;
            tma_load_2d(smem_u32(qs), up ? &tq1 : &tq0, bar, un.nt * (a.ntile * a.bits / 8), un.e * a.out_dim + kl * 64);
            tma_load_2d(smem_u32(qs + code_bytes), up ? &ts1 : &ts0, bar, kl * 64, un.e * gpe + (un.nt * a.ntile) / a.g);
          } else {
            const int nrow0 = un.e * a.out_dim + un.nt * rows_box;
            const int srow = un.e * gpe + (km * 64) / a.g;
            tma_load_2d(smem_u32(qs), &tq0, bar, km * 32, nrow0);
            tma_load_2d(smem_u32(qs + a.ntile * 32), &ts0, bar, un.nt * rows_box, srow);
            if (MODE == GATEUP) {
              tma_load_2d(smem_u32(qs + rows_box * 32), &tq1, bar, km * 32, nrow0);
              tma_load_2d(smem_u32(qs + a.ntile * 32 + ngrp * rows_box * 2), &ts1, bar, un.nt * rows_box, srow);
            }
          }
          pend.issued(q.stage, q.phase);
          q.next<kQSt>();
        }
        if (!ok) break;
      }
      // on an abort, wait (bounded) until every issued fill has landed
      if (aborted(abort_flag)) pend.drain(ctl->q_full);
    }
  } else if (warp < 10) {
    // ------------------------------------------------------------ A producer
    // Row gathers are spread so that 8 consecutive lanes copy the 8 16-byte
    // chunks of one 128-byte row piece: thread tid covers chunk tid % 8 of rows
    // tid / 8 + 16 j, j = 0..7.
    const int tid = threadIdx.x - 6 * 32;  // 0..127
    const int chunk = tid & 7;
    const int row0 = tid >> 3;
    Ring ra, rb;
    const uint32_t a_bytes = uint32_t(kAStageBytes);
    uint32_t b_bytes = 0;
    if (MODE == LORA_XA) b_bytes = uint32_t(2 * a.r * 128);
    if (MODE == LORA_HA) b_bytes = uint32_t(a.r * 128);
    if (MODE == ROUTER) b_bytes = uint32_t(a.ntile * 128);
    PendingFills pend_a, pend_b;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const Unit un = decode_unit(a, sc, u);
      int srow[8];   // gathered source rows of this thread's 8 tile rows
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = row0 + 16 * j;
        srow[j] = (!kATma && r < un.rows) ? __ldg(a.perm_token + un.base + r) : 0;
      }
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait<64>(&ctl->a_empty[ra.stage], ra.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
        const uint32_t st_u = smem_u32(a_base + size_t(ra.stage) * kAStageBytes);
        uint64_t* full = &ctl->a_full[ra.stage];
        if (kb < a.nkb_lora) {
          // rank-space A tile: s*xA / s*hA / dhA / dxa rows, zero-filled past lora_k
          const int col = kb * 64 + chunk * 8;
          const bool in = col < a.lora_k;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int r = row0 + 16 * j;
            if (r < un.rows)
              cp_async16(st_u + sw128_offset(r, chunk), a.a_lora + size_t(un.base + r) * a.lora_ld + (in ? col : 0),
                         in ? 16u : 0u);
          }
          cp_async_arrive_noinc(full);
        } else {
          const int km = kb - a.nkb_lora;
          const int kcol = (MODE == ROUTER) ? (km % a.kb_per_piece) * 64 : km * 64;
          if (kBTma && tid == 0) {
            // the B tile of a rank-space GEMM / the router comes by TMA as well
            if (!mbar_wait<64>(&ctl->b_empty[rb.stage], rb.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
            uint64_t* bfull = &ctl->b_full[rb.stage];
            const uint32_t bst_u = smem_u32(b_base + size_t(rb.stage) * kBStride);
            mbar_arrive_expect_tx(bfull, b_bytes);
            pend_b.issued(rb.stage, rb.phase);
            if (MODE == LORA_XA) {
              tma_load_2d(bst_u, &tb0, bfull, kcol, un.e * a.r);
              tma_load_2d(bst_u + a.r * 128, &tb1, bfull, kcol, un.e * a.r);
            } else if (MODE == LORA_HA) {
              tma_load_2d(bst_u, &tb0, bfull, kcol, un.e * a.r);
            } else if (MODE == ROUTER) {
              const int piece = km / a.kb_per_piece;
              tma_load_2d(bst_u, &tb0, bfull, kcol, piece * a.n_valid + un.nt * a.ntile);
            }
          }
          if (kATma) {
            if (tid == 0) {
              mbar_arrive_expect_tx(full, a_bytes);
              tma_load_2d(st_u, &ta, full, kcol, un.base);
              pend_a.issued(ra.stage, ra.phase);
            } else {
              mbar_arrive(full);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 8; ++j) {
              const int r = row0 + 16 * j;
              if (r < un.rows)
                cp_async16(st_u + sw128_offset(r, chunk), a.a_src + size_t(srow[j]) * a.a_ld + kcol + chunk * 8, 16);
            }
            cp_async_arrive_noinc(full);
          }
          if (kBTma) rb.next<kBSt>();
        }
        ra.next<kASt>();
      }
      if (!ok) break;
    }
    cp_async_wait_all();
    // on an abort, wait (bounded) for every TMA fill issued by this thread
    if (tid == 0 && aborted(abort_flag)) {
      pend_a.drain(ctl->a_full);
      pend_b.drain(ctl->b_full);
    }
  } else if (!kBTma) {
    // ------------------------------------------------------------ B producer
    // (the modes whose B tile arrives by TMA have none: the A producer's TMA
    // issuer is the B stage's only arrival)
    const int tid = threadIdx.x - 10 * 32;  // 0..255
    const int tpr = a.ntile >= 256 ? 1 : 256 / a.ntile;   // threads per B row (forward tiles)
    const int brow = tid / tpr;                              // B row (forward tiles)
    const int part = tid % tpr;
    const int nwords = tpr >= 8 ? 1 : 8 / tpr;               // int4 words (8 K values each) per thread
    // dgrad modes: two groups of 128 threads take alternate stages
    const int grp = kBGroups > 1 ? tid >> 7 : 0;
    const int gtid = kBGroups > 1 ? tid & 127 : tid;
    Ring rb, q;
    bool inexact = false;   // a group scale whose products q * s are not exact in fp16
    bool lora_inf = false;  // an adapter value beyond the fp16 range
    int n = 0;                                               // stage counter over all units
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const Unit un = decode_unit(a, sc, u);
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb, ++n) {
        if (kBGroups > 1 && (n & 1) != grp) {
          if (kb >= a.nkb_lora) q.next<kQSt>();   // the other group consumes this stage's codes
          rb.next<kBSt>();
          continue;
        }
        if (!mbar_wait_warp(&ctl->b_empty[rb.stage], rb.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
        uint8_t* bst = b_base + size_t(rb.stage) * kBStride;
        uint64_t* full = &ctl->b_full[rb.stage];
        if (kb < a.nkb_lora) {
          if (MODE == GATEUP) {
            // rank-space B^T rows as fp16, K' columns [kb*64, kb*64+64); gate rows hold
            // Bg^T in [0, r), up rows hold Bu^T in [r, 2r) (block-diagonal)
            if (brow < a.ntile) {
              const int half = a.ntile >> 1;
              for (int i = 0; i < nwords; ++i) {
                const int c = part * nwords + i;
                const int col = kb * 64 + c * 8;
                uint4 v = make_uint4(0, 0, 0, 0);
                const bool gate = brow < half;
                const int n = un.nt * half + (gate ? brow : brow - half);
                const int cc = gate ? col : col - a.r;
                if (cc >= 0 && cc < a.r)
                  v = __ldg(reinterpret_cast<const uint4*>((gate ? a.b0 : a.b1) + (size_t(un.e) * a.out_dim + n) * a.r +
                                                           cc));
                *reinterpret_cast<uint4*>(bst + sw128_offset(brow, c)) = bf16x8_to_f16x8_chk(v, lora_inf);
              }
            }
          } else if (kTrans) {
            // dgrad rank-space step, MN-major: B row rr (the K index) = A^T[rr][n0 ..
            // n0 + ntile) of the adapter (stored [r][features], bf16 -> fp16); rows
            // past lora_k are zero. Thread gtid: row gtid / 2, half gtid % 2 of the row.
            const int rr = kb * 64 + (gtid >> 1);
            const int half = gtid & 1;
            const int cpt = a.ntile >> 4;                      // 16-byte chunks per half row
            const uint16_t* src = nullptr;
            if (rr < a.r) src = a.lb0 + (size_t(un.e) * a.r + rr) * a.lb_ld;
            else if (MODE == DX && rr < 2 * a.r) src = a.lb1 + (size_t(un.e) * a.r + (rr - a.r)) * a.lb_ld;
            for (int j = 0; j < cpt; ++j) {
              const int J = half * cpt + j;                    // chunk of 8 features within the tile
              uint4 v = make_uint4(0, 0, 0, 0);
              if (src) v = bf16x8_to_f16x8_chk(__ldg(reinterpret_cast<const uint4*>(src + un.nt * a.ntile + J * 8)),
                                               lora_inf);
              *reinterpret_cast<uint4*>(bst + mn_tile_offset(gtid >> 1, J)) = v;
            }
          }
          fence_proxy_async_smem();
          mbar_arrive_warp(full);
        } else if (kTrans) {
          if (!mbar_wait_warp(&ctl->q_full[q.stage], q.phase, abort_flag, a.status)) { ok = false; break; }
          const uint8_t* qs = q_base + size_t(q.stage) * kQStageBytes;
          // The code tile holds W rows n (the K index) with the tile's ntile
          // features contiguous: exactly the MN-major operand, so each thread
          // dequantises half a row (8 features per int4 word) straight into it.
          // Thread gtid: row gtid / 2, half gtid % 2.
          const int k = gtid >> 1, half = gtid & 1;
          const int n0 = un.nt * a.ntile;
          const int rowb = a.ntile * a.bits / 8;            // bytes per code row (128 for the wide tiles)
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(qs + 64 * rowb);
          // 16-byte code chunks of this thread's half row: 128-byte rows come
          // 128B-swizzled (conflict-free reads), 64-byte rows plain
          const int cph = rowb >> 5;
          for (int j = 0; j < cph; ++j) {
            const int cc = half * cph + j;                   // code chunk within the row
            const int pos = (rowb == 128) ? (cc ^ (k & 7)) : cc;
            const uint4 w4 = *reinterpret_cast<const uint4*>(qs + k * rowb + pos * 16);
            const uint32_t wv[4] = {w4.x, w4.y, w4.z, w4.w};
            if (a.bits == 4) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const int Jw = cc * 4 + i;                   // word = features n0 + 8 Jw .. + 7
                const int gi = (n0 + Jw * 8) / a.g - n0 / a.g;
                *reinterpret_cast<uint4*>(bst + mn_tile_offset(k, Jw)) =
                    dequant_word(wv[i], scale_pair_chk(sc[gi * 64 + k], inexact));
              }
            } else {
              // int8: a chunk is 16 features = two 8-feature output chunks
#pragma unroll
              for (int i = 0; i < 2; ++i) {
                const int Jo = cc * 2 + i;                   // output chunk = features n0 + 8 Jo .. + 7
                const uint32_t s2 = scale_pair_chk(sc[((n0 + Jo * 8) / a.g - n0 / a.g) * 64 + k], inexact);
                const uint2 lo = dequant_word8(wv[2 * i], s2), hi = dequant_word8(wv[2 * i + 1], s2);
                *reinterpret_cast<uint4*>(bst + mn_tile_offset(k, Jo)) = make_uint4(lo.x, lo.y, hi.x, hi.y);
              }
            }
          }
          // hand the code slot back only after its values were consumed, behind a
          // proxy fence (its next TMA fill and the tensor-core reads are async-proxy)
          fence_proxy_async_smem();
          mbar_arrive_warp(&ctl->q_empty[q.stage]);
          q.next<kQSt>();
          mbar_arrive_warp(full);
        } else if (kDequant) {
          if (!mbar_wait_warp(&ctl->q_full[q.stage], q.phase, abort_flag, a.status)) { ok = false; break; }
          const uint8_t* qs = q_base + size_t(q.stage) * kQStageBytes;
          const uint16_t* sc = reinterpret_cast<const uint16_t*>(qs + a.ntile * 32);
          const int half = a.ntile >> 1;
          // scale pairs of this row's group(s) in this K-block (two 32-wide groups when g == 32)
          const int ngrp = a.g >= 64 ? 1 : 64 / a.g;
          const int sidx = (MODE == GATEUP) ? (brow / half) * ngrp * half + (brow % half) : brow;
          const int sstride = (MODE == GATEUP) ? half : a.ntile;
          const uint32_t s_lo = scale_pair_chk(sc[sidx], inexact);
          const uint32_t s_hi = (a.g == 32) ? scale_pair_chk(sc[sidx + sstride], inexact) : s_lo;
          if (nwords == 8) dequant_row<8>(qs, bst, brow, part, s_lo, s_hi);
          else dequant_row<4>(qs, bst, brow, part, s_lo, s_hi);
          fence_proxy_async_smem();
          mbar_arrive_warp(&ctl->q_empty[q.stage]);
          q.next<kQSt>();
          mbar_arrive_warp(full);
        }
        rb.next<kBSt>();
      }
      if (!ok) break;
    }
    if (__any_sync(0xFFFFFFFFu, inexact) && lane == 0) raise_status(a.status, TQP_STATUS_RANGE);
    if (__any_sync(0xFFFFFFFFu, lora_inf) && lane == 0) raise_status(a.status, TQP_STATUS_NONFINITE);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ----------------------------------------------------------------------------
// small helper kernels
// ----------------------------------------------------------------------------

// mb_prefix[e] = sum_{e' < e} ceil(count(e') / block), one thread block.
__global__ void schedule_kernel(const int32_t* __restrict__ offsets, int E, int32_t* __restrict__ mb_prefix,
                                int block) {
  __shared__ int32_t warp_sums[32];
  const int nt = blockDim.x;
  const int per = (E + nt - 1) / nt;
  const int lo = threadIdx.x * per;
  const int hi = min(E, lo + per);
  int local = 0;
  for (int e = lo; e < hi; ++e) local += (offsets[e + 1] - offsets[e] + block - 1) / block;
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
    if (lane < (nt >> 5)) warp_sums[lane] = s;
  }
  __syncthreads();
  int run = v - local + (wid > 0 ? warp_sums[wid - 1] : 0);
  for (int e = lo; e < hi; ++e) {
    mb_prefix[e] = run;
    run += (offsets[e + 1] - offsets[e] + block - 1) / block;
  }
  if (threadIdx.x == nt - 1) mb_prefix[E] = run;
}

// Decoded work units of one expert-kernel launch: tab[u] = {expert, n-tile,
// rows, first row} for u < mb_prefix[E] * n_tiles, with blocks of `block` rows
// (units ordered as decode_unit).
__global__ void unit_table_kernel(const int32_t* __restrict__ offsets, const int32_t* __restrict__ mb_prefix, int E,
                                  int n_tiles, int block, int max_units, int4* __restrict__ tab) {
  const int u = blockIdx.x * blockDim.x + threadIdx.x;
  if (u >= max_units || u >= mb_prefix[E] * n_tiles) return;
  int lo = 0, hi = E;
  while (hi - lo > 1) {
    const int mid = (lo + hi) >> 1;
    if (mb_prefix[mid] * n_tiles <= u) lo = mid;
    else hi = mid;
  }
  const int p0 = mb_prefix[lo];
  const int nmb = mb_prefix[lo + 1] - p0;
  const int idx = u - p0 * n_tiles;
  const int nt = idx / nmb;
  const int mb = idx - nt * nmb;
  const int o0 = offsets[lo];
  const int cnt = offsets[lo + 1] - o0;
  tab[u] = make_int4(lo, nt, min(block, cnt - mb * block), o0 + mb * block);
}

// 2 bf16 values (one 32-bit word) -> 2 fp16 values in one conversion instruction.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2_pk(uint32_t w) {
  const __half2 h = __floats2half2_rn(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
  return *reinterpret_cast<const uint32_t*>(&h);
}

// 8 bf16 values -> 8 fp16 values, two per conversion instruction: a bf16 value is
// the upper half of the fp32 with the same value, and the fp32 pair is rounded to
// an fp16 pair (exact in fp16's normal range; round to nearest even below it,
// inf past it, as the scalar conversion).
__device__ __forceinline__ uint4 bf16x8_to_f16x8_pk(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __half2 h = __floats2half2_rn(__uint_as_float(w[i] << 16), __uint_as_float(w[i] & 0xFFFF0000u));
    o[i] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// bf16 -> fp16, 8 values per thread; values beyond the fp16 range (x, or a
// LoRA factor) raise TQP_STATUS_NONFINITE (status may be null).
__global__ void to_f16_kernel(const uint16_t* __restrict__ x, uint16_t* __restrict__ x16, size_t n8,
                              int32_t* status) {
  const size_t i = size_t(blockIdx.x) * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(x) + i);
  const uint4 o = bf16x8_to_f16x8_pk(v);
  reinterpret_cast<uint4*>(x16)[i] = o;
  const uint32_t w[4] = {o.x, o.y, o.z, o.w};
  bool bad = false;
#pragma unroll
  for (int j = 0; j < 4; ++j) bad |= ((w[j] & 0x7C00u) == 0x7C00u) || ((w[j] & 0x7C000000u) == 0x7C000000u);
  if (bad) raise_status(status, TQP_STATUS_NONFINITE);
}

// Expert-sorted token rows in fp16, X_perm[i] = x[perm_token[i]], one warp per
// row, 8 16-byte loads in flight per lane; values beyond the fp16 range raise
// TQP_STATUS_NONFINITE.
__global__ void __launch_bounds__(256) gather_rows_f16_kernel(const uint16_t* __restrict__ x,
                                                              const int32_t* __restrict__ perm, int A, int d,
                                                              uint16_t* __restrict__ out, int32_t* status) {
  const int row = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (row >= A) return;
  const int lane = threadIdx.x & 31;
  const int n16 = d / 8;   // 16-byte pieces per row
  const uint4* src = reinterpret_cast<const uint4*>(x + size_t(__ldg(perm + row)) * d);
  uint4* dst = reinterpret_cast<uint4*>(out + size_t(row) * d);
  uint32_t bad = 0;
  for (int c0 = 0; c0 < n16; c0 += 256) {
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = c0 + 32 * i + lane;
      v[i] = c < n16 ? __ldg(src + c) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int c = c0 + 32 * i + lane;
      if (c < n16) {
        const uint4 o = bf16x8_to_f16x8_pk(v[i]);
        dst[c] = o;
        bad |= f16x2_nonfinite(o.x) | f16x2_nonfinite(o.y) | f16x2_nonfinite(o.z) | f16x2_nonfinite(o.w);
      }
    }
  }
  if (__any_sync(0xFFFFFFFFu, bad != 0) && lane == 0) raise_status(status, TQP_STATUS_NONFINITE);
}

// Router: one group covering all T tokens; split W_r into three exact bf16 parts.
__global__ void router_prep_kernel(const float* __restrict__ wr, int n, int T, uint16_t* __restrict__ parts,
                                   int32_t* __restrict__ offsets2, int32_t* __restrict__ mbp2) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i == 0) {
    offsets2[0] = 0;
    offsets2[1] = T;
    mbp2[0] = 0;
    mbp2[1] = (T + kMBlock - 1) / kMBlock;
  }
  if (i >= n) return;
  const float w = wr[i];
  const uint16_t hi = f32_to_bf16(w);
  const float r1 = w - bf16_to_f32(hi);
  const uint16_t mid = f32_to_bf16(r1);
  const float r2 = r1 - bf16_to_f32(mid);
  const uint16_t lo = f32_to_bf16(r2);
  parts[i] = hi;
  parts[size_t(n) + i] = mid;
  parts[2 * size_t(n) + i] = lo;
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D tensor map; swizzle = 0 (none), 32, 64 or 128 bytes.
static bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* ptr, uint64_t inner, uint64_t outer,
                     uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, int swizzle = 0) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            swizzle == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
            : swizzle == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
            : swizzle == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                            : CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 128B-swizzled K-major tile map of a row-major 16-bit matrix [rows][cols]: box {64, box_rows}.
bool make_tile_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, uint32_t box_rows) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT16, ptr, cols, rows, cols * 2, 64, box_rows, 128);
}

int num_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  return n;
}


template <int MODE>
static int run_gemm(GemmArgs a, const Maps& mp, int units_upper, cudaStream_t s) {
  static DeviceFlags attr_done;
  if (!attr_done.test_and_set_device(grouped_gemm_kernel<MODE>, int(kSmemBytes))) return TQP_ERR_CUDA;
  a.wait_ns = wait_limit_ns();
  const int grid = units_upper < num_sms() ? (units_upper > 0 ? units_upper : 1) : num_sms();
  grouped_gemm_kernel<MODE><<<grid, kThreads, kSmemBytes, s>>>(a, mp.m[0], mp.m[1], mp.m[2], mp.m[3], mp.m[4],
                                                                mp.m[5], mp.m[6]);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

size_t router_ws_bytes(int T, const tqp_moe_weights* w) {
  (void)T;
  return align_up(size_t(3) * w->E * w->d * 2, 256) + 256;
}

int launch_router_gemm(const uint16_t* x, int T, const tqp_moe_weights* w, float* logits, void* ws,
                       int32_t* status, cudaStream_t s) {
  if (T == 0) return TQP_OK;
  uint16_t* parts = static_cast<uint16_t*>(ws);
  int32_t* ctl = reinterpret_cast<int32_t*>(static_cast<char*>(ws) + align_up(size_t(3) * w->E * w->d * 2, 256));
  const int n = w->E * w->d;
  router_prep_kernel<<<(n + 255) / 256, 256, 0, s>>>(w->router_w, n, T, parts, ctl, ctl + 2);
  GemmArgs a{};
  a.E = 1;
  a.kb_per_piece = w->d / 64;
  a.nkb_main = 3 * a.kb_per_piece;
  a.ntile = w->E <= 128 ? ((w->E + 15) / 16) * 16 : 256;
  a.n_tiles = (w->E + a.ntile - 1) / a.ntile;
  a.g = 64;
  a.offsets = ctl;
  a.mb_prefix = ctl + 2;
  a.out = logits;
  a.out_ld = w->E;
  a.n_valid = w->E;
  a.bias = w->router_bias;
  a.status = status;
  Maps mp{};
  if (!make_tile_map(&mp.m[TA], x, uint64_t(T), uint64_t(w->d), 128) ||
      !make_tile_map(&mp.m[TB0], parts, 3 * uint64_t(w->E), uint64_t(w->d), uint32_t(a.ntile)))
    return TQP_ERR_CUDA;
  const int units = ((T + kMBlock - 1) / kMBlock) * a.n_tiles;
  return run_gemm<ROUTER>(a, mp, units, s);
}

// Upper bound on the work units of one expert-kernel launch (128-row blocks x
// 128-feature tiles of the wider projection).
static size_t ffn_unit_upper(int T, const tqp_moe_weights* w) {
  const size_t A = size_t(T) * w->top_k;
  const size_t mb_upper = (A + kMBlock - 1) / kMBlock + size_t(w->E);
  const int wide = w->d > w->ffn ? w->d : w->ffn;
  return mb_upper * size_t((wide + 127) / 128);
}

size_t ffn_ws_bytes(int T, const tqp_moe_weights* w) {
  const size_t A = size_t(T) * w->top_k;
  size_t b = 2 * align_up(size_t(w->E + 1) * 4, 256);          // block prefixes (128- and 256-row blocks)
  b += align_up(A * w->d * 2, 256);                            // X_perm (or x) in fp16
  if (w->rank > 0) {
    b += align_up(A * 2 * w->rank * 2, 256);                    // xa [A][2r]
    b += align_up(A * w->rank * 2, 256);                        // ha [A][r]
    b += align_up(size_t(w->E) * w->rank * w->ffn * 2, 256);   // Ad^T in fp16
  }
  b += align_up(ffn_unit_upper(T, w) * 16, 256);                 // decoded units of one expert launch
  return b + 256;
}

FfnBufs ffn_carve(void* ws, int T, const tqp_moe_weights* w) {
  const size_t A = size_t(T) * w->top_k;
  char* p = static_cast<char*>(ws);
  FfnBufs b{};
  b.mb_prefix = reinterpret_cast<int32_t*>(p);
  p += align_up(size_t(w->E + 1) * 4, 256);
  b.mb_prefix256 = reinterpret_cast<int32_t*>(p);
  p += align_up(size_t(w->E + 1) * 4, 256);
  b.x16 = reinterpret_cast<uint16_t*>(p);
  b.xperm = b.x16;
  p += align_up(A * w->d * 2, 256);
  if (w->rank > 0) {
    b.xa = reinterpret_cast<uint16_t*>(p);
    p += align_up(A * 2 * w->rank * 2, 256);
    b.ha = reinterpret_cast<uint16_t*>(p);
    p += align_up(A * w->rank * 2, 256);
    b.adT16 = reinterpret_cast<uint16_t*>(p);
    p += align_up(size_t(w->E) * w->rank * w->ffn * 2, 256);
  }
  b.unit_tab = reinterpret_cast<int4*>(p);
  return b;
}

static int build_unit_table(const GemmArgs& a, int block, int max_units, int4* tab, cudaStream_t s) {
  if (max_units <= 0) return TQP_OK;
  unit_table_kernel<<<(max_units + 255) / 256, 256, 0, s>>>(a.offsets, a.mb_prefix, a.E, a.n_tiles, block, max_units,
                                                           tab);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

static int to_f16(const uint16_t* src, uint16_t* dst, size_t n, int32_t* status, cudaStream_t s) {
  const size_t n8 = n / 8;
  if (n8 == 0) return TQP_OK;
  to_f16_kernel<<<unsigned((n8 + 255) / 256), 256, 0, s>>>(src, dst, n8, status);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

// One part of the grouped FFN (parts run in order on one workspace):
//   0 prepare : m-block schedule, x and Ad^T in fp16, xa = s X [Ag | Au]
//   1 gate/up : H = silu(G) * U
//   2 rank    : ha = s H Ad
//   3 down    : O = H Wd^T + ha Bd
int launch_grouped_ffn_part(int part, const uint16_t* x, int T, const int32_t* offsets, const int32_t* perm_token,
                            const tqp_moe_weights* w, uint16_t* h, uint16_t* out_perm, void* ws, int32_t* status,
                            cudaStream_t s, uint16_t* aux_gu) {
  if (T == 0) return TQP_OK;
  const size_t A = size_t(T) * w->top_k;
  const FfnBufs fb = ffn_carve(ws, T, w);
  const int d = w->d, f = w->ffn, r = w->rank;
  int rc;
  if (part == 0) {
    schedule_kernel<<<1, 1024, 0, s>>>(offsets, w->E, fb.mb_prefix, kMBlock);
    schedule_kernel<<<1, 1024, 0, s>>>(offsets, w->E, fb.mb_prefix256, 256);
    if (cudaGetLastError() != cudaSuccess) return TQP_ERR_CUDA;
    if (f % 128 == 0) {   // the wide gate/up kernel reads expert-sorted rows by TMA
      gather_rows_f16_kernel<<<unsigned((A + 7) / 8), 256, 0, s>>>(x, perm_token, int(A), d, fb.xperm, status);
      if (cudaGetLastError() != cudaSuccess) return TQP_ERR_CUDA;
    } else if ((rc = to_f16(x, fb.x16, size_t(T) * d, status, s)) != TQP_OK) {
      return rc;
    }
    if (r > 0 && (rc = to_f16(w->lora_a[2], fb.adT16, size_t(w->E) * r * f, status, s)) != TQP_OK) return rc;
  }
  // an upper bound on the number of work units (grid sizing only)
  const int mb_upper = int((A + kMBlock - 1) / kMBlock) + w->E;

  GemmArgs base{};
  base.E = w->E;
  base.g = w->group;
  base.r = r;
  base.lora_scale = w->lora_scale;
  base.offsets = offsets;
  base.mb_prefix = fb.mb_prefix;
  base.perm_token = perm_token;
  base.status = status;
  base.kb_per_piece = 1;
  base.bits = w->bits == 8 ? 8 : 4;
  const int bB = base.bits;

  if (part == 0 && r > 0) {  // xa = s * X [Ag | Au]   (bf16 operands)
    GemmArgs a = base;
    a.nkb_main = d / 64;
    a.ntile = 2 * r < 16 ? 16 : 2 * r;
    a.n_tiles = 1;
    a.a_src = x;
    a.a_ld = d;
    a.out = fb.xa;
    a.out_ld = 2 * r;
    a.n_valid = 2 * r;
    Maps mp{};
    if (!make_tile_map(&mp.m[TB0], w->lora_a[0], uint64_t(w->E) * r, uint64_t(d), uint32_t(r)) ||
        !make_tile_map(&mp.m[TB1], w->lora_a[1], uint64_t(w->E) * r, uint64_t(d), uint32_t(r)))
      return TQP_ERR_CUDA;
    if ((rc = run_gemm<LORA_XA>(a, mp, mb_upper, s)) != TQP_OK) return rc;
  }
  // The forward projections run with the weights in TMEM (expert_gateup.cu,
  // expert_down.cu) when the hidden width is a multiple of 128, else on the
  // shared-memory engine.
  const bool tm = (f % 128 == 0);
  if (part == 1 && tm) {  // H = silu(G) * U: wide units of up to 256 rows (expert_gateup.cu)
    GemmArgs a = base;
    a.mb_prefix = fb.mb_prefix256;
    a.nkb_main = d / 64;
    a.nkb_lora = r > 0 ? (2 * r + 63) / 64 : 0;
    a.lora_k = 2 * r;
    a.n_tiles = f / kGateUpUnitFeatures;
    a.in_dim = d;
    a.out_dim = f;
    a.b0 = w->lora_b[0];
    a.b1 = w->lora_b[1];
    a.out = h;
    a.out_ld = f;
    a.n_valid = f;
    a.aux = aux_gu;
    a.f_dim = f;
    const int ngrp = w->group >= 64 ? 1 : 64 / w->group;
    const uint32_t cbox = uint32_t(8 * bB);   // 64 K values: 32-byte int4 / 64-byte int8 code rows
    const uint64_t crow = uint64_t(d) * bB / 8;
    Maps mp{};
    bool ok = make_map(&mp.m[TQ0], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[0], crow, uint64_t(w->E) * f, crow, cbox, 64,
                       int(cbox)) &&
              make_map(&mp.m[TQ1], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[1], crow, uint64_t(w->E) * f, crow, cbox, 64,
                       int(cbox)) &&
              make_map(&mp.m[TS0], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[0], f, uint64_t(w->E) * (d / w->group),
                       uint64_t(f) * 2, 64, ngrp) &&
              make_map(&mp.m[TS1], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[1], f, uint64_t(w->E) * (d / w->group),
                       uint64_t(f) * 2, 64, ngrp) &&
              make_tile_map(&mp.m[TA], fb.xperm, uint64_t(A), uint64_t(d), 128);
    // the rank-space rows: 2r columns, the rest of each 64-wide box zero-filled
    if (ok && r > 0) ok = make_tile_map(&mp.m[TB0], fb.xa, uint64_t(A), uint64_t(2 * r), 128);
    if (!ok) return TQP_ERR_CUDA;
    const int units_upper = int((A + 255) / 256 + w->E) * a.n_tiles;
    if ((rc = build_unit_table(a, 256, units_upper, fb.unit_tab, s)) != TQP_OK) return rc;
    a.unit_tab = fb.unit_tab;
    a.wait_ns = wait_limit_ns();
    if ((rc = run_expert_gateup_wide(a, mp, units_upper, s)) != TQP_OK) return rc;
  }
  if (part == 1 && !tm) {  // H = silu(G) * U on the shared-memory engine
    GemmArgs a = base;
    a.nkb_main = d / 64;
    a.nkb_lora = r > 0 ? (2 * r + 63) / 64 : 0;
    a.lora_k = 2 * r;
    a.ntile = 128;
    a.n_tiles = f / (a.ntile / 2);
    a.in_dim = d;
    a.out_dim = f;
    a.a_src = fb.x16;
    a.a_ld = d;
    a.a_lora = fb.xa;
    a.lora_ld = 2 * r;
    a.b0 = w->lora_b[0];
    a.b1 = w->lora_b[1];
    a.out = h;
    a.out_ld = f;
    a.n_valid = f;
    a.aux = aux_gu;
    a.f_dim = f;
    const int ngrp = w->group >= 64 ? 1 : 64 / w->group;
    const uint32_t rows_box = uint32_t(a.ntile / 2);
    const uint32_t cbox = uint32_t(8 * bB);
    const uint64_t crow = uint64_t(d) * bB / 8;
    Maps mp{};
    bool ok = make_map(&mp.m[TQ0], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[0], crow, uint64_t(w->E) * f, crow, cbox,
                       rows_box) &&
              make_map(&mp.m[TQ1], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[1], crow, uint64_t(w->E) * f, crow, cbox,
                       rows_box) &&
              make_map(&mp.m[TS0], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[0], f, uint64_t(w->E) * (d / w->group),
                       uint64_t(f) * 2, rows_box, ngrp) &&
              make_map(&mp.m[TS1], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[1], f, uint64_t(w->E) * (d / w->group),
                       uint64_t(f) * 2, rows_box, ngrp);
    if (!ok) return TQP_ERR_CUDA;
    a.wait_ns = wait_limit_ns();
    if ((rc = run_gemm<GATEUP>(a, mp, mb_upper * a.n_tiles, s)) != TQP_OK) return rc;
  }
  if (part == 2 && r > 0) {  // ha = s * H Ad
    GemmArgs a = base;
    a.nkb_main = f / 64;
    a.ntile = r < 16 ? 16 : r;
    a.n_tiles = 1;
    a.out = fb.ha;
    a.out_ld = r;
    a.n_valid = r;
    Maps mp{};
    if (!make_tile_map(&mp.m[TA], h, uint64_t(A), uint64_t(f), 128) ||
        !make_tile_map(&mp.m[TB0], fb.adT16, uint64_t(w->E) * r, uint64_t(f), uint32_t(r)))
      return TQP_ERR_CUDA;
    if ((rc = run_gemm<LORA_HA>(a, mp, mb_upper, s)) != TQP_OK) return rc;
  }
  if (part == 3) {  // O = H Wd^T + (s H Ad) Bd: blocks of up to 256 rows, weights in TMEM (expert_down.cu)
    GemmArgs a = base;
    a.mb_prefix = fb.mb_prefix256;
    a.nkb_main = f / 64;
    a.nkb_lora = r > 0 ? 1 : 0;   // r <= 64: one 64-wide rank-space stage
    a.lora_k = r;
    a.ntile = 128;
    a.n_tiles = d / 128;
    a.in_dim = f;
    a.out_dim = d;
    a.a_lora = fb.ha;
    a.lora_ld = r;
    a.b0 = w->lora_b[2];
    a.out = out_perm;
    a.out_ld = d;
    a.n_valid = d;
    const int ngrp = w->group >= 64 ? 1 : 64 / w->group;
    Maps mp{};
    bool ok = make_tile_map(&mp.m[TA], h, uint64_t(A), uint64_t(f), 128) &&
              make_map(&mp.m[TQ0], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[2], uint64_t(f) * bB / 8, uint64_t(w->E) * d,
                       uint64_t(f) * bB / 8, uint32_t(8 * bB), 128, 8 * bB) &&
              make_map(&mp.m[TS0], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[2], d, uint64_t(w->E) * (f / w->group),
                       uint64_t(d) * 2, 128, ngrp);
    // the rank-space rows s H Ad: r columns, the rest of each 64-wide box zero-filled
    if (ok && r > 0) ok = make_tile_map(&mp.m[TB0], fb.ha, uint64_t(A), uint64_t(r), 128);
    if (!ok) return TQP_ERR_CUDA;
    const int units_upper = int((A + 255) / 256 + w->E) * a.n_tiles;
    if ((rc = build_unit_table(a, 256, units_upper, fb.unit_tab, s)) != TQP_OK) return rc;
    a.unit_tab = fb.unit_tab;
    a.wait_ns = wait_limit_ns();
    if ((rc = run_expert_down_wide(a, mp, units_upper, s)) != TQP_OK) return rc;
  }
  return TQP_OK;
}

int launch_grouped_ffn(const uint16_t* x, int T, const int32_t* offsets, const int32_t* perm_token,
                       const tqp_moe_weights* w, uint16_t* h, uint16_t* out_perm, void* ws, int32_t* status,
                       cudaStream_t s, uint16_t* aux_gu) {
  for (int part = 0; part < 4; ++part) {
    const int rc = launch_grouped_ffn_part(part, x, T, offsets, perm_token, w, h, out_perm, ws, status, s, aux_gu);
    if (rc != TQP_OK) return rc;
  }
  return TQP_OK;
}

// dH = dO Wd + dhA Ad^T (SwiGLU backward fused: writes dG | dU) or
// dX = [dG | dU] [Wg ; Wu] + dxa [Ag^T ; Au^T]^T, per expert, on the tensor cores
// with the int4 base dequantised into MN-major shared-memory tiles.
// K-major fp16 copy of a backward rank-space B operand, [E][n][K], one block
// per (64-wide K slice, expert):
//   which 0: Bd, stored B^T [E][d][r]  ->  [E][r][d]             (n = r,  K = d)
//   which 1: blockdiag(Bg, Bu), each stored B^T [E][f][r]  ->  [E][2r][2f], Bg in
//            rows [0, r) x columns [0, f), Bu in rows [r, 2r) x columns [f, 2f)
// The r values of a source row arrive as 16-byte pieces and land transposed in
// shared memory as fp16; each output row's 64 K values leave as 16-byte pieces.
__global__ void __launch_bounds__(256) rank_b_kernel(const uint16_t* __restrict__ b0, const uint16_t* __restrict__ b1,
                                                     int which, int r, int f, int K, uint16_t* __restrict__ out) {
  __shared__ __align__(16) uint16_t tile[64][72];   // [j][k], fp16; j < r <= 64, row pitch 144 B
  const int e = blockIdx.y, k0 = blockIdx.x * 64;
  const int n = which == 0 ? r : 2 * r;
  const bool up = which == 1 && k0 >= f;   // f % 64 == 0: a slice lies in one half
  const uint16_t* src = which == 0 ? b0 + (size_t(e) * K + k0) * r
                                   : (up ? b1 + (size_t(e) * f + (k0 - f)) * r : b0 + (size_t(e) * f + k0) * r);
  const int r8 = r >> 3;   // r % 8 == 0
  for (int i = threadIdx.x; i < 64 * r8; i += blockDim.x) {   // 64 source rows of r
    const int kk = i / r8, j8 = i - kk * r8;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t h = bf16x2_to_f16x2_pk(wv[q]);
      tile[j8 * 8 + 2 * q][kk] = uint16_t(h & 0xFFFFu);
      tile[j8 * 8 + 2 * q + 1][kk] = uint16_t(h >> 16);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < n * 8; i += blockDim.x) {
    const int j = i >> 3, c = i & 7;
    uint4 o = make_uint4(0, 0, 0, 0);
    if (which == 0) {
      o = *reinterpret_cast<const uint4*>(&tile[j][c * 8]);
    } else if ((j >= r) == up) {
      o = *reinterpret_cast<const uint4*>(&tile[up ? j - r : j][c * 8]);
    }
    *reinterpret_cast<uint4*>(out + (size_t(e) * n + j) * K + k0 + c * 8) = o;
  }
}

// Row copy of the adapter A factors for the rank-space stage of the dgrads, in fp16:
//   which 0 (dH): out[e][n][j] = Ad^T[e][j][n]                                  [E][f][r]
//   which 1 (dX): out[e][m][j] = Ag^T[e][j][m] (j < r), Au^T[e][j - r][m] (r <= j < 2r)   [E][d][2r]
// so that a tensor-memory lane (one input feature) loads its values as one
// contiguous row. One block per (64 input features, expert), transposed through
// shared memory; a value beyond the fp16 range raises TQP_STATUS_NONFINITE.
__global__ void __launch_bounds__(256) lora_a_rows_kernel(const uint16_t* __restrict__ a0,
                                                          const uint16_t* __restrict__ a1, int which, int r, int in,
                                                          uint16_t* __restrict__ out, int32_t* status) {
  // [feature][j], fp16; j < 2r <= 128, row pitch 272 B. The 8-value pieces of row f
  // are rotated by (f / 8) mod pieces, so that the eight threads that write one j
  // of eight feature groups hit different banks.
  __shared__ __align__(16) uint16_t tile[64][136];
  const int e = blockIdx.y, m0 = blockIdx.x * 64;
  const int w = which == 0 ? r : 2 * r;
  const int pcs = w >> 3;   // 16-byte pieces per output row (r % 8 == 0)
  bool bad = false;
  for (int i = threadIdx.x; i < w * 8; i += blockDim.x) {   // source rows j: 64 features = 8 pieces
    const int j = i >> 3, c = i & 7;
    const uint16_t* src = (j < r ? a0 + (size_t(e) * r + j) * in : a1 + (size_t(e) * r + (j - r)) * in) + m0 + c * 8;
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src));
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    const int jp = (((j >> 3) + c) % pcs) * 8 + (j & 7);   // rotation of row group c (rows 8c .. 8c + 7)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t h = bf16x2_to_f16x2_pk(wv[q]);
      bad |= f16x2_nonfinite(h) != 0u;
      tile[c * 8 + 2 * q][jp] = uint16_t(h & 0xFFFFu);
      tile[c * 8 + 2 * q + 1][jp] = uint16_t(h >> 16);
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < 64 * pcs; i += blockDim.x) {
    const int f = i / pcs, c = i - f * pcs;
    *reinterpret_cast<uint4*>(out + (size_t(e) * in + m0 + f) * w + c * 8) =
        *reinterpret_cast<const uint4*>(&tile[f][((c + (f >> 3)) % pcs) * 8]);
  }
  if (__syncthreads_or(bad) && threadIdx.x == 0) raise_status(status, TQP_STATUS_NONFINITE);
}

int launch_lora_a_rows(int which, const tqp_moe_weights* w, uint16_t* out, int32_t* status, cudaStream_t s) {
  const int r = w->rank;
  if (r == 0) return TQP_OK;
  const int in = which == 0 ? w->ffn : w->d;   // multiples of 64
  lora_a_rows_kernel<<<dim3(unsigned(in / 64), unsigned(w->E)), 256, 0, s>>>(
      which == 0 ? w->lora_a[2] : w->lora_a[0], which == 0 ? w->lora_a[2] : w->lora_a[1], which, r, in, out, status);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

int launch_rank_bwd(int which, const uint16_t* P, const int32_t* offsets, const int32_t* mb_prefix,
                    const tqp_moe_weights* w, int T, uint16_t* bk16, uint16_t* C, int32_t* status, cudaStream_t s) {
  const int r = w->rank, d = w->d, f = w->ffn;
  if (T == 0 || r == 0) return TQP_OK;
  const size_t A = size_t(T) * w->top_k;
  const int K = which == 0 ? d : 2 * f;
  const int n = which == 0 ? r : 2 * r;
  rank_b_kernel<<<dim3(unsigned(K / 64), unsigned(w->E)), 256, 0, s>>>(w->lora_b[which == 0 ? 2 : 0], w->lora_b[1],
                                                                       which, r, f, K, bk16);
  if (cudaGetLastError() != cudaSuccess) return TQP_ERR_CUDA;
  // C = s * P B_e^T on the rank-space engine mode: A = P rows by TMA, B = n rows of bk16 per expert
  GemmArgs a{};
  a.E = w->E;
  a.g = w->group;
  a.r = n;
  a.lora_scale = w->lora_scale;
  a.offsets = offsets;
  a.mb_prefix = mb_prefix;
  a.status = status;
  a.kb_per_piece = 1;
  a.nkb_main = K / 64;
  a.ntile = n < 16 ? 16 : n;
  a.n_tiles = 1;
  a.out = C;
  a.out_ld = n;
  a.n_valid = n;
  Maps mp{};
  if (!make_tile_map(&mp.m[TA], P, uint64_t(A), uint64_t(K), 128) ||
      !make_tile_map(&mp.m[TB0], bk16, uint64_t(w->E) * n, uint64_t(K), uint32_t(n)))
    return TQP_ERR_CUDA;
  const int mb_upper = int((A + kMBlock - 1) / kMBlock) + w->E;
  return run_gemm<LORA_HA>(a, mp, mb_upper, s);
}

int launch_dgrad(int which, const uint16_t* a_src, const uint16_t* a_lora, const int32_t* offsets,
                 const int32_t* mb_prefix, const tqp_moe_weights* w, int T, const uint16_t* aux_gu, uint16_t* out,
                 int32_t* status, cudaStream_t s, const int32_t* mb_prefix256, int4* unit_tab, const uint16_t* a_rows) {
  if (T == 0) return TQP_OK;
  const size_t A = size_t(T) * w->top_k;
  const int d = w->d, f = w->ffn, r = w->rank;
  const int mb_upper = int((A + kMBlock - 1) / kMBlock) + w->E;
  GemmArgs a{};
  a.E = w->E;
  a.g = w->group;
  a.r = r;
  a.lora_scale = w->lora_scale;
  a.offsets = offsets;
  a.mb_prefix = mb_prefix;
  a.kb_per_piece = 1;
  a.status = status;
  a.f_dim = f;
  a.a_lora = a_lora;
  a.out = out;
  a.bits = w->bits == 8 ? 8 : 4;
  const int bB = a.bits;   // code bits: a tile row of ntile features is ntile * bits / 8 bytes
  Maps mp{};
  if (which == 0 && mb_prefix256 && unit_tab && f % 128 == 0) {
    // dH with Wd^T in tensor memory (expert_dgrad.cu): units of 128 hidden features
    // x up to 256 rows; K = r rank-space columns, then the d rows of Wd; the
    // SwiGLU backward writes [dG | dU]
    a.mb_prefix = mb_prefix256;
    a.nkb_main = d / 64;
    a.half_kb = d / 64;   // one weight matrix
    a.nkb_lora = r > 0 ? (r + 63) / 64 : 0;
    a.lora_k = r;
    a.n_tiles = f / 128;
    a.in_dim = f;
    a.out_dim = d;
    a.lb0 = w->lora_a[2];
    a.lb_ld = f;
    a.lt = r > 0 ? a_rows : nullptr;
    a.lt_w = r;
    a.aux = const_cast<uint16_t*>(aux_gu);
    a.out_ld = 2 * f;
    a.n_valid = f;
    const uint32_t cbox = uint32_t(128 * bB / 8);   // one tile's 128 features of a code row
    const uint32_t srows = uint32_t(w->group >= 128 ? 1 : 128 / w->group);
    const uint64_t crow = uint64_t(f) * bB / 8;
    bool ok = make_map(&mp.m[TQ0], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[2], crow, uint64_t(w->E) * d, crow, cbox, 64,
                       int(cbox)) &&
              make_map(&mp.m[TS0], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[2], d, uint64_t(w->E) * (f / w->group),
                       uint64_t(d) * 2, 64, srows) &&
              make_tile_map(&mp.m[TA], a_src, uint64_t(A), uint64_t(d), 128);
    if (ok && r > 0) ok = make_tile_map(&mp.m[TB0], a_lora, uint64_t(A), uint64_t(r), 128);
    if (!ok) return TQP_ERR_CUDA;
    mp.m[TQ1] = mp.m[TQ0];   // one weight matrix: the second map slot repeats the first
    mp.m[TS1] = mp.m[TS0];
    const int units_upper = int((A + 255) / 256 + w->E) * a.n_tiles;
    int rc = build_unit_table(a, 256, units_upper, unit_tab, s);
    if (rc != TQP_OK) return rc;
    a.unit_tab = unit_tab;
    a.wait_ns = wait_limit_ns();
    return run_expert_dgrad(DH, a, mp, units_upper, s);
  }
  // dH runs only on the tensor-memory kernel (the backward requires ffn % 128 == 0)
  if (which == 0) return TQP_ERR_UNSUPPORTED;
  if (mb_prefix256 && unit_tab && d % 128 == 0) {
    // DX with W^T in tensor memory (expert_dgrad.cu): units of 128 input features x
    // up to 256 rows; K = 2r rank-space columns, then the f gate and f up rows of W
    a.mb_prefix = mb_prefix256;
    a.nkb_main = 2 * f / 64;
    a.half_kb = f / 64;
    a.nkb_lora = r > 0 ? (2 * r + 63) / 64 : 0;
    a.lora_k = 2 * r;
    a.n_tiles = d / 128;
    a.in_dim = d;
    a.out_dim = f;
    a.lb0 = w->lora_a[0];
    a.lb1 = w->lora_a[1];
    a.lb_ld = d;
    a.lt = r > 0 ? a_rows : nullptr;
    a.lt_w = 2 * r;
    a.out_ld = d;
    a.n_valid = d;
    const uint32_t cbox = uint32_t(128 * bB / 8);   // one tile's 128 features of a code row
    const uint32_t srows = uint32_t(w->group >= 128 ? 1 : 128 / w->group);
    const uint64_t crow = uint64_t(d) * bB / 8;
    bool ok = make_map(&mp.m[TQ0], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[0], crow, uint64_t(w->E) * f, crow, cbox, 64,
                       int(cbox)) &&
              make_map(&mp.m[TQ1], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[1], crow, uint64_t(w->E) * f, crow, cbox, 64,
                       int(cbox)) &&
              make_map(&mp.m[TS0], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[0], f, uint64_t(w->E) * (d / w->group),
                       uint64_t(f) * 2, 64, srows) &&
              make_map(&mp.m[TS1], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[1], f, uint64_t(w->E) * (d / w->group),
                       uint64_t(f) * 2, 64, srows) &&
              make_tile_map(&mp.m[TA], a_src, uint64_t(A), uint64_t(2 * f), 128);
    if (ok && r > 0) ok = make_tile_map(&mp.m[TB0], a_lora, uint64_t(A), uint64_t(2 * r), 128);
    if (!ok) return TQP_ERR_CUDA;
    const int units_upper = int((A + 255) / 256 + w->E) * a.n_tiles;
    int rc = build_unit_table(a, 256, units_upper, unit_tab, s);
    if (rc != TQP_OK) return rc;
    a.unit_tab = unit_tab;
    a.wait_ns = wait_limit_ns();
    return run_expert_dgrad(DX, a, mp, units_upper, s);
  }
  // DX on the shared-memory engine: K = 2f (gate rows then up rows of W), N = d
  a.ntile = (d % 256 == 0 && bB == 4) ? 256 : 128;
  const int ngn = w->group >= a.ntile ? 1 : a.ntile / w->group;
  a.nkb_main = 2 * f / 64;
  a.half_kb = f / 64;
  a.nkb_lora = r > 0 ? (2 * r + 63) / 64 : 0;
  a.lora_k = 2 * r;
  a.lora_ld = 2 * r;
  a.n_tiles = d / a.ntile;
  a.in_dim = d;
  a.out_dim = f;
  a.lb0 = w->lora_a[0];
  a.lb1 = w->lora_a[1];
  a.lb_ld = d;
  a.out_ld = d;
  a.n_valid = d;
  bool ok = make_tile_map(&mp.m[TA], a_src, uint64_t(A), uint64_t(2 * f), 128) &&
            make_map(&mp.m[TQ0], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[0], uint64_t(d) * bB / 8, uint64_t(w->E) * f,
                     uint64_t(d) * bB / 8, uint32_t(a.ntile * bB / 8), 64, a.ntile * bB / 8 == 128 ? 128 : 0) &&
            make_map(&mp.m[TQ1], CU_TENSOR_MAP_DATA_TYPE_UINT8, w->wq[1], uint64_t(d) * bB / 8, uint64_t(w->E) * f,
                     uint64_t(d) * bB / 8, uint32_t(a.ntile * bB / 8), 64, a.ntile * bB / 8 == 128 ? 128 : 0) &&
            make_map(&mp.m[TS0], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[0], f, uint64_t(w->E) * (d / w->group),
                     uint64_t(f) * 2, 64, ngn) &&
            make_map(&mp.m[TS1], CU_TENSOR_MAP_DATA_TYPE_UINT16, w->wscale[1], f, uint64_t(w->E) * (d / w->group),
                     uint64_t(f) * 2, 64, ngn);
  if (!ok) return TQP_ERR_CUDA;
  return run_gemm<DX>(a, mp, mb_upper * a.n_tiles, s);
}

}  // namespace tqp
