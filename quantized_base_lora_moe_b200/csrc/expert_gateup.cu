// Gate/up expert projection of the TQP MoE layer with wide token blocks and the
// dequantised base weights in tensor memory (sm_100a, tcgen05):
//   [G|U] = X_e [Wg|Wu]^T + (s X [Ag|Au]) [Bg|Bu],  H = silu(G) * U
// (low-rank adapters trained per expert over frozen quantised base expert
// weights: "Reversible Sparse MoE Single Node", Pattern 3; SwiGLU experts, TQP
// Quantization).
//
// The contraction runs transposed, D[feature][token] = W[feature][:] . X[token][:].
// A work unit is (expert e, feature tile, block of up to 256 routed rows). In
// each CTA the A operand (128 TMEM lanes) stacks the gate rows of 64 features
// on their 64 up rows, so one MMA serves both projections and SwiGLU pairs
// lane j with lane 64 + j in the same CTA. Each weight tile is dequantised once
// per 256-row block (once per expert for all but the largest experts). The token
// rows come expert-sorted (X_perm, written by the prepare step) as TMA boxes of
// 128 rows, so no thread gathers rows.
//
// The kernel runs on CTA pairs (a cluster of 2, kGateUpPair): one tcgen05.mma of
// 256 x N x 16 (cta_group::2, issued by the even CTA, N = the block's rows
// rounded up to 32) covers the unit's 128 features. Each CTA holds its 64
// features' weight rows in its own TMEM and half of the token rows in its own
// shared memory, and receives the accumulator of its 64 features for all N
// tokens. Per SM that halves the token bytes per MMA against a single CTA with
// the same tile, and doubles the token ring's depth in stages. Without pairs
// (kGateUpPair false) a CTA takes a unit of 64 features and all its rows alone.
//
// Per CTA (1 per SM, 896 threads):
//   warps 0-3, 24-27  epilogue, two groups taking alternate 32-token chunks:
//               drain the accumulator lane by lane (TMEM lane = one gate or up
//               feature), hand TMEM back, then SwiGLU and 16-byte row stores
//               through a [token][feature] tile per group
//   warp  4     TMEM allocation; one thread issuing tcgen05.mma (even CTA) or
//               relaying the odd CTA's ready stages to it
//   warp  5     TMA producer of the code / bf16 scale ring (int4 rows
//               32B-swizzled, int8 rows 64B-swizzled: conflict-free row reads)
//   warp  6     TMA producer of the token ring: X_perm boxes, and the rank-space
//               rows s X [Ag|Au] for the adapter stage
//   warps 8-23  weight producer, four groups of 4 warps on stages n % 4: each
//               thread dequantises 64 K values of one weight row (int4 or int8
//               -> fp16) into TMEM; LoRA B rows for the adapter stage
// TMEM (512 columns): one accumulator in [0, 256) (lanes 0-63 gate, 64-127 up),
// 8 weight stages of 32 columns (64 K values) in [256, 512). Token ring: 96 KB
// (3 stages of 256 rows, or 6 of 128 rows in a pair). Range: an H (or kept
// G|U) value or a LoRA B value beyond the fp16 range raises
// TQP_STATUS_NONFINITE; a group scale whose dequantised products are not exact
// in fp16 raises TQP_STATUS_RANGE. Every wait is bounded (tqp_device.cuh); on an
// abort every asynchronous copy and MMA still in flight is drained before the
// CTA frees its memory, and the two CTAs of a pair meet before either frees
// its tensor memory or exits. No TMA multicast is used.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "expert_common.cuh"
#include "gemm_common.cuh"
#include "tqp_device.cuh"
#include "tqp_launch.h"

namespace tqp {

namespace gu_wide {

constexpr int kRows = 256;            // routed rows per unit
constexpr int kF = 64;                // features per CTA and unit, of gate and of up each
constexpr int kK = 64;                // K per pipeline stage
// Token ring: a single CTA holds all of a unit's rows (3 stages of 256 rows x
// 128 B); in a CTA pair each CTA holds half of them (6 stages of 128 rows).
template <bool PAIR>
struct XCfg {
  static constexpr int kStages = PAIR ? 6 : 3;
  static constexpr int kStageBytes = (PAIR ? kRows / 2 : kRows) * kK * 2;
};
constexpr int kXStagesMax = 6;
constexpr int kXRingBytes = 3 * kRows * kK * 2;   // the same bytes either way
constexpr int kWStages = 8;
constexpr uint32_t kWCols = 32;       // TMEM columns per weight stage (64 fp16 K values)
constexpr uint32_t kWBase = 256;
constexpr int kQStagesMax = 8;
constexpr int kGroups = 4;            // weight-producer groups
constexpr int kWWarp0 = 8;            // first weight-producer warp (a multiple of 4)
constexpr int kWWarps = 16;
constexpr int kEpi1Warp0 = kWWarp0 + kWWarps;   // second epilogue group (4 warps)
constexpr int kThreads = (kEpi1Warp0 + 4) * 32;
constexpr int kDRow = 528;            // drain row: 256 tokens in fp16 + 16 B against bank conflicts
constexpr int kHRow = 144;            // chunk tile row: one token's 64 features in fp16 + 16 B
constexpr int kStaging = 128 * kDRow + 2 * 32 * kHRow;

struct Ctl {
  uint64_t x_empty[kXStagesMax];
  // stage n is ready when full[n % 8] completes: the weight group's 4 warps, the
  // token tile's TMA bytes and (pair, even CTA) the odd CTA's relay arrived
  uint64_t w_full[kWStages], w_empty[kWStages];
  uint64_t q_full[kQStagesMax], q_empty[kQStagesMax];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint64_t epi[2];
  uint32_t tmem_base;
  Abort ab;
};

// Code ring per code width: a stage holds 64 K values of the tile's 64 gate
// rows and 64 up rows (32 B per row for int4, 64 B for int8; TMA 32B / 64B
// swizzle) and up to 2 x 2 x 64 scales.
template <int BITS>
struct QCfg {
  static constexpr int kCB = 8 * BITS;                 // code bytes per row and stage
  static constexpr int kStages = BITS == 4 ? 8 : 5;
  static constexpr int kStageBytes = 128 * kCB + 512;
  // 16-byte chunk c of row r of one 64-row box, as the TMA swizzle placed it
  __device__ static __forceinline__ int chunk_offset(int r, int c) {
    return r * kCB + ((BITS == 4 ? (c ^ ((r >> 2) & 1)) : (c ^ ((r >> 1) & 3))) << 4);
  }
};

template <int BITS>
constexpr size_t smem_bytes() {
  return 1024 + size_t(kXRingBytes) + size_t(QCfg<BITS>::kStages) * QCfg<BITS>::kStageBytes + size_t(kStaging) +
         sizeof(Ctl);
}
static_assert(smem_bytes<4>() + 2 * (kSchedSmemE + 1) * 4 <= 232448, "shared memory budget");
static_assert(smem_bytes<8>() + 2 * (kSchedSmemE + 1) * 4 <= 232448, "shared memory budget");

// 16 tokens x this lane's feature (8 words of fp16 pairs, word j = tokens
// t0+2j, t0+2j+1) into the [token][64 feature] chunk tile: lane pairs trade
// halves so that each lane writes two adjacent features of one token as one
// 32-bit word.
__device__ __forceinline__ void stage16(uint8_t* tile, int t0, int feat, const uint32_t* w) {
  const bool odd = (threadIdx.x & 1) != 0;
  uint8_t* colp = tile + (feat & ~1) * 2;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, w[j], 1);
    const uint32_t v = odd ? __byte_perm(other, w[j], 0x7632) : __byte_perm(w[j], other, 0x5410);
    *reinterpret_cast<uint32_t*>(colp + (t0 + 2 * j + (odd ? 1 : 0)) * kHRow) = v;
  }
}

// PAIR: a cluster of two CTAs shares each unit. One tcgen05.mma of M = 256
// (cta_group::2, issued by the even CTA) covers 128 features: each CTA holds
// the 64 gate and 64 up rows of its 64 features in its own TMEM, half of the
// unit's token rows in its shared memory, and receives its 128 x N quarter of
// the accumulator (all N tokens of its features), so SwiGLU stays in the CTA.
// Stage n is ready when the even CTA's full barrier completes: both CTAs' weight
// groups arrive on it (the odd CTA's remotely, release at cluster scope), and
// both CTAs' token loads complete their bytes on it (the odd CTA's through the
// cta_group::2 form of the TMA load); the even CTA's token thread expects the
// bytes of both halves. The MMA completions are multicast to both CTAs.
//
// Every role arrives once per warp (after __syncwarp), and the MMA thread waits
// on one barrier per stage (weights, token bytes and the pair relay together).
template <int BITS, bool PAIR>
__global__ void __launch_bounds__(kThreads, 1)
    gateup_wide_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tq0, const __grid_constant__ CUtensorMap tq1,
                       const __grid_constant__ CUtensorMap ts0, const __grid_constant__ CUtensorMap ts1,
                       const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap txa) {
  using QC = QCfg<BITS>;
  constexpr int kQStages = QC::kStages;
  constexpr int kQStageBytes = QC::kStageBytes;
  constexpr int kCB = QC::kCB;
  constexpr int kXStages = XCfg<PAIR>::kStages;
  constexpr int kXStageBytes = XCfg<PAIR>::kStageBytes;
  constexpr int kFU = PAIR ? 2 * kF : kF;   // features of a unit (the pair's together)
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* x_base = smem;
  uint8_t* q_base = x_base + size_t(kXRingBytes);
  uint8_t* staging = q_base + size_t(kQStages) * kQStageBytes;
  Ctl* ctl = reinterpret_cast<Ctl*>(staging + kStaging);
  Abort* abort_flag = &ctl->ab;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int rank = PAIR ? int(cluster_ctarank()) : 0;   // CTA within the pair
  const int fofs = rank * kF;                           // this CTA's features within the unit's tile
  __shared__ int32_t s_sched[2 * (kSchedSmemE + 1)];
  const Sched sc = load_sched(a, s_sched);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kXStages; ++i) mbar_init(&ctl->x_empty[i], 1);
    for (int i = 0; i < kWStages; ++i) {
      // one weight group (4 warps) + the token TMA thread; pair (even CTA): the
      // odd CTA's weight group as well (its token bytes need no arrival)
      mbar_init(&ctl->w_full[i], PAIR ? 4 + 4 + 1 : 4 + 1);
      mbar_init(&ctl->w_empty[i], 1);
    }
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_empty[i], 4);   // the 4 warps of the consuming group
    }
    mbar_init(&ctl->acc_full, 1);
    // one arrival per epilogue warp: both groups (and, pair, both CTAs)
    mbar_init(&ctl->acc_empty, PAIR ? 16 : 8);
    mbar_init(&ctl->drain, 1);
    mbar_init(&ctl->epi[0], 4);
    mbar_init(&ctl->epi[1], 4);
    abort_init(&ctl->ab, a.wait_ns);
    fence_barrier_init();
  }
  if (warp == 4) {
    if (PAIR) {
      tmem_alloc2(&ctl->tmem_base, 512);
      tmem_relinquish2();
    } else {
      tmem_alloc(&ctl->tmem_base, 512);
      tmem_relinquish();
    }
  }
  if (threadIdx.x == 5 * 32) {
    prefetch_tmap(&tq0);
    prefetch_tmap(&tq1);
    prefetch_tmap(&ts0);
    prefetch_tmap(&ts1);
  }
  if (threadIdx.x == 6 * 32) {
    prefetch_tmap(&tx);
    if (a.nkb_lora > 0) prefetch_tmap(&txa);
  }
  tc_fence_before();
  __syncthreads();
  // pair: both CTAs' barriers are initialised and their TMEM allocated before
  // any arrival, commit or MMA crosses to the other CTA
  if (PAIR) cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  const int nunits = total_units(a, sc);
  const int u0 = PAIR ? int(blockIdx.x >> 1) : int(blockIdx.x);   // both CTAs of a pair take the same units
  const int ustride = PAIR ? int(gridDim.x >> 1) : int(gridDim.x);
  UnitStream us{a.unit_tab, nunits, ustride};
  us.start(u0);
  const int nkb = a.nkb_main + a.nkb_lora;
  const int ngrp = a.g >= kK ? 1 : kK / a.g;   // scale rows per K stage

  if (warp < 4 || warp >= kEpi1Warp0) {
    // ------------------------------------------------------------ epilogue
    const int eg = warp < 4 ? 0 : 1;           // group: 32-token chunks with (c / 32) % 2 == eg
    const int lrow = 32 * (warp & 3) + lane;   // TMEM lane: gate feature lrow (< 64) or up feature lrow - 64
    const int etid = lrow;                     // thread index within the group
    const uint32_t tl = tmem_base + (uint32_t(32 * (warp & 3)) << 16);
    uint8_t* drow = staging + lrow * kDRow;
    uint8_t* ct = staging + 128 * kDRow + eg * 32 * kHRow;
    // SwiGLU assignment: feature j of the tile, tokens [16 hh, 16 hh + 16) of each chunk
    const int j = etid & 63, hh = etid >> 6;
    const uint8_t* grow = staging + j * kDRow;
    const uint8_t* urow = staging + (64 + j) * kDRow;
    EpiSyncT<true> es{&ctl->epi[eg]};
    uint32_t bad = 0;   // nonzero once an fp16 output of a valid token overflowed
    int it = 0;
    // pair: each epilogue warp's arrival goes to the even CTA's barrier
    const uint32_t acc_empty0 = PAIR ? mapa_shared(smem_u32(&ctl->acc_empty), 0) : 0u;
    for (int u = u0; u < nunits; u += ustride, ++it) {
      const Unit un = us.take(u);
      const int n16 = PAIR ? (un.rows + 31) & ~31 : (un.rows + 15) & ~15;   // accumulator columns
      if (!mbar_wait_warp<128>(&ctl->acc_full, uint32_t(it) & 1u, abort_flag, a.status)) break;
      tc_fence_after();
      // drain this group's chunks of this lane's row as fp16
#pragma unroll 1
      for (int c = 32 * eg; c < n16; c += 64) {
        float v[32];
        tmem_ld32(tl + uint32_t(c), v);
        uint4* dst = reinterpret_cast<uint4*>(drow + 2 * c);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          dst[q4] = make_uint4(f32x2_to_f16x2(v[8 * q4], v[8 * q4 + 1]), f32x2_to_f16x2(v[8 * q4 + 2], v[8 * q4 + 3]),
                               f32x2_to_f16x2(v[8 * q4 + 4], v[8 * q4 + 5]),
                               f32x2_to_f16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) mbar_arrive_cluster(acc_empty0);
        else mbar_arrive(&ctl->acc_empty);
      }
      // the group's gate and up rows of its chunks are complete
      if (!es.sync(abort_flag, a.status)) break;
      uint16_t* hout = static_cast<uint16_t*>(a.out) + un.nt * kFU + fofs;
      bool stop = false;
#pragma unroll 1
      for (int c = 32 * eg; c < n16; c += 64) {
        const int nt = min(32, un.rows - c);
        auto words8 = [&](const uint8_t* src, uint32_t* w) {
          const uint4 v0 = *reinterpret_cast<const uint4*>(src + 2 * (c + 16 * hh));
          const uint4 v1 = *reinterpret_cast<const uint4*>(src + 2 * (c + 16 * hh) + 16);
          w[0] = v0.x; w[1] = v0.y; w[2] = v0.z; w[3] = v0.w;
          w[4] = v1.x; w[5] = v1.y; w[6] = v1.z; w[7] = v1.w;
        };
        // one [32 token][64 feature] chunk through the tile: wait until the tile
        // is free, transpose into it, wait until complete, 16-byte row stores
        auto emit = [&](const uint32_t* w, uint16_t* dst, size_t ld) -> bool {
          if (!es.sync(abort_flag, a.status)) return false;
          stage16(ct, 16 * hh, j, w);
          if (!es.sync(abort_flag, a.status)) return false;
          // (only valid tokens are stored and checked: padding columns hold stale data)
          for (int p = etid; p < nt * 8; p += 128) {
            const int t = p >> 3, fg = p & 7;
            const uint4 v = *reinterpret_cast<const uint4*>(ct + t * kHRow + fg * 16);
            bad |= f16x2_nonfinite(v.x) | f16x2_nonfinite(v.y) | f16x2_nonfinite(v.z) | f16x2_nonfinite(v.w);
            *reinterpret_cast<uint4*>(dst + size_t(un.base + c + t) * ld + fg * 8) = v;
          }
          return true;
        };
        uint32_t hw[8];
        {
          uint32_t gw[8], uw[8];
          words8(grow, gw);
          words8(urow, uw);
#pragma unroll
          for (int q = 0; q < 8; ++q) hw[q] = swiglu_pair(gw[q], uw[q]);
        }
        if (!emit(hw, hout, size_t(a.out_ld))) { stop = true; break; }
        if (a.aux) {  // keep the pre-activations for the backward: G in [0, f), U in [f, 2f)
          uint16_t* aux = a.aux + un.nt * kFU + fofs;
          uint32_t w8[8];
          words8(grow, w8);
          if (!emit(w8, aux, 2 * size_t(a.f_dim))) { stop = true; break; }
          words8(urow, w8);
          if (!emit(w8, aux + a.f_dim, 2 * size_t(a.f_dim))) { stop = true; break; }
        }
      }
      if (stop) break;
    }
    if (__any_sync(0xFFFFFFFFu, bad != 0) && lane == 0) raise_status(a.status, TQP_STATUS_NONFINITE);
  } else if (warp == 4) {
    if (lane == 0 && (!PAIR || rank == 0)) {
      // ------------------------------------------------------------ MMA issuer
      Ring rx, rw;
      int it = 0;
      bool ok = true;
      // descriptors of ring stage 0; a stage's are these plus a fixed offset
      const uint64_t xdesc0 = sdesc_k_sw128(smem_u32(x_base));
      const uint32_t wa0 = tmem_base + kWBase;
      for (int u = u0; u < nunits && ok; u += ustride, ++it) {
        const Unit un = us.take(u);
        const int ncol = PAIR ? (un.rows + 31) & ~31 : (un.rows + 15) & ~15;
        const uint32_t idesc = idesc_f16(PAIR ? 256 : 128, ncol);
        if (!mbar_wait<0, PAIR>(&ctl->acc_empty, (uint32_t(it) & 1u) ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t accf = 0u;   // the unit's first MMA overwrites the accumulator
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait<0, PAIR>(&ctl->w_full[rw.stage], rw.phase, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = xdesc0 + uint64_t(rx.stage) * uint64_t(kXStageBytes >> 4);
          const uint32_t wa = wa0 + uint32_t(rw.stage) * kWCols;
          auto mma = [&](int kk) {
            if (PAIR) umma2_f16_ts(tmem_base, wa + uint32_t(8 * kk), bdesc + uint64_t(2 * kk), idesc, accf);
            else umma_f16_ts(tmem_base, wa + uint32_t(8 * kk), bdesc + uint64_t(2 * kk), idesc, accf);
            accf = 1u;
          };
          if (kb >= a.nkb_lora) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) mma(kk);
          } else {
            // the rank-space stage has only its first lora_k columns live (within the first 64)
            const int ksteps = (min(kK, a.lora_k - kb * kK) + 15) / 16;
            for (int kk = 0; kk < ksteps; ++kk) mma(kk);
          }
          if (PAIR) {
            umma2_commit_both(&ctl->x_empty[rx.stage]);
            umma2_commit_both(&ctl->w_empty[rw.stage]);
          } else {
            umma_commit(&ctl->x_empty[rx.stage]);
            umma_commit(&ctl->w_empty[rw.stage]);
          }
          rx.next<kXStages>();
          rw.next<kWStages>();
        }
        if (!ok) break;
        if (PAIR) umma2_commit_both(&ctl->acc_full);
        else umma_commit(&ctl->acc_full);
      }
      // no MMA may still read or write TMEM (of either CTA) when it is freed:
      // wait for all of them (they run to completion whether or not the CTA aborted)
      if (PAIR) umma2_commit_both(&ctl->drain);
      else umma_commit(&ctl->drain);
      mbar_drain(&ctl->drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ TMA producer (codes + scales)
    if (lane == 0) {
      Ring q;
      PendingFills pend;
      // gate codes [64 rows][kCB B] | up codes | gate scales [ngrp][64] | up scales
      const uint32_t bytes = uint32_t(128 * kCB + 256 * ngrp);
      const int gpe = a.in_dim / a.g;  // scale rows per expert
      for (int u = u0; u < nunits; u += ustride) {
        const Unit un = us.take(u);
        const int fcol = un.nt * kFU + fofs;   // first feature of this CTA's rows
        const int nrow0 = un.e * a.out_dim + fcol;
        bool ok = true;
        for (int km = 0; km < a.nkb_main; ++km) {
          if (!mbar_wait<64>(&ctl->q_empty[q.stage], q.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
          uint8_t* qs = q_base + size_t(q.stage) * kQStageBytes;
          uint64_t* bar = &ctl->q_full[q.stage];
          const int srow = un.e * gpe + (km * kK) / a.g;
          mbar_arrive_expect_tx(bar, bytes);
          tma_load_2d(smem_u32(qs), &tq0, bar, km * kCB, nrow0);
          tma_load_2d(smem_u32(qs + 64 * kCB), &tq1, bar, km * kCB, nrow0);
          tma_load_2d(smem_u32(qs + 128 * kCB), &ts0, bar, fcol, srow);
          tma_load_2d(smem_u32(qs + 128 * kCB + 128 * ngrp), &ts1, bar, fcol, srow);
          pend.issued(q.stage, q.phase);
          q.next<kQStages>();
        }
        if (!ok) break;
      }
      // on an abort, wait (bounded) until every issued fill has landed
      if (aborted(abort_flag)) pend.drain(ctl->q_full);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ TMA producer (token rows)
    if (lane == 0) {
      Ring rx, rw;
      PendingFills pend;
      for (int u = u0; u < nunits; u += ustride) {
        const Unit un = us.take(u);
        // single CTA: a second 128-row box only when the MMA reads it; pair: this
        // CTA's half of the N = rows rounded up to 32 columns, one box
        const int nbox = (!PAIR && un.rows > 128) ? 2 : 1;
        const int row0 = un.base + (PAIR ? rank * (((un.rows + 31) & ~31) >> 1) : 0);
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait<64>(&ctl->x_empty[rx.stage], rx.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
          uint8_t* st = x_base + size_t(rx.stage) * kXStageBytes;
          uint64_t* bar = &ctl->w_full[rw.stage];
          // the adapter stage reads s X [Ag|Au] (zero-filled past its 2r columns), the rest X_perm
          const CUtensorMap* map = kb < a.nkb_lora ? &txa : &tx;
          const int col = (kb < a.nkb_lora ? kb : kb - a.nkb_lora) * kK;
          if (!PAIR) {
            mbar_arrive_expect_tx(bar, uint32_t(nbox * 16384));
            tma_load_2d(smem_u32(st), map, bar, col, row0);
            if (nbox == 2) tma_load_2d(smem_u32(st + 16384), map, bar, col, row0 + 128);
          } else if (rank == 0) {
            mbar_arrive_expect_tx(bar, uint32_t(2 * 16384));   // both CTAs' halves
            tma_load_2d(smem_u32(st), map, bar, col, row0);
          } else {
            tma_load_2d_pair(smem_u32(st), map, mapa_shared(smem_u32(bar), 0), col, row0);
          }
          pend.issued(rw.stage, rw.phase);
          rx.next<kXStages>();
          rw.next<kWStages>();
        }
        if (!ok) break;
      }
      // (the odd CTA's fills complete on the even CTA's barriers, which the even
      // CTA drains before the pair's final cluster barrier)
      if (aborted(abort_flag) && (!PAIR || rank == 0)) pend.drain(ctl->w_full);
    }
  } else if (warp >= kWWarp0) {
    // ------------------------------------------------------------ weight producer
    // Four groups of 4 warps take stages n % 4, so that four stages are being
    // dequantised at any time (one stage's chain of code read -> dequant ->
    // TMEM store -> arrive is latency-bound). A thread converts 64 consecutive
    // K values (8 int4 words) of one weight row: TMEM lane lrow, the gate row
    // of feature lrow (lrow < 64) or the up row of feature lrow - 64.
    const int wi = warp - kWWarp0;            // 0..15
    const int grp = wi >> 2;                  // stages n with n % 4 == grp
    const int lrow = 32 * (warp & 3) + lane;  // TMEM lane
    const int mat = lrow >> 6;                // 0 gate, 1 up
    const int r64 = lrow & 63;                // row within the tile's gate / up box
    const uint32_t tw = tmem_base + (uint32_t(32 * (warp & 3)) << 16) + kWBase;
    const int row_off = mat * 64 * kCB;
    // scale rows of the two 32-wide K halves of this thread's slice
    const int g_hi = (ngrp == 1) ? 0 : 32 / a.g;
    const int sbase = 128 * kCB + mat * 128 * ngrp;
    const int s_lo_off = sbase + r64 * 2, s_hi_off = sbase + (g_hi * 64 + r64) * 2;
    const uint16_t* bsrc = mat ? a.b1 : a.b0;
    bool inexact = false;   // a group scale whose products q * s are not exact in fp16
    bool lora_inf = false;  // a LoRA B value beyond the fp16 range
    int n = 0;    // pipeline stage counter of this CTA
    int m = 0;    // main (code-carrying) stage counter
    for (int u = u0; u < nunits; u += ustride) {
      const Unit un = us.take(u);
      const int feat = un.nt * kFU + fofs + r64;   // output feature of this row
      bool ok = true;
      if (a.nkb_lora > 0 && grp == 0 && u + ustride < nunits) {
        // the next unit's LoRA B row into L2 (its rank-space stage comes first)
        const Unit nx = us.peek();
        const uint16_t* rowp = bsrc + (size_t(nx.e) * a.out_dim + nx.nt * kFU + fofs + r64) * a.r;
        for (int off = 0; off < a.r; off += 64) prefetch_l2(rowp + off);
      }
      for (int kb = 0; kb < nkb; ++kb, ++n) {
        const bool main_stage = kb >= a.nkb_lora;
        const int mq = m;
        if (main_stage) ++m;
        if ((n & (kGroups - 1)) != grp) continue;
        const int st = n & (kWStages - 1);
        const uint32_t ph = uint32_t(n / kWStages) & 1u;
        if (!mbar_wait_warp(&ctl->w_empty[st], ph ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t v[32];
        if (!main_stage) {
          // LoRA B rows as fp16: gate rows hold Bg in K' [0, r), up rows Bu in [r, 2r)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int colk = kb * kK + c * 8;
            const int src = mat ? colk - a.r : colk;
            uint4 w4 = make_uint4(0, 0, 0, 0);
            if (src >= 0 && src < a.r)
              w4 = bf16x8_to_f16x8_chk(
                  __ldg(reinterpret_cast<const uint4*>(bsrc + (size_t(un.e) * a.out_dim + feat) * a.r + src)), lora_inf);
            v[4 * c] = w4.x; v[4 * c + 1] = w4.y; v[4 * c + 2] = w4.z; v[4 * c + 3] = w4.w;
          }
        } else {
          const int qst = mq % kQStages;
          const uint32_t qph = uint32_t(mq / kQStages) & 1u;
          if (!mbar_wait_warp(&ctl->q_full[qst], qph, abort_flag, a.status)) { ok = false; break; }
          const uint8_t* qs = q_base + size_t(qst) * kQStageBytes;
          const uint32_t s_lo = scale_pair_chk(*reinterpret_cast<const uint16_t*>(qs + s_lo_off), inexact);
          const uint32_t s_hi = scale_pair_chk(*reinterpret_cast<const uint16_t*>(qs + s_hi_off), inexact);
          if (BITS == 4) {
            // 64 K values = 8 words of 8 codes
            const uint4 wa = *reinterpret_cast<const uint4*>(qs + row_off + QC::chunk_offset(r64, 0));
            const uint4 wb = *reinterpret_cast<const uint4*>(qs + row_off + QC::chunk_offset(r64, 1));
            const uint32_t wd[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 d4 = dequant_word(wd[c], c < 4 ? s_lo : s_hi);
              v[4 * c] = d4.x; v[4 * c + 1] = d4.y; v[4 * c + 2] = d4.z; v[4 * c + 3] = d4.w;
            }
          } else {
            // 64 K values = 16 words of 4 codes
#pragma unroll
            for (int ch = 0; ch < 4; ++ch) {
              const uint4 w4 = *reinterpret_cast<const uint4*>(qs + row_off + QC::chunk_offset(r64, ch));
              const uint32_t wd[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const uint2 d2 = dequant_word8(wd[i], ch < 2 ? s_lo : s_hi);
                v[8 * ch + 2 * i] = d2.x;
                v[8 * ch + 2 * i + 1] = d2.y;
              }
            }
          }
          // the code slot's values have been consumed; its next fill is an
          // async-proxy TMA write, hence the proxy fence before handing it back
          fence_proxy_async_smem();
          mbar_arrive_warp(&ctl->q_empty[qst]);
        }
        tmem_st32(tw + uint32_t(st) * kWCols, v);
        tmem_wait_st();
        tc_fence_before();
        if (PAIR) {   // both CTAs' groups arrive on the even CTA's barrier
          __syncwarp();
          if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&ctl->w_full[st]), 0));
        } else {
          mbar_arrive_warp(&ctl->w_full[st]);
        }
      }
      if (!ok) break;
    }
    if (__any_sync(0xFFFFFFFFu, inexact) && lane == 0) raise_status(a.status, TQP_STATUS_RANGE);
    if (__any_sync(0xFFFFFFFFu, lora_inf) && lane == 0) raise_status(a.status, TQP_STATUS_NONFINITE);
  }

  tc_fence_before();
  __syncthreads();
  // pair: neither CTA frees its TMEM or exits while the other may still send
  // it arrivals or (even CTA) run MMAs on its memory
  if (PAIR) cluster_sync();
  if (warp == 4) {
    tc_fence_after();
    if (PAIR) tmem_dealloc2(tmem_base, 512);
    else tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace gu_wide

template <int BITS, bool PAIR>
static int launch_gateup_wide(const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s) {
  static DeviceFlags attr_done;
  constexpr size_t smem = gu_wide::smem_bytes<BITS>();
  auto kern = gu_wide::gateup_wide_kernel<BITS, PAIR>;
  if (!attr_done.test_and_set_device(kern, int(smem))) return TQP_ERR_CUDA;
  const int nsm = num_sms();
  if (!PAIR) {
    const int grid = units_upper < nsm ? (units_upper > 0 ? units_upper : 1) : nsm;
    kern<<<grid, gu_wide::kThreads, smem, s>>>(a, mp.m[TQ0], mp.m[TQ1], mp.m[TS0], mp.m[TS1], mp.m[TA], mp.m[TB0]);
    return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg{};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(gu_wide::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // as many pairs as can be resident at once (persistent), at most one per unit
  int max_pairs = 0;
  cfg.gridDim = dim3(unsigned(nsm & ~1));
  if (cudaOccupancyMaxActiveClusters(&max_pairs, kern, &cfg) != cudaSuccess || max_pairs <= 0) max_pairs = nsm / 2;
  const int pairs = units_upper < max_pairs ? (units_upper > 0 ? units_upper : 1) : max_pairs;
  cfg.gridDim = dim3(unsigned(2 * pairs));
  if (cudaLaunchKernelEx(&cfg, kern, a, mp.m[TQ0], mp.m[TQ1], mp.m[TS0], mp.m[TS1], mp.m[TA], mp.m[TB0]) !=
      cudaSuccess)
    return TQP_ERR_CUDA;
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

int run_expert_gateup_wide(const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s) {
  return a.bits == 8 ? launch_gateup_wide<8, kGateUpPair>(a, mp, units_upper, s)
                     : launch_gateup_wide<4, kGateUpPair>(a, mp, units_upper, s);
}

}  // namespace tqp
