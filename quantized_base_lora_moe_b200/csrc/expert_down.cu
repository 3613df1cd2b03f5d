// Down projection of the TQP MoE experts with wide token blocks (sm_100a):
//   O = H_e Wd^T + (s H Ad) Bd
// (low-rank adapters trained per expert over frozen quantised base expert
// weights: "Reversible Sparse MoE Single Node", Pattern 3; SwiGLU experts, TQP
// Quantization).
//
// As in the gate/up kernel (expert_gateup.cu), the contraction runs transposed, D[feature][token] =
// Wd[feature][:] . H[token][:], with the dequantised 128-feature weight tile as
// the tcgen05.mma A operand in TMEM and the expert's routed rows as the B
// operand in shared memory. Here a unit takes up to 256 rows of one expert, so
// that an expert of the 460-expert configuration (about 214 rows on average)
// is one block: every MMA is 128 x N x 16 with N up to 256 (half as many MMA
// instructions per expert as 128-row blocks, each near the compute-bound
// rate), and every weight tile is dequantised once per expert instead of once
// per 128-row block.
//
// Work unit = (expert e, 128-feature tile, block of up to 256 routed rows),
// ordered (expert, tile, block) over a persistent grid. Per CTA (1 per SM, 960
// threads):
//   warps 0-3, 26-29  epilogue, two groups taking alternate 32-token chunks:
//               drain the accumulator row by row (one feature per thread,
//               16-byte shared-memory stores), hand TMEM back, then send their
//               chunks out through a [token][feature] tile per group as
//               16-byte row pieces (the single accumulator is released after
//               half the drain time)
//   warp  4     TMEM allocation + one thread issuing tcgen05.mma
//   warp  5     TMA producer of the code / bf16 scale ring (int4 rows
//               32B-swizzled, int8 rows 64B-swizzled, read without bank conflicts)
//   warp  6     TMA producer of the token ring: two boxes of 128 H rows per
//               64-wide K stage, and the rank-space rows s H Ad (zero-filled
//               past their r columns) for the adapter stage
//   warps 7-9   idle
//   warps 10-25 weight producer, four groups of 4 warps on stages n % 4: each
//               thread dequantises the 64 K values of one weight row per stage
//               (int4 or int8 -> fp16) into TMEM; LoRA B rows
// TMEM (512 columns): one accumulator in [0, 256), 8 weight stages of 32
// columns (64 K values) in [256, 512). Token ring: 3 stages of 32 KB. Stage n is
// ready when full[n % 8] completes (the weight group's 4 warps and the token
// tile's TMA bytes), so the MMA thread waits once per stage; every role arrives
// once per warp.
// An O value of a routed row or a LoRA B value beyond the fp16 range raises
// TQP_STATUS_NONFINITE; a group scale whose dequantised products are not exact
// in fp16 raises TQP_STATUS_RANGE. Every wait is bounded (tqp_device.cuh); on an abort every
// asynchronous copy and MMA still in flight is drained before the CTA frees
// its memory. No TMA multicast is used.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "expert_common.cuh"
#include "gemm_common.cuh"
#include "tqp_device.cuh"
#include "tqp_launch.h"

namespace tqp {
namespace down_wide {

constexpr int kWWarp0 = 10;
constexpr int kWWarps = 16;
constexpr int kEpi1Warp0 = kWWarp0 + kWWarps;   // second epilogue group (4 warps)
constexpr int kThreads = (kEpi1Warp0 + 4) * 32;
constexpr int kRows = 256;             // routed rows per unit
constexpr int kK = 64;                 // K per pipeline stage
constexpr int kXStages = 3;
constexpr int kXStageBytes = kRows * kK * 2;   // 256 rows x 128 B, 128B-swizzled
constexpr int kWStages = 8;
constexpr uint32_t kWCols = 32;        // TMEM columns per weight stage
constexpr uint32_t kWBase = 256;
constexpr int kQStagesMax = 8;
constexpr int kDRow = 528;             // drain row: 256 tokens in fp16 + 16 B against bank conflicts
constexpr int kStaging = 128 * kDRow + 2 * 32 * kTRow;   // drain rows + one chunk tile per epilogue group

struct Ctl {
  uint64_t x_empty[kXStages];
  uint64_t w_full[kWStages], w_empty[kWStages];
  uint64_t q_full[kQStagesMax], q_empty[kQStagesMax];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint64_t epi[2];
  uint32_t tmem_base;
  Abort ab;
};

// Code ring per code width: a stage holds 64 K values of 128 weight rows (32 B
// per row for int4, 64 B for int8; TMA 32B / 64B swizzle) and up to 2 x 128 scales.
template <int BITS>
struct QCfg {
  static constexpr int kCB = 8 * BITS;                 // code bytes per row and stage
  static constexpr int kStages = BITS == 4 ? 8 : 4;
  static constexpr int kStageBytes = 128 * kCB + 512;
  // 16-byte chunk c of row r, as the TMA swizzle placed it
  __device__ static __forceinline__ int chunk_offset(int r, int c) {
    return r * kCB + ((BITS == 4 ? (c ^ ((r >> 2) & 1)) : (c ^ ((r >> 1) & 3))) << 4);
  }
};

template <int BITS>
constexpr size_t smem_bytes() {
  return 1024 + size_t(kXStages) * kXStageBytes + size_t(QCfg<BITS>::kStages) * QCfg<BITS>::kStageBytes +
         size_t(kStaging) + sizeof(Ctl);
}
static_assert(smem_bytes<4>() + 2 * (kSchedSmemE + 1) * 4 <= 232448, "shared memory budget");
static_assert(smem_bytes<8>() + 2 * (kSchedSmemE + 1) * 4 <= 232448, "shared memory budget");

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
    down_wide_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap ts,
                     const __grid_constant__ CUtensorMap th, const __grid_constant__ CUtensorMap tha) {
  using QC = QCfg<BITS>;
  constexpr int kQStages = QC::kStages;
  constexpr int kQStageBytes = QC::kStageBytes;
  constexpr int kCB = QC::kCB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* x_base = smem;
  uint8_t* q_base = x_base + size_t(kXStages) * kXStageBytes;
  uint8_t* staging = q_base + size_t(kQStages) * kQStageBytes;
  Ctl* ctl = reinterpret_cast<Ctl*>(staging + kStaging);
  Abort* abort_flag = &ctl->ab;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  __shared__ int32_t s_sched[2 * (kSchedSmemE + 1)];
  const Sched sc = load_sched(a, s_sched);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kXStages; ++i) mbar_init(&ctl->x_empty[i], 1);
    for (int i = 0; i < kWStages; ++i) {
      mbar_init(&ctl->w_full[i], 4 + 1);   // one weight-producer group (4 warps) + the token TMA thread
      mbar_init(&ctl->w_empty[i], 1);
    }
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_empty[i], 4);
    }
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->acc_empty, 8);   // one arrival per epilogue warp, both groups
    mbar_init(&ctl->drain, 1);
    mbar_init(&ctl->epi[0], 4);
    mbar_init(&ctl->epi[1], 4);
    abort_init(&ctl->ab, a.wait_ns);
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 5 * 32) {
    prefetch_tmap(&tq);
    prefetch_tmap(&ts);
  }
  if (threadIdx.x == 6 * 32) {
    prefetch_tmap(&th);
    if (a.nkb_lora > 0) prefetch_tmap(&tha);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  const int nunits = total_units(a, sc);
  UnitStream us{a.unit_tab, nunits, int(gridDim.x)};
  us.start(blockIdx.x);
  const int nkb = a.nkb_main + a.nkb_lora;
  const int ngrp = a.g >= kK ? 1 : kK / a.g;   // scale rows per K stage

  if (warp < 4 || warp >= kEpi1Warp0) {
    // ------------------------------------------------------------ epilogue
    const int eg = warp < 4 ? 0 : 1;          // group: 32-token chunks with (c / 32) % 2 == eg
    const int row = 32 * (warp & 3) + lane;   // feature within the tile = TMEM lane
    const int etid = row;                     // thread index within the group
    const uint32_t tl = tmem_base + (uint32_t(32 * (warp & 3)) << 16);
    uint8_t* drow = staging + row * kDRow;
    uint8_t* ct = staging + 128 * kDRow + eg * 32 * kTRow;
    EpiSyncT<true> es{&ctl->epi[eg]};
    uint32_t bad = 0;   // nonzero once an fp16 output of a valid token overflowed
    int it = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
      const Unit un = us.take(u);
      const int n16 = (un.rows + 15) & ~15;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait<128>(&ctl->acc_full, uint32_t(it) & 1u, abort_flag, a.status))) break;
      tc_fence_after();
      // drain this group's chunks of this thread's feature row as fp16
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
      mbar_arrive_warp(&ctl->acc_empty);
      // this group's 32-token chunks through its [token][feature] tile, 16-byte row stores
      uint16_t* out = static_cast<uint16_t*>(a.out) + un.nt * 128;
      bool stop = false;
#pragma unroll 1
      for (int c = 32 * eg; c < n16; c += 64) {
        uint32_t w[16];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          const uint4 v4 = *reinterpret_cast<const uint4*>(drow + 2 * c + 16 * q4);
          w[4 * q4] = v4.x; w[4 * q4 + 1] = v4.y; w[4 * q4 + 2] = v4.z; w[4 * q4 + 3] = v4.w;
        }
        if (!es.sync(abort_flag, a.status)) { stop = true; break; }   // the chunk tile is free
        stage_tokens<16>(ct, 0, row, w);
        if (!es.sync(abort_flag, a.status)) { stop = true; break; }   // the chunk tile is complete
        const int nt = min(32, un.rows - c);
        // (only valid tokens are stored and checked: padding columns hold stale data)
        for (int p = etid; p < nt * 16; p += 128) {
          const int t = p >> 4, fg = p & 15;
          const uint4 v = *reinterpret_cast<const uint4*>(ct + t * kTRow + fg * 16);
          bad |= f16x2_nonfinite(v.x) | f16x2_nonfinite(v.y) | f16x2_nonfinite(v.z) | f16x2_nonfinite(v.w);
          *reinterpret_cast<uint4*>(out + size_t(un.base + c + t) * a.out_ld + fg * 8) = v;
        }
      }
      if (stop) break;
    }
    if (__any_sync(0xFFFFFFFFu, bad != 0) && lane == 0) raise_status(a.status, TQP_STATUS_NONFINITE);
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      Ring rx, rw;
      int it = 0;
      bool ok = true;
      // descriptors of ring stage 0; a stage's are these plus a fixed offset
      const uint64_t xdesc0 = sdesc_k_sw128(smem_u32(x_base));
      const uint32_t wa0 = tmem_base + kWBase;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++it) {
        const Unit un = us.take(u);
        const int n16 = (un.rows + 15) & ~15;
        const uint32_t idesc = idesc_f16(128, n16);
        if (!mbar_wait(&ctl->acc_empty, (uint32_t(it) & 1u) ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t accf = 0u;   // the unit's first MMA overwrites the accumulator
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&ctl->w_full[rw.stage], rw.phase, abort_flag, a.status)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t bdesc = xdesc0 + uint64_t(rx.stage) * uint64_t(kXStageBytes >> 4);
          const uint32_t wa = wa0 + uint32_t(rw.stage) * kWCols;
          if (kb >= a.nkb_lora) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              umma_f16_ts(tmem_base, wa + uint32_t(8 * kk), bdesc + uint64_t(2 * kk), idesc, accf);
              accf = 1u;
            }
          } else {
            const int ksteps = (min(kK, a.lora_k - kb * kK) + 15) / 16;
            for (int kk = 0; kk < ksteps; ++kk) {
              umma_f16_ts(tmem_base, wa + uint32_t(8 * kk), bdesc + uint64_t(2 * kk), idesc, accf);
              accf = 1u;
            }
          }
          umma_commit(&ctl->x_empty[rx.stage]);
          umma_commit(&ctl->w_empty[rw.stage]);
          rx.next<kXStages>();
          rw.next<kWStages>();
        }
        if (!ok) break;
        umma_commit(&ctl->acc_full);
      }
      // no MMA may still read or write TMEM when it is freed: wait for all of
      // them (they run to completion whether or not the CTA aborted)
      umma_commit(&ctl->drain);
      mbar_drain(&ctl->drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ TMA producer (int4 + scales)
    if (lane == 0) {
      Ring q;
      PendingFills pend;
      const uint32_t bytes = uint32_t(128 * kCB + 256 * ngrp);
      const int gpe = a.in_dim / a.g;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit un = us.take(u);
        const int nrow0 = un.e * a.out_dim + un.nt * 128;
        bool ok = true;
        for (int km = 0; km < a.nkb_main; ++km) {
          if (!mbar_wait<64>(&ctl->q_empty[q.stage], q.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
          uint8_t* qs = q_base + size_t(q.stage) * kQStageBytes;
          uint64_t* bar = &ctl->q_full[q.stage];
          mbar_arrive_expect_tx(bar, bytes);
          tma_load_2d(smem_u32(qs), &tq, bar, km * kCB, nrow0);
          tma_load_2d(smem_u32(qs + 128 * kCB), &ts, bar, un.nt * 128, un.e * gpe + (km * kK) / a.g);
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
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit un = us.take(u);
        const int nbox = un.rows > 128 ? 2 : 1;   // a second 128-row box only when the MMA reads it
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait<64>(&ctl->x_empty[rx.stage], rx.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
          uint8_t* st = x_base + size_t(rx.stage) * kXStageBytes;
          uint64_t* bar = &ctl->w_full[rw.stage];
          // the adapter stage reads s H Ad (zero-filled past its r columns), the rest H
          const CUtensorMap* map = kb < a.nkb_lora ? &tha : &th;
          const int col = (kb < a.nkb_lora ? kb : kb - a.nkb_lora) * kK;
          mbar_arrive_expect_tx(bar, uint32_t(nbox * (kXStageBytes / 2)));
          tma_load_2d(smem_u32(st), map, bar, col, un.base);
          if (nbox == 2) tma_load_2d(smem_u32(st + kXStageBytes / 2), map, bar, col, un.base + 128);
          pend.issued(rw.stage, rw.phase);
          rx.next<kXStages>();
          rw.next<kWStages>();
        }
        if (!ok) break;
      }
      if (aborted(abort_flag)) pend.drain(ctl->w_full);
    }
  } else if (warp >= kWWarp0) {
    // ------------------------------------------------------------ weight producer
    // Four groups of 4 warps take stages n % 4, so that four stages are being
    // dequantised at any time (one stage's chain of code read -> dequant ->
    // TMEM store -> arrive is latency-bound). A thread converts the 64 K
    // values of one weight row (TMEM lane lrow) per stage.
    const int wi = warp - kWWarp0;            // 0..15
    const int grp = wi >> 2;                  // stages n with n % 4 == grp
    const int lrow = 32 * (warp & 3) + lane;  // TMEM lane = feature within the tile
    const uint32_t tw = tmem_base + (uint32_t(32 * (warp & 3)) << 16) + kWBase;
    // scale rows of the two 32-wide K halves of this thread's slice
    const int g_hi = (ngrp == 1) ? 0 : 32 / a.g;
    const int s_lo_off = 128 * kCB + lrow * 2, s_hi_off = 128 * kCB + (g_hi * 128 + lrow) * 2;
    bool inexact = false;   // a group scale whose products q * s are not exact in fp16
    bool lora_inf = false;  // a LoRA B value beyond the fp16 range
    int n = 0;   // stage counter
    int m = 0;   // main (code-carrying) stage counter
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const Unit un = us.take(u);
      const int feat = un.nt * 128 + lrow;
      bool ok = true;
      if (a.nkb_lora > 0 && grp == 0 && u + int(gridDim.x) < nunits) {
        // the next unit's LoRA B row into L2 (its rank-space stage comes first)
        const Unit nx = us.peek();
        const uint16_t* row = a.b0 + (size_t(nx.e) * a.out_dim + nx.nt * 128 + lrow) * a.r;
        for (int off = 0; off < a.r; off += 64) prefetch_l2(row + off);
      }
      for (int kb = 0; kb < nkb; ++kb, ++n) {
        const bool main_stage = kb >= a.nkb_lora;
        const int mq = m;
        if (main_stage) ++m;
        if ((n & 3) != grp) continue;
        const int st = n % kWStages;
        const uint32_t ph = uint32_t(n / kWStages) & 1u;
        if (!mbar_wait_warp(&ctl->w_empty[st], ph ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t v[32];
        if (!main_stage) {
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int colk = kb * kK + c * 8;
            uint4 w4 = make_uint4(0, 0, 0, 0);
            if (colk < a.r)
              w4 = bf16x8_to_f16x8_chk(
                  __ldg(reinterpret_cast<const uint4*>(a.b0 + (size_t(un.e) * a.out_dim + feat) * a.r + colk)), lora_inf);
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
            const uint4 wa = *reinterpret_cast<const uint4*>(qs + QC::chunk_offset(lrow, 0));
            const uint4 wb = *reinterpret_cast<const uint4*>(qs + QC::chunk_offset(lrow, 1));
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
              const uint4 w4 = *reinterpret_cast<const uint4*>(qs + QC::chunk_offset(lrow, ch));
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
        mbar_arrive_warp(&ctl->w_full[st]);
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

}  // namespace down_wide

template <int BITS>
static int launch_down(const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s) {
  static DeviceFlags attr_done;
  constexpr size_t smem = down_wide::smem_bytes<BITS>();
  if (!attr_done.test_and_set_device(down_wide::down_wide_kernel<BITS>, int(smem))) return TQP_ERR_CUDA;
  const int grid = units_upper < num_sms() ? (units_upper > 0 ? units_upper : 1) : num_sms();
  down_wide::down_wide_kernel<BITS><<<grid, down_wide::kThreads, smem, s>>>(a, mp.m[TQ0], mp.m[TS0], mp.m[TA],
                                                                             mp.m[TB0]);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

int run_expert_down_wide(const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s) {
  return a.bits == 8 ? launch_down<8>(a, mp, units_upper, s) : launch_down<4>(a, mp, units_upper, s);
}

}  // namespace tqp
