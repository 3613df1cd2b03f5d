// Gate/up expert projection of the TQP MoE layer with the dequantised base
// weights held in tensor memory (sm_100a, tcgen05):
//   [G|U] = X_e [Wg|Wu]^T + (s X [Ag|Au]) [Bg|Bu],  H = silu(G) * U
// (low-rank adapters trained per expert over frozen quantised base expert
// weights: "Reversible Sparse MoE Single Node", Pattern 3; SwiGLU experts, TQP
// Quantization).
//
// The contraction runs transposed: D[feature][token] = W[feature][:] . X[token][:],
// with W (M = 128 output features of one tile) as the tcgen05.mma A operand in
// TMEM and the token rows (N = the unit's routed rows rounded up to 16) as the B
// operand in 128B-swizzled shared memory. The int4 codes are dequantised by
// registers -> tcgen05.st straight into TMEM, so the dequantised tile never
// touches shared memory, and a ragged expert block costs at most 15 idle
// columns instead of a padded 128-row tile.
//
// Work unit = (expert e, 128-feature tile, block of up to 128 routed rows);
// units are ordered (expert, tile, block) over a persistent grid. One K stage
// is 8 tcgen05.mma of 128 x N x 16 (64 K for gate and for up), so that one
// barrier round trip is amortised over 8 MMAs. Per CTA (1 per SM, 832 threads):
//   warps 0-3   epilogue (TMEM lanes 32w..32w+31 = features of the tile)
//   warp  4     TMEM allocation + one thread issuing tcgen05.mma
//   warp  5     TMA producer of the code / bf16 scale ring (int4 code rows come
//               32B-swizzled, int8 rows 64B-swizzled, so the row reads below
//               are free of bank conflicts)
//   warps 6-9   token producer: cp.async row gathers (rows picked by perm_token)
//               and the rank-space rows
//   warps 10-25 weight producer, two groups of 8 warps on alternate stages:
//               each thread dequantises 64 K values of one weight row (int4 or
//               int8 -> fp16) into TMEM; LoRA B rows
// TMEM (512 columns): accumulators in [0, 256) (gate cols [0,128), up
// [128,256)), 4 weight stages of 64 columns in [256, 512), each holding gate 32
// | up 32 columns. A pipeline stage pairs one token tile (shared memory) with
// one weight stage (TMEM): one "full" barrier collects both producers'
// arrivals and one commit per stage frees both. The epilogue drains G and U as
// fp16 rows (one feature per thread, 16-byte stores) into shared memory, hands
// TMEM back, and then, while the next unit runs, computes SwiGLU in 32-token
// chunks transposed through a [token][feature] tile for 16-byte row stores.
//
// Range: an H (or kept G|U) value or a LoRA B value beyond the fp16 range
// raises TQP_STATUS_NONFINITE; a group scale whose dequantised products are not
// exact in fp16 raises TQP_STATUS_RANGE. Every wait is bounded (tqp_device.cuh); on
// an abort every asynchronous copy and MMA still in flight is drained before
// the CTA frees its memory. No TMA multicast is used.
#include <cstdint>
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "expert_common.cuh"
#include "gemm_common.cuh"
#include "tqp_device.cuh"
#include "tqp_launch.h"

namespace tqp {
namespace tmem_ffn {

constexpr int kWWarp0 = 10;           // first weight-producer warp
constexpr int kWWarps = 16;
constexpr int kThreads = (kWWarp0 + kWWarps) * 32;
constexpr int kQStagesMax = 8;
constexpr uint32_t kWBase = 256;      // first TMEM column of the weight stages
constexpr int kStages = 4;            // pipeline stages (token tile + weight stage)
constexpr uint32_t kWCols = 64;       // TMEM columns per weight stage
constexpr int kK = 64;                // K per stage
constexpr int kXBytes = 16384;        // 128 token rows x 128 B
constexpr int kStaging = (2 * 128 + 32) * kTRow;   // G rows | U rows | chunk tile

// Code ring per code width: a stage holds 64 K values of 128 gate rows and 128
// up rows (32 B per row for int4, 64 B for int8; TMA 32B / 64B swizzle) and up
// to 2 x 2 x 128 scales.
template <int BITS>
struct QCfg {
  static constexpr int kCB = 8 * BITS;                 // code bytes per row and stage
  static constexpr int kStages = BITS == 4 ? 8 : 4;
  static constexpr int kStageBytes = 256 * kCB + 1024;
  // 16-byte chunk c of row r, as the TMA swizzle placed it
  __device__ static __forceinline__ int chunk_offset(int r, int c) {
    return r * kCB + ((BITS == 4 ? (c ^ ((r >> 2) & 1)) : (c ^ ((r >> 1) & 3))) << 4);
  }
};

struct Ctl {
  uint64_t full[kStages], empty[kStages];
  uint64_t q_full[kQStagesMax], q_empty[kQStagesMax];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint64_t epi;
  uint32_t tmem_base;
  Abort ab;
};

template <int BITS>
constexpr size_t smem_bytes() {
  return 1024 + size_t(kStages) * kXBytes + size_t(QCfg<BITS>::kStages) * QCfg<BITS>::kStageBytes + size_t(kStaging) +
         sizeof(Ctl);
}
static_assert(smem_bytes<4>() + 2 * (kSchedSmemE + 1) * 4 <= 232448, "shared memory budget");
static_assert(smem_bytes<8>() + 2 * (kSchedSmemE + 1) * 4 <= 232448, "shared memory budget");

template <int BITS>
__global__ void __launch_bounds__(kThreads, 1)
    gateup_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tq0, const __grid_constant__ CUtensorMap tq1,
                  const __grid_constant__ CUtensorMap ts0, const __grid_constant__ CUtensorMap ts1) {
  using QC = QCfg<BITS>;
  constexpr int kQStages = QC::kStages;
  constexpr int kQStageBytes = QC::kStageBytes;
  constexpr int kCB = QC::kCB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* x_base = smem;
  uint8_t* q_base = x_base + size_t(kStages) * kXBytes;
  uint8_t* staging = q_base + size_t(kQStages) * kQStageBytes;
  Ctl* ctl = reinterpret_cast<Ctl*>(staging + kStaging);
  Abort* abort_flag = &ctl->ab;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  __shared__ int32_t s_sched[2 * (kSchedSmemE + 1)];
  const Sched sc = load_sched(a, s_sched);

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&ctl->full[i], 128 + kWWarps * 16);   // token producer + one weight-producer group
      mbar_init(&ctl->empty[i], 1);
    }
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_empty[i], kWWarps * 16);
    }
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->acc_empty, 128);
    mbar_init(&ctl->drain, 1);
    mbar_init(&ctl->epi, 128);
    abort_init(&ctl->ab, a.wait_ns);
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(&ctl->tmem_base, 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 5 * 32) {
    prefetch_tmap(&tq0);
    prefetch_tmap(&ts0);
    prefetch_tmap(&tq1);
    prefetch_tmap(&ts1);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  const int nunits = total_units(a, sc);
  UnitStream us{a.unit_tab, nunits, int(gridDim.x)};
  us.start(blockIdx.x);
  const int nkb = a.nkb_main + a.nkb_lora;
  // scale rows per K stage (one per quantisation group it spans)
  const int ngrp = a.g >= kK ? 1 : kK / a.g;

  if (warp < 4) {
    // ------------------------------------------------------------ epilogue
    const int row = warp * 32 + lane;   // feature within the tile = TMEM lane
    const uint32_t tl = tmem_base + (uint32_t(warp * 32) << 16);
    int it = 0;
    EpiSync es{&ctl->epi};
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
      const Unit un = us.take(u);
      const int n16 = (un.rows + 15) & ~15;
      if (!__all_sync(0xFFFFFFFFu, mbar_wait<128>(&ctl->acc_full, uint32_t(it) & 1u, abort_flag, a.status))) break;
      tc_fence_after();
      // staging: G rows [feature][token] | U rows | chunk tile [32 tokens][feature]
      uint8_t* grow_s = staging + row * kTRow;
      uint8_t* urow_s = staging + (128 + row) * kTRow;
      uint8_t* ht = staging + 256 * kTRow;
      // drain: this thread's feature row of G and U as fp16 (16-byte stores)
#pragma unroll 1
      for (int c = 0; c < n16; c += 32) {
#pragma unroll
        for (int m2 = 0; m2 < 2; ++m2) {
          float v[32];
          tmem_ld32(tl + uint32_t(128 * m2 + c), v);
          uint4* dst = reinterpret_cast<uint4*>((m2 ? urow_s : grow_s) + 2 * c);
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4)
            dst[q4] = make_uint4(f32x2_to_f16x2(v[8 * q4], v[8 * q4 + 1]), f32x2_to_f16x2(v[8 * q4 + 2], v[8 * q4 + 3]),
                                 f32x2_to_f16x2(v[8 * q4 + 4], v[8 * q4 + 5]),
                                 f32x2_to_f16x2(v[8 * q4 + 6], v[8 * q4 + 7]));
        }
      }
      tc_fence_before();
      mbar_arrive(&ctl->acc_empty);
      // SwiGLU per 32-token chunk (own feature row), transposed through the chunk
      // tile, then 16-byte row stores; overlaps the next unit's main loop
      uint16_t* hout = static_cast<uint16_t*>(a.out) + un.nt * 128;
      bool stop = false;
#pragma unroll 1
      for (int c = 0; c < n16; c += 32) {
        // 16 words (32 tokens) of this thread's staged row
        auto row_words = [&](const uint8_t* src, uint32_t* w) {
#pragma unroll
          for (int q4 = 0; q4 < 4; ++q4) {
            const uint4 v4 = *reinterpret_cast<const uint4*>(src + 2 * c + 16 * q4);
            w[4 * q4] = v4.x; w[4 * q4 + 1] = v4.y; w[4 * q4 + 2] = v4.z; w[4 * q4 + 3] = v4.w;
          }
        };
        uint32_t hw[16];
        {
          uint32_t gw[16], uw[16];
          row_words(grow_s, gw);
          row_words(urow_s, uw);
#pragma unroll
          for (int j = 0; j < 16; ++j) hw[j] = swiglu_pair(gw[j], uw[j]);
        }
        const int nt = min(32, un.rows - c);
        // one [32 token][128 feature] chunk through the tile: wait until the tile
        // is free, transpose into it, wait until complete, 16-byte row stores
        auto emit = [&](const uint32_t* w, uint16_t* dst, size_t ld) -> bool {
          if (!es.sync(abort_flag, a.status)) return false;
          stage_tokens<16>(ht, 0, row, w);
          if (!es.sync(abort_flag, a.status)) return false;
          // (only valid tokens are stored and checked: padding columns hold stale data)
          for (int p = threadIdx.x; p < nt * 16; p += 128) {
            const int t = p >> 4, fg = p & 15;
            const uint4 v = *reinterpret_cast<const uint4*>(ht + t * kTRow + fg * 16);
            if (f16x2_nonfinite(v.x) | f16x2_nonfinite(v.y) | f16x2_nonfinite(v.z) | f16x2_nonfinite(v.w))
              raise_status(a.status, TQP_STATUS_NONFINITE);   // rare: reported where it happens
            *reinterpret_cast<uint4*>(dst + size_t(un.base + c + t) * ld + fg * 8) = v;
          }
          return true;
        };
        if (!emit(hw, hout, size_t(a.out_ld))) { stop = true; break; }
        if (a.aux) {  // keep the pre-activations for the backward (re-read from the staged rows)
          uint16_t* aux = a.aux + un.nt * 128;
          uint32_t w16[16];
          row_words(grow_s, w16);
          if (!emit(w16, aux, 2 * size_t(a.f_dim))) { stop = true; break; }
          row_words(urow_s, w16);
          if (!emit(w16, aux + a.f_dim, 2 * size_t(a.f_dim))) { stop = true; break; }
        }
      }
      if (stop) break;
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      Ring rs;
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++it) {
        const Unit un = us.take(u);
        const int n16 = (un.rows + 15) & ~15;
        const uint32_t idesc = idesc_f16(128, n16);
        if (!mbar_wait(&ctl->acc_empty, (uint32_t(it) & 1u) ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t dacc = tmem_base;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait(&ctl->full[rs.stage], rs.phase, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bdesc = sdesc_k_sw128(smem_u32(x_base + size_t(rs.stage) * kXBytes));
          const uint32_t wa = tmem_base + kWBase + uint32_t(rs.stage) * kWCols;
          // the rank-space stage has only its first lora_k columns live (within the first 64)
          const int ksteps = (kb >= a.nkb_lora) ? 4 : (min(kK, a.lora_k - kb * kK) + 15) / 16;
          for (int kk = 0; kk < ksteps; ++kk) {
            const uint32_t acc = (kb > 0 || kk > 0) ? 1u : 0u;
            umma_f16_ts(dacc, wa + uint32_t(8 * kk), bdesc + uint64_t(2 * kk), idesc, acc);
            umma_f16_ts(dacc + 128, wa + 32 + uint32_t(8 * kk), bdesc + uint64_t(2 * kk), idesc, acc);
          }
          umma_commit(&ctl->empty[rs.stage]);
          rs.next<kStages>();
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
      // gate codes [128 rows][kCB B] | up codes | gate scales [ngrp][128] | up scales
      const uint32_t bytes = uint32_t(256 * kCB + 512 * ngrp);
      const int gpe = a.in_dim / a.g;  // scale rows per expert
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit un = us.take(u);
        const int nrow0 = un.e * a.out_dim + un.nt * 128;
        bool ok = true;
        for (int km = 0; km < a.nkb_main; ++km) {
          if (!mbar_wait<64>(&ctl->q_empty[q.stage], q.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
          uint8_t* qs = q_base + size_t(q.stage) * kQStageBytes;
          uint64_t* bar = &ctl->q_full[q.stage];
          const int srow = un.e * gpe + (km * kK) / a.g;
          mbar_arrive_expect_tx(bar, bytes);
          tma_load_2d(smem_u32(qs), &tq0, bar, km * kCB, nrow0);
          tma_load_2d(smem_u32(qs + 128 * kCB), &tq1, bar, km * kCB, nrow0);
          tma_load_2d(smem_u32(qs + 256 * kCB), &ts0, bar, un.nt * 128, srow);
          tma_load_2d(smem_u32(qs + 256 * kCB + 256 * ngrp), &ts1, bar, un.nt * 128, srow);
          pend.issued(q.stage, q.phase);
          q.next<kQStages>();
        }
        if (!ok) break;
      }
      // on an abort, wait (bounded) until every issued fill has landed
      if (aborted(abort_flag)) pend.drain(ctl->q_full);
    }
  } else if (warp < kWWarp0) {
    // ------------------------------------------------------------ token producer
    // Row gathers are spread so that 8 consecutive lanes copy the 8 16-byte
    // chunks of one 128-byte row piece (one coalesced request per row piece):
    // thread tid covers chunk tid % 8 of rows tid / 8 + 16 j, j = 0..7.
    const int tid = threadIdx.x - 6 * 32;  // 0..127
    const int chunk = tid & 7;
    const int row0 = tid >> 3;             // 0..15
    Ring rx;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const Unit un = us.take(u);
      // source token rows of this thread's 8 tile rows
      int tok[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int r = row0 + 16 * j;
        tok[j] = r < un.rows ? __ldg(a.perm_token + un.base + r) : 0;
      }
      bool ok = true;
      for (int kb = 0; kb < nkb; ++kb) {
        if (!mbar_wait<64>(&ctl->empty[rx.stage], rx.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
        const uint32_t st_u = smem_u32(x_base + size_t(rx.stage) * kXBytes);
        uint64_t* full = &ctl->full[rx.stage];
        if (kb < a.nkb_lora) {
          // rank-space rows s X[Ag|Au], zero-filled past lora_k (lora_k <= 128)
          const int colk = kb * kK + chunk * 8;
          const bool in = colk < a.lora_k;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int r = row0 + 16 * j;
            if (r < un.rows)
              cp_async16(st_u + sw128_offset(r, chunk), a.a_lora + size_t(un.base + r) * a.lora_ld + (in ? colk : 0),
                         in ? 16u : 0u);
          }
        } else {
          const int km = kb - a.nkb_lora;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int r = row0 + 16 * j;
            if (r < un.rows)
              cp_async16(st_u + sw128_offset(r, chunk), a.a_src + size_t(tok[j]) * a.a_ld + km * 64 + chunk * 8, 16);
          }
        }
        cp_async_arrive_noinc(full);
        rx.next<kStages>();
      }
      if (!ok) break;
    }
    cp_async_wait_all();
  } else {
    // ------------------------------------------------------------ weight producer
    // Two groups of 8 warps take alternate pipeline stages, so that two stages
    // are being dequantised at any time (one stage's chain of code read ->
    // dequant -> TMEM store -> arrive is latency-bound). Within a group, a
    // thread converts 64 consecutive K values (8 int4 words) of one weight row:
    // row lrow of the gate (mat 0) or up (mat 1) tile.
    const int wi = warp - kWWarp0;            // 0..15
    const int grp = wi >> 3;                  // stage parity handled by this group
    const int gw = wi & 7;
    const int lrow = 32 * (warp & 3) + lane;  // TMEM lane = feature within the tile
    const int mat = gw >> 2;                  // 0 gate, 1 up
    const uint32_t tw = tmem_base + (uint32_t(32 * (warp & 3)) << 16) + kWBase + uint32_t(mat * 32);
    // this thread's code row inside a stage (TMA-swizzled rows of kCB bytes)
    const int row_off = mat * 128 * kCB;
    // scale rows of the two 32-wide K halves of this thread's slice
    const int g_lo = 0, g_hi = (ngrp == 1) ? 0 : 32 / a.g;
    const int sbase = 256 * kCB + mat * 256 * ngrp;
    const int s_lo_off = sbase + (g_lo * 128 + lrow) * 2, s_hi_off = sbase + (g_hi * 128 + lrow) * 2;
    const bool is_up = mat == 1;
    bool inexact = false;   // a group scale whose products q * s are not exact in fp16
    bool lora_inf = false;  // a LoRA B value beyond the fp16 range
    int n = 0;    // pipeline stage counter of this CTA
    int m = 0;    // main (code-carrying) stage counter
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const Unit un = us.take(u);
      const int feat = un.nt * 128 + lrow;  // output feature
      bool ok = true;
      if (a.nkb_lora > 0 && grp == 0 && u + int(gridDim.x) < nunits) {
        // the next unit's LoRA B row into L2 (its rank-space stage comes first)
        const Unit nx = us.peek();
        const uint16_t* bsrc = is_up ? a.b1 : a.b0;
        const uint16_t* rowp = bsrc + (size_t(nx.e) * a.out_dim + nx.nt * 128 + lrow) * a.r;
        for (int off = 0; off < a.r; off += 64) prefetch_l2(rowp + off);
      }
      for (int kb = 0; kb < nkb; ++kb, ++n) {
        const bool main_stage = kb >= a.nkb_lora;
        const int mq = m;
        if (main_stage) ++m;
        if ((n & 1) != grp) continue;
        const int st = n & (kStages - 1);
        const uint32_t ph = uint32_t(n / kStages) & 1u;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait(&ctl->empty[st], ph ^ 1u, abort_flag, a.status))) { ok = false; break; }
        tc_fence_after();
        uint32_t v[32];
        if (!main_stage) {
          // LoRA B rows as fp16: gate rows hold Bg in K' [0, r), up rows Bu in [r, 2r)
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const int colk = kb * kK + c * 8;
            const int src = is_up ? colk - a.r : colk;
            uint4 w4 = make_uint4(0, 0, 0, 0);
            if (src >= 0 && src < a.r) {
              const uint16_t* bsrc = is_up ? a.b1 : a.b0;
              w4 = bf16x8_to_f16x8_chk(
                  __ldg(reinterpret_cast<const uint4*>(bsrc + (size_t(un.e) * a.out_dim + feat) * a.r + src)), lora_inf);
            }
            v[4 * c] = w4.x; v[4 * c + 1] = w4.y; v[4 * c + 2] = w4.z; v[4 * c + 3] = w4.w;
          }
        } else {
          const int qst = mq % kQStages;
          const uint32_t qph = uint32_t(mq / kQStages) & 1u;
          if (!__all_sync(0xFFFFFFFFu, mbar_wait(&ctl->q_full[qst], qph, abort_flag, a.status))) { ok = false; break; }
          const uint8_t* qs = q_base + size_t(qst) * kQStageBytes;
          const uint32_t s_lo = scale_pair_chk(*reinterpret_cast<const uint16_t*>(qs + s_lo_off), inexact);
          const uint32_t s_hi = scale_pair_chk(*reinterpret_cast<const uint16_t*>(qs + s_hi_off), inexact);
          if (BITS == 4) {
            // 64 K values = 8 words of 8 codes
            const uint4 wa = *reinterpret_cast<const uint4*>(qs + row_off + QC::chunk_offset(lrow, 0));
            const uint4 wb = *reinterpret_cast<const uint4*>(qs + row_off + QC::chunk_offset(lrow, 1));
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
              const uint4 w4 = *reinterpret_cast<const uint4*>(qs + row_off + QC::chunk_offset(lrow, ch));
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
          mbar_arrive(&ctl->q_empty[qst]);
        }
        tmem_st32(tw + uint32_t(st) * kWCols, v);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&ctl->full[st]);
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

}  // namespace tmem_ffn

template <int BITS>
static int launch_gateup(const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s) {
  static DeviceFlags attr_done;
  constexpr size_t smem = tmem_ffn::smem_bytes<BITS>();
  if (!attr_done.test_and_set_device(tmem_ffn::gateup_kernel<BITS>, int(smem))) return TQP_ERR_CUDA;
  const int grid = units_upper < num_sms() ? (units_upper > 0 ? units_upper : 1) : num_sms();
  tmem_ffn::gateup_kernel<BITS><<<grid, tmem_ffn::kThreads, smem, s>>>(a, mp.m[TQ0], mp.m[TQ1], mp.m[TS0], mp.m[TS1]);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

int run_expert_gateup(const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s) {
  return a.bits == 8 ? launch_gateup<8>(a, mp, units_upper, s) : launch_gateup<4>(a, mp, units_upper, s);
}

}  // namespace tqp
