// Input gradients of the TQP MoE expert projections with the dequantised base
// weights in tensor memory (sm_100a, tcgen05), per expert over expert-sorted rows:
//   dX : dX = dG Wg + dU Wu + dxa [Ag ; Au]^T
//   dH : dH = dO Wd + dha Ad^T, then the SwiGLU backward
//        dG = dH U silu'(G), dU = dH silu(G) (G, U kept by the forward)
// (the base weights are frozen and only the adapters train, but the input
// gradients still flow through W + s A B: "Reversible Sparse MoE Single Node",
// Principle 3 and Pattern 3; the rank-space row products dxa, dha come from
// the engine's rank-space mode).
//
// The contraction runs transposed, D[m][row] = W^T[m][:] . P[row][:], as in the
// forward expert kernels: one unit is (expert e, 128 output features m of one
// tile, block of up to 256 routed rows). A = W^T (M = 128 TMEM lanes = features
// m, K = the contraction index n) is dequantised into TMEM; B = the rows P
// ([dG | dU] for dX, dO for dH; N = rows, K-major) come by TMA from the
// expert-sorted buffers; the K loop runs over the rank-space stage, then the
// weight rows (for dX the f gate rows, then the f up rows). Each weight tile is
// dequantised once per 256-row block.
//
// W is stored with n as its row (the codes of the contraction index are rows):
// a lane (one m) needs one code from each of 64 code rows per stage. Eight lanes
// load one 32-bit word each (8 int4 codes of 8 consecutive m, from 8 different
// rows) and transpose the 8 x 8 nibble block with three shuffle stages, so that
// each lane holds the 8 codes of its m along n. The rows are loaded in the order
// 0,2,4,6,1,3,5,7, which leaves the codes in the storage order of an int4 word
// (even positions in the low half-word), so the exact fp16 dequantisation of
// the forward kernels applies with one scale pair per pair of positions (the
// group scale varies along n here: scale[m / g][n]). The lanes then hold the
// word's features in its storage order, so TMEM lane L carries feature
// lane_feature(L) and the epilogue writes each lane's output column there. int8
// codes use a 4 x 4 byte transpose and keep lane = feature. One warp converts
// each stage's bf16 scale tile to fp16 in place first.
//
// Per CTA (1 per SM, 896 threads):
//   warps 0-3, 24-27  epilogue (two groups on alternate 32-row chunks): the
//               down kernel's transposing 16-byte row stores (dX), or the
//               SwiGLU backward on the [row][feature] chunk tile (dH)
//   warp  4     TMEM allocation + one thread issuing tcgen05.mma
//   warp  5     TMA producer of the code / scale ring
//   warp  6     TMA producer of the row ring (P rows; the rank-space rows for
//               the rank-space stage, zero-filled past their width)
//   warp  7     scale converter (bf16 -> fp16 in place; range status)
//   warps 8-23  weight producer, four groups of 4 warps on stages n % 4
// TMEM: one 256-column accumulator and 8 weight stages of 32 columns. Every
// wait is bounded; on an abort the copies and MMAs in flight are drained before
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
namespace dgrad_tm {

constexpr int kWWarp0 = 8;
constexpr int kWWarps = 16;
constexpr int kEpi1Warp0 = kWWarp0 + kWWarps;
constexpr int kThreads = (kEpi1Warp0 + 4) * 32;
constexpr int kDhBatch = 2;   // dH epilogue: 16-byte pieces whose G and U loads are in flight together
constexpr int kRows = 256;
constexpr int kK = 64;
constexpr int kXStages = 3;
constexpr int kXStageBytes = kRows * kK * 2;
constexpr int kWStages = 8;
constexpr uint32_t kWCols = 32;
constexpr uint32_t kWBase = 256;
constexpr int kQStagesMax = 8;
constexpr int kDRow = 528;
constexpr int kStaging = 128 * kDRow + 2 * 32 * kTRow;

struct Ctl {
  uint64_t x_empty[kXStages];
  uint64_t w_full[kWStages], w_empty[kWStages];
  uint64_t q_full[kQStagesMax], q_conv[kQStagesMax], q_empty[kQStagesMax];
  uint64_t acc_full, acc_empty;
  uint64_t drain;
  uint64_t epi[2];
  uint32_t tmem_base;
  Abort ab;
};

// Code ring: a stage holds 64 code rows (hidden index n) of the tile's 128
// features (64 B per row for int4, 64B-swizzled; 128 B for int8, 128B-swizzled)
// and the scale rows of the tile's groups along m (up to 4 x 64 values).
template <int BITS>
struct QCfg {
  static constexpr int kRowBytes = 16 * BITS;
  static constexpr int kStages = BITS == 4 ? 8 : 4;
  static constexpr int kStageBytes = BITS == 4 ? 64 * 64 + 512 : 64 * 128 + 1024;
};

template <int BITS>
constexpr size_t smem_bytes() {
  return 1024 + size_t(kXStages) * kXStageBytes + size_t(QCfg<BITS>::kStages) * QCfg<BITS>::kStageBytes +
         size_t(kStaging) + sizeof(Ctl);
}
static_assert(smem_bytes<4>() + 2 * (kSchedSmemE + 1) * 4 <= 232448, "shared memory budget");
static_assert(smem_bytes<8>() + 2 * (kSchedSmemE + 1) * 4 <= 232448, "shared memory budget");

// Transpose of an 8 x 8 block of int4 codes held by 8 consecutive lanes (lane
// i's word: nibble k = element (i, k)) into lane j's word: nibble i = element (i, j).
__device__ __forceinline__ uint32_t transpose8_nibbles(uint32_t x, int lane) {
  uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, x, 4);
  x = (lane & 4) ? __byte_perm(o, x, 0x7632) : __byte_perm(x, o, 0x5410);
  o = __shfl_xor_sync(0xFFFFFFFFu, x, 2);
  x = (lane & 2) ? __byte_perm(o, x, 0x7351) : __byte_perm(x, o, 0x6240);
  o = __shfl_xor_sync(0xFFFFFFFFu, x, 1);
  x = (lane & 1) ? (((o >> 4) & 0x0F0F0F0Fu) | (x & 0xF0F0F0F0u)) : ((x & 0x0F0F0F0Fu) | ((o & 0x0F0F0F0Fu) << 4));
  return x;
}

// Transpose of a 4 x 4 block of int8 codes held by 4 consecutive lanes.
__device__ __forceinline__ uint32_t transpose4_bytes(uint32_t x, int lane) {
  uint32_t o = __shfl_xor_sync(0xFFFFFFFFu, x, 2);
  x = (lane & 2) ? __byte_perm(o, x, 0x7632) : __byte_perm(x, o, 0x5410);
  o = __shfl_xor_sync(0xFFFFFFFFu, x, 1);
  x = (lane & 1) ? __byte_perm(o, x, 0x7351) : __byte_perm(x, o, 0x6240);
  return x;
}

// Feature of TMEM lane L within a tile. int4 words store features 8w + 0, 2,
// 4, 6 in their low half-word and 8w + 1, 3, 5, 7 in the high one; after the
// transpose lane 8k + j holds the codes of the word's j-th nibble, i.e. feature
// 8k + p(j), p(j) = 2 (j & 3) + (j >> 2). int8 words are in feature order.
template <int BITS>
__device__ __forceinline__ int lane_feature(int L) {
  return BITS == 4 ? ((L & ~7) | (((L & 3) << 1) | ((L >> 2) & 1))) : L;
}

// 2*NW tokens x this lane's feature into the [token][feature] chunk tile, as
// stage_tokens, with the lane holding the adjacent feature at lane ^ kPair.
template <int NW, int kPair>
__device__ __forceinline__ void stage_tokens_pair(uint8_t* tile, int feat, const uint32_t* w) {
  const bool odd = (feat & 1) != 0;
  uint8_t* colp = tile + (feat & ~1) * 2;
#pragma unroll
  for (int j = 0; j < NW; ++j) {
    const uint32_t other = __shfl_xor_sync(0xFFFFFFFFu, w[j], kPair);
    const uint32_t v = odd ? __byte_perm(other, w[j], 0x7632) : __byte_perm(w[j], other, 0x5410);
    *reinterpret_cast<uint32_t*>(colp + (2 * j + (odd ? 1 : 0)) * kTRow) = v;
  }
}

// MODE: DX or DH (gemm_common.cuh).
template <int MODE, int BITS>
__global__ void __launch_bounds__(kThreads, 1)
    dgrad_kernel(const GemmArgs a, const __grid_constant__ CUtensorMap tq0, const __grid_constant__ CUtensorMap tq1,
              const __grid_constant__ CUtensorMap ts0, const __grid_constant__ CUtensorMap ts1,
              const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap txa) {
  using QC = QCfg<BITS>;
  constexpr int kQStages = QC::kStages;
  constexpr int kQStageBytes = QC::kStageBytes;
  constexpr int kRB = QC::kRowBytes;
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
      mbar_init(&ctl->w_full[i], 4 + 1);   // one weight group (4 warps) + the row TMA thread
      mbar_init(&ctl->w_empty[i], 1);
    }
    for (int i = 0; i < kQStages; ++i) {
      mbar_init(&ctl->q_full[i], 1);
      mbar_init(&ctl->q_conv[i], 1);
      mbar_init(&ctl->q_empty[i], 4);
    }
    mbar_init(&ctl->acc_full, 1);
    mbar_init(&ctl->acc_empty, 8);
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
    prefetch_tmap(&tq0);
    prefetch_tmap(&ts0);
    if (MODE == DX) {
      prefetch_tmap(&tq1);
      prefetch_tmap(&ts1);
    }
  }
  if (threadIdx.x == 6 * 32) {
    prefetch_tmap(&tx);
    if (a.nkb_lora > 0) prefetch_tmap(&txa);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;

  const int nunits = total_units(a, sc);
  UnitStream us{a.unit_tab, nunits, int(gridDim.x)};
  us.start(blockIdx.x);
  const int nkb = a.nkb_main + a.nkb_lora;
  // scale rows of a tile: the groups along m that its 128 features span
  const int srows = a.g >= 128 ? 1 : 128 / a.g;

  if (warp < 4 || warp >= kEpi1Warp0) {
    // ------------------------------------------------------------ epilogue
    const int eg = warp < 4 ? 0 : 1;
    const int row = 32 * (warp & 3) + lane;   // feature within the tile = TMEM lane
    const int etid = row;
    const uint32_t tl = tmem_base + (uint32_t(32 * (warp & 3)) << 16);
    uint8_t* drow = staging + row * kDRow;
    uint8_t* ct = staging + 128 * kDRow + eg * 32 * kTRow;
    EpiSyncT<true> es{&ctl->epi[eg]};
    uint32_t bad = 0;
    int it = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x, ++it) {
      const Unit un = us.take(u);
      const int n16 = (un.rows + 15) & ~15;
      if (!mbar_wait_warp<128>(&ctl->acc_full, uint32_t(it) & 1u, abort_flag, a.status)) break;
      tc_fence_after();
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
        stage_tokens_pair<16, BITS == 4 ? 4 : 1>(ct, lane_feature<BITS>(row), w);
        if (!es.sync(abort_flag, a.status)) { stop = true; break; }   // the chunk tile is complete
        const int nt = min(32, un.rows - c);
        if (MODE == DX) {
          for (int p = etid; p < nt * 16; p += 128) {
            const int t = p >> 4, fg = p & 15;
            const uint4 v = *reinterpret_cast<const uint4*>(ct + t * kTRow + fg * 16);
            const size_t orow = size_t(un.base + c + t) * a.out_ld;
            bad |= f16x2_nonfinite(v.x) | f16x2_nonfinite(v.y) | f16x2_nonfinite(v.z) | f16x2_nonfinite(v.w);
            *reinterpret_cast<uint4*>(out + orow + fg * 8) = v;
          }
        } else {
          // SwiGLU backward of 8 features: dG = dH U s (1 + G (1 - s)), dU = dH G s,
          // s = sigmoid(G). The G and U pieces of kDhBatch pieces are loaded before
          // any of them is used, so that their latencies overlap.
          for (int p0 = etid; p0 < nt * 16; p0 += kDhBatch * 128) {
            uint4 g4[kDhBatch], u4[kDhBatch];
#pragma unroll
            for (int i = 0; i < kDhBatch; ++i) {
              const int p = p0 + 128 * i;
              g4[i] = u4[i] = make_uint4(0u, 0u, 0u, 0u);
              if (p < nt * 16) {
                const uint16_t* gu = a.aux + size_t(un.base + c + (p >> 4)) * a.out_ld + un.nt * 128 + (p & 15) * 8;
                g4[i] = *reinterpret_cast<const uint4*>(gu);
                u4[i] = *reinterpret_cast<const uint4*>(gu + a.f_dim);
              }
            }
#pragma unroll
            for (int i = 0; i < kDhBatch; ++i) {
              const int p = p0 + 128 * i;
              if (p >= nt * 16) break;
              const int t = p >> 4, fg = p & 15;
              const uint4 v = *reinterpret_cast<const uint4*>(ct + t * kTRow + fg * 16);
              const size_t orow = size_t(un.base + c + t) * a.out_ld;
              const uint32_t hw[4] = {v.x, v.y, v.z, v.w};
              const uint32_t gw[4] = {g4[i].x, g4[i].y, g4[i].z, g4[i].w};
              const uint32_t uw[4] = {u4[i].x, u4[i].y, u4[i].z, u4[i].w};
              uint32_t dg[4], du[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float2 dh = __half22float2(*reinterpret_cast<const __half2*>(&hw[q]));
                const float2 g = __half22float2(*reinterpret_cast<const __half2*>(&gw[q]));
                const float2 uu = __half22float2(*reinterpret_cast<const __half2*>(&uw[q]));
                const float s0 = 1.0f / (1.0f + __expf(-g.x)), s1 = 1.0f / (1.0f + __expf(-g.y));
                dg[q] = f32x2_to_f16x2(dh.x * uu.x * s0 * (1.0f + g.x * (1.0f - s0)),
                                       dh.y * uu.y * s1 * (1.0f + g.y * (1.0f - s1)));
                du[q] = f32x2_to_f16x2(dh.x * g.x * s0, dh.y * g.y * s1);
                bad |= f16x2_nonfinite(dg[q]) | f16x2_nonfinite(du[q]);
              }
              uint16_t* dgu = static_cast<uint16_t*>(a.out) + orow + un.nt * 128 + fg * 8;
              *reinterpret_cast<uint4*>(dgu) = make_uint4(dg[0], dg[1], dg[2], dg[3]);
              *reinterpret_cast<uint4*>(dgu + a.f_dim) = make_uint4(du[0], du[1], du[2], du[3]);
            }
          }
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
      const uint64_t xdesc0 = sdesc_k_sw128(smem_u32(x_base));
      const uint32_t wa0 = tmem_base + kWBase;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x, ++it) {
        const Unit un = us.take(u);
        const int n16 = (un.rows + 15) & ~15;
        const uint32_t idesc = idesc_f16(128, n16);
        if (!mbar_wait(&ctl->acc_empty, (uint32_t(it) & 1u) ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        uint32_t accf = 0u;
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
      umma_commit(&ctl->drain);
      mbar_drain(&ctl->drain, 0, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------ TMA producer (codes + scales)
    if (lane == 0) {
      Ring q;
      PendingFills pend;
      const uint32_t bytes = uint32_t(64 * kRB + srows * 64 * 2);
      const int gpe = a.in_dim / a.g;   // scale rows per expert
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit un = us.take(u);
        const int m0 = un.nt * 128;
        bool ok = true;
        for (int km = 0; km < a.nkb_main; ++km) {
          if (!mbar_wait<64>(&ctl->q_empty[q.stage], q.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
          const int mat = km >= a.half_kb ? 1 : 0;
          const int n0 = (km - mat * a.half_kb) * kK;
          uint8_t* qs = q_base + size_t(q.stage) * kQStageBytes;
          uint64_t* bar = &ctl->q_full[q.stage];
          mbar_arrive_expect_tx(bar, bytes);
          tma_load_2d(smem_u32(qs), mat ? &tq1 : &tq0, bar, m0 * BITS / 8, un.e * a.out_dim + n0);
          tma_load_2d(smem_u32(qs + 64 * kRB), mat ? &ts1 : &ts0, bar, n0, un.e * gpe + m0 / a.g);
          pend.issued(q.stage, q.phase);
          q.next<kQStages>();
        }
        if (!ok) break;
      }
      if (aborted(abort_flag)) pend.drain(ctl->q_full);
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------ TMA producer (rows)
    if (lane == 0) {
      Ring rx, rw;
      PendingFills pend;
      for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
        const Unit un = us.take(u);
        const int nbox = un.rows > 128 ? 2 : 1;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait<64>(&ctl->x_empty[rx.stage], rx.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
          uint8_t* st = x_base + size_t(rx.stage) * kXStageBytes;
          uint64_t* bar = &ctl->w_full[rw.stage];
          const CUtensorMap* map = kb < a.nkb_lora ? &txa : &tx;
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
  } else if (warp == 7) {
    // ------------------------------------------------------------ scale converter
    // Each stage's bf16 scale tile becomes fp16 in place (one fp16 rounding-free
    // conversion: the range check flags scales whose products q * s would not be
    // exact in fp16).
    Ring q;
    bool inexact = false;
    const int nwords = srows * 32;   // scale pairs in a stage
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      bool ok = true;
      for (int km = 0; km < a.nkb_main; ++km) {
        if (!mbar_wait_warp(&ctl->q_full[q.stage], q.phase, abort_flag, a.status)) { ok = false; break; }
        uint32_t* sw = reinterpret_cast<uint32_t*>(q_base + size_t(q.stage) * kQStageBytes + 64 * kRB);
        for (int i = lane; i < nwords; i += 32) {
          const uint32_t b2 = sw[i];
          const uint32_t lo = scale_pair_chk(uint16_t(b2 & 0xFFFFu), inexact) & 0xFFFFu;
          const uint32_t hi = scale_pair_chk(uint16_t(b2 >> 16), inexact) & 0xFFFFu;
          sw[i] = lo | (hi << 16);
        }
        // the slot's next fill is an async-proxy TMA write
        fence_proxy_async_smem();
        mbar_arrive_warp(&ctl->q_conv[q.stage]);
        q.next<kQStages>();
      }
      if (!ok) break;
    }
    if (__any_sync(0xFFFFFFFFu, inexact) && lane == 0) raise_status(a.status, TQP_STATUS_RANGE);
  } else if (warp >= kWWarp0) {
    // ------------------------------------------------------------ weight producer
    const int wi = warp - kWWarp0;            // 0..15
    const int grp = wi >> 2;                  // stages n with n % 4 == grp
    const int q4 = warp & 3;                  // TMEM lane quarter
    const int lrow = 32 * q4 + lane;          // TMEM lane = feature within the tile
    const uint32_t tw = tmem_base + (uint32_t(32 * q4) << 16) + kWBase;
    // this feature's scale row within the tile's groups (lane_feature stays within the lane's 8-group)
    const int sr = lrow / (a.g >= 128 ? 128 : a.g);
    bool lora_inf = false;
    int n = 0, m = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const Unit un = us.take(u);
      const int feat = un.nt * 128 + lane_feature<BITS>(lrow);   // input feature m of this lane
      bool ok = true;
      if (a.nkb_lora > 0 && !a.lt && grp == 0 && u + int(gridDim.x) < nunits) {
        // the next unit's rank-space columns into L2: for each j, this warp's 32
        // features are one 64-byte piece of row j of Ag^T / Au^T (Ad^T)
        const Unit nx = us.peek();
        const size_t col = size_t(nx.nt) * 128 + 32 * q4;
        for (int j = lane; j < a.lora_k; j += 32) {
          const uint16_t* src = j < a.r ? a.lb0 + (size_t(nx.e) * a.r + j) * a.lb_ld
                                        : a.lb1 + (size_t(nx.e) * a.r + (j - a.r)) * a.lb_ld;
          prefetch_l2(src + col);
        }
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
        if (!main_stage && a.lt) {
          // rank-space stage from the row copy: this feature's lt_w fp16 values are one
          // contiguous row, loaded as up to eight 16-byte pieces at once; column c of
          // the stage holds the pair j = 2c, 2c + 1 (zero past lora_k)
          const uint4* rowp =
              reinterpret_cast<const uint4*>(a.lt + (size_t(un.e) * a.in_dim + feat) * a.lt_w + kb * kK);
          const int npc = (min(kK, a.lt_w - kb * kK)) >> 3;   // 16-byte pieces in this stage (lt_w % 8 == 0)
          uint32_t v[32];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const uint4 p4 = q < npc ? __ldg(rowp + q) : make_uint4(0, 0, 0, 0);
            v[4 * q] = p4.x; v[4 * q + 1] = p4.y; v[4 * q + 2] = p4.z; v[4 * q + 3] = p4.w;
          }
          tmem_st32(tw + uint32_t(st) * kWCols, v);
        } else if (!main_stage) {
          // rank-space stage: A[m][j] = Ag^T[j][m] (j < r), Au^T[j - r][m] (r <= j < 2r), else 0,
          // written to TMEM in eight pieces of 4 columns (8 K values each)
          // dX: Ag^T then Au^T (lora_k = 2r); dH: Ad^T (lora_k = r)
          const uint16_t* pg = a.lb0 + size_t(un.e) * a.r * a.lb_ld + feat;
          const uint16_t* pu = MODE == DX ? a.lb1 + size_t(un.e) * a.r * a.lb_ld + feat : pg;
#pragma unroll 1
          for (int qv = 0; qv < 8; ++qv) {
            // 8 loads are issued together (addresses selected, invalid columns read
            // a valid element and are zeroed), then converted into 4 columns
            uint16_t raw[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) {
              const int j = kb * kK + 8 * qv + t;
              const uint16_t* ptr = (j < a.r) ? pg + size_t(j) * a.lb_ld : pu + size_t(j - a.r) * a.lb_ld;
              raw[t] = __ldg(j < a.lora_k ? ptr : pg);
            }
            uint32_t w4[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int j = kb * kK + 8 * qv + 2 * c;
              const uint32_t lo = j < a.lora_k ? bf16_to_f16_bits_chk(raw[2 * c], lora_inf) : 0u;
              const uint32_t hi = j + 1 < a.lora_k ? bf16_to_f16_bits_chk(raw[2 * c + 1], lora_inf) : 0u;
              w4[c] = lo | (hi << 16);
            }
            tmem_st4(tw + uint32_t(st) * kWCols + uint32_t(4 * qv), w4);
          }
        } else {
          uint32_t v[32];
          const int qst = mq % kQStages;
          const uint32_t qph = uint32_t(mq / kQStages) & 1u;
          if (!mbar_wait_warp(&ctl->q_conv[qst], qph, abort_flag, a.status)) { ok = false; break; }
          const uint8_t* qs = q_base + size_t(qst) * kQStageBytes;
          const uint8_t* sct = qs + 64 * kRB + sr * 128;   // this feature's fp16 scales along n
          if (BITS == 4) {
            // 8 blocks of 8 code rows; lane (k, i) = (lane >> 3, lane & 7) loads word
            // 4 q4 + k (features 32 q4 + 8 k .. + 7) of row 8 b + t(i), t = 0,2,4,6,1,3,5,7
            const int i = lane & 7, k = lane >> 3;
            const int rsub = ((i & 3) << 1) | (i >> 2);
#pragma unroll
            for (int b = 0; b < 8; ++b) {
              const int row = 8 * b + rsub;
              const int chunk = q4 ^ ((row >> 1) & 3);   // 64B swizzle of the TMA box
              const uint32_t x = *reinterpret_cast<const uint32_t*>(qs + row * 64 + (chunk << 4) + 4 * k);
              const uint32_t y = transpose8_nibbles(x, lane);
              const uint4 s4 = *reinterpret_cast<const uint4*>(sct + 16 * b);   // scales of rows 8b .. 8b+7
              const uint32_t sp[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
              for (int p = 0; p < 4; ++p) {
                const uint32_t q2 = ((y >> (4 * p)) & 0x000F000Fu) ^ 0x64086408u;   // fp16 pair 1032 + q
                v[4 * b + p] = f16x2_mul(f16x2_sub(q2, 0x64086408u), sp[p]);
              }
            }
          } else {
            // 16 blocks of 4 code rows; lane (k, i) = (lane >> 2, lane & 3) loads word
            // 8 q4 + k (features 32 q4 + 4 k .. + 3) of row 4 b + i
            const int i = lane & 3, k = lane >> 2;
#pragma unroll
            for (int b = 0; b < 16; ++b) {
              const int row = 4 * b + i;
              const int chunk = (2 * q4 + (k >> 2)) ^ (row & 7);   // 128B swizzle of the TMA box
              const uint32_t x = *reinterpret_cast<const uint32_t*>(qs + row * 128 + (chunk << 4) + 4 * (k & 3));
              const uint32_t y = transpose4_bytes(x, lane) ^ 0x80808080u;
              const uint2 s2 = *reinterpret_cast<const uint2*>(sct + 8 * b);   // scales of rows 4b .. 4b+3
              const uint32_t lo = __byte_perm(y, 0x64646464u, 0x4140);
              const uint32_t hi = __byte_perm(y, 0x64646464u, 0x4342);
              v[2 * b] = f16x2_mul(f16x2_sub(lo, 0x64806480u), s2.x);
              v[2 * b + 1] = f16x2_mul(f16x2_sub(hi, 0x64806480u), s2.y);
            }
          }
          fence_proxy_async_smem();
          mbar_arrive_warp(&ctl->q_empty[qst]);
          tmem_st32(tw + uint32_t(st) * kWCols, v);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(&ctl->w_full[st]);
      }
      if (!ok) break;
    }
    if (__any_sync(0xFFFFFFFFu, lora_inf) && lane == 0) raise_status(a.status, TQP_STATUS_NONFINITE);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace dgrad_tm

template <int MODE, int BITS>
static int launch_dgrad_tm(const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s) {
  static DeviceFlags attr_done;
  constexpr size_t smem = dgrad_tm::smem_bytes<BITS>();
  auto kern = dgrad_tm::dgrad_kernel<MODE, BITS>;
  if (!attr_done.test_and_set_device(kern, int(smem))) return TQP_ERR_CUDA;
  const int grid = units_upper < num_sms() ? (units_upper > 0 ? units_upper : 1) : num_sms();
  kern<<<grid, dgrad_tm::kThreads, smem, s>>>(a, mp.m[TQ0], mp.m[TQ1], mp.m[TS0], mp.m[TS1], mp.m[TA], mp.m[TB0]);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

int run_expert_dgrad(int mode, const GemmArgs& a, const Maps& mp, int units_upper, cudaStream_t s) {
  if (mode == DX) return a.bits == 8 ? launch_dgrad_tm<DX, 8>(a, mp, units_upper, s) : launch_dgrad_tm<DX, 4>(a, mp, units_upper, s);
  return a.bits == 8 ? launch_dgrad_tm<DH, 8>(a, mp, units_upper, s) : launch_dgrad_tm<DH, 4>(a, mp, units_upper, s);
}

}  // namespace tqp
