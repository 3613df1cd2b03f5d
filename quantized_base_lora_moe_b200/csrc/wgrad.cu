// Adapter gradients of the TQP layer's backward on the tensor cores (sm_100a).
//
// Every adapter gradient is, per expert e, a contraction over the rows routed
// to e (base and router frozen: only the adapters get gradients, "Reversible
// Sparse MoE Single Node", Principle 3 / Pattern 3):
//   C[m][j] = sum_{rows of e} P[row][m] * Q[row][j]
// with P the wide operand (m over d or f) and Q the rank-space operand (j over
// r or 2r). Four kinds of units, all in one launch:
//   kind 0  dB_down[e][m][j]  = sum dO[row][m]  * ha[row][j]       (m < d,  j < r)
//   kind 1  dA_down[e][j][m]  = sum h[row][m]   * dha[row][j]      (m < f,  j < r)
//   kind 2  dB_gate[e][m][j]  = sum dG[row][m]  * xa[row][j]       (m < f,  j < r)
//           dB_up[e][m][j]    = sum dU[row][m]  * xa[row][r + j]   (dG|dU rows are [2f], xa rows [2r])
//   kind 3  dA_gate[e][j][m]  = sum x[tok][m]   * dxa[row][j]      (m < d,  j < r; x[tok] = X_perm[row],
//                                                                     or x[perm[row]] when perm is given)
//           dA_up[e][j][m]    = sum x[tok][m]   * dxa[row][r + j]  (one unit computes both: N = 2r)
// The operands hold the fp16 intermediates of the backward, computed for the
// cotangent dy * 2^P; the fp32 results are scaled back by 2^-P.
//
// A unit is (kind, expert, 128-wide tile of m). The MMA is D[m][j] = A[m][k] B[j][k]
// with k = the routed row: both operands are stored row by row (k slow), so
// they are loaded as MN-major 128B-swizzled tiles (64 MN elements = 128 bytes
// per k row, 8 k rows per 1024-byte atom) and the instruction descriptor marks
// A and B as MN-major. Rows past the expert's last row are zero-filled, so a
// ragged tail contributes nothing. An expert with no rows gets zeros.
// Per CTA (persistent, 1 per SM, 288 threads):
//   warps 0-3  epilogue: TMEM -> registers -> fp32 stores (one m per thread)
//   warp  4    TMEM allocation + one thread issuing tcgen05.mma
//   warps 5-8  producers of 64-row stages: P (128 m) by two TMA boxes of
//              64 x 64 (128B swizzle, the MN-major atom layout), issued by one
//              thread; Q (r or 2r) by cp.async, zero-filled past the expert's
//              rows, so that the P rows a box reads past them contribute nothing.
//              (X gathered through perm: P by cp.async as well.)
// Accumulators are double-buffered in TMEM (2 x 64 columns), so ranks up to 32
// (kind 3 needs 2r columns); the MMA's N is the width rounded up to 16. Every
// wait is bounded (tqp_device.cuh); no TMA multicast is used.
#include <cstdint>
#include <cstring>
#include <cuda_runtime.h>

#include "../../include/tqp_moe.h"
#include "gemm_common.cuh"
#include "tqp_device.cuh"
#include "tqp_launch.h"

namespace tqp {
namespace wgrad {

constexpr int kThreads = 288;
constexpr int kStages = 8;
constexpr int kRowsPerStage = 64;                 // k rows (routed rows) per stage: 4 MMA K-steps
constexpr int kABytes = 2 * kRowsPerStage * 128;  // 128 m: two 64-wide MN atoms of 64 rows x 128 B
constexpr int kBBytes = kRowsPerStage * 128;      // up to 64 j: one MN atom
constexpr int kAtomCol = kRowsPerStage * 128;     // bytes between the two 64-wide MN atoms of A (LBO)
constexpr uint32_t kAccCols = 64;

struct Ctl {
  uint64_t full[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  Abort ab;
};

constexpr size_t kSmemBytes = 1024 + size_t(kStages) * (kABytes + kBBytes) + sizeof(Ctl);
static_assert(kSmemBytes <= 232448, "shared memory budget");

// Instruction descriptor: kind::f16, A = B = fp16, D = f32, both MN-major.
__host__ __device__ constexpr uint32_t idesc_f16_mn(int M, int N) {
  return (1u << 4) | (1u << 15) | (1u << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Byte offset of the 16-byte chunk holding MN elements [8c, 8c+8) of k row kk
// in a tile of 64 rows (c < 16: two MN atoms kAtomCol apart).
__device__ __forceinline__ uint32_t mn_offset(int kk, int c) {
  return uint32_t((c >> 3) * kAtomCol + (kk >> 3) * 1024 + (kk & 7) * 128 + (((c & 7) ^ (kk & 7)) << 4));
}

struct Args {
  int E, d, f, r;
  int tiles[4];          // m tiles per expert, per kind
  int tile_prefix[5];    // unit prefix over kinds (per expert: sum of tiles)
  const int32_t* offsets;
  const int32_t* perm;
  const uint16_t* dO;    // [A][d]
  const uint16_t* h;     // [A][f]
  const uint16_t* dgu;   // [A][2f]
  const uint16_t* x16;   // X_perm [A][d] (perm null), or x [T][d] gathered by perm
  const uint16_t* ha;    // [A][r]
  const uint16_t* dha;   // [A][r]
  const uint16_t* xa;    // [A][2r]
  const uint16_t* dxa;   // [A][2r]
  float* dA[3];
  float* dB[3];
  const uint32_t* dmax;  // max |dy|: results are scaled back by 2^-P
  int32_t* status;
  unsigned long long wait_ns;
};

struct WUnit {
  int kind, e, tile, base, rows;
};

__device__ __forceinline__ WUnit decode(const Args& a, int u) {
  // units are ordered (expert, kind, tile): one expert's tiles run side by side
  const int per_e = a.tile_prefix[4];
  WUnit w;
  w.e = u / per_e;
  int rem = u - w.e * per_e;
  w.kind = 0;
  while (w.kind < 3 && rem >= a.tile_prefix[w.kind + 1]) ++w.kind;
  w.tile = rem - a.tile_prefix[w.kind];
  w.base = __ldg(a.offsets + w.e);
  w.rows = __ldg(a.offsets + w.e + 1) - w.base;
  return w;
}

__device__ __forceinline__ int unit_n(const Args& a, int kind) { return kind == 3 ? 2 * a.r : a.r; }

// MMA N of a kind: its width rounded up to a multiple of 16 (the extra Q
// columns are zero-filled and their results dropped)
__device__ __forceinline__ int unit_npad(const Args& a, int kind) { return (unit_n(a, kind) + 15) & ~15; }

// 2^-P of the cotangent scale (as in layer_bwd.cu: max|dy| * 2^P in [2^7, 2^8))
__device__ __forceinline__ float inv_grad_scale(const uint32_t* dmax) {
  const float m = __uint_as_float(*dmax);
  if (!(m > 0.0f) || !isfinite(m)) return 1.0f;
  int e;
  frexpf(m, &e);
  return ldexpf(1.0f, -max(-120, min(120, 8 - e)));
}

// tp[kind]: the P matrix of each kind as a box {64 m, 64 rows} map, tq[kind] the Q
// matrix as a box {64 columns, 64 rows} map (both unused when perm is set)
__global__ void __launch_bounds__(kThreads, 1)
    wgrad_kernel(const Args a, const __grid_constant__ CUtensorMap tp0, const __grid_constant__ CUtensorMap tp1,
                 const __grid_constant__ CUtensorMap tp2, const __grid_constant__ CUtensorMap tp3,
                 const __grid_constant__ CUtensorMap tq0, const __grid_constant__ CUtensorMap tq1,
                 const __grid_constant__ CUtensorMap tq2, const __grid_constant__ CUtensorMap tq3) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* a_base = smem;
  uint8_t* b_base = a_base + size_t(kStages) * kABytes;
  Ctl* ctl = reinterpret_cast<Ctl*>(b_base + size_t(kStages) * kBBytes);
  Abort* abort_flag = &ctl->ab;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&ctl->full[i], 128);   // the producers' cp.async arrivals (the P boxes add their bytes)
      mbar_init(&ctl->empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&ctl->acc_full[i], 1);
      mbar_init(&ctl->acc_empty[i], 128);
    }
    mbar_init(&ctl->drain, 1);
    abort_init(&ctl->ab, a.wait_ns);
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(&ctl->tmem_base, 2 * kAccCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = ctl->tmem_base;
  const int nunits = a.E * a.tile_prefix[4];

  if (warp < 4) {
    // ------------------------------------------------------------ epilogue
    const int lrow = warp * 32 + lane;   // m within the tile = TMEM lane
    const uint32_t tl = tmem_base + (uint32_t(warp * 32) << 16);
    const float isc = inv_grad_scale(a.dmax);
    int it = 0;
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const WUnit w = decode(a, u);
      const int m = w.tile * 128 + lrow;
      float v[64];
      if (w.rows > 0) {
        const int ab = it & 1;
        if (!__all_sync(0xFFFFFFFFu, mbar_wait<64>(&ctl->acc_full[ab], uint32_t(it >> 1) & 1u, abort_flag, a.status)))
          break;
        tc_fence_after();
        tmem_ld32(tl + uint32_t(ab * kAccCols), v);
        if (unit_npad(a, w.kind) > 32) tmem_ld32(tl + uint32_t(ab * kAccCols + 32), v + 32);
        tc_fence_before();
        mbar_arrive(&ctl->acc_empty[ab]);
        ++it;
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] *= isc;
      } else {
#pragma unroll
        for (int j = 0; j < 64; ++j) v[j] = 0.0f;
      }
      const size_t e = size_t(w.e);
      const int r = a.r;
      // (fully unrolled over the rank with a guard, so that v stays in registers)
      if (w.kind == 0 || w.kind == 2) {
        const bool up = w.kind == 2 && m >= a.f;
        float* dst = w.kind == 0 ? a.dB[2] + (e * a.d + m) * r : (up ? a.dB[1] : a.dB[0]) + (e * a.f + (up ? m - a.f : m)) * r;
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          if (j < r) *reinterpret_cast<float4*>(dst + j) = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
      } else if (w.kind == 1) {
        float* dst = a.dA[2] + e * r * a.f + m;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < r) dst[size_t(j) * a.f] = v[j];
      } else {
        float* dg = a.dA[0] + e * r * a.d + m;
        float* du = a.dA[1] + e * r * a.d + m;
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < r) dg[size_t(j) * a.d] = v[j];
#pragma unroll
        for (int j = 0; j < 64; ++j)
          if (j >= r && j < 2 * r) du[size_t(j - r) * a.d] = v[j];
      }
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      Ring rs;
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; u < nunits && ok; u += gridDim.x) {
        const WUnit w = decode(a, u);
        if (w.rows <= 0) continue;
        const int ab = it & 1;
        if (!mbar_wait(&ctl->acc_empty[ab], (uint32_t(it >> 1) & 1u) ^ 1u, abort_flag, a.status)) { ok = false; break; }
        tc_fence_after();
        const uint32_t idesc = idesc_f16_mn(128, unit_npad(a, w.kind));
        const uint32_t dacc = tmem_base + uint32_t(ab * kAccCols);
        const int nst = (w.rows + kRowsPerStage - 1) / kRowsPerStage;
        for (int s = 0; s < nst; ++s) {
          if (!mbar_wait(&ctl->full[rs.stage], rs.phase, abort_flag, a.status)) { ok = false; break; }
          tc_fence_after();
          const uint32_t as = smem_u32(a_base + size_t(rs.stage) * kABytes);
          const uint32_t bs = smem_u32(b_base + size_t(rs.stage) * kBBytes);
          const int ksteps = (min(kRowsPerStage, w.rows - s * kRowsPerStage) + 15) / 16;
          for (int ks = 0; ks < ksteps; ++ks)
            umma_bf16(dacc, sdesc_mn_sw128(as + uint32_t(ks) * 2048u, kAtomCol),
                      sdesc_mn_sw128(bs + uint32_t(ks) * 2048u, kAtomCol), idesc, (s > 0 || ks > 0) ? 1u : 0u);
          umma_commit(&ctl->empty[rs.stage]);
          rs.next<kStages>();
        }
        if (!ok) break;
        umma_commit(&ctl->acc_full[ab]);
        ++it;
      }
      umma_commit(&ctl->drain);
      mbar_drain(&ctl->drain, 0, 100000000ull);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ producers
    const int tid = threadIdx.x - 5 * 32;   // 0..127
    const bool ptma = a.perm == nullptr;    // P rows are contiguous: TMA boxes
    Ring rs;
    PendingFills pend;
    if (tid == 0 && ptma) {
      prefetch_tmap(&tp0);
      prefetch_tmap(&tp1);
      prefetch_tmap(&tp2);
      prefetch_tmap(&tp3);
      prefetch_tmap(&tq0);
      prefetch_tmap(&tq1);
      prefetch_tmap(&tq2);
      prefetch_tmap(&tq3);
    }
    for (int u = blockIdx.x; u < nunits; u += gridDim.x) {
      const WUnit w = decode(a, u);
      if (w.rows <= 0) continue;
      const int nreal = unit_n(a, w.kind) / 8;     // 16-byte Q chunks per row with data
      const int nchunk = unit_npad(a, w.kind) / 8; // chunks per row the MMA reads (the rest zero-filled)
      // P row source and column offset of this tile; Q row source, width and column offset
      const uint16_t* P;
      int ldp, pcol = w.tile * 128;
      const uint16_t* Qs;
      int ldq, qcol = 0;
      switch (w.kind) {
        case 0: P = a.dO; ldp = a.d; Qs = a.ha; ldq = a.r; break;
        case 1: P = a.h; ldp = a.f; Qs = a.dha; ldq = a.r; break;
        case 2: P = a.dgu; ldp = 2 * a.f; Qs = a.xa; ldq = 2 * a.r; qcol = (pcol >= a.f) ? a.r : 0; break;
        default: P = a.x16; ldp = a.d; Qs = a.dxa; ldq = 2 * a.r; break;
      }
      const int nst = (w.rows + kRowsPerStage - 1) / kRowsPerStage;
      bool ok = true;
      for (int s = 0; s < nst; ++s) {
        if (!mbar_wait<32>(&ctl->empty[rs.stage], rs.phase ^ 1u, abort_flag, a.status)) { ok = false; break; }
        const uint32_t as = smem_u32(a_base + size_t(rs.stage) * kABytes);
        const uint32_t bs = smem_u32(b_base + size_t(rs.stage) * kBBytes);
        const int k0 = s * kRowsPerStage;
        // a stage whose 64 rows all belong to the expert takes Q by TMA as well;
        // the expert's last, partial stage takes Q by cp.async, zero-filled past
        // the expert's rows
        const bool qtma = ptma && k0 + kRowsPerStage <= w.rows;
        if (ptma) {
          // P: two boxes of 64 m x 64 rows (rows past the expert are read, and
          // meet Q's zero rows; rows past the matrix are zero-filled)
          if (tid == 0) {
            const CUtensorMap* map = w.kind == 0 ? &tp0 : w.kind == 1 ? &tp1 : w.kind == 2 ? &tp2 : &tp3;
            mbar_expect_tx(&ctl->full[rs.stage], uint32_t(2 * 64 * 128 + (qtma ? kBBytes : 0)));
            tma_load_2d(as, map, &ctl->full[rs.stage], pcol, w.base + k0);
            tma_load_2d(as + kAtomCol, map, &ctl->full[rs.stage], pcol + 64, w.base + k0);
            if (qtma) {
              // Q: one box of 64 columns x 64 rows (columns past the matrix zero-filled,
              // columns past the kind's width never read by the MMA)
              const CUtensorMap* qmap = w.kind == 0 ? &tq0 : w.kind == 1 ? &tq1 : w.kind == 2 ? &tq2 : &tq3;
              tma_load_2d(bs, qmap, &ctl->full[rs.stage], qcol, w.base + k0);
            }
            pend.issued(rs.stage, rs.phase);
          }
        } else {
          // P: 64 rows x 16 chunks (128 m); 16 consecutive threads read one row
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const int c = tid + 128 * i;
            const int kk = c >> 4, ch = c & 15;
            const bool in = k0 + kk < w.rows;
            int prow = w.base + k0 + kk;
            if (w.kind == 3 && in && a.perm) prow = __ldg(a.perm + prow);
            const uint16_t* src = P + size_t(in ? prow : 0) * ldp + pcol + ch * 8;
            cp_async16(as + mn_offset(kk, ch), src, in ? 16u : 0u);
          }
        }
        // Q: 64 rows x nchunk chunks
        for (int c = tid; !qtma && c < kRowsPerStage * nchunk; c += 128) {
          const int kk = c / nchunk, ch = c - kk * nchunk;
          const bool in = k0 + kk < w.rows && ch < nreal;
          const uint16_t* src = Qs + size_t(in ? w.base + k0 + kk : 0) * ldq + qcol + (in ? ch * 8 : 0);
          cp_async16(bs + mn_offset(kk, ch), src, in ? 16u : 0u);
        }
        cp_async_arrive_noinc(&ctl->full[rs.stage]);
        rs.next<kStages>();
      }
      if (!ok) break;
    }
    cp_async_wait_all();
    // on an abort, wait (bounded) for every TMA fill issued by this thread
    if (tid == 0 && aborted(abort_flag)) pend.drain(ctl->full);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 2 * kAccCols);
  }
}

}  // namespace wgrad

int launch_wgrad(const tqp_moe_weights* w, size_t A, const int32_t* offsets, const int32_t* perm, const uint16_t* dO,
                 const uint16_t* h, const uint16_t* dgu, const uint16_t* x16, const uint16_t* ha, const uint16_t* dha,
                 const uint16_t* xa, const uint16_t* dxa, const tqp_adapter_grads* g, const uint32_t* dmax,
                 int32_t* status, cudaStream_t s) {
  const int r = w->rank;
  if (r == 0) return TQP_OK;
  if (r > 32 || w->d % 128 != 0 || w->ffn % 128 != 0) return TQP_ERR_UNSUPPORTED;   // caller falls back
  wgrad::Args a{};
  a.E = w->E;
  a.d = w->d;
  a.f = w->ffn;
  a.r = r;
  a.tiles[0] = w->d / 128;
  a.tiles[1] = w->ffn / 128;
  a.tiles[2] = 2 * w->ffn / 128;
  a.tiles[3] = w->d / 128;
  a.tile_prefix[0] = 0;
  for (int k = 0; k < 4; ++k) a.tile_prefix[k + 1] = a.tile_prefix[k] + a.tiles[k];
  a.offsets = offsets;
  a.perm = perm;
  a.dO = dO;
  a.h = h;
  a.dgu = dgu;
  a.x16 = x16;
  a.ha = ha;
  a.dha = dha;
  a.xa = xa;
  a.dxa = dxa;
  for (int p = 0; p < 3; ++p) {
    a.dA[p] = g->dA[p];
    a.dB[p] = g->dB[p];
  }
  a.dmax = dmax;
  a.status = status;
  a.wait_ns = wait_limit_ns();
  static DeviceFlags attr_done;
  if (!attr_done.test_and_set_device(wgrad::wgrad_kernel, int(wgrad::kSmemBytes))) return TQP_ERR_CUDA;
  CUtensorMap tp[4], tq[4];
  std::memset(tp, 0, sizeof(tp));
  std::memset(tq, 0, sizeof(tq));
  if (!perm) {
    // the P and Q matrices are expert-sorted rows [A][width]
    const uint64_t rows = uint64_t(A);
    if (!make_tile_map(&tp[0], dO, rows, uint64_t(w->d), 64) || !make_tile_map(&tp[1], h, rows, uint64_t(w->ffn), 64) ||
        !make_tile_map(&tp[2], dgu, rows, uint64_t(2 * w->ffn), 64) ||
        !make_tile_map(&tp[3], x16, rows, uint64_t(w->d), 64) ||
        !make_tile_map(&tq[0], ha, rows, uint64_t(r), 64) || !make_tile_map(&tq[1], dha, rows, uint64_t(r), 64) ||
        !make_tile_map(&tq[2], xa, rows, uint64_t(2 * r), 64) || !make_tile_map(&tq[3], dxa, rows, uint64_t(2 * r), 64))
      return TQP_ERR_CUDA;
  }
  const int units = a.E * a.tile_prefix[4];
  const int grid = units < num_sms() ? units : num_sms();
  wgrad::wgrad_kernel<<<grid, wgrad::kThreads, wgrad::kSmemBytes, s>>>(a, tp[0], tp[1], tp[2], tp[3], tq[0], tq[1],
                                                                        tq[2], tq[3]);
  return cudaGetLastError() == cudaSuccess ? TQP_OK : TQP_ERR_CUDA;
}

}  // namespace tqp
