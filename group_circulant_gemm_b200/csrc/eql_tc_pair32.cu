// FP32 p4 (T = 4) EQ-Linear layer on the tensor cores: 3xTF32 split precision on
// SM pairs (tcgen05 cta_group::2, kind::tf32), FP32 in, FP32 accumulate, FP32 out.
//
// What it computes (Flash EQ-Linear summary, "Algorithmic approach" items 1-3):
// the same four input planes X0, X2, Xr, Xi (each times 1/4) and the same six
// per-frequency products against the prepared weight planes (A0, A2, Br, Bi) as
// the FP16 pair kernel, then the inverse DFT plus bias in the epilogue.  Each FP32
// operand v is split as v = hi + lo with hi = tf32(v) (round to nearest, 10
// mantissa bits) and lo = tf32(v - hi); a product A B^T is taken as
//   Ahi Bhi^T + Alo Bhi^T + Ahi Blo^T
// on the TF32 tensor cores with FP32 accumulation.  hi*hi is exact; the dropped
// lo*lo term and the rounding of lo are each below 2^-21 of |A||B| elementwise,
// so the result keeps about FP32 accuracy (the FP32 bar is 1e-5 of max|Y|).
//
// Input planes ("tiled FP32 hi/lo planes", written by group_dft_tf32_kernel):
// eight planes (hi of X0, X2, Xr, Xi, then lo of the same), each stored like
// the FP16 tiled planes but with 8 FP32 channels per 32-byte row: element
// (plane q, row n, channel j) at byte
//   ((q * (C / 8) + j / 8) * Np + n) * 32 + 16 * (((j % 8) / 4) ^ ((n / 4) % 2)) + 4 * (j % 4),
// Np = N rounded up to a multiple of 128.  One TMA box per stage brings the
// eight planes of one K step (8 channels) for this CTA's 128 rows (32 KB).
//
// Design (cluster of 2 CTAs, one per SM, persistent over (256-row, 64
// out-channel) tiles; K step = stage = 8 input channels):
//   warp 0     producer (both CTAs): per stage the 32 KB input box and this
//              CTA's 8 KB of the weights (32 rows of each of the 8 planes),
//              both completing on the leader's stage barrier.
//   warps 1, 3 TMEM allocation (warp 1, both CTAs); lane 0 of warps 1 and 3 of
//              the leader issue the MMAs (M = 256, N = 64, K = 8): three
//              products each (warp 1: Y0, Y1r, -Xi Bi; warp 3: Y2, Y1i, Xi Br),
//              three TF32 MMAs per product.
//   warps 4-11 epilogue (both CTAs, own 128 rows): per 8 out-channels, the four
//              FP32 accumulators from TMEM, inverse DFT + bias (+ activation),
//              one TMA store of 32 rows x 32 floats.
// TMEM holds two tiles' accumulators (2 x [Y0 | Y2 | Y1r | Y1i] x 64 columns),
// so a tile's epilogue overlaps the next tile's MMAs.  Why N = 64: with N = 128
// the four FP32 accumulators fill TMEM, and the FP32 outputs of a 128-channel
// tile do not fit in registers while it is drained.  Every wait is bounded
// (about 2 s); on expiry the CTA sets its abort flag and the plan's status word,
// drains what it issued, and both CTAs meet at the final cluster barrier.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "eql_common.cuh"
#include "eql_kernels.h"
#include "eql_tc_common.cuh"
#include "eql_tc_fwd_parts.cuh"
#include "eql_tc_pair_common.cuh"

namespace eql {
namespace {

using namespace tc;
using namespace ftc;

constexpr int P3_BD = 64;                          // out-channels per tile (N)
constexpr int P3_KC = 8;                           // input channels per K step / stage
constexpr uint32_t P3_ROWB = 32;                   // bytes per operand row (8 FP32)
constexpr uint32_t P3_XPL = 128 * P3_ROWB;         // 4 KB: one input plane, own 128 rows
constexpr uint32_t P3_XBYTES = 8 * P3_XPL;         // 32 KB: hi and lo of 4 planes
constexpr uint32_t P3_WPL = 32 * P3_ROWB;          // 1 KB: this CTA's 32 rows of a weight plane
constexpr uint32_t P3_WBYTES = 8 * P3_WPL;         // 8 KB
constexpr uint32_t P3_STAGE = P3_XBYTES + P3_WBYTES;  // 40 KB
constexpr int P3_WLINES = P3_WBYTES / 128;         // a weight stage as 128-byte lines
constexpr int P3_ST = 4;                           // ring depth
constexpr int P3_THREADS = 384;
constexpr int P3_EPI0 = 4;
constexpr uint32_t P3_STG = 4096;                  // per epilogue warp: 32 rows x 128 B
constexpr uint32_t P3_OFF_STG = P3_ST * P3_STAGE;
constexpr uint32_t P3_OFF_BIAS = P3_OFF_STG + kEpiWarps * P3_STG;
constexpr uint32_t P3_OFF_BAR = P3_OFF_BIAS + kEpiWarps * 128;
constexpr uint32_t P3_SMEM = P3_OFF_BAR + 512 + 1024;
static_assert(P3_STAGE % 1024 == 0, "stage slots stay 1024-byte aligned");
static_assert(P3_SMEM <= 232448, "shared memory budget");

struct P3Bars {
  uint64_t full[P3_ST];    // leader: both CTAs' bytes of a stage landed
  uint64_t empty[P3_ST];   // each CTA: the stage's MMAs are done
  uint64_t acc_full[2];    // each CTA: accumulator buffer b is final
  uint64_t acc_empty[2];   // leader: both CTAs' epilogues have read buffer b
  uint64_t drain[2];       // leader: every MMA an issuer issued is complete
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(P3Bars) <= 512, "barrier block");

// Instruction descriptor, kind::tf32: A = B = TF32 (format 2), D = F32, both
// K-major; bit 13 negates A.
__host__ __device__ constexpr uint32_t idesc_tf32(int M, int N, bool negate_a = false) {
  return (1u << 4) | (2u << 7) | (2u << 10) | (negate_a ? (1u << 13) : 0u) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}
__device__ __forceinline__ void umma_pair_tf32(uint32_t d_tmem, uint64_t a, uint64_t b,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// TF32 value of v, rounded to nearest (ties away), in a 32-bit container.
__device__ __forceinline__ float tf32_rna(float v) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(v));
  return __uint_as_float(r);
}

struct P3Sched {
  int64_t N;
  int n_prow, n_dt, n_ks, Cout, total;
  const float* bias;
};

template <int ACT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P3_THREADS, 1)
    eq_pair_tf32_kernel(const __grid_constant__ CUtensorMap map_x,
                        const __grid_constant__ CUtensorMap map_w,
                        const __grid_constant__ CUtensorMap map_y, P3Sched sc, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  P3Bars* bars = reinterpret_cast<P3Bars*>(smem + P3_OFF_BAR);
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cta_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P3_ST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 2);  // a multicast commit from each issuer
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars->acc_full[b], 2);
      mbar_init(&bars->acc_empty[b], 2 * kEpiWarps);
    }
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  grid_dependency_wait();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ---------------- producer: eight input planes and this CTA's weight rows ----------------
    if (lane == 0) {
      int issued_phase[P3_ST];
      for (int s = 0; s < P3_ST; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int u = pair; ok && u < sc.total; u += npairs) {
        const int prow = u / sc.n_dt, dt = u % sc.n_dt;
        const int row = prow * 256 + 128 * (int)rank;
        for (int ks = 0; ks < sc.n_ks; ++ks, ++it) {
          const int s = it % P3_ST;
          const uint32_t ph = (it / P3_ST) & 1;
          if (!(ok = wait_bounded(&bars->empty[s], ph ^ 1, abort_flag, status))) break;
          const uint32_t full_leader = peer_addr(smem_u32(&bars->full[s]), 0);
          if (rank == 0) mbar_expect_tx(&bars->full[s], 2 * P3_STAGE);
          const uint32_t slot = sbase + s * P3_STAGE;
          tma_load_4d_pair(slot, &map_x, full_leader, 0, row / 4, ks, 0);
          const int wline = ((dt * sc.n_ks + ks) * 2 + (int)rank) * P3_WLINES;
          tma_load_2d_pair(slot + P3_XBYTES, &map_w, full_leader, 0, wline);
          issued_phase[s] = (int)ph;
        }
      }
      if (!ok && rank == 0) {
        for (int s = 0; s < P3_ST; ++s)
          if (issued_phase[s] >= 0) drain_wait(&bars->full[s], (uint32_t)issued_phase[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 3) {
    // ---------------- MMA issuers (leader CTA) ----------------
    if (rank == 0 && lane == 0) {
      const int who = warp == 1 ? 0 : 1;
      const uint32_t id_pos = idesc_tf32(256, P3_BD), id_neg = idesc_tf32(256, P3_BD, true);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int u = pair; ok && u < sc.total; u += npairs, ++tcount) {
        const uint32_t b = tcount & 1;
        if (!(ok = wait_bounded(&bars->acc_empty[b], ((tcount >> 1) & 1) ^ 1, abort_flag, status)))
          break;
        tc_fence_after();
        const uint32_t acc = tmem + b * 4 * P3_BD;  // [Y0 | Y2 | Y1r | Y1i], 64 columns each
        for (int ks = 0; ks < sc.n_ks; ++ks, ++it) {
          const int s = it % P3_ST;
          if (!(ok = wait_bounded(&bars->full[s], (it / P3_ST) & 1, abort_flag, status))) break;
          tc_fence_after();
          const uint32_t xs = sbase + s * P3_STAGE, ws = xs + P3_XBYTES;
#pragma unroll
          for (int combo = 0; combo < 3; ++combo) {
            // (A part, B part): (hi, hi), (lo, hi), (hi, lo)
            const uint32_t ha = combo == 1 ? 4u : 0u, hb = combo == 2 ? 4u : 0u;
            const uint32_t first = (ks == 0 && combo == 0) ? 0u : 1u;
            const uint64_t xr = desc_kmajor<32>(xs + (ha + 2) * P3_XPL);
            const uint64_t xi = desc_kmajor<32>(xs + (ha + 3) * P3_XPL);
            const uint64_t br = desc_kmajor<32>(ws + (hb + 2) * P3_WPL);
            const uint64_t bi = desc_kmajor<32>(ws + (hb + 3) * P3_WPL);
            if (who == 0) {
              umma_pair_tf32(acc + 0, desc_kmajor<32>(xs + (ha + 0) * P3_XPL),
                             desc_kmajor<32>(ws + (hb + 0) * P3_WPL), id_pos, first);   // Y0
              umma_pair_tf32(acc + 2 * P3_BD, xr, br, id_pos, first);                  // Y1r
              umma_pair_tf32(acc + 2 * P3_BD, xi, bi, id_neg, 1u);                     // -Xi Bi
            } else {
              umma_pair_tf32(acc + P3_BD, desc_kmajor<32>(xs + (ha + 1) * P3_XPL),
                             desc_kmajor<32>(ws + (hb + 1) * P3_WPL), id_pos, first);   // Y2
              umma_pair_tf32(acc + 3 * P3_BD, xr, bi, id_pos, first);                  // Y1i
              umma_pair_tf32(acc + 3 * P3_BD, xi, br, id_pos, 1u);                     // Xi Br
            }
          }
          umma_commit_pair(&bars->empty[s], 3);
        }
        if (ok) umma_commit_pair(&bars->acc_full[b], 3);
      }
      umma_commit_pair(&bars->drain[who], 1);
      drain_wait(&bars->drain[who], 0);
    }
    __syncwarp();
  } else if (warp >= P3_EPI0 && warp < P3_EPI0 + kEpiWarps) {
    // ---------------- epilogue (both CTAs, own rows) ----------------
    const int q = warp & 3;                // TMEM lane quarter = rows 32q..32q+31
    const int ch = (warp - P3_EPI0) >> 2;  // 32-channel half of the 64-channel tile
    uint8_t* stg = smem + P3_OFF_STG + (warp - P3_EPI0) * P3_STG;
    const uint32_t stg_s = smem_u32(stg);
    float* bsm = reinterpret_cast<float*>(smem + P3_OFF_BIAS + (warp - P3_EPI0) * 128);
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    uint32_t tcount = 0;
    for (int u = pair; u < sc.total; u += npairs, ++tcount) {
      const int prow = u / sc.n_dt, dt = u % sc.n_dt;
      const int64_t row0 = (int64_t)prow * 256 + 128 * rank + 32 * q;
      const int dbase = dt * P3_BD + 32 * ch;
      const uint32_t b = tcount & 1;
      bsm[lane] = (sc.bias && dbase + lane < sc.Cout) ? sc.bias[dbase + lane] : 0.f;
      __syncwarp();
      if (!warp_wait(&bars->acc_full[b], (tcount >> 1) & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t acc = lane_base + b * 4 * P3_BD + 32 * ch;
#pragma unroll 1
      for (int k = 0; k < 4; ++k) {
        const int d0 = dbase + 8 * k;
        if (d0 >= sc.Cout) break;
        uint32_t v[4][8];
#pragma unroll
        for (int p = 0; p < 4; ++p) tmem_ld_32x32b<8>(acc + p * P3_BD + 8 * k, v[p]);
        tmem_wait_ld();
        // both operands carry 1/4: the accumulators hold Y/16; inverse transform
        // terms 4 acc (real frequencies) and 8 acc (complex)
        float4 o[8];
#pragma unroll
        for (int m = 0; m < 8; ++m) {
          const float a0 = __uint_as_float(v[0][m]), a2 = __uint_as_float(v[1][m]);
          const float ar = __uint_as_float(v[2][m]), ai = __uint_as_float(v[3][m]);
          const float sb = fmaf(4.f, a0, bsm[8 * k + m]);
          const float ev = fmaf(4.f, a2, sb), od = fmaf(-4.f, a2, sb);
          o[m] = make_float4(act_fn<ACT>(fmaf(8.f, ar, ev)), act_fn<ACT>(fmaf(-8.f, ai, od)),
                             act_fn<ACT>(fmaf(-8.f, ar, ev)), act_fn<ACT>(fmaf(8.f, ai, od)));
        }
        if (lane == 0) bulk_wait_read_all();  // the previous store has read the staging
        __syncwarp();
        uint8_t* rowp = stg + lane * 128;
#pragma unroll
        for (int m = 0; m < 8; ++m)
          *reinterpret_cast<float4*>(rowp + ((m ^ (lane & 7)) << 4)) = o[m];
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0 && row0 < sc.N) {
          tma_store_3d(&map_y, stg_s, 0, d0 / 8, (int)row0);
          bulk_commit();
        }
      }
      // buffer b is read (or holds nothing for this warp): hand it back; relaxed,
      // as every TMEM load of this warp completed above
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_remote_relaxed(peer_addr(smem_u32(&bars->acc_empty[b]), 0));
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// Group DFT of p4 FP32 rows into the hi/lo planes (layout above), each value
// times 1/4, rows N..Np-1 zero.  A warp takes 4 rows and up to 4 blocks of 8
// channels; per block a lane loads one channel's four group elements (16 bytes;
// lane l: row 4r + l/8, channel l%8), so each load instruction reads 4 whole
// 128-byte row segments, and per plane a lane stores 4 bytes, so each store
// instruction writes 128 contiguous bytes.
__global__ void group_dft_tf32_kernel(const float4* __restrict__ X, int64_t N, int64_t Np, int C,
                                      uint8_t* __restrict__ out) {
  constexpr int G = 4;
  grid_dependency_wait();
  grid_launch_dependents();
  const int KB = C / 8;
  const int KBG = (KB + G - 1) / G;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= Np / 4 * KBG) return;
  const int lane = (int)(threadIdx.x & 31);
  const int kb0 = (int)(w % KBG) * G;
  const int64_t n = (w / KBG) * 4 + (lane >> 3);
  const int piece = lane & 7;
  float4 v[G];
#pragma unroll
  for (int g = 0; g < G; ++g) {
    v[g] = make_float4(0.f, 0.f, 0.f, 0.f);
    if (n < N && kb0 + g < KB) v[g] = X[n * C + (int64_t)(kb0 + g) * 8 + piece];
  }
  const int64_t inrow = n * 32 + (((piece >> 2) ^ (int)((n >> 2) & 1)) << 4) + (piece & 3) * 4;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    if (kb0 + g >= KB) break;
    const float x0 = v[g].x, x1 = v[g].y, x2 = v[g].z, x3 = v[g].w;
    const float a = x0 + x2, b = x1 + x3;
    const float pl[4] = {(a + b) * 0.25f, (a - b) * 0.25f, (x0 - x2) * 0.25f, (x3 - x1) * 0.25f};
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      const float hi = tf32_rna(pl[p]);
      const float lo = tf32_rna(pl[p] - hi);
      *reinterpret_cast<float*>(out + ((int64_t)p * KB + kb0 + g) * Np * 32 + inrow) = hi;
      *reinterpret_cast<float*>(out + ((int64_t)(4 + p) * KB + kb0 + g) * Np * 32 + inrow) = lo;
    }
  }
}

// Prepared FP32 planes [P][Cout][Cin] (A0, A2, Br, Bi first) -> the 3xTF32
// kernel's weight stages: blob (dt, ks, rank) = 8 planes (hi of A0, A2, Br, Bi,
// then lo) x 32 rows x 8 channels (32 bytes, 32-byte swizzle: 16-byte piece ^=
// (row / 4) % 2); row r of a plane = out-channel dt*64 + 32*rank + r, channels
// 8ks ..; zero past the matrix.  One thread per 16-byte piece.
__global__ void pair_tf32_tile_weights_kernel(const float* __restrict__ planes, int Cin, int Cout,
                                              int n_ks, int64_t n_pieces,
                                              float4* __restrict__ tiles) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_pieces) return;
  const int piece = (int)(idx & 1);
  const int r = (int)((idx >> 1) & 31);
  const int plane = (int)((idx >> 6) & 3);
  const int hl = (int)((idx >> 8) & 1);
  const int64_t blob = idx >> 9;  // (dt, ks, rank)
  const int rank = (int)(blob & 1);
  const int64_t dk = blob >> 1;
  const int dt = (int)(dk / n_ks), ks = (int)(dk % n_ks);
  const int d = dt * P3_BD + 32 * rank + r;
  const int c0 = ks * P3_KC + piece * 4;
  float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
  if (d < Cout && c0 < Cin) {  // Cin % 8 == 0: the 4 channels are all in range
    const float4 w = *reinterpret_cast<const float4*>(planes + ((int64_t)plane * Cout + d) * Cin + c0);
    const float e[4] = {w.x, w.y, w.z, w.w};
    float t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float h = tf32_rna(e[i]);
      t[i] = hl ? tf32_rna(e[i] - h) : h;
    }
    v = make_float4(t[0], t[1], t[2], t[3]);
  }
  const int64_t dst = blob * P3_WBYTES + (hl * 4 + plane) * P3_WPL + r * P3_ROWB +
                      ((piece ^ ((r >> 2) & 1)) << 4);
  tiles[dst >> 4] = v;
}

template <int ACT>
cudaError_t set_tf32_attr() {
  return cudaFuncSetAttribute(eq_pair_tf32_kernel<ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              P3_SMEM);
}

int tf32_capacity(const void* kernel, int num_sms) {
  static int max_pairs = 0;
  if (max_pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)(num_sms / 2));
    cfg.blockDim = dim3(P3_THREADS);
    cfg.dynamicSmemBytes = P3_SMEM;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms / 2;
    }
    max_pairs = n < num_sms / 2 ? n : num_sms / 2;
  }
  return max_pairs;
}

int tf32_n_dt(int Cout) { return (Cout + P3_BD - 1) / P3_BD; }

}  // namespace

bool pair_tf32_supported(int64_t N, int Cin, int Cout) {
  return N >= 1 && N <= 0x7fffff00LL && Cin % 8 == 0 && Cout % 8 == 0 && Cin >= 8 && Cout >= 8;
}

size_t tiled_tf32_planes_bytes(int64_t N, int channels) {
  return (size_t)8 * (size_t)((N + 127) / 128 * 128) * (size_t)channels * 4;
}

size_t pair_tf32_tile_bytes(int Cin, int Cout) {
  return (size_t)tf32_n_dt(Cout) * (size_t)(Cin / P3_KC) * 2 * P3_WBYTES;
}

cudaError_t launch_pair_tf32_tile_weights(const void* planes, int Cin, int Cout, void* tiles,
                                          cudaStream_t st) {
  if (Cin % 8 != 0 || Cout % 8 != 0) return cudaErrorInvalidValue;
  const int64_t n_pieces = (int64_t)pair_tf32_tile_bytes(Cin, Cout) / 16;
  pair_tf32_tile_weights_kernel<<<(unsigned)((n_pieces + 255) / 256), 256, 0, st>>>(
      static_cast<const float*>(planes), Cin, Cout, Cin / P3_KC, n_pieces,
      static_cast<float4*>(tiles));
  return cudaGetLastError();
}

cudaError_t launch_group_dft_tf32(const void* X, int64_t N, int C, void* out, cudaStream_t st) {
  if (N <= 0) return cudaSuccess;
  if (C % 8 != 0) return cudaErrorInvalidValue;
  const int64_t Np = (N + 127) / 128 * 128;
  const int64_t threads = Np / 4 * ((C / 8 + 3) / 4) * 32;
  return launch_dependent(group_dft_tf32_kernel, dim3((unsigned)((threads + 255) / 256)), dim3(256),
                          0, st, static_cast<const float4*>(X), N, Np, C,
                          static_cast<uint8_t*>(out));
}

cudaError_t launch_pair_tf32(const void* Xt, int64_t N, int Cin, int Cout, const void* tiles,
                             const void* bias, void* Y, int* status, int num_sms, int act,
                             cudaStream_t st) {
  if (!pair_tf32_supported(N, Cin, Cout) || !tiles) return cudaErrorNotSupported;
  if (act != 0 && act != 1) return cudaErrorInvalidValue;
  auto encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  const int64_t Np = (N + 127) / 128 * 128;
  CUtensorMap mx, mw, my;
  {
    // input planes: (32 floats of a 128-byte line, Np/4 lines, Cin/8 blocks, 8 planes);
    // box = 32 lines (128 rows) x 1 block x 8 planes = 32 KB
    cuuint64_t dims[4] = {32, (cuuint64_t)(Np / 4), (cuuint64_t)(Cin / 8), 8};
    cuuint64_t strides[3] = {128, (cuuint64_t)Np * 32, (cuuint64_t)Np * 32 * (Cin / 8)};
    cuuint32_t box[4] = {32, 32, 1, 8};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<void*>(Xt), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // weight stages as 128-byte lines, box = one stage of this CTA (64 lines)
    cuuint64_t dims[2] = {32, (cuuint64_t)(pair_tf32_tile_bytes(Cin, Cout) / 128)};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {32, P3_WLINES};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(tiles), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    // Y [N][Cout*4] FP32: (32 floats = 8 channels, Cout/8 chunks, N rows); box = 32 rows
    cuuint64_t dims[3] = {32, (cuuint64_t)(Cout / 8), (cuuint64_t)N};
    cuuint64_t strides[2] = {128, (cuuint64_t)Cout * 4 * 4};
    cuuint32_t box[3] = {32, 1, 32};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, Y, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static bool attrs = false;
  if (!attrs) {
    cudaError_t e = set_tf32_attr<0>();
    if (e == cudaSuccess) e = set_tf32_attr<1>();
    if (e != cudaSuccess) return e;
    attrs = true;
  }
  P3Sched sc = {};
  sc.N = N;
  sc.n_prow = (int)((N + 255) / 256);
  sc.n_dt = tf32_n_dt(Cout);
  sc.n_ks = Cin / P3_KC;
  sc.Cout = Cout;
  if ((int64_t)sc.n_prow * sc.n_dt > 0x7fffffffLL) return cudaErrorInvalidValue;
  sc.total = sc.n_prow * sc.n_dt;
  sc.bias = static_cast<const float*>(bias);
  auto kernel = act ? eq_pair_tf32_kernel<1> : eq_pair_tf32_kernel<0>;
  int npairs = tf32_capacity((const void*)kernel, num_sms);
  if (npairs > sc.total) npairs = sc.total;
  return launch_dependent(kernel, dim3(2 * npairs), dim3(P3_THREADS), P3_SMEM, st, mx, mw, my, sc,
                          status);
}

}  // namespace eql
