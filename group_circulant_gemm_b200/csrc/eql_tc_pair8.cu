// Eight-plane layers on SM pairs (tcgen05 cta_group::2, kind::f16): the cyclic
// T = 8 EQ-Linear layer and the layer over the dihedral group D4, FP16 in, FP32
// accumulate, FP16 out, for sm_100a.
//
// What it computes (Flash EQ-Linear summary, "Algorithmic approach" items 1-3;
// the D4 form as read in "Limitations and future work"): the input arrives as
// its group Fourier transform, eight FP16 planes (each times 1/8) in the tiled
// layout of the p4 pair kernel; per frequency the real products against the
// prepared weight planes; then the inverse transform plus bias (and activation)
// in the epilogue.
//   cyclic T = 8 (planes V0, V4, Re/Im V1, V2, V3 of the DFT; the weights hold
//   conj(DFT(W))/8 in the same order): 2 real products and 4 per complex
//   frequency, 14 in all, into 8 accumulators (frequencies 0 and 4, Re/Im of
//   1, 2, 3);
//   D4 (planes: the four characters, then the 2 x 2 representation's entries
//   X[i][j] at 4 + 2i + j; weight entry W[k][j] at 4 + k + 2j): 4 character
//   products and Y[i][k] += X[i][j] W[k][j], 12 in all, into 8 accumulators.
// Eight accumulators of 64 columns fill TMEM, so a tile is 256 rows x 64
// out-channels, every MMA is M = 256, N = 64, K = 16.
//
// Design (cluster of 2 CTAs, one per SM, persistent over (256-row, 64
// out-channel) tiles; stage = one K step of 16 input channels):
//   warp 0     producer (both CTAs): per stage one 4-D TMA box of the tiled
//              planes (its 128 rows x 1 channel block x 8 planes = 32 KB) and its
//              8 KB of the weights (32 rows of each plane), completing on the
//              leader's stage barrier; a 4-deep ring.
//   warps 1, 3 TMEM allocation (warp 1, both CTAs); lane 0 of warps 1 and 3 of
//              the leader issue the products, each owning four accumulators.
//   warps 4-11 epilogue (both CTAs, own 128 rows): per 4 out-channels the eight
//              accumulators from TMEM, inverse transform + bias (+ activation),
//              FP16; per 8 channels one TMA store of 32 rows x 128 bytes.
// The loads (40 KB per stage against 448 cycles of MMA) bound the main loop;
// the epilogue holds TMEM while it drains, during which the producer refills
// the ring for the next tile.  Every wait is bounded (about 2 s); on expiry the
// CTA sets its abort flag and the plan's status word, drains what it issued,
// and both CTAs meet at the final cluster barrier.
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

constexpr int P8_BD = 64;                          // out-channels per tile (N)
constexpr int P8_KC = 16;                          // input channels per K step / stage
constexpr uint32_t P8_ROWB = 32;                   // bytes per operand row (16 halves)
constexpr uint32_t P8_XPL = 128 * P8_ROWB;         // 4 KB: one input plane, own 128 rows
constexpr uint32_t P8_XBYTES = 8 * P8_XPL;         // 32 KB
constexpr uint32_t P8_WPL = 32 * P8_ROWB;          // 1 KB: this CTA's 32 rows of a weight plane
constexpr uint32_t P8_WBYTES = 8 * P8_WPL;         // 8 KB
constexpr uint32_t P8_STAGE = P8_XBYTES + P8_WBYTES;  // 40 KB
constexpr int P8_WLINES = P8_WBYTES / 128;
constexpr int P8_ST = 4;
constexpr int P8_THREADS = 384;
constexpr int P8_EPI0 = 4;
// per epilogue warp: 32 rows x 128 B of Y, or (next-layer planes) 8 planes x 32
// rows x 32 B of one 16-channel block
constexpr uint32_t P8_STG = 8192;
constexpr uint32_t P8_OFF_STG = P8_ST * P8_STAGE;
constexpr uint32_t P8_OFF_BIAS = P8_OFF_STG + kEpiWarps * P8_STG;
constexpr uint32_t P8_OFF_BAR = P8_OFF_BIAS + kEpiWarps * 128;
constexpr uint32_t P8_SMEM = P8_OFF_BAR + 512 + 1024;
static_assert(P8_STAGE % 1024 == 0, "stage slots stay 1024-byte aligned");
static_assert(P8_SMEM <= 232448, "shared memory budget");

struct P8Bars {
  uint64_t full[P8_ST];
  uint64_t empty[P8_ST];
  uint64_t acc_full;
  uint64_t acc_empty;
  uint64_t drain[2];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(P8Bars) <= 512, "barrier block");

// One product: accumulator, input plane, weight plane, negate A, and whether it
// is the first product into its accumulator within a K step.
struct Prod {
  int acc, xp, wp, neg, first;
};
// The products of one K step for issuer WHO (seven for cyclic T = 8, six for
// D4; each issuer owns its accumulators).
template <int G, int WHO>
__device__ __forceinline__ void issue8(uint32_t tmem, uint32_t xs, uint32_t ws, int ks,
                                       uint32_t id_pos, uint32_t id_neg) {
  constexpr Prod cyc[2][7] = {
      {{0, 0, 0, 0, 1}, {2, 2, 2, 0, 1}, {2, 3, 3, 1, 0}, {3, 2, 3, 0, 1}, {3, 3, 2, 0, 0},
       {4, 4, 4, 0, 1}, {4, 5, 5, 1, 0}},
      {{1, 1, 1, 0, 1}, {5, 4, 5, 0, 1}, {5, 5, 4, 0, 0}, {6, 6, 6, 0, 1}, {6, 7, 7, 1, 0},
       {7, 6, 7, 0, 1}, {7, 7, 6, 0, 0}}};
  // D4: Y[i][k] (accumulator 4 + 2i + k) += X[i][j] (plane 4 + 2i + j) W[k][j]
  // (weight plane 4 + k + 2j)
  constexpr Prod dih[2][6] = {
      {{0, 0, 0, 0, 1}, {1, 1, 1, 0, 1}, {4, 4, 4, 0, 1}, {4, 5, 6, 0, 0}, {5, 4, 5, 0, 1},
       {5, 5, 7, 0, 0}},
      {{2, 2, 2, 0, 1}, {3, 3, 3, 0, 1}, {6, 6, 4, 0, 1}, {6, 7, 6, 0, 0}, {7, 6, 5, 0, 1},
       {7, 7, 7, 0, 0}}};
  constexpr int n = G ? 6 : 7;
#pragma unroll
  for (int j = 0; j < n; ++j) {
    const Prod pr = G ? dih[WHO][j < 6 ? j : 5] : cyc[WHO][j];
    umma_pair(tmem + pr.acc * P8_BD, desc_kmajor<32>(xs + pr.xp * P8_XPL),
              desc_kmajor<32>(ws + pr.wp * P8_WPL), pr.neg ? id_neg : id_pos,
              (ks > 0 || !pr.first) ? 1u : 0u);
  }
}

struct P8Sched {
  int64_t N;
  int n_dt, n_ks, Cout, total;
  const __half* bias;
  int64_t Np;     // rows of the tiled planes
};

// The group Fourier transform of one channel's eight elements x[t] (FP32), in
// the plane order of the tiled layout (not yet times 1/8):
//   G = 0, cyclic T = 8: V0, V4, Re V1, Im V1, Re V2, Im V2, Re V3, Im V3 of
//   V[k] = sum_t x_t e^{-2 pi i k t / 8} (radix 2: a_t = x_t + x_{t+4},
//   b_t = x_t - x_{t+4}, one twiddle sqrt(2)/2);
//   G = 1, D4 (t = a + 4b for r^a m^b): the characters (chi(r), chi(m)) =
//   (+,+), (+,-), (-,+), (-,-), then X[i][j] = sum_t x_t rho(t)_ij of
//   r -> [[0,-1],[1,0]], m -> diag(1,-1), at 4 + 2i + j.
template <int G>
__device__ __forceinline__ void dft8(const float (&x)[8], float (&val)[8]) {
  if constexpr (G == 1) {
    const float e0 = x[0] + x[2], o0 = x[1] + x[3];
    const float e1 = x[4] + x[6], o1 = x[5] + x[7];
    const float d0 = x[0] - x[2], d1 = x[1] - x[3];
    const float d4 = x[4] - x[6], d5 = x[5] - x[7];
    val[0] = (e0 + o0) + (e1 + o1);
    val[1] = (e0 + o0) - (e1 + o1);
    val[2] = (e0 - o0) + (e1 - o1);
    val[3] = (e0 - o0) - (e1 - o1);
    val[4] = d0 + d4;
    val[5] = d5 - d1;
    val[6] = d1 + d5;
    val[7] = d0 - d4;
  } else {
    const float h = 0.70710678118654752f;
    const float a0 = x[0] + x[4], a1 = x[1] + x[5], a2 = x[2] + x[6], a3 = x[3] + x[7];
    const float b0 = x[0] - x[4], b1 = x[1] - x[5], b2 = x[2] - x[6], b3 = x[3] - x[7];
    // rounded products (never fused into the adds), so every caller forms the
    // same values
    const float s13 = __fmul_rn(h, b1 - b3), t13 = __fmul_rn(h, b1 + b3);
    val[0] = (a0 + a2) + (a1 + a3);
    val[1] = (a0 + a2) - (a1 + a3);
    val[2] = b0 + s13;
    val[3] = -b2 - t13;
    val[4] = a0 - a2;
    val[5] = a3 - a1;
    val[6] = b0 - s13;
    val[7] = b2 - t13;
  }
}

// NEXT = 1: the output is written as the tiled planes of act(Y) (the next
// layer's input): each value of Y is rounded to FP16 first and then transformed
// with group_dft8_tiled_kernel's arithmetic (dft8), so the planes are those of
// the spatial output passed through that kernel; rows N..Np-1 are zero.
template <int G, int ACT, int NEXT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(P8_THREADS, 1)
    eq_pair8_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                       const __grid_constant__ CUtensorMap map_w,
                       const __grid_constant__ CUtensorMap map_y, P8Sched sc, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  P8Bars* bars = reinterpret_cast<P8Bars*>(smem + P8_OFF_BAR);
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cta_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < P8_ST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], 2);
    }
    mbar_init(&bars->acc_full, 2);
    mbar_init(&bars->acc_empty, 2 * kEpiWarps);
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
    // ---------------- producer ----------------
    if (lane == 0) {
      int issued_phase[P8_ST];
      for (int s = 0; s < P8_ST; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int u = pair; ok && u < sc.total; u += npairs) {
        const int prow = u / sc.n_dt, dt = u % sc.n_dt;
        const int row = prow * 256 + 128 * (int)rank;
        for (int ks = 0; ks < sc.n_ks; ++ks, ++it) {
          const int s = it % P8_ST;
          const uint32_t ph = (it / P8_ST) & 1;
          if (!(ok = wait_bounded(&bars->empty[s], ph ^ 1, abort_flag, status))) break;
          const uint32_t full_leader = peer_addr(smem_u32(&bars->full[s]), 0);
          if (rank == 0) mbar_expect_tx(&bars->full[s], 2 * P8_STAGE);
          const uint32_t slot = sbase + s * P8_STAGE;
          tma_load_4d_pair(slot, &map_x, full_leader, 0, row / 4, ks, 0);
          const int wline = ((dt * sc.n_ks + ks) * 2 + (int)rank) * P8_WLINES;
          tma_load_2d_pair(slot + P8_XBYTES, &map_w, full_leader, 0, wline);
          issued_phase[s] = (int)ph;
        }
      }
      if (!ok && rank == 0) {
        for (int s = 0; s < P8_ST; ++s)
          if (issued_phase[s] >= 0) drain_wait(&bars->full[s], (uint32_t)issued_phase[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1 || warp == 3) {
    // ---------------- MMA issuers (leader CTA) ----------------
    if (rank == 0 && lane == 0) {
      const int who = warp == 1 ? 0 : 1;
      const uint32_t id_pos = idesc_f16(256, P8_BD), id_neg = idesc_f16(256, P8_BD, true);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int u = pair; ok && u < sc.total; u += npairs, ++tcount) {
        if (!(ok = wait_bounded(&bars->acc_empty, (tcount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int ks = 0; ks < sc.n_ks; ++ks, ++it) {
          const int s = it % P8_ST;
          if (!(ok = wait_bounded(&bars->full[s], (it / P8_ST) & 1, abort_flag, status))) break;
          tc_fence_after();
          const uint32_t xs = sbase + s * P8_STAGE, ws = xs + P8_XBYTES;
          if (who == 0)
            issue8<G, 0>(tmem, xs, ws, ks, id_pos, id_neg);
          else
            issue8<G, 1>(tmem, xs, ws, ks, id_pos, id_neg);
          umma_commit_pair(&bars->empty[s], 3);
        }
        if (ok) umma_commit_pair(&bars->acc_full, 3);
      }
      umma_commit_pair(&bars->drain[who], 1);
      drain_wait(&bars->drain[who], 0);
    }
    __syncwarp();
  } else if (warp >= P8_EPI0 && warp < P8_EPI0 + kEpiWarps) {
    // ---------------- epilogue (both CTAs, own rows) ----------------
    const int q = warp & 3;
    const int ch = (warp - P8_EPI0) >> 2;  // 32-channel half of the tile
    uint8_t* stg = smem + P8_OFF_STG + (warp - P8_EPI0) * P8_STG;
    const uint32_t stg_s = smem_u32(stg);
    __half* bsm = reinterpret_cast<__half*>(smem + P8_OFF_BIAS + (warp - P8_EPI0) * 128);
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
    const uint32_t acc_empty_leader = peer_addr(smem_u32(&bars->acc_empty), 0);
    uint32_t tcount = 0;
    for (int u = pair; u < sc.total; u += npairs, ++tcount) {
      const int prow = u / sc.n_dt, dt = u % sc.n_dt;
      const int64_t row0 = (int64_t)prow * 256 + 128 * rank + 32 * q;
      const int dbase = dt * P8_BD + 32 * ch;
      bsm[lane] = (sc.bias && dbase + lane < sc.Cout) ? sc.bias[dbase + lane] : __float2half(0.f);
      __syncwarp();
      if (!warp_wait(&bars->acc_full, tcount & 1, abort_flag, status)) break;
      tc_fence_after();
#pragma unroll 1
      for (int k = 0; k < 4; ++k) {
        const int d0 = dbase + 8 * k;
        if (d0 >= sc.Cout) break;
        uint4 oa[4], ob[4];
        epi_half<8, P8_BD, ACT, G>(lane_addr, 32 * ch + 8 * k, bsm + 8 * k, oa);
        epi_half<8, P8_BD, ACT, G>(lane_addr, 32 * ch + 8 * k + 4, bsm + 8 * k + 4, ob);
        if constexpr (NEXT) {
          // this lane's row: the 8 channels' Y (FP16) -> 8 planes x 8 channels,
          // one 16-byte half row per plane, staged as the tiled layout's image
          // ([plane][32 rows][32 B], halves swapped when (row / 4) % 2); the
          // 16-channel block goes out as one TMA store after its second half
          const int64_t n = row0 + lane;
          {
            uint32_t pl[8][4];
#pragma unroll
            for (int cp = 0; cp < 4; ++cp) {  // channel pair 2cp, 2cp + 1
              float val[2][8];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int c = 2 * cp + e;
                const uint4 y = c < 4 ? oa[c] : ob[c - 4];
                const float2 y01 = unpack_h2(y.x), y23 = unpack_h2(y.y);
                const float2 y45 = unpack_h2(y.z), y67 = unpack_h2(y.w);
                const float x[8] = {y01.x, y01.y, y23.x, y23.y, y45.x, y45.y, y67.x, y67.y};
                dft8<G>(x, val[e]);
              }
#pragma unroll
              for (int p = 0; p < 8; ++p)
                pl[p][cp] = n < sc.N ? pack_h2(val[0][p] * 0.125f, val[1][p] * 0.125f) : 0u;
            }
            const int half = k & 1;  // d0 % 16 / 8: dbase is a multiple of 16
            if (half == 0) {
              if (lane == 0) bulk_wait_read_all();  // the previous store has read the staging
              __syncwarp();
            }
            uint8_t* rowp = stg + lane * 32 + ((half ^ ((lane >> 2) & 1)) << 4);
#pragma unroll
            for (int p = 0; p < 8; ++p)
              *reinterpret_cast<uint4*>(rowp + p * 1024) =
                  make_uint4(pl[p][0], pl[p][1], pl[p][2], pl[p][3]);
            if (half == 1) {
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              __syncwarp();
              // rows past Np fall outside the map and are not written
              if (lane == 0 && row0 < sc.Np) {
                tma_store_4d(&map_y, stg_s, 0, (int)(row0 / 4), d0 / 16, 0);
                bulk_commit();
              }
            }
          }
          continue;
        }
        if (lane == 0) bulk_wait_read_all();  // the previous store has read the staging
        __syncwarp();
        uint8_t* rowp = stg + lane * 128;
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          *reinterpret_cast<uint4*>(rowp + ((m ^ (lane & 7)) << 4)) = oa[m];
          *reinterpret_cast<uint4*>(rowp + (((4 + m) ^ (lane & 7)) << 4)) = ob[m];
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0 && row0 < sc.N) {
          tma_store_3d(&map_y, stg_s, 0, d0 / 8, (int)row0);
          bulk_commit();
        }
      }
      // every TMEM load of this warp for the tile has completed (epi_half waits)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_remote_relaxed(acc_empty_leader);
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

// Fourier transform of eight-element group rows into eight tiled planes, each
// value times 1/8 (FP32 arithmetic, one rounding), rows N..Np-1 zero.
//   G = 0, cyclic T = 8: V0, V4, Re V1, Im V1, Re V2, Im V2, Re V3, Im V3 of the
//   DFT V[k] = sum_t x_t e^{-2 pi i k t / 8} (radix 2: a_t = x_t + x_{t+4},
//   b_t = x_t - x_{t+4}, one twiddle sqrt(2)/2);
//   G = 1, D4 (g = a + 4b for r^a m^b): the characters (chi(r), chi(m)) =
//   (+,+), (+,-), (-,+), (-,-), then X[i][j] = sum_g x_g rho(g)_ij of r ->
//   [[0,-1],[1,0]], m -> diag(1,-1), plane 4 + 2i + j.
// A warp takes 4 rows and up to 4 blocks of 16 channels; per block a lane loads
// two channels' eight group elements (32 bytes; lane l: row 4r + l/8, channels
// 2(l%8), 2(l%8)+1 of the block) and stores 4 bytes per plane, so each store
// instruction writes 128 contiguous bytes.
template <int G>
__global__ void group_dft8_tiled_kernel(const uint4* __restrict__ X, int64_t N, int64_t Np, int C,
                                        uint8_t* __restrict__ out) {
  constexpr int GB = 4;
  grid_dependency_wait();
  grid_launch_dependents();
  const int KB = C / 16;
  const int KBG = (KB + GB - 1) / GB;
  const int64_t w = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (w >= Np / 4 * KBG) return;
  const int lane = (int)(threadIdx.x & 31);
  const int kb0 = (int)(w % KBG) * GB;
  const int64_t n = (w / KBG) * 4 + (lane >> 3);
  const int piece = lane & 7;
  uint4 v[GB][2];
#pragma unroll
  for (int g = 0; g < GB; ++g) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      v[g][e] = make_uint4(0u, 0u, 0u, 0u);
      if (n < N && kb0 + g < KB) v[g][e] = X[n * C + (int64_t)(kb0 + g) * 16 + 2 * piece + e];
    }
  }
  const int64_t inrow = n * 32 + (((piece >> 2) ^ (int)((n >> 2) & 1)) << 4) + (piece & 3) * 4;
#pragma unroll
  for (int g = 0; g < GB; ++g) {
    if (kb0 + g >= KB) break;
    float val[2][8];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const float2 p01 = unpack_h2(v[g][e].x), p23 = unpack_h2(v[g][e].y);
      const float2 p45 = unpack_h2(v[g][e].z), p67 = unpack_h2(v[g][e].w);
      const float x[8] = {p01.x, p01.y, p23.x, p23.y, p45.x, p45.y, p67.x, p67.y};
      dft8<G>(x, val[e]);
    }
#pragma unroll
    for (int p = 0; p < 8; ++p)
      *reinterpret_cast<uint32_t*>(out + ((int64_t)p * KB + kb0 + g) * Np * 32 + inrow) =
          pack_h2(val[0][p] * 0.125f, val[1][p] * 0.125f);
  }
}

// Prepared planes -> the eight-plane pair kernel's weight stages: blob (dt, ks,
// rank) = 8 planes x 32 rows x 16 channels (32 bytes, 32-byte swizzle: 16-byte
// piece ^= (row / 4) % 2); row r of a plane = out-channel dt*64 + 32*rank + r,
// channels 16ks ..; zero past the matrix.  One thread per 16-byte piece.
// Normal: planes [P][Cout][Cin], the first eight in the kernel's plane order.
// Adjoint of a D4 layer (dX = the D4 layer of dY with W'[c][d][v] = W[d][c][v^-1]):
// its planes are the forward planes [8][Cin][Cout] read transposed, with the
// 2 x 2 block's off-diagonal entries exchanged (v -> v^-1 maps rho(v) to
// rho(v)^T and keeps every character).
__global__ void pair8_tile_weights_kernel(const __half* __restrict__ planes, int Cin, int Cout,
                                          int n_ks, int64_t n_pieces, int d4_adjoint,
                                          uint4* __restrict__ tiles) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_pieces) return;
  const int piece = (int)(idx & 1);
  const int r = (int)((idx >> 1) & 31);
  const int plane = (int)((idx >> 6) & 7);
  const int64_t blob = idx >> 9;  // (dt, ks, rank)
  const int rank = (int)(blob & 1);
  const int64_t dk = blob >> 1;
  const int dt = (int)(dk / n_ks), ks = (int)(dk % n_ks);
  const int d = dt * P8_BD + 32 * rank + r;
  const int c0 = ks * P8_KC + piece * 8;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (d < Cout && c0 < Cin) {
    if (!d4_adjoint) {
      v = *reinterpret_cast<const uint4*>(planes + ((int64_t)plane * Cout + d) * Cin + c0);
    } else {
      const int src = plane == 5 ? 6 : (plane == 6 ? 5 : plane);
      __half e[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) e[i] = planes[((int64_t)src * Cin + c0 + i) * Cout + d];
      v = *reinterpret_cast<const uint4*>(e);
    }
  }
  const int64_t dst = blob * P8_WBYTES + plane * P8_WPL + r * P8_ROWB + ((piece ^ ((r >> 2) & 1)) << 4);
  tiles[dst >> 4] = v;
}

template <int G, int ACT, int NEXT>
cudaError_t set_p8_attr() {
  return cudaFuncSetAttribute(eq_pair8_tc_kernel<G, ACT, NEXT>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, P8_SMEM);
}

int p8_capacity(const void* kernel, int num_sms) {
  static int max_pairs = 0;
  if (max_pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)(num_sms / 2));
    cfg.blockDim = dim3(P8_THREADS);
    cfg.dynamicSmemBytes = P8_SMEM;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms / 2;
    }
    max_pairs = n < num_sms / 2 ? n : num_sms / 2;
  }
  return max_pairs;
}

}  // namespace

bool pair8_supported(int64_t N, int Cin, int Cout) {
  return N >= 1 && N <= 0x7fffff00LL && Cin % 16 == 0 && Cout % 16 == 0 && Cin >= 16 &&
         Cout >= 16;
}

size_t tiled8_planes_bytes(int64_t N, int channels) {
  return (size_t)8 * (size_t)((N + 127) / 128 * 128) * (size_t)channels * 2;
}

size_t pair8_tile_bytes(int Cin, int Cout) {
  return (size_t)((Cout + P8_BD - 1) / P8_BD) * (size_t)(Cin / P8_KC) * 2 * P8_WBYTES;
}

cudaError_t launch_pair8_tile_weights(const void* planes, int Cin, int Cout, void* tiles,
                                      cudaStream_t st, int d4_adjoint) {
  if (Cin % 16 != 0 || Cout % 16 != 0) return cudaErrorInvalidValue;
  const int64_t n_pieces = (int64_t)pair8_tile_bytes(Cin, Cout) / 16;
  pair8_tile_weights_kernel<<<(unsigned)((n_pieces + 255) / 256), 256, 0, st>>>(
      static_cast<const __half*>(planes), Cin, Cout, Cin / P8_KC, n_pieces, d4_adjoint,
      static_cast<uint4*>(tiles));
  return cudaGetLastError();
}

cudaError_t launch_group_dft8_tiled(const void* X, int64_t N, int C, int group, void* out,
                                    cudaStream_t st) {
  if (N <= 0) return cudaSuccess;
  if (C % 16 != 0) return cudaErrorInvalidValue;
  const int64_t Np = (N + 127) / 128 * 128;
  const int64_t threads = Np / 4 * ((C / 16 + 3) / 4) * 32;
  const dim3 grid((unsigned)((threads + 255) / 256)), block(256);
  auto kernel = group ? group_dft8_tiled_kernel<1> : group_dft8_tiled_kernel<0>;
  return launch_dependent(kernel, grid, block, 0, st, static_cast<const uint4*>(X), N, Np, C,
                          static_cast<uint8_t*>(out));
}

cudaError_t launch_pair8_tc(const void* Xt, int64_t N, int Cin, int Cout, const void* tiles,
                            const void* bias, void* Y, int* status, int num_sms, int act,
                            int group, cudaStream_t st, int next_planes) {
  if (!pair8_supported(N, Cin, Cout) || !tiles) return cudaErrorNotSupported;
  if (act != 0 && act != 1) return cudaErrorInvalidValue;
  auto encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  const int64_t Np = (N + 127) / 128 * 128;
  CUtensorMap mx, mw, my;
  {
    // planes: (64 halves of a 128-byte line, Np/4 lines, Cin/16 blocks, 8 planes);
    // box = 32 lines (128 rows) x 1 block x 8 planes = 32 KB
    cuuint64_t dims[4] = {64, (cuuint64_t)(Np / 4), (cuuint64_t)(Cin / 16), 8};
    cuuint64_t strides[3] = {128, (cuuint64_t)Np * 32, (cuuint64_t)Np * 32 * (Cin / 16)};
    cuuint32_t box[4] = {64, 32, 1, 8};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(Xt), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  {
    cuuint64_t dims[2] = {64, (cuuint64_t)(pair8_tile_bytes(Cin, Cout) / 128)};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {64, P8_WLINES};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(tiles), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (!next_planes) {
    // Y [N][Cout*8]: (64 halves = 8 channels, Cout/8 chunks, N rows); box = 32 rows
    cuuint64_t dims[3] = {64, (cuuint64_t)(Cout / 8), (cuuint64_t)N};
    cuuint64_t strides[2] = {128, (cuuint64_t)Cout * 8 * 2};
    cuuint32_t box[3] = {64, 1, 32};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, Y, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  } else {
    // the next layer's tiled planes: (64 halves of a 128-byte line, Np/4 lines,
    // Cout/16 blocks, 8 planes); box = 8 lines (32 rows) x 1 block x 8 planes
    cuuint64_t dims[4] = {64, (cuuint64_t)(Np / 4), (cuuint64_t)(Cout / 16), 8};
    cuuint64_t strides[3] = {128, (cuuint64_t)Np * 32, (cuuint64_t)Np * 32 * (Cout / 16)};
    cuuint32_t box[4] = {64, 8, 1, 8};
    cuuint32_t estr[4] = {1, 1, 1, 1};
    if (encode(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, Y, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static bool attrs = false;
  if (!attrs) {
    cudaError_t e = set_p8_attr<0, 0, 0>();
    if (e == cudaSuccess) e = set_p8_attr<0, 1, 0>();
    if (e == cudaSuccess) e = set_p8_attr<1, 0, 0>();
    if (e == cudaSuccess) e = set_p8_attr<1, 1, 0>();
    if (e == cudaSuccess) e = set_p8_attr<0, 0, 1>();
    if (e == cudaSuccess) e = set_p8_attr<0, 1, 1>();
    if (e == cudaSuccess) e = set_p8_attr<1, 0, 1>();
    if (e == cudaSuccess) e = set_p8_attr<1, 1, 1>();
    if (e != cudaSuccess) return e;
    attrs = true;
  }
  P8Sched sc = {};
  sc.N = N;
  const int n_prow = (int)((N + 255) / 256);
  sc.n_dt = (Cout + P8_BD - 1) / P8_BD;
  sc.n_ks = Cin / P8_KC;
  sc.Cout = Cout;
  if ((int64_t)n_prow * sc.n_dt > 0x7fffffffLL) return cudaErrorInvalidValue;
  sc.total = n_prow * sc.n_dt;
  sc.bias = static_cast<const __half*>(bias);
  sc.Np = Np;
  using K = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, P8Sched, int*);
  const K table[2][2][2] = {
      {{eq_pair8_tc_kernel<0, 0, 0>, eq_pair8_tc_kernel<0, 0, 1>},
       {eq_pair8_tc_kernel<0, 1, 0>, eq_pair8_tc_kernel<0, 1, 1>}},
      {{eq_pair8_tc_kernel<1, 0, 0>, eq_pair8_tc_kernel<1, 0, 1>},
       {eq_pair8_tc_kernel<1, 1, 0>, eq_pair8_tc_kernel<1, 1, 1>}}};
  const K kernel = table[group ? 1 : 0][act ? 1 : 0][next_planes ? 1 : 0];
  int npairs = p8_capacity((const void*)kernel, num_sms);
  if (npairs > sc.total) npairs = sc.total;
  return launch_dependent(kernel, dim3(2 * npairs), dim3(P8_THREADS), P8_SMEM, st, mx, mw, my, sc,
                          status);
}

}  // namespace eql
