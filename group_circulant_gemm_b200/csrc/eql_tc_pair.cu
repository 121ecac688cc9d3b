// Pair-CTA tcgen05 forward of the p4 (T = 4) EQ-Linear layer from spectral
// input planes, FP16 in, FP32 accumulate, FP16 out, for sm_100a.
//
// What it computes (Flash EQ-Linear summary, "Algorithmic approach" items 1-3
// and "Specialisation for p4"): the input arrives as its group DFT, four FP16
// planes X0, X2, Xr, Xi (each times 1/4) in the tiled layout below; per
// frequency the real products against the prepared weight planes (A0, A2, Br,
// Bi, and -Bi):
//   Y0 = X0 A0^T,  Y2 = X2 A2^T,
//   [Y1r | Y1i] = Xr [Br | Bi]^T + Xi [-Bi | Br]^T
// (the complex product (Xr + i Xi)(Br - i Bi) as two real products of twice the
// width), then the inverse DFT plus bias (and activation) in the epilogue,
// written as Y [N][Cout*4] or as the next layer's planes.
//
// Why a CTA pair: with one CTA per tile, an M = 128 MMA reads both operands
// from its own SM's shared memory at about the rate that memory delivers, so
// every byte the TMA writes or another warp moves slows the tensor core.  With
// tcgen05.mma.cta_group::2 two SMs compute a 256-row tile: each holds its own
// 128 rows of the A operand (the input planes) and half of the B rows (the
// weights), so each SM reads half the weight bytes and its TMA fetches half of
// the weight tile from L2.  The inputs are already transformed, so nothing but
// the TMA and the tensor core touches the operand ring.
//
// Tiled planes (the layout of eqlinear_group_dft's output): the planes are
// stored in HBM exactly as the MMA reads them from shared memory, so every
// load is whole 128-byte lines (a TMA fetches a box line by line; 32-byte rows
// cost as many requests as 128-byte ones).  Rows are padded to Np, a multiple
// of 128; element (plane p, row n, channel c) sits at byte
//   ((p * (C / 16) + c / 16) * Np + n) * 32 + ((h ^ ((n / 4) % 2)) * 16) + (c % 8) * 2,
// h = (c % 16) / 8: per 16-channel block, 32-byte rows with the 32-byte
// swizzle of the MMA's K-major operand layout.
//
// Design (cluster of 2 CTAs, one per SM, persistent over (256-row, 128
// out-channel) tiles; K step = 16 input channels):
//   warp 0    producer (both CTAs): per K step one 4-D TMA box of the tiled
//             planes (16 channels x 128 own rows x 4 planes = 4 x 4 KB) and one
//             box of this CTA's half of the weight tile (12 KB), both completing
//             on the leader CTA's stage barrier (cta_group::2 loads).
//   warp 1    TMEM allocation (both); lane 0 of the leader issues the four pair
//             MMAs of each K step and commits each stage's release to both CTAs.
//   warps 4-11 epilogue (both CTAs, own 128 rows): read the tile's four FP32
//             accumulators from TMEM, inverse DFT + bias, pack to FP16; the
//             first 16 out-channels go to the staging buffer and the other 48
//             stay in registers, so TMEM is handed back to the MMA issuer before
//             any store drains; then four TMA stores of 32 rows x 16 channels.
// TMEM per CTA: Y0 [0,128) | Y2 [128,256) | Y1r [256,384) | Y1i [384,512).
// Every wait is bounded (about 2 s); on expiry the CTA sets its abort flag and
// the plan's status word, drains what it issued, and both CTAs meet at the
// final cluster barrier, so a stuck pipeline never hangs the GPU.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "eql_kernels.h"
#include "eql_tc_common.cuh"
#include "eql_tc_fwd_parts.cuh"

namespace eql {
namespace {

using namespace tc;
using namespace ftc;

constexpr int PR_BD = 128;                       // out-channels per tile
constexpr int PR_KC = 16;                        // input channels per K step (stage)
constexpr int PR_ROWB = 32;                      // bytes per operand row (16 halves)
constexpr uint32_t PR_XPLANE = BM * PR_ROWB;     // 4 KB: one plane, own 128 rows
constexpr uint32_t PR_XBYTES = 4 * PR_XPLANE;    // 16 KB
constexpr int PR_WROWS = 384;                    // this CTA's weight rows per stage
constexpr uint32_t PR_WBYTES = PR_WROWS * PR_ROWB;  // 12 KB
constexpr int PR_WLINES = PR_WBYTES / 128;       // the weight stage as 128-byte lines
constexpr uint32_t PR_STAGE = PR_XBYTES + PR_WBYTES;  // 28 KB
constexpr int PR_ST = 6;                         // ring depth
// warps: 0 producer, 1 TMEM + MMA, 2-3 idle, 4-11 epilogue (lane quarter =
// warp % 4); 168 registers a thread (three warps per SM sub-partition)
constexpr int PR_THREADS = 384;
constexpr int PR_EPI0 = 4;
constexpr uint32_t PR_OFF_STG = PR_ST * PR_STAGE;
constexpr uint32_t PR_OFF_BIAS = PR_OFF_STG + kEpiWarps * kStgBytes;
constexpr uint32_t PR_OFF_BAR = PR_OFF_BIAS + kEpiWarps * 128;
constexpr uint32_t PR_SMEM = PR_OFF_BAR + 512 + 1024;
static_assert(PR_STAGE % 1024 == 0, "stage slots stay 1024-byte aligned");
static_assert(PR_SMEM <= 232448, "shared memory budget");
// weight regions inside a stage (byte offsets): A0 half, A2 half (64 rows each),
// then 128 rows of [Br | Bi] and 128 rows of [-Bi | Br] (which half: CTA rank)
constexpr uint32_t PR_R0 = 0, PR_R1 = 64 * PR_ROWB, PR_R2 = 128 * PR_ROWB, PR_R3 = 256 * PR_ROWB;

struct PairBars {
  uint64_t full[PR_ST];   // leader: both CTAs' bytes of a stage landed
  uint64_t empty[PR_ST];  // each CTA: the stage's MMAs are done (multicast commit)
  uint64_t acc_full;      // each CTA: the tile's accumulators are final
  uint64_t acc_empty;     // leader: both CTAs' epilogues have read TMEM
  uint64_t drain;         // leader: every MMA it issued is complete
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(PairBars) <= 512, "barrier block");

struct PairInfo {
  int n_dt;       // out-channel tiles
  int num_tiles;  // 256-row tiles x out-channel tiles
  int n_ks;       // K steps = Cin / 16
  int64_t N;
  int Cout;
};

__device__ __forceinline__ uint32_t cta_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\t"
               "barrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}
__device__ __forceinline__ void arrive_remote(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}
// TMA tile loads whose completion is counted on a barrier of either CTA of the
// pair (the leader's); the destination is this CTA's shared memory.
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int x, int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void tma_load_4d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int x, int y, int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
__device__ __forceinline__ void tma_store_4d(const CUtensorMap* map, uint32_t src, int x, int y,
                                             int z, int w) {
  asm volatile(
      "cp.async.bulk.tensor.4d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5}], [%1];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(x), "r"(y), "r"(z), "r"(w)
      : "memory");
}
// Stores of the next layer's tiled planes: 32 rows (row0 a multiple of 32) x 16
// channels x 4 planes, one 4-D box; rows of the padding past N are written too
// (they belong to the buffer), tiles wholly past N are skipped.
struct TiledStore {
  const CUtensorMap* map;
  int64_t row0, N;
  __device__ __forceinline__ void operator()(uint32_t src, int d0) const {
    if (row0 < N) tma_store_4d(map, src, 0, (int)(row0 / 4), d0 / 16, 0);
  }
};
template <int IO>
using PairStoreOf = typename std::conditional<IO == kIoSpectralOut, TiledStore, RowStore<4>>::type;

__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const CUtensorMap* map,
                                                 uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void umma_pair(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive (once the MMAs issued so far complete) on the barrier at `bar`'s offset
// in every CTA of `mask`.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// Two 8-channel slices (16 out-channels) of this lane's row into the warp's
// staging buffer, in the layout of one TMA store box: spatial Y (32 rows x
// 128 B, 128-byte swizzle) or spectral planes ([plane][32 rows][32 B], 32-byte
// swizzle).
template <int IO>
__device__ __forceinline__ void stage_two(uint8_t* stg, int lane, const uint4 (&a)[4],
                                          const uint4 (&b)[4]) {
  if constexpr (IO == kIoSpectralOut) {
    const int sw = (lane >> 2) & 1;
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      *reinterpret_cast<uint4*>(stg + p * 1024 + lane * 32 + ((0 ^ sw) << 4)) = a[p];
      *reinterpret_cast<uint4*>(stg + p * 1024 + lane * 32 + ((1 ^ sw) << 4)) = b[p];
    }
  } else {
    uint8_t* row = stg + lane * 128;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      *reinterpret_cast<uint4*>(row + ((m ^ (lane & 7)) << 4)) = a[m];
      *reinterpret_cast<uint4*>(row + (((4 + m) ^ (lane & 7)) << 4)) = b[m];
    }
  }
}

template <int IO, int ACT>
__device__ __forceinline__ void slice_out(uint32_t lane_addr, int c0, const __half* bs,
                                          uint4 (&o)[4]) {
  if constexpr (IO == kIoSpectralOut)
    epi_half_spec<PR_BD, ACT>(lane_addr, c0, bs, o);
  else
    epi_half<4, PR_BD, ACT>(lane_addr, c0, bs, o);
}

template <int ACT, int IO>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PR_THREADS, 1)
    eq_pair_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                      const __grid_constant__ CUtensorMap map_w,
                      const __grid_constant__ CUtensorMap map_y, const __half* __restrict__ bias,
                      PairInfo pi, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  PairBars* bars = reinterpret_cast<PairBars*>(smem + PR_OFF_BAR);
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cta_rank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PR_ST; ++s) {
      mbar_init(&bars->full[s], 1);   // the leader's producer arrives (with both CTAs' bytes)
      mbar_init(&bars->empty[s], 1);  // one multicast commit
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, 2 * kEpiWarps);  // one arrival per epilogue warp of each CTA
    mbar_init(&bars->drain, 1);
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
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA completion
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ---------------- producer: planes and this CTA's half of the weights ----------------
    if (lane == 0) {
      int issued_phase[PR_ST];
      for (int s = 0; s < PR_ST; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int u = pair; ok && u < pi.num_tiles; u += npairs) {
        const int prow = u / pi.n_dt, dt = u % pi.n_dt;
        const int row = prow * 256 + 128 * (int)rank;
        for (int ks = 0; ks < pi.n_ks; ++ks, ++it) {
          const int s = it % PR_ST;
          const uint32_t ph = (it / PR_ST) & 1;
          if (!(ok = wait_bounded(&bars->empty[s], ph ^ 1, abort_flag, status))) break;
          const uint32_t full_leader = peer_addr(smem_u32(&bars->full[s]), 0);
          if (rank == 0) mbar_expect_tx(&bars->full[s], 2 * PR_STAGE);
          const uint32_t slot = sbase + s * PR_STAGE;
          // planes: lines row/4 .. +32 of channel block ks, all four planes
          tma_load_4d_pair(slot, &map_x, full_leader, 0, row / 4, ks, 0);
          const int wline = ((dt * pi.n_ks + ks) * 2 + (int)rank) * PR_WLINES;
          tma_load_2d_pair(slot + PR_XBYTES, &map_w, full_leader, 0, wline);
          issued_phase[s] = (int)ph;
        }
      }
      if (!ok && rank == 0) {
        // wait (bounded) for the loads this CTA pair put in flight on the leader's barriers
        for (int s = 0; s < PR_ST; ++s)
          if (issued_phase[s] >= 0) drain_wait(&bars->full[s], (uint32_t)issued_phase[s]);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- MMA issuer (leader CTA) ----------------
    if (rank == 0 && lane == 0) {
      const uint32_t id_n1 = idesc_f16(256, PR_BD);
      const uint32_t id_n2 = idesc_f16(256, 2 * PR_BD);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      for (int u = pair; ok && u < pi.num_tiles; u += npairs, ++tcount) {
        if (!(ok = wait_bounded(&bars->acc_empty, (tcount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int ks = 0; ks < pi.n_ks; ++ks, ++it) {
          const int s = it % PR_ST;
          if (!(ok = wait_bounded(&bars->full[s], (it / PR_ST) & 1, abort_flag, status))) break;
          tc_fence_after();
          const uint32_t xa = sbase + s * PR_STAGE, wb = xa + PR_XBYTES;
          const uint32_t acc = ks > 0 ? 1u : 0u;
          umma_pair(tmem + 0, desc_kmajor<32>(xa + 0 * PR_XPLANE), desc_kmajor<32>(wb + PR_R0),
                    id_n1, acc);
          umma_pair(tmem + PR_BD, desc_kmajor<32>(xa + 1 * PR_XPLANE),
                    desc_kmajor<32>(wb + PR_R1), id_n1, acc);
          umma_pair(tmem + 2 * PR_BD, desc_kmajor<32>(xa + 2 * PR_XPLANE),
                    desc_kmajor<32>(wb + PR_R2), id_n2, acc);
          umma_pair(tmem + 2 * PR_BD, desc_kmajor<32>(xa + 3 * PR_XPLANE),
                    desc_kmajor<32>(wb + PR_R3), id_n2, 1u);
          umma_commit_pair(&bars->empty[s], 3);
        }
        if (ok) umma_commit_pair(&bars->acc_full, 3);
      }
      // every MMA this thread issued completes before TMEM is freed
      umma_commit_pair(&bars->drain, 1);
      drain_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= PR_EPI0 && warp < PR_EPI0 + kEpiWarps) {
    // ---------------- epilogue (both CTAs, own rows) ----------------
    const int q = warp & 3;               // TMEM lane quarter = rows 32q..32q+31
    const int ch = (warp - PR_EPI0) >> 2;  // out-channel half of the tile
    uint8_t* stg = smem + PR_OFF_STG + (warp - PR_EPI0) * kStgBytes;
    const uint32_t stg_s = smem_u32(stg);
    __half* bsm = reinterpret_cast<__half*>(smem + PR_OFF_BIAS + (warp - PR_EPI0) * 128);
    const uint32_t acc_empty_leader = peer_addr(smem_u32(&bars->acc_empty), 0);
    const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
    uint32_t tcount = 0;
    for (int u = pair; u < pi.num_tiles; u += npairs, ++tcount) {
      const int prow = u / pi.n_dt, dt = u % pi.n_dt;
      const int64_t row0 = (int64_t)prow * 256 + 128 * rank + 32 * q;
      const int dbase = dt * PR_BD + (PR_BD / 2) * ch;
      if (2 * lane < PR_BD / 2) {
        const int d = dbase + 2 * lane;
        uint32_t v = 0u;
        if (bias && d < pi.Cout) v = *reinterpret_cast<const uint32_t*>(bias + d);  // Cout even
        reinterpret_cast<uint32_t*>(bsm)[lane] = v;
      }
      __syncwarp();
      if (!warp_wait(&bars->acc_full, tcount & 1, abort_flag, status)) break;
      tc_fence_after();
      // read the whole tile share out of TMEM: slices 0-1 into staging, 2-7 held
      uint4 held[3][2][4];
      {
        uint4 a[4], b[4];
        slice_out<IO, ACT>(lane_addr, (PR_BD / 2) * ch, bsm, a);
        slice_out<IO, ACT>(lane_addr, (PR_BD / 2) * ch + 8, bsm + 8, b);
        if (lane == 0) bulk_wait_read_all();  // the previous tile's last store has read stg
        __syncwarp();
        stage_two<IO>(stg, lane, a, b);
      }
#pragma unroll
      for (int sc = 1; sc < 4; ++sc) {
        slice_out<IO, ACT>(lane_addr, (PR_BD / 2) * ch + 16 * sc, bsm + 16 * sc, held[sc - 1][0]);
        slice_out<IO, ACT>(lane_addr, (PR_BD / 2) * ch + 16 * sc + 8, bsm + 16 * sc + 8,
                           held[sc - 1][1]);
      }
      // TMEM is free for the next tile's MMAs once every warp of both CTAs got here
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_remote(acc_empty_leader);
      // stores: 16 out-channels x 32 rows each, while the next tile's MMAs run
      PairStoreOf<IO> store{&map_y, row0, pi.N};
#pragma unroll
      for (int sc = 0; sc < 4; ++sc) {
        const int d0 = dbase + 16 * sc;
        if (sc > 0) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          stage_two<IO>(stg, lane, held[sc - 1][0], held[sc - 1][1]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0 && d0 < pi.Cout) {
          store(stg_s, d0);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its pair may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

// Prepared planes [P][Cout][Cin] (P = 5 at T = 4: A0, A2, Br, Bi, -Bi) -> the
// pair kernel's weight stages: blob (dt, ks, rank) = 384 rows x 16 channels
// (32 bytes, 32-byte swizzle: 16-byte piece ^= (row / 4) % 2), rows 0-63 plane 0
// and 64-127 plane 1 at out-channels dt*128 + 64*rank + r, rows 128-255 plane 2
// (rank 0) or 3 (rank 1), rows 256-383 plane 4 (rank 0) or 2 (rank 1) at
// out-channels dt*128 + r; zero past the matrix.  One thread per 16-byte piece.
__global__ void pair_tile_weights_kernel(const __half* __restrict__ planes, int Cin, int Cout,
                                         int n_ks, int64_t n_pieces, uint4* __restrict__ tiles) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_pieces) return;
  const int piece = (int)(idx & 1);
  const int r = (int)((idx >> 1) % PR_WROWS);
  const int64_t blob = (idx >> 1) / PR_WROWS;
  const int rank = (int)(blob & 1);
  const int64_t dk = blob >> 1;
  const int dt = (int)(dk / n_ks), ks = (int)(dk % n_ks);
  int plane, d;
  if (r < 128) {
    plane = r < 64 ? 0 : 1;
    d = dt * PR_BD + 64 * rank + (r & 63);
  } else if (r < 256) {
    plane = rank == 0 ? 2 : 3;
    d = dt * PR_BD + (r - 128);
  } else {
    plane = rank == 0 ? 4 : 2;
    d = dt * PR_BD + (r - 256);
  }
  const int c0 = ks * PR_KC + piece * 8;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (d < Cout && c0 < Cin)  // Cin % 16 == 0: the 8 channels are all in range
    v = *reinterpret_cast<const uint4*>(planes + ((int64_t)plane * Cout + d) * Cin + c0);
  const int64_t dst = blob * PR_WBYTES + r * PR_ROWB + ((piece ^ ((r >> 2) & 1)) << 4);
  tiles[dst >> 4] = v;
}

// Group DFT of p4 rows into tiled planes (layout above): X [N][C*4] -> the
// four planes, each value times 1/4 (FP32 arithmetic, one rounding), rows
// N..Np-1 zero.  A thread takes one row and 8 channels (64 bytes of X, four
// 16-byte plane pieces); a warp covers 16 rows x one 16-channel block, so its
// reads are whole 128-byte row segments and its writes 512 contiguous bytes
// per plane.
__global__ void group_dft_tiled_kernel(const uint4* __restrict__ X, int64_t N, int64_t Np, int C,
                                       uint8_t* __restrict__ out) {
  const int KB = C / 16;
  const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t groups = Np / 16 * KB;  // (16-row group, channel block) pairs
  const int64_t g = t >> 5;
  if (g >= groups) return;
  const int lane = (int)(t & 31);
  const int kb = (int)(g % KB);
  const int64_t n = (g / KB) * 16 + (lane >> 1);
  const int h = lane & 1;
  uint32_t o[4][4];
  if (n < N) {
    const uint4* src = X + (n * C * 4 + (int64_t)kb * 64 + h * 32) / 8;
#pragma unroll
    for (int q = 0; q < 4; ++q) {  // piece q: channels 2q, 2q+1 of the 8
      const uint4 v = src[q];
      const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
      float f0[2], fh[2], fr[2], fi[2];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float2 lo = unpack_h2(w4[2 * e]), hi = unpack_h2(w4[2 * e + 1]);
        const float x0 = lo.x, x1 = lo.y, x2 = hi.x, x3 = hi.y;
        const float a = x0 + x2, b = x1 + x3;
        f0[e] = (a + b) * 0.25f;
        fh[e] = (a - b) * 0.25f;
        fr[e] = (x0 - x2) * 0.25f;
        fi[e] = (x3 - x1) * 0.25f;
      }
      o[0][q] = pack_h2(f0[0], f0[1]);
      o[1][q] = pack_h2(fh[0], fh[1]);
      o[2][q] = pack_h2(fr[0], fr[1]);
      o[3][q] = pack_h2(fi[0], fi[1]);
    }
  } else {
#pragma unroll
    for (int p = 0; p < 4; ++p)
#pragma unroll
      for (int q = 0; q < 4; ++q) o[p][q] = 0u;
  }
  const int64_t inrow = n * 32 + ((h ^ (int)((n >> 2) & 1)) << 4);
#pragma unroll
  for (int p = 0; p < 4; ++p)
    *reinterpret_cast<uint4*>(out + ((int64_t)p * KB + kb) * Np * 32 + inrow) =
        make_uint4(o[p][0], o[p][1], o[p][2], o[p][3]);
}

// 4-D view of tiled planes: (64 halves of a 128-byte line, Np/4 lines of a
// channel block, C/16 blocks, 4 planes); box = `lines` lines x all 4 planes.
bool encode_tiled_map(CUtensorMap* m, const void* base, int channels, int64_t Np, uint32_t lines) {
  auto encode = encode_fn();
  cuuint64_t dims[4] = {64, (cuuint64_t)(Np / 4), (cuuint64_t)(channels / 16), 4};
  cuuint64_t strides[3] = {128, (cuuint64_t)Np * 32, (cuuint64_t)Np * 32 * (channels / 16)};
  cuuint32_t box[4] = {64, lines, 1, 4};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int ACT, int IO>
cudaError_t set_pair_attr() {
  return cudaFuncSetAttribute(eq_pair_tc_kernel<ACT, IO>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, PR_SMEM);
}

}  // namespace

int64_t tiled_rows(int64_t N) { return (N + 127) / 128 * 128; }

size_t tiled_planes_bytes(int64_t N, int channels) {
  return (size_t)4 * (size_t)tiled_rows(N) * (size_t)channels * 2;
}

cudaError_t launch_group_dft_tiled(const void* X, int64_t N, int C, void* out, cudaStream_t st) {
  if (N <= 0) return cudaSuccess;
  if (C % 16 != 0) return cudaErrorInvalidValue;
  const int64_t Np = tiled_rows(N);
  const int64_t threads = Np / 16 * (C / 16) * 32;
  group_dft_tiled_kernel<<<(unsigned)((threads + 255) / 256), 256, 0, st>>>(
      static_cast<const uint4*>(X), N, Np, C, static_cast<uint8_t*>(out));
  return cudaGetLastError();
}

bool pair_tc_supported(int64_t N, int Cin, int Cout) {
  return N >= 1 && N <= 0x7fffff00LL && Cin % 16 == 0 && Cout % 16 == 0 && Cin >= 16 &&
         Cout >= 16;
}

size_t pair_tile_bytes(int Cin, int Cout) {
  const size_t n_dt = (size_t)(Cout + PR_BD - 1) / PR_BD, n_ks = (size_t)(Cin + PR_KC - 1) / PR_KC;
  return n_dt * n_ks * 2 * PR_WBYTES;
}

cudaError_t launch_pair_tile_weights(const void* planes, int Cin, int Cout, void* tiles,
                                     cudaStream_t st) {
  const int n_ks = (Cin + PR_KC - 1) / PR_KC;
  const int64_t n_pieces = (int64_t)pair_tile_bytes(Cin, Cout) / 16;
  pair_tile_weights_kernel<<<(unsigned)((n_pieces + 255) / 256), 256, 0, st>>>(
      static_cast<const __half*>(planes), Cin, Cout, n_ks, n_pieces, static_cast<uint4*>(tiles));
  return cudaGetLastError();
}

cudaError_t launch_pair_tc(const void* Xhat, int64_t N, int Cin, int Cout, const void* tiles,
                           const void* bias, void* Y, int* status, int num_sms, int act,
                           int spectral_out, cudaStream_t st) {
  if (!pair_tc_supported(N, Cin, Cout) || !tiles) return cudaErrorNotSupported;
  if (act != 0 && act != 1) return cudaErrorInvalidValue;
  auto encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  CUtensorMap mx, mw, my;
  const int64_t Np = tiled_rows(N);
  // input planes (tiled): box = 32 lines (128 rows) x 4 planes, copied verbatim
  if (!encode_tiled_map(&mx, Xhat, Cin, Np, 32)) return cudaErrorInvalidValue;
  {
    // weight stages as 128-byte lines, copied verbatim (already swizzled)
    const uint64_t lines = pair_tile_bytes(Cin, Cout) / 128;
    cuuint64_t dims[2] = {64, (cuuint64_t)lines};
    cuuint64_t strides[1] = {128};
    cuuint32_t box[2] = {64, PR_WLINES};
    cuuint32_t estr[2] = {1, 1};
    if (encode(&mw, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(tiles), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  if (spectral_out) {
    // next layer's tiled planes: store box = 8 lines (32 rows) x 4 planes
    if (!encode_tiled_map(&my, Y, Cout, Np, 8)) return cudaErrorInvalidValue;
  } else {
    // Y row = Cout*4/64 chunks of 128 B; store box = 1 chunk x 32 rows
    cuuint64_t ydims[3] = {64, (cuuint64_t)Cout * 4 / 64, (cuuint64_t)N};
    cuuint64_t ystrides[2] = {128, (cuuint64_t)Cout * 4 * 2};
    cuuint32_t ybox[3] = {64, 1, 32};
    cuuint32_t estr[3] = {1, 1, 1};
    if (encode(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, Y, ydims, ystrides, ybox, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  PairInfo pi;
  pi.n_dt = (Cout + PR_BD - 1) / PR_BD;
  const int64_t n_prow = (N + 255) / 256;
  if (n_prow * pi.n_dt > 0x7fffffffLL) return cudaErrorInvalidValue;
  pi.num_tiles = (int)(n_prow * pi.n_dt);
  pi.n_ks = Cin / PR_KC;
  pi.N = N;
  pi.Cout = Cout;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = set_pair_attr<0, kIoSpatial>();
    if (e == cudaSuccess) e = set_pair_attr<1, kIoSpatial>();
    if (e == cudaSuccess) e = set_pair_attr<0, kIoSpectralOut>();
    if (e == cudaSuccess) e = set_pair_attr<1, kIoSpectralOut>();
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  auto kernel = act ? (spectral_out ? eq_pair_tc_kernel<1, kIoSpectralOut>
                                    : eq_pair_tc_kernel<1, kIoSpatial>)
                    : (spectral_out ? eq_pair_tc_kernel<0, kIoSpectralOut>
                                    : eq_pair_tc_kernel<0, kIoSpatial>);
  // as many pairs as can be resident at once (a cluster must fit inside one GPC,
  // so this can be below num_sms / 2); the tiles are spread over them statically
  static int max_pairs = 0;
  if (max_pairs == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (unsigned)(num_sms / 2));
    cfg.blockDim = dim3(PR_THREADS);
    cfg.dynamicSmemBytes = PR_SMEM;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = num_sms / 2;
    }
    max_pairs = n < num_sms / 2 ? n : num_sms / 2;
  }
  int npairs = max_pairs;
  if (npairs > pi.num_tiles) npairs = pi.num_tiles;
  kernel<<<2 * npairs, PR_THREADS, PR_SMEM, st>>>(mx, mw, my, static_cast<const __half*>(bias),
                                                  pi, status);
  return cudaGetLastError();
}

}  // namespace eql
