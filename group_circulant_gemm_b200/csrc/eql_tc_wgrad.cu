// tcgen05/TMEM tensor-core weight gradient of the cyclic-group EQ-Linear layer
// for T = 4 (the p4 rotation group): FP16 X and dY in, FP32 partial spectra out.
//
// What it computes (Flash EQ-Linear summary, "Algorithmic approach": the
// backward pass is the same per-frequency product, transposed).  With G the
// DFT of dY and Xh the DFT of X over the group axis (G0 = g0+g1+g2+g3,
// G2 = g0-g1+g2-g3, Gr = g0-g2, Gi = g3-g1, likewise for X):
//   Q0 = G0^T Xh0,  Q2 = G2^T Xh2,
//   Qr = Gr^T Xr + Gi^T Xi,  Qi = Gr^T Xi - Gi^T Xr        (D x C each, K = rows)
// summed over a range of rows and stored as FP32 partial planes; dbias partials
// are the FP32 column sums of G0.  A finalize kernel adds a tile's partials in a
// fixed order, applies the inverse group DFT and casts, so the result is
// deterministic.  The FP16 operand planes hold G/4 and Xh/4 (exact), like every
// stored plane of the library, so no legal FP16 input overflows them; the
// partials are therefore Q/16 and the finalize multiplies by 16.
//
// Work split (stream-K over rows): the (tile, 32-row stage) space, tile = 128
// out-channels x 128 in-channels, is cut into equal contiguous ranges, one per
// CTA, so every SM does the same number of stages.  The space is ordered row
// block by row block (block = as many stages as a range, the last block
// shorter), then tile, then stage: the CTAs that run at the same time then
// read the same rows, so each row of X (read once per out-channel tile) and of
// dY (once per in-channel tile) comes from DRAM about once and from L2 after.
// A range can end one (block, tile) pair and start the next; each piece (a
// "segment") accumulates in TMEM and writes its own partial slot
// part[pair][j][4][128 c][128 d] (j = which of the pair's ranges; out-channel
// fastest, so each warp store writes 128 contiguous bytes).
//
// Design (one CTA per SM; stage = 32 rows):
//   warp 0      TMA producer: per stage one 3-D box of dY (32 rows x 1 KB: the
//               128 out-channels x 4 group elements of the tile) and one of X.
//   warp 1      TMEM allocator; lane 0 issues the MMAs: M = out-channel, N =
//               in-channel, K = row.  Per K step (16 rows): N = 128 for Q0 and
//               Q2, N = 256 for Gr [Xr|Xi], N = 128 for Gi Xi and (negated A)
//               Gi Xr.
//   warps 4-7   epilogue: tcgen05.ld of the four accumulators (one out-channel
//               per lane), FP32 stores of the partial planes.
//   warps 8-23  transform, two groups of 8 warps working on the same stage in
//               parallel (8-15: the dY tile, 16-23: the X tile): each thread takes
//               8 rows x one channel pair, forms the group DFT in FP32, rounds once
//               to FP16 and writes it transposed (rows become the K dimension) as
//               K-major 64-byte swizzled operand planes over the raw tile it came
//               from.
// TMEM (512 columns): Q0 at [0,128), Q2 at [128,256), Qr at [256,384), Qi at
// [384,512).  Every mbarrier wait is bounded (about 2 s); on expiry the CTA sets
// the plan's status word, drains what it issued and returns.
//
// Planes variant (PL): the group DFTs of X and dY arrive precomputed as FP16
// planes [4][N][C] and [4][N][D] (written by the forward and dX kernels while
// they transform the same tensors), so no transform runs here.  A ring slot is
// one 32-row stage: one 4-D TMA box per operand, (64 channels, 32 rows, 2 blocks
// of 64 channels, 4 planes), 128-byte swizzled, landing as [plane][block][32
// rows][128 B]: the rows are the MMA's K dimension and the channels are
// contiguous, i.e. MN-major operands (64-channel blocks 4 KB apart, 8-row groups
// 1 KB apart, so the N = 256 [Xr | Xi] operand spans planes 2 and 3 at a uniform
// stride).  Warps 8-11 sum plane 0 of dY's spectrum for dbias; warps 4-7 and
// 12-15 drain planes 0-1 and 2-3 of the accumulators.  Needs C and D
// multiples of 64.
//
// A convolution's taps (planes variant, launch_wgrad_tc_conv): the spectra of X
// and dY on the convolution's padded pixel grid, the taps as further in-channel
// tiles of the same stream-K problem.  Tap t = i * kw + j loads X's rows
// i * wp + j further on than dY's (the TMA box reads zeros past the end), and
// the finalize writes tap t's block of dW (grid.z = t).
//
// Tiled variant (PL, TL): the same spectra in the tiled layout of the SM-pair
// kernels ([plane][channel / 16][Np rows][16 channels], 32-byte rows stored with
// the 32-byte swizzle, written by the group-DFT pass).  One 4-D box per operand
// (8 lines of 4 rows, 8 blocks of 16 channels, 4 planes) lands as [plane][block]
// [32 rows][32 B], which is already the MN-major 32-byte-swizzled operand image:
// 16-channel blocks 1 KB apart (LBO), 8-row K groups 256 B apart (SBO), so the
// N = 256 [Xr | Xi] operand again spans planes 2 and 3 at a uniform stride.
// Channel counts need only be multiples of 16 (the box reads zeros past C).
//
// SM-pair variant (wgrad_pair_kernel, tiled planes only): a cluster of two CTAs
// takes (256 out-channel, 128 in-channel) tiles with tcgen05 cta_group::2 MMAs,
// M = 256 out-channels (each CTA its own 128 of dY's planes) and N = 128
// in-channels (each CTA holds 64 of X's): per 32-row stage a CTA loads 48 KB
// instead of 64 KB for the same MMA work, which is what bounds this kernel (the
// SMs' L2 ports).  Each CTA writes the partial slot of its own 128 x 128 block;
// the finalize is shared.  Six N = 128 products per K step on two issuing
// threads of the leader (the [Xr | Xi] operand of the one-CTA kernel would put
// Xr and Xi in different CTAs).  The dbias warps of both CTAs read dY's plane 0
// from their own shared memory once the stage's MMAs have completed (a commit
// multicast to both CTAs) and release the slot with the MMAs.

#include <algorithm>

#include "eql_kernels.h"
#include "eql_tc_common.cuh"
#include "eql_tc_pair_common.cuh"

namespace eql {
namespace {

using namespace tc;

constexpr int WG_BD = 128;                   // out-channels per unit (MMA M)
constexpr int WG_BC = 128;                   // in-channels per unit (MMA N per plane)
constexpr int WG_BR = 32;                    // rows per stage (two MMA K steps)
constexpr int WG_ST = 3;                     // ring depth
constexpr uint32_t WG_TILE = WG_BR * 1024;   // raw dY (or X) tile: 32 rows x 1 KB
constexpr uint32_t WG_STAGE = 2 * WG_TILE;   // dY tile, then X tile
constexpr uint32_t WG_ROWB = WG_BR * 2;      // operand row: 32 rows of K, FP16
constexpr uint32_t WG_PLANE = 128 * WG_ROWB; // one operand plane (128 channels)
constexpr uint32_t WG_OFF_BAR = WG_ST * WG_STAGE;
constexpr uint32_t WG_SMEM = WG_OFF_BAR + 512 + 1024;
constexpr int WG_THREADS = 768;
// Planes variant: no transform warps; warps 8..11 sum dbias, warps 4..7 and
// 12..15 drain the accumulators.  Its ring has the same 192 KB; PL_SUB = 2
// would split each stage into two 16-row slots (6 deep), which measured slower.
constexpr int WG_THREADS_PL = 512;
constexpr int WG_BIASW = 4;
constexpr int PL_SUB = 1;                         // slots per 32-row stage
constexpr int PL_ST = 3 * PL_SUB;                 // ring depth
constexpr int PL_ROWS = WG_BR / PL_SUB;           // rows per slot
constexpr uint32_t PL_BLOCK = PL_ROWS * 128;      // 64 channels x PL_ROWS rows (the LBO)
constexpr uint32_t PL_PLANE = 2 * PL_BLOCK;       // 128 channels
constexpr uint32_t PL_TILE = 4 * PL_PLANE;        // one operand's 4 planes
constexpr uint32_t PL_SLOT = 2 * PL_TILE;         // dY spectrum, then X spectrum
constexpr int WG_RING_MAX = PL_ST;
constexpr int WG_EPI0 = 4, WG_EPIW = 4;      // warps 4..7: one per TMEM lane quarter
constexpr int WG_XF0 = 8, WG_XFW = 8;        // warps 8..15 (dY tile), 16..23 (X tile)
static_assert(4 * WG_PLANE == WG_TILE, "planes replace the raw tile in place");
static_assert(PL_ST * PL_SLOT == WG_ST * WG_STAGE, "both rings fill the same bytes");
static_assert(WG_SMEM <= 232448, "shared memory budget");

// MN-major operand of a planes slot: 64-channel blocks `lbo` bytes apart, 8-row
// K groups 1 KB apart (SBO), 128-byte swizzle (layout type 2), descriptor v1.
__device__ __forceinline__ uint64_t desc_mn128(uint32_t saddr, uint32_t lbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(1024u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)2u << 61);
}
// MN-major operand of a tiled slot: 16-channel blocks 1 KB apart (LBO), 8-row K
// groups 256 B apart (SBO), 32-byte swizzle (layout type 6), descriptor v1.
__device__ __forceinline__ uint64_t desc_mn32(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(1024u >> 4) << 16) |
         ((uint64_t)(256u >> 4) << 32) | ((uint64_t)1u << 46) | ((uint64_t)6u << 61);
}
// kind::f16 instruction descriptor with both operands MN-major (bits 15, 16).
__host__ __device__ constexpr uint32_t idesc_f16_mn(int M, int N, bool negate_a = false) {
  return idesc_f16(M, N, negate_a) | (1u << 15) | (1u << 16);
}

struct WgBars {
  uint64_t full[WG_RING_MAX], read_g[WG_RING_MAX], read_x[WG_RING_MAX], ready[WG_RING_MAX],
      empty[WG_RING_MAX];
  uint64_t acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(WgBars) <= 512, "barrier block");

struct WgInfo {
  int n_dt, n_ct;      // out-channel and in-channel tiles
  // (convolution, planes variant) the in-channel tiles are taps x nct_tap: tile
  // ct is channel block ct % nct_tap of tap ct / nct_tap, whose X rows are read
  // (tap / tap_kw) * tap_wp + tap % tap_kw rows further on; one tap otherwise
  int nct_tap, tap_kw, tap_wp;
  int spt;             // 32-row stages per tile, ceil(N / 32)
  int bst;             // stages per row block (the last block: spt - (nb - 1) * bst)
  int nb;              // row blocks
  int per_unit;        // stages per CTA range
  int maxj;            // partial slots per (block, tile) pair
  int64_t total;       // tiles * spt
};

__host__ __device__ inline int ct_block(int ct, const WgInfo& wi) { return ct % wi.nct_tap; }
__host__ __device__ inline int ct_row_offset(int ct, const WgInfo& wi) {
  const int tap = ct / wi.nct_tap;
  return (tap / wi.tap_kw) * wi.tap_wp + tap % wi.tap_kw;
}

// One segment of a CTA's range: stages [r0 / 32, r0 / 32 + stages) of one tile.
struct Unit {
  int dt, ct, tile, slot;  // slot = pair * maxj + (range index within the pair)
  int64_t r0;
  int stages;
};

__host__ __device__ inline int block_len(int b, const WgInfo& wi) {
  return b == wi.nb - 1 ? wi.spt - b * wi.bst : wi.bst;
}
// Global index of the first stage of pair (block b, tile t).
__host__ __device__ inline int64_t pair_start(int b, int t, const WgInfo& wi) {
  return (int64_t)b * (wi.n_dt * wi.n_ct) * wi.bst + (int64_t)t * block_len(b, wi);
}
// The CTA ranges that touch pair (b, t): first .. last.  The layout keeps the
// stage count below 2^31, so 32-bit unsigned division suffices (the finalize
// evaluates these per output element).
__host__ __device__ inline int first_range_of_pair(int b, int t, const WgInfo& wi) {
  return (int)((uint32_t)pair_start(b, t, wi) / (uint32_t)wi.per_unit);
}
__host__ __device__ inline int last_range_of_pair(int b, int t, const WgInfo& wi) {
  return (int)((uint32_t)(pair_start(b, t, wi) + block_len(b, wi) - 1) / (uint32_t)wi.per_unit);
}

struct SegIter {
  int64_t g, g1;
  int u;
  __device__ SegIter(const WgInfo& wi, int u_) : u(u_) {
    g = (int64_t)u * wi.per_unit;
    g1 = g + wi.per_unit < wi.total ? g + wi.per_unit : wi.total;
  }
  __device__ bool next(const WgInfo& wi, Unit& x) {
    if (g >= g1) return false;
    const int tiles = wi.n_dt * wi.n_ct;
    const int64_t per_block = (int64_t)tiles * wi.bst;
    const int b = (int)(g / per_block < wi.nb - 1 ? g / per_block : wi.nb - 1);
    const int64_t off = g - (int64_t)b * per_block;
    const int len = block_len(b, wi);
    x.tile = (int)(off / len);
    const int s0 = (int)(off % len);
    const int64_t room = len - s0;
    x.stages = (int)(room < g1 - g ? room : g1 - g);
    x.dt = x.tile / wi.n_ct;
    x.ct = x.tile % wi.n_ct;
    x.slot = (b * tiles + x.tile) * wi.maxj + (u - first_range_of_pair(b, x.tile, wi));
    x.r0 = ((int64_t)b * wi.bst + s0) * WG_BR;
    g += x.stages;
    return true;
  }
};

// One transform item: rows 8q..8q+7 of the raw tile, channel pair pd = 8w + j.
// The raw tile is [row][128-byte chunk][128 B] with 128-byte swizzle (16-byte
// piece j of chunk c sits at j ^ c); chunk w holds channel pairs 8w..8w+7.
// Output: plane p, operand row (channel) ch, K piece q of the 64-byte row,
// swizzled as piece ^ ((ch / 2) % 4).  Phases of 8 lanes (fixed q) read 8
// distinct pieces and write 8 distinct bank groups (half the lanes write the
// odd channel of their pair first).
template <bool kBias>
__device__ __forceinline__ void wg_transform(uint8_t* tile, int w, int j, int q, uint64_t* read_bar,
                                             uint32_t parity, float (&bsum)[2], bool& ok,
                                             int* abort_flag, int* status) {
  uint4 v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    v[i] = *reinterpret_cast<const uint4*>(tile + (8 * q + i) * 1024 + (w << 7) + ((j ^ w) << 4));
  uint32_t o[4][2][4];  // [plane][channel of the pair][row pair]
#pragma unroll
  for (int m = 0; m < 4; ++m) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float p0[2], p2[2], pr[2], pi[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 a = v[2 * m + h];
        const float2 lo = unpack_h2(e ? a.z : a.x), hi = unpack_h2(e ? a.w : a.y);
        const float g0 = lo.x, g1 = lo.y, g2 = hi.x, g3 = hi.y;
        const float s02 = g0 + g2, s13 = g1 + g3;
        p0[h] = s02 + s13;
        p2[h] = s02 - s13;
        pr[h] = g0 - g2;
        pi[h] = g3 - g1;
        if (kBias) bsum[e] += p0[h];  // dbias: the unscaled FP32 G0
        // stored planes carry 1/4 (exact)
        p0[h] *= 0.25f;
        p2[h] *= 0.25f;
        pr[h] *= 0.25f;
        pi[h] *= 0.25f;
      }
      o[0][e][m] = pack_h2(p0[0], p0[1]);
      o[1][e][m] = pack_h2(p2[0], p2[1]);
      o[2][e][m] = pack_h2(pr[0], pr[1]);
      o[3][e][m] = pack_h2(pi[0], pi[1]);
    }
  }
  // every raw piece of the tile is in registers before any plane overwrites it
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(read_bar);
  if (!(ok = warp_wait(read_bar, parity, abort_flag, status))) return;
  const int pd = 8 * w + j;
  const int first = (j >> 2) & 1;
#pragma unroll
  for (int ord = 0; ord < 2; ++ord) {
    const int e = ord ^ first;
    const int ch = 2 * pd + e;
    const uint32_t off = ch * WG_ROWB + ((q ^ ((ch >> 1) & 3)) << 4);
#pragma unroll
    for (int p = 0; p < 4; ++p) {
      // select o[p][e] without dynamic register indexing
      const uint4 val = e ? make_uint4(o[p][1][0], o[p][1][1], o[p][1][2], o[p][1][3])
                          : make_uint4(o[p][0][0], o[p][0][1], o[p][0][2], o[p][0][3]);
      *reinterpret_cast<uint4*>(tile + p * WG_PLANE + off) = val;
    }
  }
}

template <bool PL, bool TL = false>
__global__ void __launch_bounds__(PL ? WG_THREADS_PL : WG_THREADS, 1)
    wgrad_tc_kernel(const __grid_constant__ CUtensorMap map_g,
                    const __grid_constant__ CUtensorMap map_x, int64_t N, int C, int D,
                    WgInfo wi, float* __restrict__ part, float* __restrict__ bpart, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  WgBars* bars = reinterpret_cast<WgBars*>(smem + WG_OFF_BAR);
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  constexpr int RING = PL ? PL_ST : WG_ST;           // ring slots
  constexpr int SUB = PL ? PL_SUB : 1;               // slots per 32-row stage
  constexpr uint32_t SLOT = PL ? PL_SLOT : WG_STAGE;  // bytes per slot
  constexpr uint32_t TILEB = PL ? PL_TILE : WG_TILE;  // one operand's bytes in a slot
  constexpr int EPIW = PL ? 2 * WG_EPIW : WG_EPIW;   // accumulator-draining warps

  if (threadIdx.x == 0) {
    for (int s = 0; s < RING; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->read_g[s], WG_XFW);
      mbar_init(&bars->read_x[s], WG_XFW);
      mbar_init(&bars->ready[s], 2 * WG_XFW);
      // PL: the MMA commit and the dbias warps both release the slot
      mbar_init(&bars->empty[s], PL ? 1 + WG_BIASW : 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, EPIW * 32);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int issued_phase[RING];
      for (int s = 0; s < RING; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      SegIter si(wi, blockIdx.x);
      Unit un;
      while (ok && si.next(wi, un)) {
        for (int s = 0; ok && s < un.stages * SUB; ++s, ++it) {
          const int slot = it % RING;
          const uint32_t ph = (it / RING) & 1;
          if (!(ok = wait_bounded(&bars->empty[slot], ph ^ 1, abort_flag, status))) break;
          mbar_expect_tx(&bars->full[slot], SLOT);
          const int row = (int)(un.r0 + (int64_t)(WG_BR / SUB) * s);
          const uint32_t dst = sbase + slot * SLOT;
          if constexpr (PL && TL) {
            // 4-D tiled views (128-byte line = 4 rows, line, 16-channel block, plane)
            tma_load_4d(dst, &map_g, &bars->full[slot], 0, row / 4, 8 * un.dt, 0);
            tma_load_4d(dst + TILEB, &map_x, &bars->full[slot], 0, row / 4, 8 * un.ct, 0);
          } else if constexpr (PL) {
            // 4-D planes views (64 channels, row, 64-channel block, plane)
            tma_load_4d(dst, &map_g, &bars->full[slot], 0, row, 2 * un.dt, 0);
            tma_load_4d(dst + TILEB, &map_x, &bars->full[slot], 0, row + ct_row_offset(un.ct, wi),
                        2 * ct_block(un.ct, wi), 0);
          } else {
            // 3-D views (64 halves, 128-byte chunk of the row, row); a unit's tile is
            // chunks 8*tile .. 8*tile+7 (128 channels x 4 group elements)
            tma_load_3d(dst, &map_g, &bars->full[slot], 0, 8 * un.dt, row);
            tma_load_3d(dst + WG_TILE, &map_x, &bars->full[slot], 0, 8 * un.ct, row);
          }
          issued_phase[slot] = (int)ph;
        }
      }
      if (!ok)
        for (int s = 0; s < RING; ++s)
          if (issued_phase[s] >= 0) drain_wait(&bars->full[s], (uint32_t)issued_phase[s]);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, ucount = 0;
      bool ok = true;
      const uint32_t id_n1 = PL ? idesc_f16_mn(128, WG_BC) : idesc_f16(128, WG_BC);
      const uint32_t id_n1_neg =
          PL ? idesc_f16_mn(128, WG_BC, true) : idesc_f16(128, WG_BC, true);
      const uint32_t id_n2 = PL ? idesc_f16_mn(128, 2 * WG_BC) : idesc_f16(128, 2 * WG_BC);
      SegIter si(wi, blockIdx.x);
      Unit un;
      for (; ok && si.next(wi, un); ++ucount) {
        if (!(ok = wait_bounded(&bars->acc_empty, (ucount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int s = 0; s < un.stages * SUB; ++s, ++it) {
          const int slot = it % RING;
          uint64_t* rbar = PL ? &bars->full[slot] : &bars->ready[slot];
          if (!(ok = wait_bounded(rbar, (it / RING) & 1, abort_flag, status))) break;
          tc_fence_after();
          const uint32_t g = sbase + slot * SLOT;  // G planes (A: M = out-channels)
          const uint32_t x = g + TILEB;            // Xh planes (B: N = in-channels)
#pragma unroll
          for (int kk = 0; kk < WG_BR / 16 / SUB; ++kk) {
            const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
            // transform path: K-major planes, K step = 32 B of a row; planes path:
            // MN-major planes, K step = 16 rows x 128 B (tiled: 16 rows x 32 B)
            auto A = [&](int p) {
              return PL ? (TL ? desc_mn32(g + p * PL_PLANE + 512u * kk)
                              : desc_mn128(g + p * PL_PLANE + 2048u * kk, PL_BLOCK))
                        : desc_kmajor<WG_ROWB>(g + p * WG_PLANE + 32u * kk);
            };
            auto B = [&](int p) {
              return PL ? (TL ? desc_mn32(x + p * PL_PLANE + 512u * kk)
                              : desc_mn128(x + p * PL_PLANE + 2048u * kk, PL_BLOCK))
                        : desc_kmajor<WG_ROWB>(x + p * WG_PLANE + 32u * kk);
            };
            umma(tmem + 0, A(0), B(0), id_n1, acc);              // Q0
            umma(tmem + WG_BC, A(1), B(1), id_n1, acc);          // Q2
            umma(tmem + 2 * WG_BC, A(2), B(2), id_n2, acc);      // [Qr|Qi] += Gr [Xr|Xi]
            umma(tmem + 2 * WG_BC, A(3), B(3), id_n1, 1u);       // Qr += Gi Xi
            umma(tmem + 3 * WG_BC, A(3), B(2), id_n1_neg, 1u);   // Qi -= Gi Xr
          }
          umma_commit(&bars->empty[slot]);
        }
        if (ok) umma_commit(&bars->acc_full);
      }
      umma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if ((warp >= WG_EPI0 && warp < WG_EPI0 + WG_EPIW) ||
             (PL && warp >= WG_XF0 + WG_BIASW && warp < WG_XF0 + WG_BIASW + WG_EPIW)) {
    // ---------------- epilogue: accumulators -> FP32 partial planes ----------------
    // Warp w reads TMEM lane quarter q = w % 4: lane l holds out-channel
    // 32q + l; two 32x32b loads (one wait) give it 32 consecutive in-channels
    // of one plane, and each store writes 32 consecutive out-channels (128 B).
    // Planes variant: warps 4-7 take planes 0-1, warps 12-15 planes 2-3.
    const int q = warp & 3;
    const int p0 = PL ? (warp >= WG_XF0 ? 2 : 0) : 0;
    const int p1 = PL ? p0 + 2 : 4;
    uint32_t ucount = 0;
    SegIter si(wi, blockIdx.x);
    Unit un;
    for (; si.next(wi, un); ++ucount) {
      if (!warp_wait(&bars->acc_full, ucount & 1, abort_flag, status)) break;
      tc_fence_after();
      const int dl = 32 * q + lane;  // out-channel within the tile
      const int d = un.dt * WG_BD + dl;
      const uint32_t lrow = tmem + ((uint32_t)(32 * q) << 16);
      float* slot_base = part + (int64_t)un.slot * (4 * WG_BC * WG_BD);
#pragma unroll 1
      for (int p = p0; p < p1; ++p) {
        float* dst_plane = slot_base + p * (WG_BC * WG_BD);
#pragma unroll 1
        for (int gq = 0; gq < WG_BC / 16; gq += 2) {
          const int c = ct_block(un.ct, wi) * WG_BC + 16 * gq;
          if (c >= C) break;  // warp-uniform; C % 16 == 0: the 16 columns are all in range
          const bool two = c + 16 < C;  // the second group of 16 columns is in range
          uint32_t r[16], r2[16];
          tmem_ld_32x32b<16>(lrow + p * WG_BC + 16 * gq, r);
          if (two) tmem_ld_32x32b<16>(lrow + p * WG_BC + 16 * gq + 16, r2);
          tmem_wait_ld();
          if (d < D) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
              dst_plane[(16 * gq + k) * WG_BD + dl] = __uint_as_float(r[k]);
            if (two) {
#pragma unroll
              for (int k = 0; k < 16; ++k)
                dst_plane[(16 * gq + 16 + k) * WG_BD + dl] = __uint_as_float(r2[k]);
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
    }
  } else if (PL && warp >= WG_XF0 && warp < WG_XF0 + WG_BIASW) {
    // ---------------- planes variant: dbias partials from plane 0 of dY's spectrum ----------------
    // thread = out-channel dl of the tile; plane 0 sits at [block dl / 64][row][128 B],
    // 16-byte piece (dl % 64) / 8 swizzled with row % 8 (tiled: [block dl / 16][row]
    // [32 B], piece (dl % 16) / 8 swizzled with (row / 4) % 2)
    const int dl = (warp - WG_XF0) * 32 + lane;
    uint32_t it = 0;
    bool ok = true;
    SegIter si(wi, blockIdx.x);
    Unit un;
    while (ok && si.next(wi, un)) {
      float b = 0.f;
      for (int s = 0; s < un.stages * SUB; ++s, ++it) {
        const int slot = it % RING;
        if (!(ok = warp_wait(&bars->full[slot], (it / RING) & 1, abort_flag, status))) break;
        if (un.ct == 0) {
          if constexpr (TL) {
            const uint8_t* blk = smem + slot * SLOT + (dl >> 4) * 1024;
            const int piece = (dl & 15) >> 3, within = (dl & 7) * 2;
#pragma unroll 8
            for (int r = 0; r < PL_ROWS; ++r)
              b += __half2float(*reinterpret_cast<const __half*>(
                  blk + r * 32 + ((piece ^ ((r >> 2) & 1)) << 4) + within));
          } else {
            const uint8_t* blk = smem + slot * SLOT + (dl >> 6) * PL_BLOCK;
            const int piece = (dl & 63) >> 3, within = (dl & 7) * 2;
#pragma unroll 8
            for (int r = 0; r < PL_ROWS; ++r)
              b += __half2float(*reinterpret_cast<const __half*>(
                  blk + r * 128 + ((piece ^ (r & 7)) << 4) + within));
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->empty[slot]);
      }
      if (!ok) break;
      // the saved plane 0 holds G0/4: the sum times 4 (exact) is the sum of G0
      if (un.ct == 0) bpart[(int64_t)un.slot * WG_BD + dl] = 4.f * b;
    }
  } else if (!PL && warp >= WG_XF0) {
    // ---------------- transform: group DFT, transposed into the operand planes ----------------
    const int grp = (warp - WG_XF0) >> 3;  // 0: dY tile (and the dbias sums), 1: X tile
    const int w = (warp - WG_XF0) & 7;     // raw chunk = channel pairs 8w..8w+7
    const int j = lane & 7, q = lane >> 3;
    uint32_t it = 0;
    bool ok = true;
    SegIter si(wi, blockIdx.x);
    Unit un;
    while (ok && si.next(wi, un)) {
      float bsum[2] = {0.f, 0.f}, unused[2] = {0.f, 0.f};
      for (int s = 0; s < un.stages; ++s, ++it) {
        const int slot = it % WG_ST;
        const uint32_t ph = (it / WG_ST) & 1;
        if (!(ok = warp_wait(&bars->full[slot], ph, abort_flag, status))) break;
        uint8_t* st = smem + slot * WG_STAGE;
        if (grp == 0)
          wg_transform<true>(st, w, j, q, &bars->read_g[slot], ph, bsum, ok, abort_flag, status);
        else
          wg_transform<false>(st + WG_TILE, w, j, q, &bars->read_x[slot], ph, unused, ok,
                              abort_flag, status);
        if (!ok) break;
        // make the generic-proxy stores visible to the tensor core (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->ready[slot]);
      }
      if (!ok) break;
      // dbias partial of this split: sum over the four row groups (lanes j, j+8, j+16, j+24)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        bsum[e] += __shfl_xor_sync(0xffffffffu, bsum[e], 8);
        bsum[e] += __shfl_xor_sync(0xffffffffu, bsum[e], 16);
      }
      if (grp == 0 && un.ct == 0 && q == 0) {
        const int dl = 2 * (8 * w + j);
        bpart[(int64_t)un.slot * WG_BD + dl] = bsum[0];
        bpart[(int64_t)un.slot * WG_BD + dl + 1] = bsum[1];
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

__device__ __forceinline__ void store_dw4(__half* p, const float* w) {
  // one 8-byte store (p is 8-byte aligned: dW is 16-byte aligned, entries are 4 halves)
  const __half2 lo = __floats2half2_rn(w[0], w[1]), hi = __floats2half2_rn(w[2], w[3]);
  *reinterpret_cast<uint2*>(p) =
      make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
}
__device__ __forceinline__ void store_dw4(float* p, const float* w) {
  *reinterpret_cast<float4*>(p) = make_float4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void store_one(__half* p, float v) { *p = __float2half_rn(v); }
__device__ __forceinline__ void store_one(float* p, float v) { *p = v; }

// Sum of a tile's partial slots (fixed order: row block, then range), inverse
// group DFT, cast to Out: dW[d][c][u] from part[pair][j][4][128 c][128 d];
// dbias[d] from bpart[pair][j][128] of the tiles with in-channel tile 0.
// A block takes 32 out-channels x 8 in-channels (inside one 128 x 128 tile), one
// entry per thread: lanes read the partials along d, the results pass through
// shared memory, and groups of 8 lanes write dW along c (each entry 4
// contiguous values), so both sides are coalesced.
// ---------------------------------------------------------------------------
// SM-pair weight gradient from tiled planes
// ---------------------------------------------------------------------------
constexpr int WP_ST = 4;                          // ring depth
constexpr uint32_t WP_GPLANE = 8 * 1024;          // dY: 8 blocks of 16 out-channels x 32 rows
constexpr uint32_t WP_XPLANE = 4 * 1024;          // X: this CTA's 4 blocks of 16 in-channels
constexpr uint32_t WP_G = 4 * WP_GPLANE;          // 32 KB
constexpr uint32_t WP_STAGE = WP_G + 4 * WP_XPLANE;  // 48 KB
constexpr uint32_t WP_OFF_BAR = WP_ST * WP_STAGE;
constexpr uint32_t WP_SMEM = WP_OFF_BAR + 512 + 1024;
constexpr int WP_THREADS = 512;
constexpr int WP_EPI0 = 4, WP_EPIW = 8;           // warps 4..11 drain the accumulators
constexpr int WP_BIAS0 = 12, WP_BIASW = 4;        // warps 12..15 sum dbias
static_assert(WP_SMEM <= 232448, "shared memory budget");
static_assert(WP_STAGE % 1024 == 0, "stage slots stay 1024-byte aligned");

struct WpBars {
  uint64_t full[WP_ST];   // leader: both CTAs' loads of the stage landed
  uint64_t empty[WP_ST];  // each CTA: the stage's MMAs and its dbias warps are done with it
  uint64_t done[WP_ST];   // each CTA: the stage's MMAs completed (its data is in place)
  uint64_t acc_full, acc_empty, drain[2];
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(WpBars) <= 512, "barrier block");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(WP_THREADS, 1)
    wgrad_pair_kernel(const __grid_constant__ CUtensorMap map_g,
                      const __grid_constant__ CUtensorMap map_x, int C, int D, WgInfo wi,
                      float* __restrict__ part, float* __restrict__ bpart, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  WpBars* bars = reinterpret_cast<WpBars*>(smem + WP_OFF_BAR);
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cta_rank();
  const int unit = blockIdx.x >> 1;  // the cluster's stream-K range

  if (threadIdx.x == 0) {
    for (int s = 0; s < WP_ST; ++s) {
      mbar_init(&bars->full[s], 1);              // the leader's producer (both CTAs' bytes)
      mbar_init(&bars->empty[s], 2 + WP_BIASW);  // both issuers' commits + the dbias warps
      mbar_init(&bars->done[s], 2);              // both issuers' commits
    }
    mbar_init(&bars->acc_full, 2);
    mbar_init(&bars->acc_empty, 2 * WP_EPIW);  // one arrival per epilogue warp of each CTA
    mbar_init(&bars->drain[0], 1);
    mbar_init(&bars->drain[1], 1);
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(512));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any remote arrive or TMA completion
  tc_fence_after();
  grid_dependency_wait();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    // ---------------- producer (both CTAs): own 128 out-channels of dY, own 64 in-channels of X
    if (lane == 0) {
      int issued_phase[WP_ST];
      for (int s = 0; s < WP_ST; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      SegIter si(wi, unit);
      Unit un;
      while (ok && si.next(wi, un)) {
        for (int s = 0; s < un.stages; ++s, ++it) {
          const int slot = it % WP_ST;
          const uint32_t ph = (it / WP_ST) & 1;
          if (!(ok = wait_bounded(&bars->empty[slot], ph ^ 1, abort_flag, status))) break;
          const uint32_t full_leader = peer_addr(smem_u32(&bars->full[slot]), 0);
          if (rank == 0) mbar_expect_tx(&bars->full[slot], 2 * WP_STAGE);
          const int line = (int)((un.r0 + (int64_t)WG_BR * s) / 4);
          const uint32_t dst = sbase + slot * WP_STAGE;
          // (128-byte line = 4 rows, line, 16-channel block, plane)
          tma_load_4d_pair(dst, &map_g, full_leader, 0, line, 16 * un.dt + 8 * (int)rank, 0);
          tma_load_4d_pair(dst + WP_G, &map_x, full_leader, 0, line, 8 * un.ct + 4 * (int)rank, 0);
          issued_phase[slot] = (int)ph;
        }
      }
      if (!ok && rank == 0)
        for (int s = 0; s < WP_ST; ++s)
          if (issued_phase[s] >= 0) drain_wait(&bars->full[s], (uint32_t)issued_phase[s]);
    }
    __syncwarp();
  } else if (warp == 1 || warp == 3) {
    // ---------------- MMA issuers (leader): Q0 and Qr on warp 1, Q2 and Qi on warp 3 ----------------
    if (rank == 0 && lane == 0) {
      const int who = warp == 1 ? 0 : 1;
      const uint32_t id = idesc_f16_mn(256, WG_BC), id_neg = idesc_f16_mn(256, WG_BC, true);
      uint32_t it = 0, ucount = 0;
      bool ok = true;
      SegIter si(wi, unit);
      Unit un;
      for (; ok && si.next(wi, un); ++ucount) {
        if (!(ok = wait_bounded(&bars->acc_empty, (ucount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int s = 0; s < un.stages; ++s, ++it) {
          const int slot = it % WP_ST;
          if (!(ok = wait_bounded(&bars->full[slot], (it / WP_ST) & 1, abort_flag, status))) break;
          tc_fence_after();
          const uint32_t g = sbase + slot * WP_STAGE, x = g + WP_G;
#pragma unroll
          for (int kk = 0; kk < WG_BR / 16; ++kk) {
            const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
            const uint64_t a2 = desc_mn32(g + 2 * WP_GPLANE + 512u * kk);
            const uint64_t a3 = desc_mn32(g + 3 * WP_GPLANE + 512u * kk);
            const uint64_t b2 = desc_mn32(x + 2 * WP_XPLANE + 512u * kk);
            const uint64_t b3 = desc_mn32(x + 3 * WP_XPLANE + 512u * kk);
            if (who == 0) {
              umma_pair(tmem + 0, desc_mn32(g + 512u * kk), desc_mn32(x + 512u * kk), id, acc);
              umma_pair(tmem + 2 * WG_BC, a2, b2, id, acc);        // Qr += Gr Xr
              umma_pair(tmem + 2 * WG_BC, a3, b3, id, 1u);         // Qr += Gi Xi
            } else {
              umma_pair(tmem + WG_BC, desc_mn32(g + WP_GPLANE + 512u * kk),
                        desc_mn32(x + WP_XPLANE + 512u * kk), id, acc);  // Q2
              umma_pair(tmem + 3 * WG_BC, a2, b3, id, acc);        // Qi += Gr Xi
              umma_pair(tmem + 3 * WG_BC, a3, b2, id_neg, 1u);     // Qi -= Gi Xr
            }
          }
          umma_commit_pair(&bars->done[slot], 3);
          umma_commit_pair(&bars->empty[slot], 3);
        }
        if (ok) umma_commit_pair(&bars->acc_full, 3);
      }
      // every MMA this thread issued completes before TMEM is freed
      umma_commit_pair(&bars->drain[who], 1);
      drain_wait(&bars->drain[who], 0);
    }
    __syncwarp();
  } else if (warp >= WP_EPI0 && warp < WP_EPI0 + WP_EPIW) {
    // ---------------- epilogue (both CTAs): accumulators -> FP32 partial planes ----------------
    // lane = out-channel 32q + lane of this CTA's 128; column j = in-channel 128 ct + j
    const int q = warp & 3;
    const int p0 = 2 * ((warp - WP_EPI0) >> 2);
    const uint32_t acc_empty_leader = peer_addr(smem_u32(&bars->acc_empty), 0);
    uint32_t ucount = 0;
    SegIter si(wi, unit);
    Unit un;
    for (; si.next(wi, un); ++ucount) {
      if (!warp_wait(&bars->acc_full, ucount & 1, abort_flag, status)) break;
      tc_fence_after();
      const int dl = 32 * q + lane;
      const int d = (2 * un.dt + (int)rank) * WG_BD + dl;
      const uint32_t lrow = tmem + ((uint32_t)(32 * q) << 16);
      float* slot_base = part + ((int64_t)un.slot * 2 + rank) * (4 * WG_BC * WG_BD);
#pragma unroll 1
      for (int p = p0; p < p0 + 2; ++p) {
        float* dst_plane = slot_base + p * (WG_BC * WG_BD);
#pragma unroll 1
        for (int gq = 0; gq < WG_BC / 16; gq += 2) {
          const int c = un.ct * WG_BC + 16 * gq;
          if (c >= C) break;  // warp-uniform; C % 16 == 0
          const bool two = c + 16 < C;
          uint32_t r[16], r2[16];
          tmem_ld_32x32b<16>(lrow + p * WG_BC + 16 * gq, r);
          if (two) tmem_ld_32x32b<16>(lrow + p * WG_BC + 16 * gq + 16, r2);
          tmem_wait_ld();
          if (d < D) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
              dst_plane[(16 * gq + k) * WG_BD + dl] = __uint_as_float(r[k]);
            if (two) {
#pragma unroll
              for (int k = 0; k < 16; ++k)
                dst_plane[(16 * gq + 16 + k) * WG_BD + dl] = __uint_as_float(r2[k]);
            }
          }
        }
      }
      // TMEM goes back once every warp of both CTAs has read it (its loads have
      // completed, so a relaxed arrive suffices)
      tc_fence_before();
      __syncwarp();
      if (lane == 0) arrive_remote_relaxed(acc_empty_leader);
    }
  } else if (warp >= WP_BIAS0 && warp < WP_BIAS0 + WP_BIASW) {
    // ---------------- dbias (both CTAs): sums of dY's plane 0, own 128 out-channels ----------------
    // plane 0 sits at [block dl / 16][row][32 B], piece (dl % 16) / 8 swizzled with (row / 4) % 2
    const int dl = (warp - WP_BIAS0) * 32 + lane;
    uint32_t it = 0;
    bool ok = true;
    SegIter si(wi, unit);
    Unit un;
    while (ok && si.next(wi, un)) {
      float b = 0.f;
      for (int s = 0; s < un.stages; ++s, ++it) {
        const int slot = it % WP_ST;
        if (!(ok = warp_wait(&bars->done[slot], (it / WP_ST) & 1, abort_flag, status))) break;
        if (un.ct == 0) {
          const uint8_t* blk = smem + slot * WP_STAGE + (dl >> 4) * 1024;
          const int piece = (dl & 15) >> 3, within = (dl & 7) * 2;
#pragma unroll 8
          for (int r = 0; r < WG_BR; ++r)
            b += __half2float(*reinterpret_cast<const __half*>(
                blk + r * 32 + ((piece ^ ((r >> 2) & 1)) << 4) + within));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->empty[slot]);
      }
      if (!ok) break;
      // the planes hold G0/4: the sum times 4 (exact) is the sum of G0
      if (un.ct == 0) bpart[((int64_t)un.slot * 2 + rank) * WG_BD + dl] = 4.f * b;
    }
  }

  grid_launch_dependents();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA leaves while its pair may still touch its shared memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512));
  }
}

constexpr int FZ_D = 32, FZ_C = 8;
constexpr int FZ_U = 8;  // row blocks summed side by side
template <typename Out>
__global__ void __launch_bounds__(256)
    wgrad_tc_finalize_kernel(const float* __restrict__ part, const float* __restrict__ bpart,
                             WgInfo wi, int C, int D, Out* __restrict__ dW,
                             Out* __restrict__ dbias, Twiddles tw, int pairs) {
  __shared__ __align__(16) float s[FZ_C][FZ_D * 4 + 4];  // [c][d][u], rows padded by 16 B
  const int d0 = blockIdx.x * FZ_D, c0 = blockIdx.y * FZ_C;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;  // 8 warps
  // pairs: a stream-K tile is 256 out-channels; its CTA `half` wrote this block.
  // blockIdx.z: the convolution tap (its dW block follows the previous taps')
  const int mult = pairs ? 2 : 1, half = pairs ? (d0 / WG_BD) & 1 : 0;
  const int tile = (d0 / WG_BD / mult) * wi.n_ct + blockIdx.z * wi.nct_tap + c0 / WG_BC;
  dW += (size_t)blockIdx.z * D * C * 4;
  {
    const int d = d0 + lane, c = c0 + w;  // lane = out-channel, warp = in-channel
    if (d < D && c < C) {
      const int64_t off = (int64_t)(c % WG_BC) * WG_BD + (d % WG_BD);
      // Row blocks in groups of FZ_U: each block's slots go to their own
      // accumulators (the first slot's loads of the whole group issued together,
      // so a thread has FZ_U x 4 loads in flight), then the FZ_U partial sums are
      // added in a fixed order.  A few output tiles and many row blocks (a small
      // layer over many rows) would otherwise leave a long chain of dependent
      // loads per thread.
      float qa[FZ_U][4];
#pragma unroll
      for (int u = 0; u < FZ_U; ++u)
#pragma unroll
        for (int p = 0; p < 4; ++p) qa[u][p] = 0.f;
      for (int b0 = 0; b0 < wi.nb; b0 += FZ_U) {
        float v[FZ_U][4];
#pragma unroll
        for (int u = 0; u < FZ_U; ++u) {
          const int b = b0 + u;
#pragma unroll
          for (int p = 0; p < 4; ++p) v[u][p] = 0.f;
          if (b < wi.nb) {
            const int pair = b * wi.n_dt * wi.n_ct + tile;
            const float* slot =
                part + ((int64_t)pair * wi.maxj * mult + half) * (4 * WG_BC * WG_BD);
#pragma unroll
            for (int p = 0; p < 4; ++p) v[u][p] = slot[p * (WG_BC * WG_BD) + off];
          }
        }
#pragma unroll
        for (int u = 0; u < FZ_U; ++u)
#pragma unroll
          for (int p = 0; p < 4; ++p) qa[u][p] += v[u][p];
        // a row block's further slots (ranges that started inside it)
#pragma unroll
        for (int u = 0; u < FZ_U; ++u) {
          const int b = b0 + u;
          if (b >= wi.nb) continue;
          const int pair = b * wi.n_dt * wi.n_ct + tile;
          const int n = last_range_of_pair(b, tile, wi) - first_range_of_pair(b, tile, wi);
          for (int j = 1; j <= n; ++j) {
            const float* slot =
                part + (((int64_t)pair * wi.maxj + j) * mult + half) * (4 * WG_BC * WG_BD);
#pragma unroll
            for (int p = 0; p < 4; ++p) qa[u][p] += slot[p * (WG_BC * WG_BD) + off];
          }
        }
      }
      float qv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int u = 0; u < FZ_U; ++u)
#pragma unroll
        for (int p = 0; p < 4; ++p) qv[p] += qa[u][p];
      // both operand planes carried 1/4: the partial sums are Q/16
#pragma unroll
      for (int p = 0; p < 4; ++p) qv[p] *= 16.f;
      float wv[4];
      group_idft<4>(qv, wv, tw);
      *reinterpret_cast<float4*>(&s[w][4 * lane]) = make_float4(wv[0], wv[1], wv[2], wv[3]);
    }
  }
  __syncthreads();
  {
    const int cl = threadIdx.x & (FZ_C - 1), dl = threadIdx.x / FZ_C;
    const int c = c0 + cl, d = d0 + dl;
    if (d < D && c < C) store_dw4(dW + ((int64_t)d * C + c) * 4, &s[cl][4 * dl]);
  }
  if (dbias && blockIdx.y == 0 && blockIdx.z == 0 && w == 0 && d0 + lane < D) {
    const int d = d0 + lane;
    const int tile0 = (d / WG_BD / mult) * wi.n_ct;
    float ba[FZ_U];
#pragma unroll
    for (int u = 0; u < FZ_U; ++u) ba[u] = 0.f;
    for (int rb0 = 0; rb0 < wi.nb; rb0 += FZ_U) {
#pragma unroll
      for (int u = 0; u < FZ_U; ++u) {
        const int rb = rb0 + u;
        if (rb >= wi.nb) continue;
        const int pair = rb * wi.n_dt * wi.n_ct + tile0;
        const int n = last_range_of_pair(rb, tile0, wi) - first_range_of_pair(rb, tile0, wi);
        for (int j = 0; j <= n; ++j)
          ba[u] += bpart[(((int64_t)pair * wi.maxj + j) * mult + half) * WG_BD + d % WG_BD];
      }
    }
    float b = 0.f;
#pragma unroll
    for (int u = 0; u < FZ_U; ++u) b += ba[u];
    store_one(dbias + d, b);
  }
}

bool encode_rows_map(CUtensorMap* m, const void* base, int channels, int64_t N) {
  auto encode = encode_fn();
  if (!encode) return false;
  // (64 halves, 128-byte chunk, row); box = 8 chunks (128 channels x 4) x 32 rows
  cuuint64_t dims[3] = {64, (cuuint64_t)channels * 4 / 64, (cuuint64_t)N};
  cuuint64_t strides[2] = {128, (cuuint64_t)channels * 4 * 2};
  cuuint32_t box[3] = {64, 8, WG_BR};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Spectral planes [4][N][channels] viewed as (64 channels, row, 64-channel
// block, plane); box = (64, PL_ROWS rows, 2 blocks, 4 planes), 128-byte swizzle.
// The block dimension steps by 128 B inside a row, so channels % 64 == 0 keeps
// every block inside its row.
// plane_rows: the rows between one plane and the next (N when the planes are
// [4][N][channels]; more when N rows are read from inside larger planes).
bool encode_planes4_map(CUtensorMap* m, const void* base, int channels, int64_t N,
                        int64_t plane_rows) {
  auto encode = encode_fn();
  if (!encode || channels % 64 != 0 || plane_rows < N) return false;
  cuuint64_t dims[4] = {64, (cuuint64_t)N, (cuuint64_t)channels / 64, 4};
  cuuint64_t strides[3] = {(cuuint64_t)channels * 2, 128,
                           (cuuint64_t)plane_rows * channels * 2};
  cuuint32_t box[4] = {64, PL_ROWS, 2, 4};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiled planes (tiled_rows(N) rows per 16-channel block) viewed as (64 halves of
// a 128-byte line, line, 16-channel block, plane); box = (64, 8 lines, 8 blocks,
// 4 planes), no swizzle (the rows are stored swizzled).
bool encode_tiled4_map(CUtensorMap* m, const void* base, int channels, int64_t N,
                       uint32_t blocks = 8) {
  auto encode = encode_fn();
  if (!encode || channels % 16 != 0) return false;
  const int64_t Np = tiled_rows(N);
  const int kb = channels / 16;
  cuuint64_t dims[4] = {64, (cuuint64_t)(Np / 4), (cuuint64_t)kb, 4};
  cuuint64_t strides[3] = {128, (cuuint64_t)Np * 32, (cuuint64_t)Np * 32 * kb};
  cuuint32_t box[4] = {64, PL_ROWS / 4, blocks, 4};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 4, const_cast<void*>(base), dims, strides,
                box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// The stream-K layout for N rows: equal contiguous ranges of (tile, stage), one
// per CTA, and the number of partial slots a tile can need.
// pairs: tiles of 256 out-channels, one range per cluster of two SMs.
// taps > 1 (planes variant only): a convolution's taps as in-channel tiles, tap t
// reading X (t / kw) * wp + t % kw rows further on.
bool wgrad_tc_layout(int64_t N, int C, int D, int num_sms, WgInfo* wi, int* grid,
                     bool pairs = false, int taps = 1, int kw = 1, int wp = 0) {
  if (N <= 0 || taps < 1 || kw < 1) return false;
  if (pairs) num_sms /= 2;
  if (num_sms < 1) return false;
  wi->n_dt = (D + (pairs ? 2 : 1) * WG_BD - 1) / ((pairs ? 2 : 1) * WG_BD);
  wi->nct_tap = (C + WG_BC - 1) / WG_BC;
  wi->n_ct = taps * wi->nct_tap;
  wi->tap_kw = kw;
  wi->tap_wp = wp;
  const int64_t spt = (N + WG_BR - 1) / WG_BR;
  if (spt > 0x3fffffffLL) return false;
  wi->spt = (int)spt;
  wi->total = (int64_t)wi->n_dt * wi->n_ct * spt;
  if (wi->total > 0x7fffffffLL) return false;  // stage indices stay 32-bit
  const int64_t want = std::min<int64_t>(num_sms, wi->total);
  int64_t per = (wi->total + want - 1) / want;
  // at least 16 stages (512 rows) per range, or a whole tile, so the 256 KB
  // partial a range writes is amortised
  per = std::max<int64_t>(per, std::min<int64_t>(spt, 16));
  if (per > 0x3fffffffLL) return false;
  wi->per_unit = (int)per;
  *grid = (int)((wi->total + per - 1) / per);
  // row blocks of one range's length: in every full block, range u covers
  // exactly pair u, so the CTAs of a block step through its rows together
  wi->bst = (int)std::min<int64_t>(per, spt);
  wi->nb = (int)((spt + wi->bst - 1) / wi->bst);
  // slots per pair: the number of ranges that touch it (exact maximum)
  const int tiles = wi->n_dt * wi->n_ct;
  int64_t maxj = 1;
  for (int b = 0; b < wi->nb; ++b)
    for (int t = 0; t < tiles; ++t)
      maxj = std::max<int64_t>(maxj, last_range_of_pair(b, t, *wi) -
                                         first_range_of_pair(b, t, *wi) + 1);
  wi->maxj = (int)maxj;
  return true;
}

}  // namespace

bool wgrad_tc_supported(int T, DType dt, int64_t N, int C, int D, const void* X, const void* dY) {
  return T == 4 && dt == DType::F16 && N >= 1 && N <= 0x7fffff00LL && C % 16 == 0 &&
         D % 16 == 0 && C >= 16 && D >= 16 && ((reinterpret_cast<uintptr_t>(X) & 15) == 0) &&
         ((reinterpret_cast<uintptr_t>(dY) & 15) == 0);
}

// Enough for the one-CTA layout and the SM-pair one (two 128 x 128 blocks per slot).
size_t wgrad_tc_workspace(int64_t N, int C, int D, int num_sms) {
  size_t need = 0;
  for (int pairs = 0; pairs < 2; ++pairs) {
    WgInfo wi;
    int grid = 0;
    if (!wgrad_tc_layout(N, C, D, num_sms, &wi, &grid, pairs != 0)) continue;
    const size_t slots = (size_t)wi.nb * wi.n_dt * wi.n_ct * wi.maxj * (pairs ? 2 : 1);
    need = std::max(need, slots * ((size_t)4 * WG_BC * WG_BD + WG_BD) * sizeof(float));
  }
  return need;
}

bool wgrad_tc_planes_supported(int64_t N, int C, int D, const void* Xhat, const void* Ghat) {
  return wgrad_tc_supported(4, DType::F16, N, C, D, Xhat, Ghat) && C % 64 == 0 && D % 64 == 0;
}

namespace {
cudaError_t wgrad_attrs() {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(wgrad_tc_kernel<false>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, WG_SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(wgrad_tc_kernel<true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, WG_SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(wgrad_tc_kernel<true, true>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize, WG_SMEM);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(wgrad_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               WP_SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  return cudaSuccess;
}
}  // namespace

cudaError_t launch_wgrad_tc(const void* X, const void* dY, int64_t N, int C, int D,
                            void* workspace, DType out_dt, void* dW, void* dbias, int* status,
                            int num_sms, const Twiddles& tw, cudaStream_t st, int planes,
                            int64_t plane_rows) {
  WgInfo wi;
  int grid = 0;
  if (planes < 0 || planes > 2) return cudaErrorInvalidValue;
  // tiled planes: SM pairs (the one-CTA tiled variant if the pair layout fails)
  const bool pairs = planes == 2 && wgrad_tc_layout(N, C, D, num_sms, &wi, &grid, true);
  if (!pairs && !wgrad_tc_layout(N, C, D, num_sms, &wi, &grid)) return cudaErrorInvalidValue;
  if (planes == 1 && (C % 64 != 0 || D % 64 != 0)) return cudaErrorNotSupported;
  CUtensorMap mg, mx;
  if (planes == 2) {
    if (!encode_tiled4_map(&mg, dY, D, N) ||
        !encode_tiled4_map(&mx, X, C, N, pairs ? 4u : 8u))
      return cudaErrorInvalidValue;
  } else if (planes == 1) {
    const int64_t pr = plane_rows > 0 ? plane_rows : N;
    if (!encode_planes4_map(&mg, dY, D, N, pr) || !encode_planes4_map(&mx, X, C, N, pr))
      return cudaErrorInvalidValue;
  } else if (!encode_rows_map(&mg, dY, D, N) || !encode_rows_map(&mx, X, C, N)) {
    return cudaErrorInvalidValue;
  }
  float* part = static_cast<float*>(workspace);
  float* bpart =
      part + (size_t)wi.nb * wi.n_dt * wi.n_ct * wi.maxj * (pairs ? 2 : 1) * (4 * WG_BC * WG_BD);
  cudaError_t ea = wgrad_attrs();
  if (ea != cudaSuccess) return ea;
  if (pairs) {
    cudaError_t e = launch_dependent(wgrad_pair_kernel, dim3(2 * grid), dim3(WP_THREADS), WP_SMEM,
                                     st, mg, mx, C, D, wi, part, bpart, status);
    if (e != cudaSuccess) return e;
  } else if (planes == 2)
    wgrad_tc_kernel<true, true><<<grid, WG_THREADS_PL, WG_SMEM, st>>>(mg, mx, N, C, D, wi, part,
                                                                      bpart, status);
  else if (planes == 1)
    wgrad_tc_kernel<true><<<grid, WG_THREADS_PL, WG_SMEM, st>>>(mg, mx, N, C, D, wi, part, bpart,
                                                                status);
  else
    wgrad_tc_kernel<false><<<grid, WG_THREADS, WG_SMEM, st>>>(mg, mx, N, C, D, wi, part, bpart,
                                                              status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 fgrid((D + FZ_D - 1) / FZ_D, (C + FZ_C - 1) / FZ_C);
  if (out_dt == DType::F32)
    wgrad_tc_finalize_kernel<float><<<fgrid, 256, 0, st>>>(
        part, bpart, wi, C, D, static_cast<float*>(dW), static_cast<float*>(dbias), tw,
        pairs ? 1 : 0);
  else
    wgrad_tc_finalize_kernel<__half><<<fgrid, 256, 0, st>>>(
        part, bpart, wi, C, D, static_cast<__half*>(dW), static_cast<__half*>(dbias), tw,
        pairs ? 1 : 0);
  return cudaGetLastError();
}

size_t wgrad_tc_conv_workspace(int64_t R, int C, int D, int taps, int num_sms) {
  WgInfo wi;
  int grid = 0;
  if (!wgrad_tc_layout(R, C, D, num_sms, &wi, &grid, false, taps, 1, 0)) return 0;
  const size_t slots = (size_t)wi.nb * wi.n_dt * wi.n_ct * wi.maxj;
  return slots * ((size_t)4 * WG_BC * WG_BD + WG_BD) * sizeof(float);
}

cudaError_t launch_wgrad_tc_conv(const void* Xs, const void* Gs, int64_t R, int C, int D,
                                 int taps, int kw, int wp, void* workspace, DType out_dt,
                                 void* dW, void* dbias, int* status, int num_sms,
                                 const Twiddles& tw, cudaStream_t st) {
  WgInfo wi;
  int grid = 0;
  if (C % 64 != 0 || D % 64 != 0) return cudaErrorNotSupported;
  if (!wgrad_tc_layout(R, C, D, num_sms, &wi, &grid, false, taps, kw, wp))
    return cudaErrorInvalidValue;
  // both plane sets whole: a tap's X rows past R read the map's zero fill
  CUtensorMap mg, mx;
  if (!encode_planes4_map(&mg, Gs, D, R, R) || !encode_planes4_map(&mx, Xs, C, R, R))
    return cudaErrorInvalidValue;
  float* part = static_cast<float*>(workspace);
  float* bpart = part + (size_t)wi.nb * wi.n_dt * wi.n_ct * wi.maxj * (4 * WG_BC * WG_BD);
  cudaError_t e = wgrad_attrs();
  if (e != cudaSuccess) return e;
  wgrad_tc_kernel<true><<<grid, WG_THREADS_PL, WG_SMEM, st>>>(mg, mx, R, C, D, wi, part, bpart,
                                                              status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 fgrid((D + FZ_D - 1) / FZ_D, (C + FZ_C - 1) / FZ_C, taps);
  if (out_dt == DType::F32)
    wgrad_tc_finalize_kernel<float><<<fgrid, 256, 0, st>>>(
        part, bpart, wi, C, D, static_cast<float*>(dW), static_cast<float*>(dbias), tw, 0);
  else
    wgrad_tc_finalize_kernel<__half><<<fgrid, 256, 0, st>>>(
        part, bpart, wi, C, D, static_cast<__half*>(dW), static_cast<__half*>(dbias), tw, 0);
  return cudaGetLastError();
}

}  // namespace eql
