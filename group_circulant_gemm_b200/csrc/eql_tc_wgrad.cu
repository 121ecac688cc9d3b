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
// deterministic.
//
// Work split (stream-K over rows): the (tile, 32-row stage) space, tile = 128
// out-channels x 128 in-channels, is cut into equal contiguous ranges, one per
// CTA, so every SM does the same number of stages.  A range can end one tile
// and start the next; each piece (a "segment") accumulates in TMEM and writes
// its own partial slot part[tile][j][4][128 c][128 d] (j = which of the tile's
// ranges; out-channel fastest, so each warp store writes 128 contiguous bytes).
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
#include <algorithm>

#include "eql_kernels.h"
#include "eql_tc_common.cuh"

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
constexpr int WG_EPI0 = 4, WG_EPIW = 4;      // warps 4..7: one per TMEM lane quarter
constexpr int WG_XF0 = 8, WG_XFW = 8;        // warps 8..15 (dY tile), 16..23 (X tile)
static_assert(4 * WG_PLANE == WG_TILE, "planes replace the raw tile in place");
static_assert(WG_SMEM <= 232448, "shared memory budget");

struct WgBars {
  uint64_t full[WG_ST], read_g[WG_ST], read_x[WG_ST], ready[WG_ST], empty[WG_ST];
  uint64_t acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(WgBars) <= 512, "barrier block");

struct WgInfo {
  int n_dt, n_ct;      // out-channel and in-channel tiles
  int spt;             // 32-row stages per tile, ceil(N / 32)
  int per_unit;        // stages per CTA range
  int maxj;            // partial slots per tile
  int64_t total;       // tiles * spt
};

// One segment of a CTA's range: stages [r0 / 32, r0 / 32 + stages) of one tile.
struct Unit {
  int dt, ct, tile, slot;  // slot = tile * maxj + (range index within the tile)
  int64_t r0;
  int stages;
};

__host__ __device__ inline int first_range_of_tile(int64_t tile, const WgInfo& wi) {
  return (int)(tile * wi.spt / wi.per_unit);
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
    x.tile = (int)(g / wi.spt);
    const int s0 = (int)(g % wi.spt);
    const int64_t room = wi.spt - s0;
    x.stages = (int)(room < g1 - g ? room : g1 - g);
    x.dt = x.tile / wi.n_ct;
    x.ct = x.tile % wi.n_ct;
    x.slot = x.tile * wi.maxj + (u - first_range_of_tile(x.tile, wi));
    x.r0 = (int64_t)s0 * WG_BR;
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
        if (kBias) bsum[e] += p0[h];
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

__global__ void __launch_bounds__(WG_THREADS, 1)
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

  if (threadIdx.x == 0) {
    for (int s = 0; s < WG_ST; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->read_g[s], WG_XFW);
      mbar_init(&bars->read_x[s], WG_XFW);
      mbar_init(&bars->ready[s], 2 * WG_XFW);
      mbar_init(&bars->empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, WG_EPIW * 32);
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
      int issued_phase[WG_ST];
      for (int s = 0; s < WG_ST; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      SegIter si(wi, blockIdx.x);
      Unit un;
      while (ok && si.next(wi, un)) {
        for (int s = 0; s < un.stages; ++s, ++it) {
          const int slot = it % WG_ST;
          const uint32_t ph = (it / WG_ST) & 1;
          if (!(ok = wait_bounded(&bars->empty[slot], ph ^ 1, abort_flag, status))) break;
          mbar_expect_tx(&bars->full[slot], WG_STAGE);
          const int row = (int)(un.r0 + (int64_t)WG_BR * s);
          const uint32_t dst = sbase + slot * WG_STAGE;
          // 3-D views (64 halves, 128-byte chunk of the row, row); a unit's tile is
          // chunks 8*tile .. 8*tile+7 (128 channels x 4 group elements)
          tma_load_3d(dst, &map_g, &bars->full[slot], 0, 8 * un.dt, row);
          tma_load_3d(dst + WG_TILE, &map_x, &bars->full[slot], 0, 8 * un.ct, row);
          issued_phase[slot] = (int)ph;
        }
      }
      if (!ok)
        for (int s = 0; s < WG_ST; ++s)
          if (issued_phase[s] >= 0) drain_wait(&bars->full[s], (uint32_t)issued_phase[s]);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, ucount = 0;
      bool ok = true;
      const uint32_t id_n1 = idesc_f16(128, WG_BC);
      const uint32_t id_n1_neg = idesc_f16(128, WG_BC, true);
      const uint32_t id_n2 = idesc_f16(128, 2 * WG_BC);
      SegIter si(wi, blockIdx.x);
      Unit un;
      for (; ok && si.next(wi, un); ++ucount) {
        if (!(ok = wait_bounded(&bars->acc_empty, (ucount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int s = 0; s < un.stages; ++s, ++it) {
          const int slot = it % WG_ST;
          if (!(ok = wait_bounded(&bars->ready[slot], (it / WG_ST) & 1, abort_flag, status)))
            break;
          tc_fence_after();
          const uint32_t g = sbase + slot * WG_STAGE;  // G planes (A: rows = out-channels)
          const uint32_t x = g + WG_TILE;              // Xh planes (B: rows = in-channels)
#pragma unroll
          for (int kk = 0; kk < WG_BR / 16; ++kk) {
            const uint32_t ko = 32u * kk;
            const uint32_t acc = (s > 0 || kk > 0) ? 1u : 0u;
            auto A = [&](int p) { return desc_kmajor<WG_ROWB>(g + p * WG_PLANE + ko); };
            auto B = [&](int p) { return desc_kmajor<WG_ROWB>(x + p * WG_PLANE + ko); };
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
  } else if (warp >= WG_EPI0 && warp < WG_EPI0 + WG_EPIW) {
    // ---------------- epilogue: accumulators -> FP32 partial planes ----------------
    // Warp w reads TMEM lane quarter q = w % 4: lane l holds out-channel
    // 32q + l; a 32x32b load gives it 16 consecutive in-channels of one plane,
    // and each of the 16 stores writes 32 consecutive out-channels (128 B).
    const int q = warp & 3;
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
      for (int p = 0; p < 4; ++p) {
        float* dst_plane = slot_base + p * (WG_BC * WG_BD);
#pragma unroll 1
        for (int gq = 0; gq < WG_BC / 16; ++gq) {
          const int c = un.ct * WG_BC + 16 * gq;
          if (c >= C) break;  // warp-uniform; C % 16 == 0: the 16 columns are all in range
          uint32_t r[16];
          tmem_ld_32x32b<16>(lrow + p * WG_BC + 16 * gq, r);
          tmem_wait_ld();
          if (d < D) {
#pragma unroll
            for (int k = 0; k < 16; ++k)
              dst_plane[(16 * gq + k) * WG_BD + dl] = __uint_as_float(r[k]);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
    }
  } else if (warp >= WG_XF0) {
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
  __half2* out = reinterpret_cast<__half2*>(p);
  out[0] = __floats2half2_rn(w[0], w[1]);
  out[1] = __floats2half2_rn(w[2], w[3]);
}
__device__ __forceinline__ void store_dw4(float* p, const float* w) {
  *reinterpret_cast<float4*>(p) = make_float4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void store_one(__half* p, float v) { *p = __float2half_rn(v); }
__device__ __forceinline__ void store_one(float* p, float v) { *p = v; }

// Sum of a tile's partial slots (fixed order), inverse group DFT, cast to Out:
// dW[d][c][u] from part[tile][j][4][128 c][128 d]; dbias[d] from
// bpart[tile][j][128] of the tiles with in-channel tile 0.
template <typename Out>
__global__ void wgrad_tc_finalize_kernel(const float* __restrict__ part,
                                         const float* __restrict__ bpart, WgInfo wi, int C,
                                         int D, Out* __restrict__ dW, Out* __restrict__ dbias,
                                         Twiddles tw) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // c * D + d
  if (idx < (int64_t)D * C) {
    const int c = (int)(idx / D), d = (int)(idx % D);
    const int tile = (d / WG_BD) * wi.n_ct + c / WG_BC;
    const int first = first_range_of_tile(tile, wi);
    const int last = (int)(((int64_t)tile * wi.spt + wi.spt - 1) / wi.per_unit);
    const int64_t off = (int64_t)(c % WG_BC) * WG_BD + (d % WG_BD);
    float qv[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j = 0; j <= last - first; ++j) {
      const float* slot = part + ((int64_t)tile * wi.maxj + j) * (4 * WG_BC * WG_BD);
#pragma unroll
      for (int p = 0; p < 4; ++p) qv[p] += slot[p * (WG_BC * WG_BD) + off];
    }
    float wv[4];
    group_idft<4>(qv, wv, tw);
    store_dw4(dW + ((int64_t)d * C + c) * 4, wv);
  }
  if (dbias && idx < D) {
    const int d = (int)idx;
    const int tile = (d / WG_BD) * wi.n_ct;
    const int first = first_range_of_tile(tile, wi);
    const int last = (int)(((int64_t)tile * wi.spt + wi.spt - 1) / wi.per_unit);
    float b = 0.f;
    for (int j = 0; j <= last - first; ++j)
      b += bpart[((int64_t)tile * wi.maxj + j) * WG_BD + d % WG_BD];
    store_one(dbias + idx, b);
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

// The stream-K layout for N rows: equal contiguous ranges of (tile, stage), one
// per CTA, and the number of partial slots a tile can need.
bool wgrad_tc_layout(int64_t N, int C, int D, int num_sms, WgInfo* wi, int* grid) {
  if (N <= 0) return false;
  wi->n_dt = (D + WG_BD - 1) / WG_BD;
  wi->n_ct = (C + WG_BC - 1) / WG_BC;
  const int64_t spt = (N + WG_BR - 1) / WG_BR;
  if (spt > 0x3fffffffLL) return false;
  wi->spt = (int)spt;
  wi->total = (int64_t)wi->n_dt * wi->n_ct * spt;
  const int64_t want = std::min<int64_t>(num_sms, wi->total);
  int64_t per = (wi->total + want - 1) / want;
  // at least 16 stages (512 rows) per range, or a whole tile, so the 256 KB
  // partial a range writes is amortised
  per = std::max<int64_t>(per, std::min<int64_t>(spt, 16));
  if (per > 0x3fffffffLL) return false;
  wi->per_unit = (int)per;
  *grid = (int)((wi->total + per - 1) / per);
  // slots per tile: the number of ranges that touch it (exact maximum)
  const int64_t tiles = (int64_t)wi->n_dt * wi->n_ct;
  int64_t maxj = 1;
  for (int64_t t = 0; t < tiles; ++t) {
    const int64_t first = t * spt / per, last = (t * spt + spt - 1) / per;
    maxj = std::max(maxj, last - first + 1);
  }
  wi->maxj = (int)maxj;
  return true;
}

}  // namespace

bool wgrad_tc_supported(int T, DType dt, int64_t N, int C, int D, const void* X, const void* dY) {
  return T == 4 && dt == DType::F16 && N >= 1 && N <= 0x7fffff00LL && C % 16 == 0 &&
         D % 16 == 0 && C >= 16 && D >= 16 && ((reinterpret_cast<uintptr_t>(X) & 15) == 0) &&
         ((reinterpret_cast<uintptr_t>(dY) & 15) == 0);
}

size_t wgrad_tc_workspace(int64_t N, int C, int D, int num_sms) {
  WgInfo wi;
  int grid = 0;
  if (!wgrad_tc_layout(N, C, D, num_sms, &wi, &grid)) return 0;
  const size_t slots = (size_t)wi.n_dt * wi.n_ct * wi.maxj;
  return slots * ((size_t)4 * WG_BC * WG_BD + WG_BD) * sizeof(float);
}

cudaError_t launch_wgrad_tc(const void* X, const void* dY, int64_t N, int C, int D,
                            void* workspace, DType out_dt, void* dW, void* dbias, int* status,
                            int num_sms, const Twiddles& tw, cudaStream_t st) {
  WgInfo wi;
  int grid = 0;
  if (!wgrad_tc_layout(N, C, D, num_sms, &wi, &grid)) return cudaErrorInvalidValue;
  CUtensorMap mg, mx;
  if (!encode_rows_map(&mg, dY, D, N) || !encode_rows_map(&mx, X, C, N))
    return cudaErrorInvalidValue;
  float* part = static_cast<float*>(workspace);
  float* bpart = part + (size_t)wi.n_dt * wi.n_ct * wi.maxj * (4 * WG_BC * WG_BD);
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(wgrad_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, WG_SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  wgrad_tc_kernel<<<grid, WG_THREADS, WG_SMEM, st>>>(mg, mx, N, C, D, wi, part, bpart, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t total = std::max<int64_t>((int64_t)C * D, D);
  const unsigned fblocks = (unsigned)((total + 255) / 256);
  if (out_dt == DType::F32)
    wgrad_tc_finalize_kernel<float><<<fblocks, 256, 0, st>>>(
        part, bpart, wi, C, D, static_cast<float*>(dW), static_cast<float*>(dbias), tw);
  else
    wgrad_tc_finalize_kernel<__half><<<fblocks, 256, 0, st>>>(
        part, bpart, wi, C, D, static_cast<__half*>(dW), static_cast<__half*>(dbias), tw);
  return cudaGetLastError();
}

}  // namespace eql
