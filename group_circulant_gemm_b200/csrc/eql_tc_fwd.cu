// tcgen05/TMEM tensor-core forward of the cyclic-group EQ-Linear layer for
// T = 4 (the p4 rotation group) and T = 8, FP16 in, FP32 accumulate, FP16 out,
// for sm_100a.  Also used for dX (the same product with the adjoint weights).
//
// What it computes (Flash EQ-Linear summary, "Algorithmic approach" items 1-3
// and "Specialisation for p4"): per row n and input channel c the real DFT of
// the group vector x[0..T) (FP32, one rounding to FP16), one real GEMM per real
// frequency and four per complex frequency against the prepared weight planes
// (conjugated spectrum of W), and the inverse DFT plus bias:
//   real k:     Y_k  = X_k A_k^T
//   complex k:  Y_kr = Xr_k Br_k^T - Xi_k Bi_k^T,  Y_ki = Xr_k Bi_k^T + Xi_k Br_k^T
//   y[s] = (Y_0 + (-1)^s Y_{T/2}) / T + (2/T) sum_k (Y_kr cos(2 pi k s/T) - Y_ki sin(2 pi k s/T))
// For T = 4 the transforms are adds only (X0 = x0+x1+x2+x3, X2 = x0-x1+x2-x3,
// Xr = x0-x2, Xi = x3-x1); for T = 8 a radix-2 split leaves one non-dyadic
// twiddle, sqrt(2)/2.  The inverse's factors 1/T and 2/T are folded into the
// weight tiles, so the epilogue is adds only.
//
// Template parameters: ACT = output activation (0 none, 1 GELU, fused into the
// epilogue); IO (T = 4) = spatial X and Y, or Y written as the next layer's
// spectral operand planes [4][N][Cout], or X read as such planes (then the TMA
// box lands directly as the operand planes and the transform warps are idle).
//
// Design (one persistent CTA per SM; tile = 128 rows x BD out-channels; K stage
// = BK input channels, whose raw X tile is always 128 rows x 256 B = 32 KB):
//   warp 0      TMA producer: the raw X tile of a stage, one 3-D box
//               (64 halves x 2 row chunks x 128 rows, 128B-swizzled), 3-deep ring.
//   warp 2      weight producer: one bulk copy per stage of a blob that
//               prepare_weights pre-arranged in the MMA operand layout.
//   warp 1      TMEM allocator; lane 0 issues the MMAs of each K step:
//               N = BD for each real frequency, N = 2 BD for Xr_k [Br_k|Bi_k],
//               and N = BD for -Xi_k Bi_k (negate-A bit) and Xi_k Br_k.
//   warps 12-19 transform: group DFT in FP32, one rounding to FP16, written as
//               T K-major swizzled operand planes over the raw tile of the same
//               slot (the planes take exactly the raw tile's 32 KB).
//   warps 4-11  epilogue: the tile's biases staged in shared memory while the
//               main loop runs; tcgen05.ld 32x32b (one row per lane), inverse
//               DFT + bias (+ activation), FP16 pack into a per-warp 4 KB
//               staging buffer, one TMA store per 32 rows x 128 bytes of Y (or
//               per 32 rows x 16 channels x 4 planes for spectral output).
// TMEM (T * BD = 512 columns): real frequency 0 at [0, BD), real frequency T/2
// at [BD, 2 BD), complex frequency k at [2 BD k, 2 BD k + 2 BD) as (re | im).
// Every mbarrier wait is bounded (about 2 s of %globaltimer); on expiry the CTA
// sets a shared abort flag and the plan's status word, drains what it issued and
// returns, so a stuck pipeline never hangs the GPU.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "eql_kernels.h"
#include "eql_tc_common.cuh"

namespace eql {
namespace {

using namespace tc;

constexpr int BM = 128;          // rows per tile = MMA M
constexpr int X_ST = 3;          // X ring: raw tile in, transformed operand planes out (in place)
constexpr uint32_t X_STAGE_BYTES = BM * 256;   // 128 rows x 256 B raw X per stage
constexpr int kThreads = 640;
constexpr int kEpiWarp0 = 4;     // warps 4..11: two per TMEM lane quarter
constexpr int kEpiWarps = 8;
constexpr int kXfWarp0 = 12;     // warps 12..19
constexpr int kXfWarps = 8;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kStgBytes = 4096;  // per epilogue warp: 32 rows x 128 B of Y
// Input/output forms (T = 4): spatial X and Y; Y written as the next layer's
// spectral operand planes; X read as spectral operand planes.
constexpr int kIoSpatial = 0, kIoSpectralOut = 1, kIoSpectralIn = 2;

// Per-group shape of the pipeline.
template <int T>
struct Cfg;
template <>
struct Cfg<4> {
  static constexpr int BD = 128;        // out-channels per tile
  static constexpr int BK = 32;         // in-channels per stage (two MMA K steps)
  static constexpr int W_ST = 3;        // weight-tile ring depth
};
template <>
struct Cfg<8> {
  static constexpr int BD = 64;
  static constexpr int BK = 16;         // one MMA K step
  static constexpr int W_ST = 6;
};
template <int T>
struct Shape : Cfg<T> {
  using Cfg<T>::BD;
  using Cfg<T>::BK;
  using Cfg<T>::W_ST;
  static constexpr int NPL = T;                           // operand planes = weight regions
  static constexpr int NC = T / 2 - 1;                    // complex frequencies
  static constexpr int ROWB = BK * 2;                     // bytes per operand row
  static constexpr int KSTEPS = BK / 16;
  static constexpr uint32_t PLANE_BYTES = BM * ROWB;
  static constexpr uint32_t WREG_BYTES = BD * ROWB;
  static constexpr uint32_t W_STAGE_BYTES = NPL * WREG_BYTES;
  static constexpr uint32_t OFF_X = 0;
  static constexpr uint32_t OFF_W = OFF_X + X_ST * X_STAGE_BYTES;
  static constexpr uint32_t OFF_STG = OFF_W + W_ST * W_STAGE_BYTES;
  static constexpr uint32_t OFF_BIAS = OFF_STG + kEpiWarps * kStgBytes;
  static constexpr uint32_t OFF_BAR = OFF_BIAS + kEpiWarps * 128;
  static constexpr uint32_t SMEM_BYTES = OFF_BAR + 512 + 1024;  // barriers + alignment slack
  static_assert(NPL * PLANE_BYTES == X_STAGE_BYTES, "planes replace the raw tile in place");
  static_assert(BK * T * 2 == 256, "a raw stage row is two 128-byte chunks");
  static_assert(T * BD == (int)kTmemCols, "accumulators fill TMEM");
  static_assert(SMEM_BYTES <= 232448, "shared memory budget");
};

template <int T>
struct Bars {
  uint64_t x_full[X_ST], x_read[X_ST], x_ready[X_ST], x_empty[X_ST];
  uint64_t w_full[Shape<T>::W_ST], w_empty[Shape<T>::W_ST];
  uint64_t acc_full, acc_empty, drain;
  uint32_t tmem_base;
  int abort_flag;
};


struct TileInfo {
  int n_dt;       // d tiles
  int num_tiles;  // row tiles x d tiles
  int k_stages;   // ceil(Cin / BK)
  int drop_w;     // fault injection for tests: CTA 0 never issues weight stage drop_w (-1: off)
};

// ---------------------------------------------------------------------------
// Transform: the raw stage is [row][128-byte chunk c][128 B], every 128-byte
// line L = 2r + c swizzled by (L % 8).  A thread reads eight 16-byte pieces and,
// once every transform warp holds its pieces, writes its share of the planes.
// Lane mapping: an 8-lane phase covers 4 rows x both chunks, so its swizzled
// reads and writes hit 8 distinct bank groups.
// ---------------------------------------------------------------------------
__device__ __forceinline__ float2 f2(uint32_t u) { return unpack_h2(u); }

// T = 4: a chunk holds 16 channels (2 per piece); a unit is one row x 8 channels
// (half hq of chunk c), two units per thread.
template <int T>
__device__ __forceinline__ void xf_read(const uint8_t* slot, int xt, uint4 (&v)[8]) {
  if constexpr (T == 4) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int unit = xt + 256 * u;
      const int c = unit & 1, r = (unit >> 1) & (BM - 1), hq = unit >> 8;
      const int line = 2 * r + c;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = hq * 4 + i;
        v[4 * u + i] = *reinterpret_cast<const uint4*>(slot + line * 128 + ((j ^ (line & 7)) << 4));
      }
    }
  } else {
    // T = 8: a chunk holds 8 channels (1 per piece); one unit = one line per thread
    const int c = xt & 1, r = (xt >> 1) & (BM - 1);
    const int line = 2 * r + c;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      v[j] = *reinterpret_cast<const uint4*>(slot + line * 128 + ((j ^ (line & 7)) << 4));
  }
}

template <int T>
__device__ __forceinline__ void xf_write(uint8_t* slot, int xt, const uint4 (&v)[8]) {
  using S = Shape<T>;
  if constexpr (T == 4) {
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int unit = xt + 256 * u;
      const int c = unit & 1, r = (unit >> 1) & (BM - 1), hq = unit >> 8;
      const int q = 2 * c + hq;
      // piece i holds channels 2i (.x = x0,x1  .y = x2,x3) and 2i+1 (.z, .w)
      uint32_t o0[4], o2[4], orr[4], oi[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        float f0[2], fh[2], fr[2], fi[2];
        const uint32_t w4[4] = {v[4 * u + i].x, v[4 * u + i].y, v[4 * u + i].z, v[4 * u + i].w};
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const float2 lo = f2(w4[2 * hh]), hi = f2(w4[2 * hh + 1]);
          const float x0 = lo.x, x1 = lo.y, x2 = hi.x, x3 = hi.y;
          const float a = x0 + x2, b = x1 + x3;
          f0[hh] = a + b;
          fh[hh] = a - b;
          fr[hh] = x0 - x2;
          fi[hh] = x3 - x1;
        }
        o0[i] = pack_h2(f0[0], f0[1]);
        o2[i] = pack_h2(fh[0], fh[1]);
        orr[i] = pack_h2(fr[0], fr[1]);
        oi[i] = pack_h2(fi[0], fi[1]);
      }
      // K-major 64 B rows: 16-byte piece q at (q ^ ((r / 2) % 4))
      const uint32_t off = r * 64 + ((q ^ ((r >> 1) & 3)) << 4);
      *reinterpret_cast<uint4*>(slot + 0 * S::PLANE_BYTES + off) = make_uint4(o0[0], o0[1], o0[2], o0[3]);
      *reinterpret_cast<uint4*>(slot + 1 * S::PLANE_BYTES + off) = make_uint4(o2[0], o2[1], o2[2], o2[3]);
      *reinterpret_cast<uint4*>(slot + 2 * S::PLANE_BYTES + off) =
          make_uint4(orr[0], orr[1], orr[2], orr[3]);
      *reinterpret_cast<uint4*>(slot + 3 * S::PLANE_BYTES + off) = make_uint4(oi[0], oi[1], oi[2], oi[3]);
    }
  } else {
    // T = 8: piece j = channel j of the chunk, x0..x7 in .x .y .z .w (pairs).
    // Radix-2: a_t = x_t + x_{t+4}, b_t = x_t - x_{t+4};
    //   X0 = a0+a1+a2+a3, X4 = a0-a1+a2-a3, X2 = (a0-a2) + i (a3-a1),
    //   X1 = b0 + h(b1-b3) + i(-b2 - h(b1+b3)),  X3 = b0 - h(b1-b3) + i(b2 - h(b1+b3)),
    // h = sqrt(2)/2; plane order X0, X4, Re X1, Im X1, Re X2, Im X2, Re X3, Im X3.
    const float h = 0.70710678118654752f;
    const int c = xt & 1, r = (xt >> 1) & (BM - 1);
    uint32_t o[8][4];  // [plane][channel pair]
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      float val[8][2];
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint4 w = v[2 * pr + hh];
        const float2 p01 = f2(w.x), p23 = f2(w.y), p45 = f2(w.z), p67 = f2(w.w);
        const float a0 = p01.x + p45.x, a1 = p01.y + p45.y, a2 = p23.x + p67.x, a3 = p23.y + p67.y;
        const float b0 = p01.x - p45.x, b1 = p01.y - p45.y, b2 = p23.x - p67.x, b3 = p23.y - p67.y;
        const float s13 = h * (b1 - b3), t13 = h * (b1 + b3);
        val[0][hh] = (a0 + a2) + (a1 + a3);
        val[1][hh] = (a0 + a2) - (a1 + a3);
        val[2][hh] = b0 + s13;
        val[3][hh] = -b2 - t13;
        val[4][hh] = a0 - a2;
        val[5][hh] = a3 - a1;
        val[6][hh] = b0 - s13;
        val[7][hh] = b2 - t13;
      }
#pragma unroll
      for (int p = 0; p < 8; ++p) o[p][pr] = pack_h2(val[p][0], val[p][1]);
    }
    // K-major 32 B rows: 16-byte piece c at (c ^ ((r / 4) % 2))
    const uint32_t off = r * 32 + ((c ^ ((r >> 2) & 1)) << 4);
#pragma unroll
    for (int p = 0; p < 8; ++p)
      *reinterpret_cast<uint4*>(slot + p * S::PLANE_BYTES + off) =
          make_uint4(o[p][0], o[p][1], o[p][2], o[p][3]);
  }
}

// ---------------------------------------------------------------------------
// Epilogue of 32/T out-channels (starting at tile column c0 = out-channel d0)
// for this lane's row: T accumulator planes -> inverse DFT + bias -> 64 bytes of
// FP16 output (four 16-byte pieces, in Y's channel-major, group-minor order).
// Plane p of out-channel c sits in TMEM column p * BD + c.
// ---------------------------------------------------------------------------
template <int T, int BD, int ACT>
__device__ __forceinline__ void epi_half(uint32_t lane_addr, int c0, const __half* bsm,
                                         uint4 (&o)[4]) {
  constexpr int NCH = 32 / T;
  uint32_t v[T][NCH];
#pragma unroll
  for (int p = 0; p < T; ++p) tmem_ld_32x32b<NCH>(lane_addr + p * BD + c0, v[p]);
  // the slice's biases (staged in shared memory before the accumulators were ready)
  float b[NCH];
  if constexpr (NCH == 8) {
    const uint4 bb = *reinterpret_cast<const uint4*>(bsm);
    const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = unpack_h2(bw[i]);
      b[2 * i] = f.x;
      b[2 * i + 1] = f.y;
    }
  } else {
    const uint2 bb = *reinterpret_cast<const uint2*>(bsm);
    const float2 f0 = unpack_h2(bb.x), f1 = unpack_h2(bb.y);
    b[0] = f0.x; b[1] = f0.y; b[2] = f1.x; b[3] = f1.y;
  }
  tmem_wait_ld();
  if constexpr (T == 4) {
    // accumulators arrive scaled (Y0/4, Y2/4, Yr/2, Yi/2):
    // y0 = Y0'+Y2'+Yr', y1 = Y0'-Y2'-Yi', y2 = Y0'+Y2'-Yr', y3 = Y0'-Y2'+Yi' (+ bias)
    uint32_t w[2 * NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const float s = __uint_as_float(v[0][i]) + b[i];
      const float y2 = __uint_as_float(v[1][i]);
      const float yr = __uint_as_float(v[2][i]), yi = __uint_as_float(v[3][i]);
      const float e = s + y2, od = s - y2;
      w[2 * i] = pack_h2(act_fn<ACT>(e + yr), act_fn<ACT>(od - yi));
      w[2 * i + 1] = pack_h2(act_fn<ACT>(e - yr), act_fn<ACT>(od + yi));
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) o[m] = make_uint4(w[4 * m], w[4 * m + 1], w[4 * m + 2], w[4 * m + 3]);
  } else {
    // accumulators arrive scaled (frequencies 0 and 4 by 1/8, complex by 1/4);
    // y_s = A_s + B_s, y_{s+4} = A_s - B_s (A: frequencies 0, 2, 4; B: 1, 3)
    const float h = 0.70710678118654752f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      float Yv[8];
#pragma unroll
      for (int p = 0; p < 8; ++p) Yv[p] = __uint_as_float(v[p][i]);
      const float s = Yv[0] + b[i];
      const float E = s + Yv[1], O = s - Yv[1];
      const float A0 = E + Yv[4], A2 = E - Yv[4];
      const float A1 = O - Yv[5], A3 = O + Yv[5];
      const float B0 = Yv[2] + Yv[6];
      const float B1 = h * (Yv[2] - Yv[3] - Yv[6] - Yv[7]);
      const float B2 = Yv[7] - Yv[3];
      const float B3 = h * (-Yv[2] - Yv[3] + Yv[6] - Yv[7]);
      o[i] = make_uint4(pack_h2(act_fn<ACT>(A0 + B0), act_fn<ACT>(A1 + B1)),
                        pack_h2(act_fn<ACT>(A2 + B2), act_fn<ACT>(A3 + B3)),
                        pack_h2(act_fn<ACT>(A0 - B0), act_fn<ACT>(A1 - B1)),
                        pack_h2(act_fn<ACT>(A2 - B2), act_fn<ACT>(A3 - B3)));
    }
  }
}

// T = 4 epilogue of 8 out-channels written as the NEXT layer's input in the
// frequency domain: per channel the four outputs y_s = act(IDFT + bias) are
// transformed again, X0 = y0+y1+y2+y3, X2 = y0-y1+y2-y3, Xr = y0-y2, Xi = y3-y1
// (FP32, one rounding to FP16); o[p] = plane p of the 8 channels (16 bytes).
template <int BD, int ACT>
__device__ __forceinline__ void epi_half_spec(uint32_t lane_addr, int c0, const __half* bsm,
                                              uint4 (&o)[4]) {
  uint32_t v[4][8];
#pragma unroll
  for (int p = 0; p < 4; ++p) tmem_ld_32x32b<8>(lane_addr + p * BD + c0, v[p]);
  const uint4 bb = *reinterpret_cast<const uint4*>(bsm);
  const uint32_t bw[4] = {bb.x, bb.y, bb.z, bb.w};
  tmem_wait_ld();
  uint32_t pl[4][4];
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    const float2 bf = unpack_h2(bw[m]);
    float q[4][2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int i = 2 * m + e;
      const float sb = __uint_as_float(v[0][i]) + (e ? bf.y : bf.x);
      const float y2 = __uint_as_float(v[1][i]);
      const float yr = __uint_as_float(v[2][i]), yi = __uint_as_float(v[3][i]);
      const float ev = sb + y2, od = sb - y2;
      const float z0 = act_fn<ACT>(ev + yr), z1 = act_fn<ACT>(od - yi);
      const float z2 = act_fn<ACT>(ev - yr), z3 = act_fn<ACT>(od + yi);
      const float a = z0 + z2, b = z1 + z3;
      q[0][e] = a + b;
      q[1][e] = a - b;
      q[2][e] = z0 - z2;
      q[3][e] = z3 - z1;
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) pl[p][m] = pack_h2(q[p][0], q[p][1]);
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) o[p] = make_uint4(pl[p][0], pl[p][1], pl[p][2], pl[p][3]);
}

template <int T, int ACT, int IO>
__global__ void __launch_bounds__(kThreads, 1)
    eq_fwd_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                     const __grid_constant__ CUtensorMap map_y, const uint8_t* __restrict__ wtiles,
                     const __half* __restrict__ bias, int64_t N, int Cin, int Cout, TileInfo ti,
                     int* status) {
  using S = Shape<T>;
  constexpr int BD = S::BD;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  // 1024-byte alignment for the swizzled TMA destinations and operand tiles
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars<T>* bars = reinterpret_cast<Bars<T>*>(smem + S::OFF_BAR);
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < X_ST; ++s) {
      mbar_init(&bars->x_full[s], 1);          // raw tile landed (TMA bytes)
      mbar_init(&bars->x_read[s], kXfWarps);   // every transform warp holds its raw pieces
      mbar_init(&bars->x_ready[s], kXfWarps);  // operand planes written (transform warps)
      mbar_init(&bars->x_empty[s], 1);         // MMAs done with the planes (tcgen05.commit)
    }
    for (int s = 0; s < S::W_ST; ++s) {
      mbar_init(&bars->w_full[s], 1);
      mbar_init(&bars->w_empty[s], 1);
    }
    mbar_init(&bars->acc_full, 1);
    mbar_init(&bars->acc_empty, kEpiWarps * 32);
    mbar_init(&bars->drain, 1);
    bars->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0 || warp == 2) {
    // ------- producers: warp 0 raw X (TMA, 3-D box), warp 2 weight tiles (bulk copy) -------
    if (lane == 0) {
      const bool is_raw = (warp == 0);
      const int depth = is_raw ? X_ST : S::W_ST;
      uint64_t* full = is_raw ? bars->x_full : bars->w_full;
      uint64_t* empty = is_raw ? bars->x_empty : bars->w_empty;
      int issued_phase[X_ST > S::W_ST ? X_ST : S::W_ST];  // last phase issued per slot
      for (int s = 0; s < depth; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ti.num_tiles; tile += gridDim.x) {
        const int row0 = (tile / ti.n_dt) * BM;
        const int dt = tile % ti.n_dt;
        for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
          const int s = it % depth;
          const uint32_t ph = (it / depth) & 1;
          if (!(ok = wait_bounded(&empty[s], ph ^ 1, abort_flag, status))) break;
          if (!is_raw && blockIdx.x == 0 && (int)it == ti.drop_w) continue;  // injected fault
          if (is_raw) {
            mbar_expect_tx(&full[s], X_STAGE_BYTES);
            if constexpr (IO == kIoSpectralIn) {
              // planes [4][N][Cin] of the previous layer: (32 channels, 128 rows, 4 planes)
              // land as the four K-major 64-byte-swizzled operand planes of this stage
              tma_load_3d(sbase + S::OFF_X + s * X_STAGE_BYTES, &map_x, &full[s], S::BK * ks,
                          row0, 0);
            } else {
              // 3-D view of X: (64 halves, 128-byte chunk of the row, row); a stage is
              // chunks 2ks, 2ks+1 of 128 rows
              tma_load_3d(sbase + S::OFF_X + s * X_STAGE_BYTES, &map_x, &full[s], 0, 2 * ks,
                          row0);
            }
          } else {
            // one pre-arranged blob per (out-channel tile, K stage)
            mbar_expect_tx(&full[s], S::W_STAGE_BYTES);
            const size_t blob = (size_t)dt * ti.k_stages + ks;
            bulk_load(sbase + S::OFF_W + s * S::W_STAGE_BYTES, wtiles + blob * S::W_STAGE_BYTES,
                      S::W_STAGE_BYTES, &full[s]);
          }
          issued_phase[s] = (int)ph;
        }
      }
      if (!ok) {
        // wait (bounded) for the copies this thread put in flight
        for (int s = 0; s < depth; ++s)
          if (issued_phase[s] >= 0) drain_wait(&full[s], (uint32_t)issued_phase[s]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      const uint32_t id_n1 = idesc_f16(BM, BD);
      const uint32_t id_n1_neg = idesc_f16(BM, BD, true);
      const uint32_t id_n2 = idesc_f16(BM, 2 * BD);
      for (int tile = blockIdx.x; ok && tile < ti.num_tiles; tile += gridDim.x, ++tcount) {
        if (!(ok = wait_bounded(&bars->acc_empty, (tcount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
          const int sx = it % X_ST, sw = it % S::W_ST;
          uint64_t* xbar = (IO == kIoSpectralIn) ? &bars->x_full[sx] : &bars->x_ready[sx];
          if (!(ok = wait_bounded(xbar, (it / X_ST) & 1, abort_flag, status))) break;
          if (!(ok = wait_bounded(&bars->w_full[sw], (it / S::W_ST) & 1, abort_flag, status)))
            break;
          tc_fence_after();
          const uint32_t pl = sbase + S::OFF_X + sx * X_STAGE_BYTES;     // planes
          const uint32_t wr = sbase + S::OFF_W + sw * S::W_STAGE_BYTES;  // weight regions
#pragma unroll
          for (int kk = 0; kk < S::KSTEPS; ++kk) {
            const uint32_t ko = 32u * kk;  // byte offset of this K step inside the rows
            const uint32_t acc = (ks > 0 || kk > 0) ? 1u : 0u;
            auto A = [&](int p) { return desc_kmajor<S::ROWB>(pl + p * S::PLANE_BYTES + ko); };
            auto B = [&](int p) { return desc_kmajor<S::ROWB>(wr + p * S::WREG_BYTES + ko); };
            // real frequencies 0 and T/2
            umma(tmem + 0, A(0), B(0), id_n1, acc);
            umma(tmem + BD, A(1), B(1), id_n1, acc);
            // complex frequencies: [Y_kr|Y_ki] += Xr_k [Br_k|Bi_k]^T ;
            // Y_kr += (-Xi_k) Bi_k^T ; Y_ki += Xi_k Br_k^T
#pragma unroll
            for (int k = 1; k <= S::NC; ++k) {
              const uint32_t col = 2 * BD * k;
              umma(tmem + col, A(2 * k), B(2 * k), id_n2, acc);
              umma(tmem + col, A(2 * k + 1), B(2 * k + 1), id_n1_neg, 1u);
              umma(tmem + col + BD, A(2 * k + 1), B(2 * k), id_n1, 1u);
            }
          }
          umma_commit(&bars->x_empty[sx]);
          umma_commit(&bars->w_empty[sw]);
        }
        if (ok) umma_commit(&bars->acc_full);
      }
      // all MMAs this thread issued must be complete before TMEM is freed
      umma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
    // ---------------- epilogue ----------------
    // Warp w reads TMEM lane quarter q = w % 4 (rows 32q..32q+31 of the tile) and
    // out-channel half ch.  The half goes out in slices of 64/T out-channels: a
    // slice row is 128 contiguous bytes of Y, staged in the warp's 4 KB buffer
    // (128-byte swizzle) and written by one TMA store, so TMEM is free for the
    // next tile as soon as its last slice is read, while the stores drain.
    const int q = warp & 3;
    const int ch = (warp - kEpiWarp0) >> 2;
    uint8_t* stg = smem + S::OFF_STG + (warp - kEpiWarp0) * kStgBytes;
    const uint32_t stg_s = smem_u32(stg);
    uint8_t* my_row = stg + lane * 128;
    __half* bsm = reinterpret_cast<__half*>(smem + S::OFF_BIAS + (warp - kEpiWarp0) * 128);
    constexpr int kSliceCh = 64 / T;
    constexpr int kSlices = (BD / 2) / kSliceCh;
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < ti.num_tiles; tile += gridDim.x, ++tcount) {
      const int64_t row0 = (int64_t)(tile / ti.n_dt) * BM + 32 * q;
      const int dbase = (tile % ti.n_dt) * BD + (BD / 2) * ch;
      // stage this warp's BD/2 biases while the mainloop runs (lane l: channels 2l, 2l+1)
      if (2 * lane < BD / 2) {
        const int d = dbase + 2 * lane;
        uint32_t v = 0u;
        if (bias && d < Cout) v = *reinterpret_cast<const uint32_t*>(bias + d);  // Cout even
        reinterpret_cast<uint32_t*>(bsm)[lane] = v;
      }
      __syncwarp();
      if (!warp_wait(&bars->acc_full, tcount & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
#pragma unroll 1
      for (int sc = 0; sc < kSlices; ++sc) {
        const int c0 = (BD / 2) * ch + sc * kSliceCh;  // column in the tile
        const int d0 = dbase + sc * kSliceCh;          // out-channel
        if (d0 >= Cout) break;  // warp-uniform: Cout is a multiple of 16
        const __half* bs = bsm + sc * kSliceCh;
        if constexpr (IO == kIoSpectralOut) {
          // staging [plane][32 rows][32 B], 32-byte swizzle (16-byte piece ^ (row / 4) % 2)
          uint4 o[4];
          epi_half_spec<BD, ACT>(lane_addr, c0, bs, o);
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
          const int sw = (lane >> 2) & 1;
#pragma unroll
          for (int p = 0; p < 4; ++p)
            *reinterpret_cast<uint4*>(stg + p * 1024 + lane * 32 + ((0 ^ sw) << 4)) = o[p];
          epi_half_spec<BD, ACT>(lane_addr, c0 + 8, bs + 8, o);
#pragma unroll
          for (int p = 0; p < 4; ++p)
            *reinterpret_cast<uint4*>(stg + p * 1024 + lane * 32 + ((1 ^ sw) << 4)) = o[p];
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          __syncwarp();
          if (lane == 0) {
            if (row0 < N) tma_store_3d(&map_y, stg_s, d0, (int)row0, 0);
            bulk_commit();
          }
          continue;
        }
        uint4 o[4];
        epi_half<T, BD, ACT>(lane_addr, c0, bs, o);
        // the previous slice's store has finished reading the buffer
        if (lane == 0) bulk_wait_read_all();
        __syncwarp();
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4*>(my_row + ((m ^ (lane & 7)) << 4)) = o[m];
        epi_half<T, BD, ACT>(lane_addr, c0 + 32 / T, bs + 32 / T, o);
#pragma unroll
        for (int m = 0; m < 4; ++m)
          *reinterpret_cast<uint4*>(my_row + (((4 + m) ^ (lane & 7)) << 4)) = o[m];
        // generic-proxy writes -> visible to the TMA (async proxy), then one store
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
          if (row0 < N) tma_store_3d(&map_y, stg_s, 0, d0 * T / 64, (int)row0);
          bulk_commit();
        }
      }
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  } else if (warp >= kXfWarp0 && IO != kIoSpectralIn) {
    // ---------------- transform: group DFT into the operand planes ----------------
    const int xt = threadIdx.x - kXfWarp0 * 32;  // 0..255
    uint32_t it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < ti.num_tiles; tile += gridDim.x) {
      for (int ks = 0; ks < ti.k_stages; ++ks, ++it) {
        const int sx = it % X_ST;
        if (!(ok = warp_wait(&bars->x_full[sx], (it / X_ST) & 1, abort_flag, status))) break;
        uint8_t* slot = smem + S::OFF_X + sx * X_STAGE_BYTES;
        uint4 v[8];
        xf_read<T>(slot, xt, v);
        // every raw piece of the slot is in registers before any plane overwrites it
        // (an mbarrier rather than a named barrier, so the wait stays bounded)
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->x_read[sx]);
        if (!(ok = warp_wait(&bars->x_read[sx], (it / X_ST) & 1, abort_flag, status))) break;
        xf_write<T>(slot, xt, v);
        // make the generic-proxy stores visible to the tensor core (async proxy)
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars->x_ready[sx]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}


// Re-arrange prepared planes [P][Cout][Cin] into the kernel's per-stage weight
// image: blob (dt, ks) = regions 0..T-1 (prepared planes 0..T-1: real frequency
// 0, real frequency T/2, then Re and Im of each complex frequency), each BD rows
// x BK channels in the K-major swizzled layout the MMAs read; rows and channels
// past the matrix are zero.  One thread per 16-byte piece.
template <int T>
__global__ void tile_weights_kernel(const __half* __restrict__ planes, int Cin, int Cout,
                                    int n_ks, int64_t n_chunks, uint4* __restrict__ tiles) {
  using S = Shape<T>;
  constexpr int kPieces = S::ROWB / 16;  // 16-byte pieces per row
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= n_chunks) return;
  const int piece = (int)(idx % kPieces);
  const int r = (int)((idx / kPieces) % S::BD);
  const int region = (int)((idx / kPieces) / S::BD % S::NPL);
  const int64_t blob = (idx / kPieces) / S::BD / S::NPL;
  const int dt = (int)(blob / n_ks), ks = (int)(blob % n_ks);
  const int d = dt * S::BD + r, c0 = ks * S::BK + piece * 8;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (d < Cout && c0 < Cin) {  // Cin % 16 == 0: the 8 channels are all in range
    v = *reinterpret_cast<const uint4*>(planes + ((int64_t)region * Cout + d) * Cin + c0);
    // the inverse DFT's factors 1/T (real frequencies) and 2/T (complex), exact
    // powers of two, applied here so the epilogue needs no multiplies by them
    const __half2 s = __float2half2_rn(region < 2 ? 1.f / T : 2.f / T);
    __half2* h = reinterpret_cast<__half2*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) h[i] = __hmul2(h[i], s);
  }
  // swizzle: piece ^= (byte offset of the row >> 7) within the swizzle span
  const int swz = ((r * S::ROWB) >> 7) & (kPieces - 1);
  const int64_t dst_byte = blob * S::W_STAGE_BYTES + (int64_t)region * S::WREG_BYTES +
                           r * S::ROWB + ((piece ^ swz) << 4);
  tiles[dst_byte >> 4] = v;
}

template <typename F>
cudaError_t dispatch_tc(int T, F&& f) {
  if (T == 4) return f(std::integral_constant<int, 4>{});
  if (T == 8) return f(std::integral_constant<int, 8>{});
  return cudaErrorNotSupported;
}

}  // namespace

bool fwd_tc_supported(int T, DType dt, int64_t N, int Cin, int Cout) {
  return (T == 4 || T == 8) && dt == DType::F16 && N >= 1 && N <= 0x7fffff80LL &&
         Cin % 16 == 0 && Cout % 16 == 0 && Cin >= 16 && Cout >= 16;
}

bool tc_tiles_wanted(int T, DType dt, int C, int D) {
  return (T == 4 || T == 8) && dt == DType::F16 && C % 16 == 0 && D % 16 == 0 && C >= 16 &&
         D >= 16;
}

size_t tc_tile_bytes(int T, int Cin, int Cout) {
  size_t bytes = 0;
  dispatch_tc(T, [&](auto tcst) {
    using S = Shape<decltype(tcst)::value>;
    const size_t n_dt = (size_t)(Cout + S::BD - 1) / S::BD, n_ks = (size_t)(Cin + S::BK - 1) / S::BK;
    bytes = n_dt * n_ks * S::W_STAGE_BYTES;
    return cudaSuccess;
  });
  return bytes;
}

cudaError_t launch_tile_weights(int T, const void* planes, int Cin, int Cout, void* tiles,
                                cudaStream_t st) {
  return dispatch_tc(T, [&](auto tcst) {
    constexpr int TT = decltype(tcst)::value;
    using S = Shape<TT>;
    const int n_ks = (Cin + S::BK - 1) / S::BK;
    const int64_t n_chunks = (int64_t)tc_tile_bytes(TT, Cin, Cout) / 16;
    const unsigned blocks = (unsigned)((n_chunks + 255) / 256);
    tile_weights_kernel<TT><<<blocks, 256, 0, st>>>(static_cast<const __half*>(planes), Cin, Cout,
                                                    n_ks, n_chunks, static_cast<uint4*>(tiles));
    return cudaGetLastError();
  });
}

namespace {

// Spectral planes [4][N][channels] (FP16), viewed as (channel, row, plane).
bool encode_planes_map(CUtensorMap* m, void* base, int channels, int64_t N, uint32_t box_ch,
                       uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto encode = encode_fn();
  cuuint64_t dims[3] = {(cuuint64_t)channels, (cuuint64_t)N, 4};
  cuuint64_t strides[2] = {(cuuint64_t)channels * 2, (cuuint64_t)N * channels * 2};
  cuuint32_t box[3] = {box_ch, box_rows, 4};
  cuuint32_t estr[3] = {1, 1, 1};
  return encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, base, dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int TT, int ACT, int IO>
cudaError_t set_smem_attr() {
  return cudaFuncSetAttribute(eq_fwd_tc_kernel<TT, ACT, IO>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, Shape<TT>::SMEM_BYTES);
}

}  // namespace

cudaError_t launch_fwd_tc(int T, const void* X, int64_t N, int Cin, int Cout,
                          const void* Wtiles, const void* bias, void* Y, int* status,
                          int num_sms, int drop_w_stage, int act, int io, cudaStream_t st) {
  if (!fwd_tc_supported(T, DType::F16, N, Cin, Cout)) return cudaErrorNotSupported;
  if (!Wtiles) return cudaErrorNotSupported;
  if (io != kIoSpatial && T != 4) return cudaErrorNotSupported;
  if (act != 0 && act != 1) return cudaErrorInvalidValue;

  auto encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  return dispatch_tc(T, [&](auto tcst) {
    constexpr int TT = decltype(tcst)::value;
    using S = Shape<TT>;
    cuuint32_t estr[3] = {1, 1, 1};
    CUtensorMap mx;
    if (io == kIoSpectralIn) {
      // planes of the previous layer: box = 32 channels (64 B) x 128 rows x 4 planes
      if (!encode_planes_map(&mx, const_cast<void*>(X), Cin, N, S::BK, BM,
                             CU_TENSOR_MAP_SWIZZLE_64B))
        return cudaErrorInvalidValue;
    } else {
      // X row = Cin*T/64 chunks of 64 halves (128 B); box = 2 chunks x 128 rows
      cuuint64_t dims[3] = {64, (cuuint64_t)Cin * TT / 64, (cuuint64_t)N};
      cuuint64_t strides[2] = {128, (cuuint64_t)Cin * TT * 2};
      cuuint32_t box[3] = {64, 2, BM};
      if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(X), dims, strides,
                 box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    CUtensorMap my;
    if (io == kIoSpectralOut) {
      // planes for the next layer: store box = 16 channels (32 B) x 32 rows x 4 planes
      if (!encode_planes_map(&my, Y, Cout, N, 16, 32, CU_TENSOR_MAP_SWIZZLE_32B))
        return cudaErrorInvalidValue;
    } else {
      // Y row = Cout*T/64 chunks of 128 B; store box = 1 chunk x 32 rows
      cuuint64_t ydims[3] = {64, (cuuint64_t)Cout * TT / 64, (cuuint64_t)N};
      cuuint64_t ystrides[2] = {128, (cuuint64_t)Cout * TT * 2};
      cuuint32_t ybox[3] = {64, 1, 32};
      if (encode(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, Y, ydims, ystrides, ybox, estr,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    }
    TileInfo ti;
    ti.n_dt = (Cout + S::BD - 1) / S::BD;
    const int64_t n_rt = (N + BM - 1) / BM;
    if (n_rt * ti.n_dt > 0x7fffffffLL) return cudaErrorInvalidValue;
    ti.num_tiles = (int)(n_rt * ti.n_dt);
    ti.k_stages = (Cin + S::BK - 1) / S::BK;
    ti.drop_w = drop_w_stage;
    static bool attr_set = false;
    if (!attr_set) {
      cudaError_t e = set_smem_attr<TT, 0, kIoSpatial>();
      if (e == cudaSuccess) e = set_smem_attr<TT, 1, kIoSpatial>();
      if constexpr (TT == 4) {
        if (e == cudaSuccess) e = set_smem_attr<TT, 0, kIoSpectralOut>();
        if (e == cudaSuccess) e = set_smem_attr<TT, 1, kIoSpectralOut>();
        if (e == cudaSuccess) e = set_smem_attr<TT, 0, kIoSpectralIn>();
        if (e == cudaSuccess) e = set_smem_attr<TT, 1, kIoSpectralIn>();
      }
      if (e != cudaSuccess) return e;
      attr_set = true;
    }
    const int grid = ti.num_tiles < num_sms ? ti.num_tiles : num_sms;
    auto kernel = act == 1 ? eq_fwd_tc_kernel<TT, 1, kIoSpatial> : eq_fwd_tc_kernel<TT, 0, kIoSpatial>;
    if constexpr (TT == 4) {
      if (io == kIoSpectralOut)
        kernel = act == 1 ? eq_fwd_tc_kernel<TT, 1, kIoSpectralOut>
                          : eq_fwd_tc_kernel<TT, 0, kIoSpectralOut>;
      else if (io == kIoSpectralIn)
        kernel = act == 1 ? eq_fwd_tc_kernel<TT, 1, kIoSpectralIn>
                          : eq_fwd_tc_kernel<TT, 0, kIoSpectralIn>;
    }
    kernel<<<grid, kThreads, S::SMEM_BYTES, st>>>(
        mx, my, static_cast<const uint8_t*>(Wtiles), static_cast<const __half*>(bias), N, Cin,
        Cout, ti, status);
    return cudaGetLastError();
  });
}

}  // namespace eql
