// Device-side parts of the tcgen05/TMEM EQ-Linear forward shared by the
// one-layer kernel (eql_tc_fwd.cu) and the two-layer kernel (eql_tc_chain.cu):
// tile shapes, the shared-memory barrier block, the group-DFT transform of a
// staged X tile into operand planes, and the inverse-DFT epilogue.
#pragma once

#include <type_traits>

#include "eql_tc_common.cuh"

namespace eql {
namespace ftc {

using namespace tc;

constexpr int BM = 128;          // rows per tile = MMA M
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
// kIoSaveSpectrum: spatial X and Y, and the input's group spectrum (the operand
// planes the transform makes) also written to [4][N][Cin], for a later weight
// gradient.
constexpr int kIoSpatial = 0, kIoSpectralOut = 1, kIoSpectralIn = 2, kIoSaveSpectrum = 3;

// Per-group shape of the pipeline.
template <int T>
struct Cfg;
template <>
struct Cfg<4> {
  static constexpr int BD = 128;        // out-channels per tile
  static constexpr int BK = 32;         // in-channels per stage (two MMA K steps)
  // X ring (raw tile in, operand planes out, in place) and weight-tile ring:
  // weight stages are plain bulk copies from L2 and need less lead than the
  // X stages, which also wait for the transform (4/2 measured 1-2 % faster than
  // 3/3 in the same 192 KB)
  static constexpr int X_ST = 4;
  static constexpr int W_ST = 2;
};
template <>
struct Cfg<8> {
  static constexpr int BD = 64;
  static constexpr int BK = 16;         // one MMA K step
  static constexpr int X_ST = 3;
  static constexpr int W_ST = 6;
};
template <int T>
struct Shape : Cfg<T> {
  using Cfg<T>::BD;
  using Cfg<T>::BK;
  using Cfg<T>::X_ST;
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
  static constexpr int X_ST = Shape<T>::X_ST;
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
  // Work units: [0, full) are whole tiles; the remaining tiles (the last partial
  // wave) are split into two 64-row halves each, so that wave spreads over twice
  // as many SMs: num_units = full + 2 * (num_tiles - full).
  int full;
  int num_units;
};

// Position of work unit u: first row, out-channel tile, and which half
// (-1: the whole 128-row tile; 0, 1: rows 0-63, 64-127, computed with M = 64 MMAs).
struct UnitPos {
  int64_t row0;
  int dt, half;
};
__device__ __forceinline__ UnitPos unit_pos(int u, const TileInfo& ti) {
  int tile, half;
  if (u < ti.full) {
    tile = u;
    half = -1;
  } else {
    const int h = u - ti.full;
    tile = ti.full + (h >> 1);
    half = h & 1;
  }
  UnitPos p;
  p.dt = tile % ti.n_dt;
  p.half = half;
  p.row0 = (int64_t)(tile / ti.n_dt) * BM + (half > 0 ? 64 : 0);
  return p;
}

// ---------------------------------------------------------------------------
// Transform: the raw stage is [row][128-byte chunk c][128 B], every 128-byte
// line L = 2r + c swizzled by (L % 8).  A thread reads eight 16-byte pieces and,
// once every transform warp holds its pieces, writes its share of the planes.
// Lane mapping: an 8-lane phase covers 4 rows x both chunks, so its swizzled
// reads and writes hit 8 distinct bank groups.  The planes are the DFT times
// 1/T (T = 4, 8: exact), so an FP16 plane never exceeds the largest input
// magnitude; the weight planes carry the same factor and the epilogue
// multiplies it out.
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

// G = 1 (T = 8 layout): the group is the dihedral group D4, element g = a + 4b
// for r^a m^b; the planes are its Fourier coefficients (below).
template <int T, int G = 0>
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
          // stored planes carry 1/4 (exact), so |plane| <= max|x|
          const float a = x0 + x2, b = x1 + x3;
          f0[hh] = (a + b) * 0.25f;
          fh[hh] = (a - b) * 0.25f;
          fr[hh] = (x0 - x2) * 0.25f;
          fi[hh] = (x3 - x1) * 0.25f;
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
        if constexpr (G == 1) {
          // D4: X^(rho) = sum_g x_g rho(g).  Characters chi(r) = +-1, chi(m) = +-1
          // (planes 0..3: (+,+), (+,-), (-,+), (-,-)); the 2 x 2 representation
          // r -> [[0,-1],[1,0]], m -> diag(1,-1) (planes 4..7: entries 00, 01, 10, 11).
          const float e0 = p01.x + p23.x, o0 = p01.y + p23.y;  // x0+x2, x1+x3
          const float e1 = p45.x + p67.x, o1 = p45.y + p67.y;  // x4+x6, x5+x7
          const float d0 = p01.x - p23.x, d1 = p01.y - p23.y;  // x0-x2, x1-x3
          const float d4 = p45.x - p67.x, d5 = p45.y - p67.y;  // x4-x6, x5-x7
          val[0][hh] = (e0 + o0) + (e1 + o1);
          val[1][hh] = (e0 + o0) - (e1 + o1);
          val[2][hh] = (e0 - o0) + (e1 - o1);
          val[3][hh] = (e0 - o0) - (e1 - o1);
          val[4][hh] = d0 + d4;
          val[5][hh] = d5 - d1;
          val[6][hh] = d1 + d5;
          val[7][hh] = d0 - d4;
          continue;
        }
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
      // stored planes carry 1/8 (exact), so |plane| <= max|x|
#pragma unroll
      for (int p = 0; p < 8; ++p) o[p][pr] = pack_h2(val[p][0] * 0.125f, val[p][1] * 0.125f);
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
template <int T, int BD, int ACT, int G = 0>
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
    // Both operands carry 1/4, so the accumulators hold Y/16; the exact factors 4
    // (real frequencies) and 8 (complex) give the inverse transform's scaled terms
    // Y0' = Y0/4, Y2' = Y2/4, Yr' = Yr/2, Yi' = Yi/2:
    // y0 = Y0'+Y2'+Yr', y1 = Y0'-Y2'-Yi', y2 = Y0'+Y2'-Yr', y3 = Y0'-Y2'+Yi' (+ bias)
    uint32_t w[2 * NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      const float s = fmaf(4.f, __uint_as_float(v[0][i]), b[i]);
      const float y2 = 4.f * __uint_as_float(v[1][i]);
      const float yr = 8.f * __uint_as_float(v[2][i]), yi = 8.f * __uint_as_float(v[3][i]);
      const float e = s + y2, od = s - y2;
      w[2 * i] = pack_h2(act_fn<ACT>(e + yr), act_fn<ACT>(od - yi));
      w[2 * i + 1] = pack_h2(act_fn<ACT>(e - yr), act_fn<ACT>(od + yi));
    }
#pragma unroll
    for (int m = 0; m < 4; ++m) o[m] = make_uint4(w[4 * m], w[4 * m + 1], w[4 * m + 2], w[4 * m + 3]);
  } else {
    // Both operands carry 1/8, so the accumulators hold Y/64; the exact factors 8
    // (frequencies 0 and 4) and 16 (complex) give the inverse transform's terms
    // Y/8 and Y/4.  y_s = A_s + B_s, y_{s+4} = A_s - B_s (A: frequencies 0, 2, 4;
    // B: 1, 3)
    const float h = 0.70710678118654752f;
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
      float Yv[8];
      // cyclic T = 8: planes 0, 1 real; D4: planes 0..3 characters (both x 8)
      constexpr int kReal = (G == 1) ? 4 : 2;
#pragma unroll
      for (int p = 0; p < 8; ++p) Yv[p] = (p < kReal ? 8.f : 16.f) * __uint_as_float(v[p][i]);
      if constexpr (G == 1) {
        // D4, after the factors: characters' terms Y/8, the 2 x 2 block's Y/4:
        // y(g) = sum_p chi_p(g) c_p + sum_{i,k} rho(g)_ik m_ik  (+ bias), g = a + 4b
        const float s = Yv[0] + b[i];
        const float P = s + Yv[2], Q = s - Yv[2], U = Yv[1] + Yv[3], V = Yv[1] - Yv[3];
        const float E = Yv[4] + Yv[7], F = Yv[6] - Yv[5], Gm = Yv[4] - Yv[7],
                    H = Yv[5] + Yv[6];
        o[i] = make_uint4(pack_h2(act_fn<ACT>(P + U + E), act_fn<ACT>(Q + V + F)),
                          pack_h2(act_fn<ACT>(P + U - E), act_fn<ACT>(Q + V - F)),
                          pack_h2(act_fn<ACT>(P - U + Gm), act_fn<ACT>(Q - V + H)),
                          pack_h2(act_fn<ACT>(P - U - Gm), act_fn<ACT>(Q - V - H)));
        continue;
      }
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
// transformed again, X0 = y0+y1+y2+y3, X2 = y0-y1+y2-y3, Xr = y0-y2, Xi = y3-y1,
// each times 1/4 (FP32, one rounding to FP16); o[p] = plane p of the 8 channels
// (16 bytes).
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
      // accumulators hold Y/16: factors 4 and 8 as in epi_half
      const float sb = fmaf(4.f, __uint_as_float(v[0][i]), e ? bf.y : bf.x);
      const float y2 = 4.f * __uint_as_float(v[1][i]);
      const float yr = 8.f * __uint_as_float(v[2][i]), yi = 8.f * __uint_as_float(v[3][i]);
      const float ev = sb + y2, od = sb - y2;
      const float z0 = act_fn<ACT>(ev + yr), z1 = act_fn<ACT>(od - yi);
      const float z2 = act_fn<ACT>(ev - yr), z3 = act_fn<ACT>(od + yi);
      // the next layer's planes carry 1/4 like every stored plane
      const float a = z0 + z2, b = z1 + z3;
      q[0][e] = (a + b) * 0.25f;
      q[1][e] = (a - b) * 0.25f;
      q[2][e] = (z0 - z2) * 0.25f;
      q[3][e] = (z3 - z1) * 0.25f;
    }
#pragma unroll
    for (int p = 0; p < 4; ++p) pl[p][m] = pack_h2(q[p][0], q[p][1]);
  }
#pragma unroll
  for (int p = 0; p < 4; ++p) o[p] = make_uint4(pl[p][0], pl[p][1], pl[p][2], pl[p][3]);
}

// Epilogue of one tile for one epilogue warp: its TMEM lane quarter (lane_addr),
// out-channel half ch, in slices of 64/T out-channels (16 channels for spectral
// output); each slice is staged in the warp's 4 KB buffer and written by one TMA
// store, store(staging address, first out-channel of the slice), issued by lane 0.
// bsm holds the half's biases; dbase is the half's first out-channel.
template <int T, int BD, int ACT, int IO, class Store, int G = 0>
__device__ __forceinline__ void epi_slices(uint32_t lane_addr, int ch, int lane, uint8_t* stg,
                                           const __half* bsm, int dbase, int Cout,
                                           const Store& store) {
  constexpr int kSliceCh = 64 / T;
  constexpr int kSlices = (BD / 2) / kSliceCh;
  const uint32_t stg_s = smem_u32(stg);
  uint8_t* my_row = stg + lane * 128;
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
        store(stg_s, d0);
        bulk_commit();
      }
      continue;
    }
    uint4 o[4];
    epi_half<T, BD, ACT, G>(lane_addr, c0, bs, o);
    // the previous slice's store has finished reading the buffer
    if (lane == 0) bulk_wait_read_all();
    __syncwarp();
#pragma unroll
    for (int m = 0; m < 4; ++m)
      *reinterpret_cast<uint4*>(my_row + ((m ^ (lane & 7)) << 4)) = o[m];
    epi_half<T, BD, ACT, G>(lane_addr, c0 + 32 / T, bs + 32 / T, o);
#pragma unroll
    for (int m = 0; m < 4; ++m)
      *reinterpret_cast<uint4*>(my_row + (((4 + m) ^ (lane & 7)) << 4)) = o[m];
    // generic-proxy writes -> visible to the TMA (async proxy), then one store
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) {
      store(stg_s, d0);
      bulk_commit();
    }
  }
}

// Stores of a row-tile epilogue: 32 rows starting at row0 of an [N][Cout*T]
// activation (3-D map: 64 halves, 128-byte chunk, row), or of spectral planes
// [4][N][Cout] (3-D map: channel, row, plane).
template <int T>
struct RowStore {
  const CUtensorMap* map;
  int64_t row0, N;
  __device__ __forceinline__ void operator()(uint32_t src, int d0) const {
    if (row0 < N) tma_store_3d(map, src, 0, d0 * T / 64, (int)row0);
  }
};
struct PlaneStore {
  const CUtensorMap* map;
  int64_t row0, N;
  __device__ __forceinline__ void operator()(uint32_t src, int d0) const {
    if (row0 < N) tma_store_3d(map, src, d0, (int)row0, 0);
  }
};
template <int T, int IO>
using StoreOf = typename std::conditional<IO == kIoSpectralOut, PlaneStore, RowStore<T>>::type;

}  // namespace ftc
}  // namespace eql
