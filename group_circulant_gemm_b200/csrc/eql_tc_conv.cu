// Group-circulant convolution for T = 4 (p4), FP16 in, FP32 accumulate, FP16
// out, on tcgen05/TMEM.
//
// What it computes: the EQ-Linear layer's group-circulant channel mixing at
// every tap of a KH x KW kernel, stride 1, zero padding (the pages name
// equivariant convolution as the next operator for the per-frequency method,
// "Limitations and future work", without a formula):
//   Y[n][oy][ox][d*4+s] = act(bias[d] + sum_{i,j} sum_{c,t}
//       Wc[i][j][d][c][(t-s) mod 4] * X[n][oy+i-ph][ox+j-pw][c*4+t])
// The group DFT diagonalises every tap the same way as the 1 x 1 layer, so per
// frequency it is a convolution of the spectral planes with the conjugated
// weight spectrum, and the K dimension of the per-frequency GEMMs runs over
// (tap, channel).
//
// Design.  Every input pixel feeds KH * KW taps, so its group DFT is taken once,
// by conv_planes_kernel, into planes Xhat[4][N][H][W][C] (the same FP32
// arithmetic and single rounding as the layer's in-kernel transform), and the
// main kernel reads those planes directly as MMA operands (no transform).  An
// output tile is 8 x 16 pixels of one image x 128 out-channels; a K stage is one
// tap and 32 channels, loaded by one 5-D TMA box (32 channels, 16 x, 8 y, 1
// image, 4 planes) whose start (ox0 + j - pw, oy0 + i - ph) may lie outside the
// image: the TMA fills those pixels with zeros, which is the zero padding.  The
// MMA group and the inverse-DFT epilogue are the layer's; an epilogue warp's 32
// rows are 2 image rows x 16 pixels, written by a 5-D TMA store that clips at
// the image border.  Warps: 0 X producer, 1 MMA issuer, 2 weight producer,
// 4..11 epilogue (no transform warps).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "eql_kernels.h"
#include "eql_tc_common.cuh"
#include "eql_tc_fwd_parts.cuh"

namespace eql {
namespace {

using namespace tc;
using namespace ftc;

using S = Shape<4>;
constexpr int BD = S::BD;
constexpr int kConvThreads = 384;  // warps 0..11
constexpr int BY = 8, BX = 16;     // output tile: 8 rows x 16 pixels = 128 MMA rows

struct ConvInfo {
  int N, H, W, C, D;
  int KH, KW, ph, pw;
  int Ho, Wo;
  int n_ty, n_tx, n_dt;  // tiles along y, x, out-channels
  int ks_n;              // 32-channel stages per tap
  int num_tiles;
};

__device__ __forceinline__ void tma_load_5d(uint32_t dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2),
      "r"(c3), "r"(c4)
      : "memory");
}
__device__ __forceinline__ void tma_store_5d(const CUtensorMap* map, uint32_t src, int c0, int c1,
                                             int c2, int c3, int c4) {
  asm volatile(
      "cp.async.bulk.tensor.5d.global.shared::cta.bulk_group [%0, {%2, %3, %4, %5, %6}], [%1];" ::
          "l"(reinterpret_cast<uint64_t>(map)),
      "r"(src), "r"(c0), "r"(c1), "r"(c2), "r"(c3), "r"(c4)
      : "memory");
}

// 32 output rows = 2 image rows x 16 pixels of Y [N][Ho][Wo][D*4]
struct PixelStore {
  const CUtensorMap* map;
  int n, oy, ox0, Ho;
  __device__ __forceinline__ void operator()(uint32_t src, int d0) const {
    if (oy < Ho) tma_store_5d(map, src, 0, d0 * 4 / 64, ox0, oy, n);
  }
};

// Group DFT of every pixel's group vectors: X [P][C*4] -> planes [4][P][C]
// (X0 = x0+x1+x2+x3, X2 = x0-x1+x2-x3, Xr = x0-x2, Xi = x3-x1, each times 1/4
// like every stored plane; FP32, one rounding).  One thread per pixel and 8
// channels.
__global__ void conv_planes_kernel(const uint4* __restrict__ X, int64_t P, int C,
                                   uint4* __restrict__ planes) {
  const int groups = C / 8;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= P * groups) return;
  const int64_t p = idx / groups;
  const int g = (int)(idx % groups);
  const uint4* src = X + (p * C * 4 + g * 32) / 8;  // 8 halves per uint4
  uint32_t o[4][4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {  // piece q: channels 2q, 2q+1 of the group
    const uint4 v = src[q];
    const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
    float f0[2], fh[2], fr[2], fi[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const float2 lo = unpack_h2(w4[2 * hh]), hi = unpack_h2(w4[2 * hh + 1]);
      const float x0 = lo.x, x1 = lo.y, x2 = hi.x, x3 = hi.y;
      const float a = x0 + x2, b = x1 + x3;
      f0[hh] = (a + b) * 0.25f;
      fh[hh] = (a - b) * 0.25f;
      fr[hh] = (x0 - x2) * 0.25f;
      fi[hh] = (x3 - x1) * 0.25f;
    }
    o[0][q] = pack_h2(f0[0], f0[1]);
    o[1][q] = pack_h2(fh[0], fh[1]);
    o[2][q] = pack_h2(fr[0], fr[1]);
    o[3][q] = pack_h2(fi[0], fi[1]);
  }
#pragma unroll
  for (int pl = 0; pl < 4; ++pl)
    planes[((int64_t)pl * P * C + p * C + g * 8) / 8] = make_uint4(o[pl][0], o[pl][1], o[pl][2],
                                                                   o[pl][3]);
}

template <int ACT>
__global__ void __launch_bounds__(kConvThreads, 1)
    eq_conv_tc_kernel(const __grid_constant__ CUtensorMap map_x,
                      const __grid_constant__ CUtensorMap map_y, const uint8_t* __restrict__ wtiles,
                      const __half* __restrict__ bias, ConvInfo ci, int* status) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars<4>* bars = reinterpret_cast<Bars<4>*>(smem + S::OFF_BAR);
  int* abort_flag = &bars->abort_flag;
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int taps = ci.KH * ci.KW;
  const int k_total = taps * ci.ks_n;
  const size_t tap_blobs = (size_t)ci.n_dt * ci.ks_n;  // weight blobs per tap

  if (threadIdx.x == 0) {
    for (int s = 0; s < S::X_ST; ++s) {
      mbar_init(&bars->x_full[s], 1);
      mbar_init(&bars->x_empty[s], 1);
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
    // ------- producers: warp 0 planes (5-D TMA box per tap), warp 2 weights -------
    if (lane == 0) {
      const bool is_x = (warp == 0);
      const int depth = is_x ? S::X_ST : S::W_ST;
      uint64_t* full = is_x ? bars->x_full : bars->w_full;
      uint64_t* empty = is_x ? bars->x_empty : bars->w_empty;
      int issued_phase[S::X_ST > S::W_ST ? S::X_ST : S::W_ST];
      for (int s = 0; s < depth; ++s) issued_phase[s] = -1;
      uint32_t it = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < ci.num_tiles; tile += gridDim.x) {
        const int dt = tile % ci.n_dt;
        int rest = tile / ci.n_dt;
        const int bx = rest % ci.n_tx;
        rest /= ci.n_tx;
        const int by = rest % ci.n_ty;
        const int n = rest / ci.n_ty;
        for (int kk = 0; kk < k_total; ++kk, ++it) {
          const int s = it % depth;
          const uint32_t ph = (it / depth) & 1;
          if (!(ok = wait_bounded(&empty[s], ph ^ 1, abort_flag, status))) break;
          const int tap = kk / ci.ks_n, ks = kk % ci.ks_n;
          if (is_x) {
            const int i = tap / ci.KW, j = tap % ci.KW;
            mbar_expect_tx(&full[s], X_STAGE_BYTES);
            // (channel, x, y, image, plane); x and y may start outside the image
            tma_load_5d(sbase + S::OFF_X + s * X_STAGE_BYTES, &map_x, &full[s], S::BK * ks,
                        bx * BX + j - ci.pw, by * BY + i - ci.ph, n, 0);
          } else {
            mbar_expect_tx(&full[s], S::W_STAGE_BYTES);
            const size_t blob = tap * tap_blobs + (size_t)dt * ci.ks_n + ks;
            bulk_load(sbase + S::OFF_W + s * S::W_STAGE_BYTES, wtiles + blob * S::W_STAGE_BYTES,
                      S::W_STAGE_BYTES, &full[s]);
          }
          issued_phase[s] = (int)ph;
        }
      }
      if (!ok) {
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
      for (int tile = blockIdx.x; ok && tile < ci.num_tiles; tile += gridDim.x, ++tcount) {
        if (!(ok = wait_bounded(&bars->acc_empty, (tcount & 1) ^ 1, abort_flag, status))) break;
        tc_fence_after();
        for (int kk = 0; kk < k_total; ++kk, ++it) {
          const int sx = it % S::X_ST, sw = it % S::W_ST;
          if (!(ok = wait_bounded(&bars->x_full[sx], (it / S::X_ST) & 1, abort_flag, status)))
            break;
          if (!(ok = wait_bounded(&bars->w_full[sw], (it / S::W_ST) & 1, abort_flag, status)))
            break;
          tc_fence_after();
          const uint32_t pl = sbase + S::OFF_X + sx * X_STAGE_BYTES;
          const uint32_t wr = sbase + S::OFF_W + sw * S::W_STAGE_BYTES;
#pragma unroll
          for (int k2 = 0; k2 < S::KSTEPS; ++k2) {
            const uint32_t ko = 32u * k2;
            const uint32_t acc = (kk > 0 || k2 > 0) ? 1u : 0u;
            auto A = [&](int p) { return desc_kmajor<S::ROWB>(pl + p * S::PLANE_BYTES + ko); };
            auto B = [&](int p) { return desc_kmajor<S::ROWB>(wr + p * S::WREG_BYTES + ko); };
            umma(tmem + 0, A(0), B(0), id_n1, acc);
            umma(tmem + BD, A(1), B(1), id_n1, acc);
            umma(tmem + 2 * BD, A(2), B(2), id_n2, acc);
            umma(tmem + 2 * BD, A(3), B(3), id_n1_neg, 1u);
            umma(tmem + 3 * BD, A(3), B(2), id_n1, 1u);
          }
          umma_commit(&bars->x_empty[sx]);
          umma_commit(&bars->w_empty[sw]);
        }
        if (ok) umma_commit(&bars->acc_full);
      }
      umma_commit(&bars->drain);
      drain_wait(&bars->drain, 0);
    }
    __syncwarp();
  } else if (warp >= kEpiWarp0 && warp < kEpiWarp0 + kEpiWarps) {
    // ---------------- epilogue ----------------
    const int q4 = warp & 3;
    const int ch = (warp - kEpiWarp0) >> 2;
    uint8_t* stg = smem + S::OFF_STG + (warp - kEpiWarp0) * kStgBytes;
    __half* bsm = reinterpret_cast<__half*>(smem + S::OFF_BIAS + (warp - kEpiWarp0) * 128);
    uint32_t tcount = 0;
    for (int tile = blockIdx.x; tile < ci.num_tiles; tile += gridDim.x, ++tcount) {
      const int dt = tile % ci.n_dt;
      int rest = tile / ci.n_dt;
      const int bx = rest % ci.n_tx;
      rest /= ci.n_tx;
      const int by = rest % ci.n_ty;
      const int n = rest / ci.n_ty;
      const int dbase = dt * BD + (BD / 2) * ch;
      if (2 * lane < BD / 2) {
        const int d = dbase + 2 * lane;
        uint32_t v = 0u;
        if (bias && d < ci.D) v = *reinterpret_cast<const uint32_t*>(bias + d);
        reinterpret_cast<uint32_t*>(bsm)[lane] = v;
      }
      __syncwarp();
      if (!warp_wait(&bars->acc_full, tcount & 1, abort_flag, status)) break;
      tc_fence_after();
      const uint32_t lane_addr = tmem + ((uint32_t)(32 * q4) << 16);
      // this warp's 32 tile rows are image rows by*8 + 2 q4 (+1), 16 pixels each
      epi_slices<4, BD, ACT, kIoSpatial>(lane_addr, ch, lane, stg, bsm, dbase, ci.D,
                                         PixelStore{&map_y, n, by * BY + 2 * q4, bx * BX,
                                                    ci.Ho});
      tc_fence_before();
      mbar_arrive(&bars->acc_empty);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTmemCols));
  }
}

template <int ACT>
cudaError_t set_conv_attr() {
  return cudaFuncSetAttribute(eq_conv_tc_kernel<ACT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              S::SMEM_BYTES);
}

}  // namespace

bool conv_tc_supported(int T, DType dt, int64_t N, int H, int W, int C, int D, int KH, int KW,
                       int ph, int pw) {
  if (T != 4 || dt != DType::F16) return false;
  if (N < 1 || H < 1 || W < 1 || KH < 1 || KW < 1 || ph < 0 || pw < 0) return false;
  if (KH > 15 || KW > 15 || ph >= KH || pw >= KW) return false;
  if (C % 16 != 0 || D % 16 != 0 || C < 16 || D < 16) return false;
  const int64_t Ho = (int64_t)H + 2 * ph - KH + 1, Wo = (int64_t)W + 2 * pw - KW + 1;
  if (Ho < 1 || Wo < 1) return false;
  // TMA: coordinates and extents are 32-bit; planes and Y stay far below 2^31 rows
  return N <= 65535 && H <= 32767 && W <= 32767 && N * H * W <= 0x3fffffffLL &&
         N * Ho * Wo <= 0x3fffffffLL;
}

size_t conv_tc_planes_bytes(int64_t N, int H, int W, int C) {
  return (size_t)4 * N * H * W * C * 2;
}

cudaError_t launch_conv_tc(const void* X, int64_t N, int H, int W, int C, int D, int KH, int KW,
                           int ph, int pw, const void* Wtiles, const void* bias, void* Y,
                           void* planes, int* status, int num_sms, int act, cudaStream_t st) {
  if (!conv_tc_supported(4, DType::F16, N, H, W, C, D, KH, KW, ph, pw))
    return cudaErrorNotSupported;
  if (!Wtiles || !planes) return cudaErrorInvalidValue;
  if (act != 0 && act != 1) return cudaErrorInvalidValue;
  auto encode = encode_fn();
  if (!encode) return cudaErrorNotSupported;
  const int Ho = H + 2 * ph - KH + 1, Wo = W + 2 * pw - KW + 1;
  const int64_t P = N * H * W;

  // planes [4][N][H][W][C] as (channel, x, y, image, plane); box = one K stage
  CUtensorMap mx, my;
  {
    cuuint64_t dims[5] = {(cuuint64_t)C, (cuuint64_t)W, (cuuint64_t)H, (cuuint64_t)N, 4};
    cuuint64_t strides[4] = {(cuuint64_t)C * 2, (cuuint64_t)W * C * 2, (cuuint64_t)H * W * C * 2,
                             (cuuint64_t)P * C * 2};
    cuuint32_t box[5] = {(cuuint32_t)S::BK, BX, BY, 1, 4};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    if (encode(&mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, planes, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  // Y [N][Ho][Wo][D*4] as (64 halves, 128-byte chunk, x, y, image); box = 16 x 2 pixels
  {
    cuuint64_t dims[5] = {64, (cuuint64_t)D * 4 / 64, (cuuint64_t)Wo, (cuuint64_t)Ho,
                          (cuuint64_t)N};
    cuuint64_t strides[4] = {128, (cuuint64_t)D * 4 * 2, (cuuint64_t)Wo * D * 4 * 2,
                             (cuuint64_t)Ho * Wo * D * 4 * 2};
    cuuint32_t box[5] = {64, 1, BX, 2, 1};
    cuuint32_t estr[5] = {1, 1, 1, 1, 1};
    if (encode(&my, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 5, Y, dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) !=
        CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  ConvInfo ci;
  ci.N = (int)N; ci.H = H; ci.W = W; ci.C = C; ci.D = D;
  ci.KH = KH; ci.KW = KW; ci.ph = ph; ci.pw = pw;
  ci.Ho = Ho; ci.Wo = Wo;
  ci.n_ty = (Ho + BY - 1) / BY;
  ci.n_tx = (Wo + BX - 1) / BX;
  ci.n_dt = (D + BD - 1) / BD;
  ci.ks_n = (C + S::BK - 1) / S::BK;
  const int64_t tiles = N * ci.n_ty * ci.n_tx * ci.n_dt;
  if (tiles > 0x7fffffffLL) return cudaErrorInvalidValue;
  ci.num_tiles = (int)tiles;

  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = set_conv_attr<0>();
    if (e == cudaSuccess) e = set_conv_attr<1>();
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  const int64_t work = P * (C / 8);
  conv_planes_kernel<<<(unsigned)((work + 255) / 256), 256, 0, st>>>(
      static_cast<const uint4*>(X), P, C, static_cast<uint4*>(planes));
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int grid = ci.num_tiles < num_sms ? ci.num_tiles : num_sms;
  auto kernel = act ? eq_conv_tc_kernel<1> : eq_conv_tc_kernel<0>;
  kernel<<<grid, kConvThreads, S::SMEM_BYTES, st>>>(mx, my, static_cast<const uint8_t*>(Wtiles),
                                                   static_cast<const __half*>(bias), ci, status);
  return cudaGetLastError();
}

namespace {
// A pixel tensor moved onto another pixel grid: out[n][oy][ox] = X[n][oy + i - ph]
// [ox + j - pw], zero where that pixel lies outside the image (the convolution's
// weight gradient puts X and dY on its padded grid this way); one thread per 16
// bytes.
__global__ void conv_shift_rows_kernel(const uint4* __restrict__ X, int64_t N, int H, int W,
                                       int c16, int i, int j, int ph, int pw, int Ho, int Wo,
                                       uint4* __restrict__ out) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = N * Ho * Wo * c16;
  if (idx >= total) return;
  const int64_t q = idx / c16;
  const int k = (int)(idx % c16);
  const int ox = (int)(q % Wo), oy = (int)((q / Wo) % Ho);
  const int64_t n = q / ((int64_t)Wo * Ho);
  const int iy = oy + i - ph, ix = ox + j - pw;
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (iy >= 0 && iy < H && ix >= 0 && ix < W) v = X[((n * H + iy) * W + ix) * c16 + k];
  out[idx] = v;
}
}  // namespace

cudaError_t launch_conv_group_planes(const void* X, int64_t P, int C, void* planes,
                                     cudaStream_t st) {
  if (C % 8 != 0) return cudaErrorInvalidValue;
  const int64_t work = P * (C / 8);
  if (work == 0) return cudaSuccess;
  conv_planes_kernel<<<(unsigned)((work + 255) / 256), 256, 0, st>>>(
      static_cast<const uint4*>(X), P, C, static_cast<uint4*>(planes));
  return cudaGetLastError();
}

cudaError_t launch_conv_shift_rows(const void* X, int64_t N, int H, int W, int c4, int i, int j,
                                   int ph, int pw, int Ho, int Wo, void* out, cudaStream_t st) {
  if (c4 % 8 != 0) return cudaErrorInvalidValue;
  const int64_t total = N * Ho * Wo * (c4 / 8);
  if (total == 0) return cudaSuccess;
  conv_shift_rows_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(
      static_cast<const uint4*>(X), N, H, W, c4 / 8, i, j, ph, pw, Ho, Wo,
      static_cast<uint4*>(out));
  return cudaGetLastError();
}

}  // namespace eql
