// Weight gradient of the layer over the dihedral group D4 on CUDA cores, FP16
// X and dY in, FP32 accumulation, FP16 or FP32 out.
//
// What it computes (the D4 layer Y[n,d,g] = bias[d] + sum_{c,h} W[d,c,g^-1 h] X[n,c,h],
// "Limitations and future work" read as the group cross-correlation over D4,
// differentiated):
//   dW[d][c][u] = sum_{n,g} dY[n][d*8+g] * X[n][c*8 + g u],
//   dbias[d]    = sum_{n,g} dY[n][d*8+g],
// elements g = a + 4b for r^a m^b with m r m = r^-1.
//
// Work split: blocks of 16 out-channels x 16 in-channels (one (d, c) pair and
// its eight u per thread) times row splits; each block stages 16 rows of dY
// and X tiles in shared memory as FP32 and accumulates 64 products per row and
// thread.  Every split writes FP32 partials; a second kernel adds the splits in
// a fixed order and casts, so the result is deterministic.
#include <algorithm>

#include "eql_common.cuh"
#include "eql_kernels.h"
#include "eql_tc_common.cuh"

namespace eql {
namespace {

using tc::unpack_h2;

constexpr int DW_B = 16;     // out-channels and in-channels per block
constexpr int DW_R = 16;     // rows staged per step

// (r^a m^b)(r^c m^e) = r^(a + (-1)^b c) m^(b+e), g = a + 4b
__host__ __device__ constexpr int d4m(int g, int h) {
  return ((((g & 3) + ((g >> 2) ? -(h & 3) : (h & 3))) & 3) + 4 * ((g >> 2) ^ (h >> 2)));
}

__global__ void __launch_bounds__(256) d4_wgrad_kernel(const __half* __restrict__ X,
                                                      const __half* __restrict__ dY, int64_t N,
                                                      int C, int D, int64_t rows_per_split,
                                                      float* __restrict__ part,
                                                      float* __restrict__ bpart) {
  __shared__ float sy[DW_R][DW_B][8];
  __shared__ float sx[DW_R][DW_B][8];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;  // in-channel, out-channel
  const int d0 = blockIdx.x * DW_B, c0 = blockIdx.y * DW_B, split = blockIdx.z;
  const int64_t n_begin = (int64_t)split * rows_per_split;
  const int64_t n_end = (n_begin + rows_per_split < N) ? n_begin + rows_per_split : N;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  float bacc = 0.f;
  for (int64_t n0 = n_begin; n0 < n_end; n0 += DW_R) {
    // stage 16 rows x 16 channels x 8 elements of dY and X (one 16-byte load each)
    {
      const int r = threadIdx.x >> 4, ch = threadIdx.x & 15;
      const int64_t n = n0 + r;
      float4 ylo = make_float4(0.f, 0.f, 0.f, 0.f), yhi = ylo, xlo = ylo, xhi = ylo;
      if (n < n_end && d0 + ch < D) {
        const uint4 v = *reinterpret_cast<const uint4*>(dY + (n * D + d0 + ch) * 8);
        const float2 a = unpack_h2(v.x), b = unpack_h2(v.y), c = unpack_h2(v.z), d = unpack_h2(v.w);
        ylo = make_float4(a.x, a.y, b.x, b.y);
        yhi = make_float4(c.x, c.y, d.x, d.y);
      }
      if (n < n_end && c0 + ch < C) {
        const uint4 v = *reinterpret_cast<const uint4*>(X + (n * C + c0 + ch) * 8);
        const float2 a = unpack_h2(v.x), b = unpack_h2(v.y), c = unpack_h2(v.z), d = unpack_h2(v.w);
        xlo = make_float4(a.x, a.y, b.x, b.y);
        xhi = make_float4(c.x, c.y, d.x, d.y);
      }
      *reinterpret_cast<float4*>(&sy[r][ch][0]) = ylo;
      *reinterpret_cast<float4*>(&sy[r][ch][4]) = yhi;
      *reinterpret_cast<float4*>(&sx[r][ch][0]) = xlo;
      *reinterpret_cast<float4*>(&sx[r][ch][4]) = xhi;
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < DW_R; ++r) {
      float y[8], x[8];
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        y[g] = sy[r][ty][g];
        x[g] = sx[r][tx][g];
      }
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        bacc += y[g];
#pragma unroll
        for (int u = 0; u < 8; ++u) acc[u] = fmaf(y[g], x[d4m(g, u)], acc[u]);
      }
    }
    __syncthreads();
  }
  const int d = d0 + ty, c = c0 + tx;
  if (d < D && c < C) {
    float4* dst = reinterpret_cast<float4*>(part + (((int64_t)split * D + d) * C + c) * 8);
    dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
    dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
  }
  if (blockIdx.y == 0 && tx == 0 && d < D) bpart[(int64_t)split * D + d] = bacc;
}

template <typename OutT>
__global__ void d4_wgrad_finalize_kernel(const float* __restrict__ part,
                                         const float* __restrict__ bpart, int splits, int C, int D,
                                         OutT* __restrict__ dW, OutT* __restrict__ dbias) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)D * C * 8;
  if (idx < total) {
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += part[(int64_t)k * total + idx];
    dW[idx] = from_f32<OutT>(s);
  }
  if (dbias && idx < D) {
    float s = 0.f;
    for (int k = 0; k < splits; ++k) s += bpart[(int64_t)k * D + idx];
    dbias[idx] = from_f32<OutT>(s);
  }
}

int d4_splits(int64_t N, int C, int D, int num_sms) {
  const int64_t tiles = (int64_t)((D + DW_B - 1) / DW_B) * ((C + DW_B - 1) / DW_B);
  const int64_t want = std::max<int64_t>(1, (4LL * num_sms + tiles - 1) / tiles);
  const int64_t by_rows = std::max<int64_t>(1, (N + 255) / 256);  // >= 256 rows per split
  return (int)std::min<int64_t>(std::min<int64_t>(want, by_rows), 64);
}

}  // namespace

size_t d4_wgrad_workspace(int64_t N, int C, int D, int num_sms) {
  const int splits = d4_splits(N, C, D, num_sms);
  return (size_t)splits * ((size_t)D * C * 8 + D) * sizeof(float);
}

cudaError_t launch_d4_wgrad(const void* X, const void* dY, int64_t N, int C, int D, DType out_dt,
                            void* dW, void* dbias, float* workspace, int num_sms,
                            cudaStream_t st) {
  const int splits = d4_splits(N, C, D, num_sms);
  float* part = workspace;
  float* bpart = workspace + (size_t)splits * D * C * 8;
  const int64_t rps = (N + splits - 1) / splits;
  if (N > 0) {
    const dim3 grid((unsigned)((D + DW_B - 1) / DW_B), (unsigned)((C + DW_B - 1) / DW_B),
                    (unsigned)splits);
    d4_wgrad_kernel<<<grid, 256, 0, st>>>(static_cast<const __half*>(X),
                                          static_cast<const __half*>(dY), N, C, D, rps, part,
                                          bpart);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  } else {
    cudaError_t e = cudaMemsetAsync(workspace, 0, d4_wgrad_workspace(N, C, D, num_sms), st);
    if (e != cudaSuccess) return e;
  }
  const int64_t total = std::max<int64_t>((int64_t)D * C * 8, D);
  const unsigned blocks = (unsigned)((total + 255) / 256);
  if (out_dt == DType::F32)
    d4_wgrad_finalize_kernel<float><<<blocks, 256, 0, st>>>(
        part, bpart, splits, C, D, static_cast<float*>(dW), static_cast<float*>(dbias));
  else
    d4_wgrad_finalize_kernel<__half><<<blocks, 256, 0, st>>>(
        part, bpart, splits, C, D, static_cast<__half*>(dW), static_cast<__half*>(dbias));
  return cudaGetLastError();
}

}  // namespace eql
