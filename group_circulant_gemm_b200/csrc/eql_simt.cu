// CUDA-core (FP32 FMA) kernels of the EQ-Linear library, for every supported T:
//   - prepare: one-time DFT of the weights into spectral planes,
//   - forward / dX: tiled per-frequency GEMM with the group DFT fused into the
//     tile load and the inverse DFT + bias fused into the store,
//   - weight gradient: split reduction over rows of per-frequency products,
//     plus a finalize kernel (fixed-order split sum, inverse DFT, cast).
// These are the FP32 path ("Implementation": FP32 and FP16 precisions) and the
// general-T path; the FP16 p4 forward on tensor cores lives in eql_tc_fwd.cu.
#include <algorithm>
#include <type_traits>

#include "eql_common.cuh"
#include "eql_kernels.h"

namespace eql {
namespace {

// ---------------------------------------------------------------------------
// prepare: W[D][C][T] -> forward planes [P][D][C] = conj(DFT(W)), adjoint planes
// [P][C][D] = DFT(W) transposed, both times 1/Tp (exact; the stored range never
// exceeds max|W|).  One thread per (d, c).
// conj(DFT(w))[k] = sum_u w[u] e^{+2 pi i k u/T}: Re = sum w cos, Im = +sum w sin.
// ---------------------------------------------------------------------------
template <int T, typename In>
__global__ void prepare_kernel(const In* __restrict__ W, int C, int D, In* __restrict__ fwd,
                               In* __restrict__ adj, Twiddles tw) {
  using S = Spec<T>;
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= (int64_t)C * D) return;
  const int d = (int)(idx / C), c = (int)(idx % C);
  float w[T];
#pragma unroll
  for (int u = 0; u < T; ++u) w[u] = to_f32(W[idx * T + u]);
  float re[S::P], im_adj[S::P];  // per plane: forward value, adjoint value
  float s0 = 0.f;
#pragma unroll
  for (int u = 0; u < T; ++u) s0 += w[u];
  re[0] = s0;
  im_adj[0] = s0;
  if constexpr (S::NR == 2) {
    float h = 0.f;
#pragma unroll
    for (int u = 0; u < T; ++u) h += (u & 1) ? -w[u] : w[u];
    re[1] = h;
    im_adj[1] = h;
  }
#pragma unroll
  for (int k = 1; k <= S::NC; ++k) {
    float a = 0.f, b = 0.f;
#pragma unroll
    for (int u = 0; u < T; ++u) {
      a = fmaf(w[u], tw.cs[k][u], a);
      b = fmaf(w[u], tw.sn[k][u], b);
    }
    re[S::re(k)] = a;        // forward Re
    re[S::im(k)] = b;        // forward Im  (conjugated spectrum: +sum w sin)
    re[S::negim(k)] = -b;    // forward -Im
    im_adj[S::re(k)] = a;    // adjoint Re
    im_adj[S::im(k)] = -b;   // adjoint Im  (plain spectrum)
    im_adj[S::negim(k)] = b; // adjoint -Im
  }
  const int64_t plane = (int64_t)C * D;
  constexpr float sc = plane_scale<T>();
#pragma unroll
  for (int j = 0; j < S::P; ++j) {
    fwd[j * plane + (int64_t)d * C + c] = from_f32<In>(re[j] * sc);
    adj[j * plane + (int64_t)c * D + d] = from_f32<In>(im_adj[j] * sc);
  }
}

// ---------------------------------------------------------------------------
// Forward (and dX) on CUDA cores.
// CTA tile: BM rows x BD out-channels, 256 threads as a 16 x 16 grid, each
// thread TM rows x TD out-channels x T spectral accumulators; K loop over
// input channels in stages of BK.  Per stage, the next stage's group vectors
// and weight planes are prefetched into registers during the FMA loop, then
// the group DFT runs in registers and writes spectral planes to smem.
// ---------------------------------------------------------------------------
template <int T>
struct SimtTile {
  static constexpr int TM = 4;
  static constexpr int TD = (T <= 4) ? 4 : 2;
  static constexpr int BM = 16 * TM;
  static constexpr int BD = 16 * TD;
  static constexpr int BK = (T <= 4) ? 16 : 8;  // keeps static smem under 48 KB
  static constexpr int XS = BM + 4;        // padded row of a spectral plane
  static constexpr int WS = BD + 4;
  static constexpr int G_PER_THREAD = BM * BK / 256;  // group vectors loaded per thread
  static constexpr int W_PER_THREAD = (T * BK * BD + 255) / 256;
  static_assert(BM * BK % 256 == 0 && BK % 8 == 0, "loader mapping");
};

template <int T, typename In>
__global__ void __launch_bounds__(256) fwd_simt_kernel(const In* __restrict__ X, int64_t N,
                                                       int Cin, int Cout,
                                                       const In* __restrict__ Wt,
                                                       const In* __restrict__ bias,
                                                       In* __restrict__ Y, Twiddles tw, int act) {
  using S = Spec<T>;
  using G = SimtTile<T>;
  __shared__ __align__(16) float xs[T][G::BK][G::XS];
  __shared__ __align__(16) float ws[T][G::BK][G::WS];

  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t row0 = (int64_t)blockIdx.x * G::BM;
  const int d0 = blockIdx.y * G::BD;
  const int64_t plane = (int64_t)Cin * Cout;
  const int64_t ldx = (int64_t)Cin * T;

  float acc[G::TM][G::TD][T];
#pragma unroll
  for (int m = 0; m < G::TM; ++m)
#pragma unroll
    for (int dd = 0; dd < G::TD; ++dd)
#pragma unroll
      for (int j = 0; j < T; ++j) acc[m][dd][j] = 0.f;

  // Loader mapping: each warp covers 8 channels x 4 rows of group vectors, so
  // its global reads are 4 contiguous row segments and its spectral-plane
  // stores (stride XS = BM + 4) hit 32 distinct banks.
  auto group_of = [&](int i, int& r, int& c) {
    const int g = tid + i * 256;
    const int cl = g & 7, rl = (g >> 3) & 3, blk = g >> 5;
    c = (blk % (G::BK / 8)) * 8 + cl;
    r = (blk / (G::BK / 8)) * 4 + rl;
  };
  float greg[G::G_PER_THREAD][T];
  float wreg[G::W_PER_THREAD];

  auto load_stage = [&](int c0) {
#pragma unroll
    for (int i = 0; i < G::G_PER_THREAD; ++i) {
      int r, c;
      group_of(i, r, c);
      const int64_t row = row0 + r;
      const bool ok = row < N && c0 + c < Cin;
      const In* src = X + row * ldx + (int64_t)(c0 + c) * T;
#pragma unroll
      for (int t = 0; t < T; ++t) greg[i][t] = ok ? to_f32(src[t]) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < G::W_PER_THREAD; ++i) {
      const int e = tid + i * 256;
      float v = 0.f;
      if (e < T * G::BK * G::BD) {
        const int j = e / (G::BK * G::BD), q = e % (G::BK * G::BD);
        const int c = c0 + q / G::BD, d = d0 + q % G::BD;
        // spectral plane j -> prepared plane: Re planes as-is, Im from the -Im slot
        int src = j;
        if (j >= S::NR && ((j - S::NR) & 1)) src = S::negim((j - S::NR) / 2 + 1);
        // the stored planes carry 1/Tp: undo it exactly here
        if (c < Cin && d < Cout)
          v = to_f32(Wt[src * plane + (int64_t)c * Cout + d]) * (float)plane_pow2(T);
      }
      wreg[i] = v;
    }
  };

  const int nst = (Cin + G::BK - 1) / G::BK;
  load_stage(0);
  for (int st = 0; st < nst; ++st) {
    // group DFT of the prefetched group vectors straight into the spectral planes
#pragma unroll
    for (int i = 0; i < G::G_PER_THREAD; ++i) {
      int r, c;
      group_of(i, r, c);
      float p[T];
      group_dft<T>(greg[i], p, tw);
#pragma unroll
      for (int j = 0; j < T; ++j) xs[j][c][r] = p[j];
    }
#pragma unroll
    for (int i = 0; i < G::W_PER_THREAD; ++i) {
      const int e = tid + i * 256;
      if (e < T * G::BK * G::BD) {
        const int j = e / (G::BK * G::BD), q = e % (G::BK * G::BD);
        ws[j][q / G::BD][q % G::BD] = wreg[i];
      }
    }
    __syncthreads();
    if (st + 1 < nst) load_stage((st + 1) * G::BK);
#pragma unroll 4
    for (int c = 0; c < G::BK; ++c) {
      float xv[T][G::TM], wv[T][G::TD];
#pragma unroll
      for (int j = 0; j < T; ++j) {
#pragma unroll
        for (int m = 0; m < G::TM; ++m) xv[j][m] = xs[j][c][ty * G::TM + m];
#pragma unroll
        for (int dd = 0; dd < G::TD; ++dd) wv[j][dd] = ws[j][c][tx * G::TD + dd];
      }
#pragma unroll
      for (int m = 0; m < G::TM; ++m) {
#pragma unroll
        for (int dd = 0; dd < G::TD; ++dd) {
#pragma unroll
          for (int j = 0; j < S::NR; ++j) acc[m][dd][j] = fmaf(xv[j][m], wv[j][dd], acc[m][dd][j]);
#pragma unroll
          for (int k = 1; k <= S::NC; ++k) {
            const int jr = S::re(k), ji = S::im(k);
            // (Wr + i Wi)(Xr + i Xi)
            float r = acc[m][dd][jr], i = acc[m][dd][ji];
            r = fmaf(wv[jr][dd], xv[jr][m], r);
            r = fmaf(-wv[ji][dd], xv[ji][m], r);
            i = fmaf(wv[ji][dd], xv[jr][m], i);
            i = fmaf(wv[jr][dd], xv[ji][m], i);
            acc[m][dd][jr] = r;
            acc[m][dd][ji] = i;
          }
        }
      }
    }
    __syncthreads();
  }

  // epilogue: inverse DFT + bias, T contiguous outputs per (row, out-channel)
  const int64_t ldy = (int64_t)Cout * T;
#pragma unroll
  for (int m = 0; m < G::TM; ++m) {
    const int64_t row = row0 + ty * G::TM + m;
    if (row >= N) continue;
#pragma unroll
    for (int dd = 0; dd < G::TD; ++dd) {
      const int d = d0 + tx * G::TD + dd;
      if (d >= Cout) continue;
      float y[T];
      group_idft<T>(acc[m][dd], y, tw);
      const float b = bias ? to_f32(bias[d]) : 0.f;
#pragma unroll
      for (int s = 0; s < T; ++s)
        Y[row * ldy + (int64_t)d * T + s] = from_f32<In>(apply_act(y[s] + b, act));
    }
  }
}

// ---------------------------------------------------------------------------
// Weight gradient on CUDA cores.  Per frequency k the product is
//   Q_k[d][c] = sum_n conj(G_k[n,d]) X_k[n,c]       (G = DFT of dY, X = DFT of X)
// real k: Q += G X;  complex k: Qr += Gr Xr + Gi Xi,  Qi += Gr Xi - Gi Xr.
// CTA tile: BD out-channels x BC in-channels, rows reduced in stages of BK,
// grid.z = row splits, each writing its own FP32 partial planes.
// ---------------------------------------------------------------------------
template <int T>
struct WgTile {
  static constexpr int TM = 4;                     // out-channels per thread
  static constexpr int TD = (T <= 4) ? 4 : 2;      // in-channels per thread
  static constexpr int BD = 16 * TM;
  static constexpr int BC = 16 * TD;
  static constexpr int BK = (T <= 4) ? 16 : 8;    // rows per stage (smem < 48 KB)
  static constexpr int GS = BD + 4;
  static constexpr int CS = BC + 4;
};

template <int T, typename In>
__global__ void __launch_bounds__(256) wgrad_simt_kernel(const In* __restrict__ X,
                                                         const In* __restrict__ dY, int64_t N,
                                                         int C, int D, int64_t rows_per_split,
                                                         float* __restrict__ part,
                                                         float* __restrict__ bpart, Twiddles tw) {
  using S = Spec<T>;
  using G = WgTile<T>;
  __shared__ __align__(16) float gs[T][G::BK][G::GS];
  __shared__ __align__(16) float xs[T][G::BK][G::CS];

  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int d0 = blockIdx.x * G::BD;
  const int c0 = blockIdx.y * G::BC;
  const int z = blockIdx.z;
  const int64_t r_begin = (int64_t)z * rows_per_split;
  const int64_t r_end = min(N, r_begin + rows_per_split);
  const int64_t ldx = (int64_t)C * T, ldy = (int64_t)D * T;

  float acc[G::TM][G::TD][T];
#pragma unroll
  for (int m = 0; m < G::TM; ++m)
#pragma unroll
    for (int dd = 0; dd < G::TD; ++dd)
#pragma unroll
      for (int j = 0; j < T; ++j) acc[m][dd][j] = 0.f;
  float bacc[G::TM];
#pragma unroll
  for (int m = 0; m < G::TM; ++m) bacc[m] = 0.f;

  for (int64_t r0 = r_begin; r0 < r_end; r0 += G::BK) {
    // DFT of dY groups (BK rows x BD channels) and X groups (BK rows x BC channels)
    for (int g = tid; g < G::BK * G::BD; g += 256) {
      const int r = g / G::BD, dl = g % G::BD;
      const int64_t row = r0 + r;
      const int d = d0 + dl;
      float x[T], p[T];
#pragma unroll
      for (int t = 0; t < T; ++t)
        x[t] = (row < r_end && d < D) ? to_f32(dY[row * ldy + (int64_t)d * T + t]) : 0.f;
      group_dft<T>(x, p, tw);
#pragma unroll
      for (int j = 0; j < T; ++j) gs[j][r][dl] = p[j];
    }
    for (int g = tid; g < G::BK * G::BC; g += 256) {
      const int r = g / G::BC, cl = g % G::BC;
      const int64_t row = r0 + r;
      const int c = c0 + cl;
      float x[T], p[T];
#pragma unroll
      for (int t = 0; t < T; ++t)
        x[t] = (row < r_end && c < C) ? to_f32(X[row * ldx + (int64_t)c * T + t]) : 0.f;
      group_dft<T>(x, p, tw);
#pragma unroll
      for (int j = 0; j < T; ++j) xs[j][r][cl] = p[j];
    }
    __syncthreads();
#pragma unroll 4
    for (int r = 0; r < G::BK; ++r) {
      float gv[T][G::TM], xv[T][G::TD];
#pragma unroll
      for (int j = 0; j < T; ++j) {
#pragma unroll
        for (int m = 0; m < G::TM; ++m) gv[j][m] = gs[j][r][ty * G::TM + m];
#pragma unroll
        for (int dd = 0; dd < G::TD; ++dd) xv[j][dd] = xs[j][r][tx * G::TD + dd];
      }
#pragma unroll
      for (int m = 0; m < G::TM; ++m) {
        bacc[m] += gv[0][m];
#pragma unroll
        for (int dd = 0; dd < G::TD; ++dd) {
#pragma unroll
          for (int j = 0; j < S::NR; ++j) acc[m][dd][j] = fmaf(gv[j][m], xv[j][dd], acc[m][dd][j]);
#pragma unroll
          for (int k = 1; k <= S::NC; ++k) {
            const int jr = S::re(k), ji = S::im(k);
            float re = acc[m][dd][jr], im = acc[m][dd][ji];
            re = fmaf(gv[jr][m], xv[jr][dd], re);
            re = fmaf(gv[ji][m], xv[ji][dd], re);
            im = fmaf(gv[jr][m], xv[ji][dd], im);
            im = fmaf(-gv[ji][m], xv[jr][dd], im);
            acc[m][dd][jr] = re;
            acc[m][dd][ji] = im;
          }
        }
      }
    }
    __syncthreads();
  }

  const int64_t plane = (int64_t)D * C;
  float* out = part + (int64_t)z * T * plane;
#pragma unroll
  for (int m = 0; m < G::TM; ++m) {
    const int d = d0 + ty * G::TM + m;
    if (d >= D) continue;
#pragma unroll
    for (int dd = 0; dd < G::TD; ++dd) {
      const int c = c0 + tx * G::TD + dd;
      if (c >= C) continue;
#pragma unroll
      for (int j = 0; j < T; ++j) out[j * plane + (int64_t)d * C + c] = acc[m][dd][j];
    }
    if (blockIdx.y == 0 && tx == 0) bpart[(int64_t)z * D + d] = bacc[m];
  }
}

template <int T, typename Out>
__global__ void wgrad_finalize_kernel(const float* __restrict__ part,
                                      const float* __restrict__ bpart, int splits, int C, int D,
                                      Out* __restrict__ dW, Out* __restrict__ dbias, Twiddles tw) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t plane = (int64_t)D * C;
  if (idx < plane) {
    float q[T];
#pragma unroll
    for (int j = 0; j < T; ++j) q[j] = 0.f;
    for (int z = 0; z < splits; ++z) {
#pragma unroll
      for (int j = 0; j < T; ++j) q[j] += part[((int64_t)z * T + j) * plane + idx];
    }
    float w[T];
    group_idft<T>(q, w, tw);
#pragma unroll
    for (int u = 0; u < T; ++u) dW[idx * T + u] = from_f32<Out>(w[u]);
  }
  if (dbias && idx < D) {
    float b = 0.f;
    for (int z = 0; z < splits; ++z) b += bpart[(int64_t)z * D + idx];
    dbias[idx] = from_f32<Out>(b);
  }
}

template <typename F>
cudaError_t dispatch_T(int T, F&& f) {
  switch (T) {
    case 1: return f(std::integral_constant<int, 1>{});
    case 2: return f(std::integral_constant<int, 2>{});
    case 3: return f(std::integral_constant<int, 3>{});
    case 4: return f(std::integral_constant<int, 4>{});
    case 5: return f(std::integral_constant<int, 5>{});
    case 6: return f(std::integral_constant<int, 6>{});
    case 7: return f(std::integral_constant<int, 7>{});
    case 8: return f(std::integral_constant<int, 8>{});
    default: return cudaErrorNotSupported;
  }
}

}  // namespace

cudaError_t launch_prepare(int T, DType dt, const void* W, int C, int D, void* fwd, void* adj,
                           const Twiddles& tw, cudaStream_t st) {
  const int64_t total = (int64_t)C * D;
  const int threads = 256;
  const unsigned blocks = (unsigned)((total + threads - 1) / threads);
  return dispatch_T(T, [&](auto tc) {
    constexpr int TT = decltype(tc)::value;
    if (dt == DType::F32)
      prepare_kernel<TT, float><<<blocks, threads, 0, st>>>((const float*)W, C, D, (float*)fwd,
                                                            (float*)adj, tw);
    else
      prepare_kernel<TT, __half><<<blocks, threads, 0, st>>>(
          (const __half*)W, C, D, (__half*)fwd, (__half*)adj, tw);
    return cudaGetLastError();
  });
}

cudaError_t launch_fwd_simt(int T, DType dt, const void* X, int64_t N, int Cin, int Cout,
                            const void* Wt, const void* bias, void* Y, const Twiddles& tw,
                            int act, cudaStream_t st) {
  if (N == 0) return cudaSuccess;
  return dispatch_T(T, [&](auto tc) {
    constexpr int TT = decltype(tc)::value;
    using G = SimtTile<TT>;
    const int64_t gx = (N + G::BM - 1) / G::BM;
    if (gx > 0x7fffffff) return cudaErrorInvalidValue;
    dim3 grid((unsigned)gx, (unsigned)((Cout + G::BD - 1) / G::BD));
    if (dt == DType::F32)
      fwd_simt_kernel<TT, float><<<grid, 256, 0, st>>>((const float*)X, N, Cin, Cout,
                                                       (const float*)Wt, (const float*)bias,
                                                       (float*)Y, tw, act);
    else
      fwd_simt_kernel<TT, __half><<<grid, 256, 0, st>>>((const __half*)X, N, Cin, Cout,
                                                        (const __half*)Wt, (const __half*)bias,
                                                        (__half*)Y, tw, act);
    return cudaGetLastError();
  });
}

int wgrad_simt_splits(int T, int64_t N, int C, int D, int num_sms) {
  const int td = (T <= 4) ? 4 : 2;
  const int64_t tiles = (int64_t)((D + 63) / 64) * ((C + 16 * td - 1) / (16 * td));
  const int64_t want = std::max<int64_t>(1, (4LL * num_sms + tiles - 1) / tiles);
  const int64_t max_by_rows = std::max<int64_t>(1, (N + 127) / 128);  // >= 128 rows per split
  return (int)std::min<int64_t>(std::min<int64_t>(want, max_by_rows), 64);
}

size_t wgrad_simt_workspace(int T, int64_t N, int C, int D, int num_sms) {
  const int splits = wgrad_simt_splits(T, N, C, D, num_sms);
  return (size_t)splits * ((size_t)T * C * D + D) * sizeof(float);
}

cudaError_t launch_wgrad_finalize(int T, DType out_dt, const float* part, const float* bpart,
                                  int splits, int C, int D, void* dW, void* dbias,
                                  const Twiddles& tw, cudaStream_t st) {
  const int64_t total = std::max<int64_t>((int64_t)C * D, D);
  const unsigned blocks = (unsigned)((total + 255) / 256);
  return dispatch_T(T, [&](auto tc) {
    constexpr int TT = decltype(tc)::value;
    if (out_dt == DType::F32)
      wgrad_finalize_kernel<TT, float><<<blocks, 256, 0, st>>>(part, bpart, splits, C, D,
                                                               (float*)dW, (float*)dbias, tw);
    else
      wgrad_finalize_kernel<TT, __half><<<blocks, 256, 0, st>>>(
          part, bpart, splits, C, D, (__half*)dW, (__half*)dbias, tw);
    return cudaGetLastError();
  });
}

cudaError_t launch_wgrad_simt(int T, DType dt, DType out_dt, const void* X, const void* dY,
                              int64_t N, int C, int D, void* dW, void* dbias, float* ws,
                              int splits, const Twiddles& tw, cudaStream_t st) {
  float* part = ws;
  float* bpart = ws + (size_t)splits * T * C * D;
  if (N > 0) {
    const int64_t rows_per_split = (N + splits - 1) / splits;
    cudaError_t e = dispatch_T(T, [&](auto tc) {
      constexpr int TT = decltype(tc)::value;
      using G = WgTile<TT>;
      dim3 grid((unsigned)((D + G::BD - 1) / G::BD), (unsigned)((C + G::BC - 1) / G::BC),
                (unsigned)splits);
      if (dt == DType::F32)
        wgrad_simt_kernel<TT, float><<<grid, 256, 0, st>>>((const float*)X, (const float*)dY, N,
                                                           C, D, rows_per_split, part, bpart, tw);
      else
        wgrad_simt_kernel<TT, __half><<<grid, 256, 0, st>>>(
            (const __half*)X, (const __half*)dY, N, C, D, rows_per_split, part, bpart, tw);
      return cudaGetLastError();
    });
    if (e != cudaSuccess) return e;
  }
  return launch_wgrad_finalize(T, out_dt, part, bpart, N > 0 ? splits : 0, C, D, dW, dbias, tw,
                               st);
}

namespace {

// Four elements per thread (16-byte loads, 8-byte stores) when both pointers
// allow it, else one.
__global__ void cast_from_f32_kernel(const float* __restrict__ src, __half* __restrict__ dst,
                                     int64_t n, int vec) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t t0 = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  int64_t done = 0;
  if (vec) {
    const int64_t n4 = n / 4;
    for (int64_t i = t0; i < n4; i += stride) {
      const float4 v = reinterpret_cast<const float4*>(src)[i];
      const __half2 lo = __floats2half2_rn(v.x, v.y), hi = __floats2half2_rn(v.z, v.w);
      uint2 o;
      o.x = *reinterpret_cast<const uint32_t*>(&lo);
      o.y = *reinterpret_cast<const uint32_t*>(&hi);
      reinterpret_cast<uint2*>(dst)[i] = o;
    }
    done = n4 * 4;
  }
  for (int64_t i = done + t0; i < n; i += stride) dst[i] = __float2half_rn(src[i]);
}

}  // namespace

cudaError_t launch_cast_from_f32(DType dt, const float* src, void* dst, int64_t n,
                                 cudaStream_t st) {
  if (n <= 0) return cudaSuccess;
  if (dt == DType::F32) {
    if (static_cast<const void*>(src) == dst) return cudaSuccess;
    return cudaMemcpyAsync(dst, src, (size_t)n * sizeof(float), cudaMemcpyDeviceToDevice, st);
  }
  const int vec = ((reinterpret_cast<uintptr_t>(src) & 15) == 0 &&
                   (reinterpret_cast<uintptr_t>(dst) & 7) == 0) ? 1 : 0;
  const int64_t want = ((vec ? n / 4 : n) + 255) / 256;
  const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>(want, 148 * 8));
  cast_from_f32_kernel<<<blocks, 256, 0, st>>>(src, static_cast<__half*>(dst), n, vec);
  return cudaGetLastError();
}

}  // namespace eql
