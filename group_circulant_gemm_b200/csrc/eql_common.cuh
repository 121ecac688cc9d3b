// Shared device-side definitions of the EQ-Linear CUDA library (sm_100a).
//
// Spectral plane convention (Flash EQ-Linear summary, "Algorithmic approach"
// items 1-2): a real group vector v[0..T) has the DFT  V[k] = sum_t v[t] e^{-2 pi i k t/T};
// conjugate symmetry leaves the non-redundant frequencies k = 0..floor(T/2).
// Those are stored as T real "spectral planes", in this order:
//   plane 0            : V[0]                     (real)
//   plane 1 (even T)   : V[T/2]                   (real)
//   then for k = 1..NC : Re V[k], Im V[k]         (NC complex frequencies)
// The prepared weights add NC more planes holding -Im of each complex frequency,
// so that a tensor-core B operand can be a contiguous stack of planes.
//
// Range: every stored plane (prepared weights, and the input planes the
// tensor-core kernels form or save) holds the DFT divided by Tp, the smallest
// power of two >= T.  |V[k]| <= T max|v|, so a stored value never exceeds the
// largest input magnitude and legal FP16 inputs cannot overflow to inf in an
// FP16 plane; the division and the matching multiplication by Tp in every
// consumer are exact (powers of two).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace eql {

constexpr int kMaxT = 8;

// DFT twiddles, computed on the host in double and rounded once to float,
// with values within 1e-7 of 0 snapped to 0 (so T = 4 is exactly 0/+-1).
struct Twiddles {
  float cs[kMaxT][kMaxT];  // cos(2 pi k t / T)
  float sn[kMaxT][kMaxT];  // sin(2 pi k t / T)
};

template <int T>
struct Spec {
  static constexpr int NR = (T % 2 == 0) ? 2 : 1;  // real frequencies (0, and T/2 for even T)
  static constexpr int NC = (T - NR) / 2;          // complex frequencies 1..NC
  static constexpr int P = T + NC;                 // prepared planes per block
  __host__ __device__ static constexpr int re(int k) { return k == 0 ? 0 : NR + 2 * (k - 1); }
  __host__ __device__ static constexpr int im(int k) { return NR + 2 * (k - 1) + 1; }
  __host__ __device__ static constexpr int negim(int k) { return T + (k - 1); }
  // number of real multiply-adds per (row, out-channel, in-channel)
  static constexpr int macs = NR + 4 * NC;
};

// Tp: smallest power of two >= T; stored planes are the DFT times 1/Tp.
__host__ __device__ constexpr int plane_pow2(int T) { return T <= 1 ? 1 : 2 * plane_pow2((T + 1) / 2); }
template <int T>
__host__ __device__ constexpr float plane_scale() { return 1.0f / plane_pow2(T); }

__host__ __device__ inline int spec_nr(int T) { return (T % 2 == 0) ? 2 : 1; }
__host__ __device__ inline int spec_nc(int T) { return (T - spec_nr(T)) / 2; }
__host__ __device__ inline int spec_planes(int T) { return T + spec_nc(T); }

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }
template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

// Real DFT of one group vector into T spectral planes (plane order above).
template <int T>
__device__ __forceinline__ void group_dft(const float (&x)[T], float (&p)[T], const Twiddles& tw) {
  using S = Spec<T>;
  float s0 = 0.f;
#pragma unroll
  for (int t = 0; t < T; ++t) s0 += x[t];
  p[0] = s0;
  if constexpr (S::NR == 2) {
    float h = 0.f;
#pragma unroll
    for (int t = 0; t < T; ++t) h += (t & 1) ? -x[t] : x[t];
    p[1] = h;
  }
#pragma unroll
  for (int k = 1; k <= S::NC; ++k) {
    float re = 0.f, im = 0.f;
#pragma unroll
    for (int t = 0; t < T; ++t) {
      re = fmaf(x[t], tw.cs[k][t], re);
      im = fmaf(-x[t], tw.sn[k][t], im);
    }
    p[S::re(k)] = re;
    p[S::im(k)] = im;
  }
}

// Inverse real DFT of T spectral planes back to a group vector:
//   y[s] = (1/T)(P0 + (-1)^s P_half) + (2/T) sum_k (Re_k cos(2pi ks/T) - Im_k sin(2pi ks/T))
template <int T>
__device__ __forceinline__ void group_idft(const float (&p)[T], float (&y)[T], const Twiddles& tw) {
  using S = Spec<T>;
  constexpr float inv = 1.0f / T;
  constexpr float two = 2.0f / T;
#pragma unroll
  for (int s = 0; s < T; ++s) {
    float v = p[0];
    if constexpr (S::NR == 2) v += (s & 1) ? -p[1] : p[1];
    v *= inv;
#pragma unroll
    for (int k = 1; k <= S::NC; ++k) {
      float c = p[S::re(k)] * tw.cs[k][s];
      c = fmaf(-p[S::im(k)], tw.sn[k][s], c);
      v = fmaf(two, c, v);
    }
    y[s] = v;
  }
}

// Output activation of the EQ-MLP block: 0 = none, 1 = GELU (exact erf form),
// y * Phi(y) = 0.5 y (1 + erf(y / sqrt 2)), in FP32 before the output rounding.
// A pointwise function of each output feature commutes with the group shift.
// erf is evaluated with Abramowitz & Stegun, Handbook of Mathematical Functions,
// formula 7.1.28 (|error| <= 3e-7 on the whole line; GELU deviates from the
// exact form by < 5e-7):
//   1 - erf(x) = (1 + a1 x + a2 x^2 + ... + a6 x^6)^-16,  x >= 0,
// with erf(-x) = -erf(x), which gives 1 + erf(x) without cancellation on the
// negative side; one reciprocal is the only special-function operation.
__device__ __forceinline__ float gelu_erf(float y) {
  const float x = fabsf(y) * 0.70710678118654752f;
  float q = fmaf(x, 0.0000430638f, 0.0002765672f);
  q = fmaf(x, q, 0.0001520143f);
  q = fmaf(x, q, 0.0092705272f);
  q = fmaf(x, q, 0.0422820123f);
  q = fmaf(x, q, 0.0705230784f);
  q = fmaf(x, q, 1.0f);
  q = q * q;
  q = q * q;
  q = q * q;
  q = q * q;                             // (polynomial)^16, inf for large x
  const float r = __fdividef(1.0f, q);   // 1 - erf(|y| / sqrt 2), 0 once q overflows
  return 0.5f * y * (y >= 0.f ? 2.0f - r : r);
}

template <int ACT>
__device__ __forceinline__ float act_fn(float y) {
  if constexpr (ACT == 1) {
    return gelu_erf(y);
  } else {
    return y;
  }
}

// Runtime-selected form for the CUDA-core kernels.
__device__ __forceinline__ float apply_act(float y, int act) {
  return act == 1 ? gelu_erf(y) : y;
}

}  // namespace eql
