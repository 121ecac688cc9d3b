// C ABI of the EQ-Linear library: plans, argument checks, kernel dispatch.
// The operations and their definitions are documented in include/eqlinear.h.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <new>

#include "../../include/eqlinear.h"
#include "eql_kernels.h"
#include "eql_plan.h"

using eql::DType;

namespace {

constexpr int kVersion = 100;  // 0.1.0

size_t elem_size(eqlinear_dtype_t dt) { return dt == EQL_F32 ? 4 : 2; }
DType to_dt(eqlinear_dtype_t dt) { return dt == EQL_F32 ? DType::F32 : DType::F16; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

void make_twiddles(int T, eql::Twiddles* tw) {
  std::memset(tw, 0, sizeof(*tw));
  const double two_pi = 6.283185307179586476925286766559;
  for (int k = 0; k < T; ++k) {
    for (int t = 0; t < T; ++t) {
      // reduce k*t mod T first so the angle is exact-ish and symmetric values match
      const int m = (k * t) % T;
      float c = (float)std::cos(two_pi * m / T);
      float s = (float)std::sin(two_pi * m / T);
      if (std::fabs(c) < 1e-7f) c = 0.f;
      if (std::fabs(s) < 1e-7f) s = 0.f;
      tw->cs[k][t] = c;
      tw->sn[k][t] = s;
    }
  }
}

eqlinear_status_t from_cuda(cudaError_t e) {
  if (e == cudaSuccess) return EQL_OK;
  if (e == cudaErrorNotSupported) return EQL_ERR_UNSUPPORTED;
  return EQL_ERR_CUDA;
}

size_t plane_elems(const eqlinear_plan_s* p) { return (size_t)p->C * p->D; }

const void* fwd_block(const eqlinear_plan_s* p, const void* W_hat) { return W_hat; }
const void* adj_block(const eqlinear_plan_s* p, const void* W_hat) {
  return static_cast<const char*>(W_hat) +
         (size_t)eql::spec_planes(p->T) * plane_elems(p) * elem_size(p->dtype);
}
bool has_tiles(const eqlinear_plan_s* p) {
  return eql::tc_tiles_wanted(p->T, to_dt(p->dtype), p->C, p->D);
}
// tensor-core operand tiles: forward (Cin = C, Cout = D) then adjoint (Cin = D, Cout = C);
// a D4 plan holds its 8 spectrum planes then the forward tiles only
const void* fwd_tiles(const eqlinear_plan_s* p, const void* W_hat) {
  if (p->group == 1) return static_cast<const char*>(W_hat) + 8 * plane_elems(p) * 2;
  return static_cast<const char*>(W_hat) +
         2 * (size_t)eql::spec_planes(p->T) * plane_elems(p) * elem_size(p->dtype);
}
const void* adj_tiles(const eqlinear_plan_s* p, const void* W_hat) {
  return static_cast<const char*>(fwd_tiles(p, W_hat)) + eql::tc_tile_bytes(p->T, p->C, p->D);
}
// p4 FP16 plans also hold the pair kernel's weight stages (forward, then adjoint)
bool has_pair_tiles(const eqlinear_plan_s* p) {
  return p->group == 0 && p->T == 4 && has_tiles(p);
}
const void* pair_fwd_tiles(const eqlinear_plan_s* p, const void* W_hat) {
  return static_cast<const char*>(adj_tiles(p, W_hat)) + eql::tc_tile_bytes(p->T, p->D, p->C);
}
const void* pair_adj_tiles(const eqlinear_plan_s* p, const void* W_hat) {
  return static_cast<const char*>(pair_fwd_tiles(p, W_hat)) + eql::pair_tile_bytes(p->C, p->D);
}
// p4 FP32 plans with C, D multiples of 8 hold the 3xTF32 pair kernel's weight
// stages after their planes (forward, then adjoint)
bool has_tf32_tiles(const eqlinear_plan_s* p) {
  return p->group == 0 && p->T == 4 && p->dtype == EQL_F32 && p->C % 8 == 0 && p->D % 8 == 0;
}
const void* tf32_fwd_tiles(const eqlinear_plan_s* p, const void* W_hat) {
  return static_cast<const char*>(W_hat) +
         2 * (size_t)eql::spec_planes(p->T) * plane_elems(p) * elem_size(p->dtype);
}
// FP16 T = 8 plans (cyclic or D4) with C, D multiples of 16 also hold the
// eight-plane pair kernel's weight stages, forward then adjoint: cyclic after the
// one-CTA tiles, D4 after its forward tiles
bool has_pair8_tiles(const eqlinear_plan_s* p) {
  return p->T == 8 && p->dtype == EQL_F16 && p->C % 16 == 0 && p->D % 16 == 0 && has_tiles(p);
}
const void* pair8_fwd_tiles(const eqlinear_plan_s* p, const void* W_hat) {
  if (p->group == 1)
    return static_cast<const char*>(fwd_tiles(p, W_hat)) + eql::tc_tile_bytes(8, p->C, p->D);
  return static_cast<const char*>(adj_tiles(p, W_hat)) + eql::tc_tile_bytes(p->T, p->D, p->C);
}
const void* pair8_adj_tiles(const eqlinear_plan_s* p, const void* W_hat) {
  return static_cast<const char*>(pair8_fwd_tiles(p, W_hat)) + eql::pair8_tile_bytes(p->C, p->D);
}
const void* tf32_adj_tiles(const eqlinear_plan_s* p, const void* W_hat) {
  return static_cast<const char*>(tf32_fwd_tiles(p, W_hat)) + eql::pair_tf32_tile_bytes(p->C, p->D);
}

// Forward-shaped product used by both eqlinear_forward (Cin=C, Cout=D) and
// eqlinear_backward_input (Cin=D, Cout=C).
//   tiles : tensor-core operand tiles of this direction (or null)
//   other : planes [P][Cin][Cout]  (CUDA-core operand)
eqlinear_status_t run_forward_like(eqlinear_plan_s* p, const void* X, int64_t N, int Cin,
                                   int Cout, const void* tiles, const void* other,
                                   const void* bias, void* Y, int act, cudaStream_t st) {
  const bool tc_ok = has_tiles(p) && eql::fwd_tc_supported(p->T, to_dt(p->dtype), N, Cin, Cout);
  if (p->kernel == EQL_KERNEL_TCGEN05 && !tc_ok) return EQL_ERR_UNSUPPORTED;
  if (p->kernel != EQL_KERNEL_SIMT && tc_ok)
    return from_cuda(eql::launch_fwd_tc(p->T, X, N, Cin, Cout, tiles, bias, Y, p->status,
                                        p->num_sms, p->debug_drop_w_stage, act, 0, st));
  return from_cuda(eql::launch_fwd_simt(p->T, to_dt(p->dtype), X, N, Cin, Cout, other, bias, Y,
                                        p->tw, act, st));
}

eqlinear_status_t check_plan_device(const eqlinear_plan_s* p) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return EQL_ERR_CUDA;
  return dev == p->device ? EQL_OK : EQL_ERR_INVALID_ARG;
}

}  // namespace

extern "C" {

int eqlinear_version(void) { return kVersion; }

const char* eqlinear_status_string(eqlinear_status_t s) {
  switch (s) {
    case EQL_OK: return "EQL_OK";
    case EQL_ERR_INVALID_ARG: return "EQL_ERR_INVALID_ARG: invalid argument";
    case EQL_ERR_UNSUPPORTED: return "EQL_ERR_UNSUPPORTED: no kernel for this T/dtype/shape";
    case EQL_ERR_ALIGNMENT: return "EQL_ERR_ALIGNMENT: device pointer not 16-byte aligned";
    case EQL_ERR_WORKSPACE: return "EQL_ERR_WORKSPACE: workspace missing or too small";
    case EQL_ERR_CUDA: return "EQL_ERR_CUDA: CUDA runtime error";
    case EQL_ERR_TIMEOUT: return "EQL_ERR_TIMEOUT: a device-side bounded wait gave up";
  }
  return "EQL_ERR_UNKNOWN";
}

eqlinear_status_t eqlinear_plan_create(int T, int C, int D, eqlinear_dtype_t dtype,
                                       eqlinear_plan_t* out) {
  if (!out || C <= 0 || D <= 0 || T <= 0) return EQL_ERR_INVALID_ARG;
  if (dtype != EQL_F32 && dtype != EQL_F16) return EQL_ERR_INVALID_ARG;
  if (T > eql::kMaxT) return EQL_ERR_UNSUPPORTED;
  if ((int64_t)C * T > 0x7fffffff || (int64_t)D * T > 0x7fffffff) return EQL_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return EQL_ERR_CUDA;
  int sms = 0;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return EQL_ERR_CUDA;
  eqlinear_plan_s* p = new (std::nothrow) eqlinear_plan_s();
  if (!p) return EQL_ERR_INVALID_ARG;
  p->T = T;
  p->C = C;
  p->D = D;
  p->dtype = dtype;
  p->kernel = EQL_KERNEL_AUTO;
  p->device = dev;
  p->num_sms = sms;
  // Test hook for the failure-detection path: with EQL_DEBUG_DROP_W_STAGE=k in the
  // environment at plan creation, the tensor-core kernel's CTA 0 skips weight
  // stage k; its bounded waits then expire and eqlinear_get_status reports
  // EQL_ERR_TIMEOUT.  Unset (the normal case) it is off.
  p->debug_drop_w_stage = -1;
  if (const char* e = std::getenv("EQL_DEBUG_DROP_W_STAGE")) p->debug_drop_w_stage = std::atoi(e);
  make_twiddles(T, &p->tw);
  if (cudaMalloc(&p->status, sizeof(int)) != cudaSuccess) {
    delete p;
    return EQL_ERR_CUDA;
  }
  if (cudaMemset(p->status, 0, sizeof(int)) != cudaSuccess) {
    cudaFree(p->status);
    delete p;
    return EQL_ERR_CUDA;
  }
  *out = p;
  return EQL_OK;
}

void eqlinear_plan_destroy(eqlinear_plan_t p) {
  if (!p) return;
  if (p->status) cudaFree(p->status);
  delete p;
}

eqlinear_status_t eqlinear_plan_create_dihedral4(int C, int D, eqlinear_dtype_t dtype,
                                                 eqlinear_plan_t* out) {
  eqlinear_status_t s = eqlinear_plan_create(8, C, D, dtype, out);
  if (s == EQL_OK) (*out)->group = 1;
  return s;
}

// The D4 layer runs on the tensor cores only (FP16, C and D multiples of 16).
static bool d4_ok(eqlinear_plan_t p) {
  return p->dtype == EQL_F16 && p->kernel != EQL_KERNEL_SIMT && has_tiles(p);
}

eqlinear_status_t eqlinear_plan_set_kernel(eqlinear_plan_t p, eqlinear_kernel_t which) {
  if (!p) return EQL_ERR_INVALID_ARG;
  if (which != EQL_KERNEL_AUTO && which != EQL_KERNEL_SIMT && which != EQL_KERNEL_TCGEN05)
    return EQL_ERR_INVALID_ARG;
  p->kernel = which;
  return EQL_OK;
}

const char* eqlinear_forward_kernel_name(eqlinear_plan_t p, int64_t N) {
  if (!p) return "unsupported";
  const bool tc_ok = has_tiles(p) && eql::fwd_tc_supported(p->T, to_dt(p->dtype), N, p->C, p->D);
  if (p->group == 1) return d4_ok(p) && tc_ok ? "tcgen05" : "unsupported";
  if (p->kernel == EQL_KERNEL_TCGEN05) return tc_ok ? "tcgen05" : "unsupported";
  if (p->kernel == EQL_KERNEL_AUTO && tc_ok) return "tcgen05";
  return "simt";
}

// The tensor-core weight gradient needs 16-byte aligned X and dY (TMA); the
// name query assumes aligned buffers, as every torch allocation is.
static bool wgrad_tc_ok(eqlinear_plan_t p, int64_t N, const void* X, const void* dY) {
  return eql::wgrad_tc_supported(p->T, to_dt(p->dtype), N, p->C, p->D, X, dY);
}

static bool wgrad_use_tc(eqlinear_plan_t p, int64_t N, const void* X, const void* dY) {
  return p->kernel != EQL_KERNEL_SIMT && wgrad_tc_ok(p, N, X, dY);
}

const char* eqlinear_backward_weight_kernel_name(eqlinear_plan_t p, int64_t N) {
  if (!p) return "unsupported";
  if (p->group == 1) return p->kernel == EQL_KERNEL_TCGEN05 ? "unsupported" : "simt";
  const void* aligned = reinterpret_cast<const void*>(uintptr_t(256));
  const bool tc_ok = wgrad_tc_ok(p, N, aligned, aligned);
  if (p->kernel == EQL_KERNEL_TCGEN05) return tc_ok ? "tcgen05" : "unsupported";
  if (p->kernel == EQL_KERNEL_AUTO && tc_ok) return "tcgen05";
  return "simt";
}

size_t eqlinear_prepared_weight_bytes(eqlinear_plan_t p) {
  if (!p) return 0;
  if (p->group == 1)
    return d4_ok(p) ? 8 * plane_elems(p) * 2 + eql::tc_tile_bytes(8, p->C, p->D) +
                          (has_pair8_tiles(p) ? eql::pair8_tile_bytes(p->C, p->D) +
                                                    eql::pair8_tile_bytes(p->D, p->C)
                                              : 0)
                    : 0;
  size_t bytes = 2 * (size_t)eql::spec_planes(p->T) * plane_elems(p) * elem_size(p->dtype);
  if (has_tiles(p)) bytes += eql::tc_tile_bytes(p->T, p->C, p->D) + eql::tc_tile_bytes(p->T, p->D, p->C);
  if (has_pair_tiles(p)) bytes += eql::pair_tile_bytes(p->C, p->D) + eql::pair_tile_bytes(p->D, p->C);
  if (has_tf32_tiles(p))
    bytes += eql::pair_tf32_tile_bytes(p->C, p->D) + eql::pair_tf32_tile_bytes(p->D, p->C);
  if (has_pair8_tiles(p)) bytes += eql::pair8_tile_bytes(p->C, p->D) + eql::pair8_tile_bytes(p->D, p->C);
  return bytes;
}

eqlinear_status_t eqlinear_prepare_weights(eqlinear_plan_t p, const void* W, void* W_hat,
                                           void* stream) {
  EQL_TRACE();
  if (!p || !W || !W_hat) return EQL_ERR_INVALID_ARG;
  if (!aligned16(W) || !aligned16(W_hat)) return EQL_ERR_ALIGNMENT;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  void* fwd = W_hat;
  void* adj = const_cast<void*>(adj_block(p, W_hat));
  cudaStream_t st = (cudaStream_t)stream;
  if (p->group == 1) {
    if (!d4_ok(p)) return EQL_ERR_UNSUPPORTED;
    s = from_cuda(eql::launch_prepare_d4(W, p->C, p->D, fwd, st));
    if (s != EQL_OK) return s;
    s = from_cuda(eql::launch_tile_weights(8, fwd, p->C, p->D,
                                           const_cast<void*>(fwd_tiles(p, W_hat)), st, 1));
    if (s != EQL_OK || !has_pair8_tiles(p)) return s;
    s = from_cuda(eql::launch_pair8_tile_weights(
        fwd, p->C, p->D, const_cast<void*>(pair8_fwd_tiles(p, W_hat)), st));
    if (s != EQL_OK) return s;
    return from_cuda(eql::launch_pair8_tile_weights(
        fwd, p->D, p->C, const_cast<void*>(pair8_adj_tiles(p, W_hat)), st, 1));
  }
  s = from_cuda(eql::launch_prepare(p->T, to_dt(p->dtype), W, p->C, p->D, fwd, adj, p->tw, st));
  if (s == EQL_OK && has_tf32_tiles(p)) {
    s = from_cuda(eql::launch_pair_tf32_tile_weights(
        fwd, p->C, p->D, const_cast<void*>(tf32_fwd_tiles(p, W_hat)), st));
    if (s == EQL_OK)
      s = from_cuda(eql::launch_pair_tf32_tile_weights(
          adj, p->D, p->C, const_cast<void*>(tf32_adj_tiles(p, W_hat)), st));
    return s;
  }
  if (s != EQL_OK || !has_tiles(p)) return s;
  s = from_cuda(eql::launch_tile_weights(p->T, fwd, p->C, p->D, const_cast<void*>(fwd_tiles(p, W_hat)),
                                         st));
  if (s != EQL_OK) return s;
  s = from_cuda(eql::launch_tile_weights(p->T, adj, p->D, p->C,
                                         const_cast<void*>(adj_tiles(p, W_hat)), st));
  if (s == EQL_OK && has_pair8_tiles(p)) {
    s = from_cuda(eql::launch_pair8_tile_weights(
        fwd, p->C, p->D, const_cast<void*>(pair8_fwd_tiles(p, W_hat)), st));
    if (s == EQL_OK)
      s = from_cuda(eql::launch_pair8_tile_weights(
          adj, p->D, p->C, const_cast<void*>(pair8_adj_tiles(p, W_hat)), st));
    return s;
  }
  if (s != EQL_OK || !has_pair_tiles(p)) return s;
  s = from_cuda(eql::launch_pair_tile_weights(fwd, p->C, p->D,
                                              const_cast<void*>(pair_fwd_tiles(p, W_hat)), st));
  if (s != EQL_OK) return s;
  return from_cuda(eql::launch_pair_tile_weights(adj, p->D, p->C,
                                                 const_cast<void*>(pair_adj_tiles(p, W_hat)), st));
}

eqlinear_status_t eqlinear_forward(eqlinear_plan_t p, const void* X, int64_t N,
                                   const void* W_hat, const void* bias, void* Y, void* stream) {
  EQL_TRACE();
  return eqlinear_forward_act(p, X, N, W_hat, bias, EQL_ACT_NONE, Y, stream);
}

eqlinear_status_t eqlinear_forward_act(eqlinear_plan_t p, const void* X, int64_t N,
                                       const void* W_hat, const void* bias, eqlinear_act_t act,
                                       void* Y, void* stream) {
  EQL_TRACE();
  if (!p || N < 0) return EQL_ERR_INVALID_ARG;
  if (act != EQL_ACT_NONE && act != EQL_ACT_GELU) return EQL_ERR_INVALID_ARG;
  if (N == 0) return EQL_OK;
  if (!X || !W_hat || !Y) return EQL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_hat) || !aligned16(Y) || (bias && !aligned16(bias)))
    return EQL_ERR_ALIGNMENT;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  if (p->group == 1) {
    if (!d4_ok(p) || !eql::fwd_tc_supported(8, to_dt(p->dtype), N, p->C, p->D))
      return EQL_ERR_UNSUPPORTED;
    return from_cuda(eql::launch_fwd_tc(8, X, N, p->C, p->D, fwd_tiles(p, W_hat), bias, Y,
                                        p->status, p->num_sms, p->debug_drop_w_stage, (int)act,
                                        0, (cudaStream_t)stream, 1));
  }
  return run_forward_like(p, X, N, p->C, p->D, fwd_tiles(p, W_hat), adj_block(p, W_hat), bias,
                          Y, (int)act, (cudaStream_t)stream);
}

static bool spectral_ok(eqlinear_plan_t p, int64_t N) {
  return p->T == 4 && p->dtype == EQL_F16 && p->kernel != EQL_KERNEL_SIMT && has_tiles(p) &&
         eql::fwd_tc_supported(p->T, to_dt(p->dtype), N, p->C, p->D);
}

size_t eqlinear_spectral_bytes(eqlinear_plan_t p, int64_t N) {
  if (!p || N < 0) return 0;
  return (size_t)4 * (size_t)N * (size_t)p->D * 2;
}

static eqlinear_status_t forward_spectral_io(eqlinear_plan_t p, const void* X, int64_t N,
                                             const void* W_hat, const void* bias,
                                             eqlinear_act_t act, void* Y, int io, void* stream) {
  if (!p || N < 0) return EQL_ERR_INVALID_ARG;
  if (act != EQL_ACT_NONE && act != EQL_ACT_GELU) return EQL_ERR_INVALID_ARG;
  if (N == 0) return EQL_OK;
  if (!X || !W_hat || !Y) return EQL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W_hat) || !aligned16(Y) || (bias && !aligned16(bias)))
    return EQL_ERR_ALIGNMENT;
  if (!spectral_ok(p, N)) return EQL_ERR_UNSUPPORTED;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  return from_cuda(eql::launch_fwd_tc(p->T, X, N, p->C, p->D, fwd_tiles(p, W_hat), bias, Y,
                                      p->status, p->num_sms, p->debug_drop_w_stage, (int)act, io,
                                      (cudaStream_t)stream));
}

eqlinear_status_t eqlinear_forward_to_spectral(eqlinear_plan_t p, const void* X, int64_t N,
                                               const void* W_hat, const void* bias,
                                               eqlinear_act_t act, void* Xhat_next,
                                               void* stream) {
  EQL_TRACE();
  return forward_spectral_io(p, X, N, W_hat, bias, act, Xhat_next, 1, stream);
}

eqlinear_status_t eqlinear_forward_from_spectral(eqlinear_plan_t p, const void* Xhat, int64_t N,
                                                 const void* W_hat, const void* bias,
                                                 eqlinear_act_t act, void* Y, void* stream) {
  EQL_TRACE();
  return forward_spectral_io(p, Xhat, N, W_hat, bias, act, Y, 2, stream);
}

size_t eqlinear_tiled_spectrum_bytes(eqlinear_plan_t p, int64_t N, int channels) {
  if (!p || N < 0 || channels <= 0) return 0;
  if (p->dtype == EQL_F32) return eql::tiled_tf32_planes_bytes(N, channels);
  if (p->T == 8) return eql::tiled8_planes_bytes(N, channels);
  return eql::tiled_planes_bytes(N, channels);
}

// Tiled spectral input through the pair kernel: forward (adjoint = false:
// Cin = C, Cout = D, bias and act allowed) or dX (adjoint: Cin = D, Cout = C).
static eqlinear_status_t pair_io(eqlinear_plan_t p, const void* Xt, int64_t N, const void* W_hat,
                                 const void* bias, eqlinear_act_t act, void* out,
                                 int spectral_out, bool adjoint, void* stream) {
  if (!p || N < 0) return EQL_ERR_INVALID_ARG;
  if (act != EQL_ACT_NONE && act != EQL_ACT_GELU) return EQL_ERR_INVALID_ARG;
  if (N == 0) return EQL_OK;
  if (!Xt || !W_hat || !out) return EQL_ERR_INVALID_ARG;
  if (!aligned16(Xt) || !aligned16(W_hat) || !aligned16(out) || (bias && !aligned16(bias)))
    return EQL_ERR_ALIGNMENT;
  const int Cin = adjoint ? p->D : p->C, Cout = adjoint ? p->C : p->D;
  if (p->T == 8) {
    // eight-plane pair kernel; spatial output or the next layer's tiled planes
    if (!has_pair8_tiles(p) || p->kernel == EQL_KERNEL_SIMT ||
        !eql::pair8_supported(N, Cin, Cout))
      return EQL_ERR_UNSUPPORTED;
    eqlinear_status_t s = check_plan_device(p);
    if (s != EQL_OK) return s;
    return from_cuda(eql::launch_pair8_tc(
        Xt, N, Cin, Cout, adjoint ? pair8_adj_tiles(p, W_hat) : pair8_fwd_tiles(p, W_hat), bias,
        out, p->status, p->num_sms, (int)act, p->group, (cudaStream_t)stream,
        spectral_out ? 1 : 0));
  }
  if (p->dtype == EQL_F32) {
    // 3xTF32 on SM pairs; the output is spatial only
    if (!has_tf32_tiles(p) || p->kernel == EQL_KERNEL_SIMT || spectral_out ||
        !eql::pair_tf32_supported(N, Cin, Cout))
      return EQL_ERR_UNSUPPORTED;
    eqlinear_status_t s = check_plan_device(p);
    if (s != EQL_OK) return s;
    return from_cuda(eql::launch_pair_tf32(
        Xt, N, Cin, Cout, adjoint ? tf32_adj_tiles(p, W_hat) : tf32_fwd_tiles(p, W_hat), bias, out,
        p->status, p->num_sms, (int)act, (cudaStream_t)stream));
  }
  if (!has_pair_tiles(p) || p->kernel == EQL_KERNEL_SIMT ||
      !eql::pair_tc_supported(N, Cin, Cout))
    return EQL_ERR_UNSUPPORTED;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  return from_cuda(eql::launch_pair_tc(Xt, N, Cin, Cout,
                                       adjoint ? pair_adj_tiles(p, W_hat) : pair_fwd_tiles(p, W_hat),
                                       bias, out, p->status, p->num_sms, (int)act, spectral_out,
                                       (cudaStream_t)stream));
}

eqlinear_status_t eqlinear_group_dft(eqlinear_plan_t p, const void* X, int64_t N, int channels,
                                     void* Xt, void* stream) {
  EQL_TRACE();
  if (!p || N < 0) return EQL_ERR_INVALID_ARG;
  if (channels != p->C && channels != p->D) return EQL_ERR_INVALID_ARG;
  const bool f32 = p->dtype == EQL_F32;
  const bool eight = p->T == 8 && !f32 && channels % 16 == 0;
  if (!eight && (p->T != 4 || p->group != 0 || channels % (f32 ? 8 : 16) != 0))
    return EQL_ERR_UNSUPPORTED;
  if (N == 0) return EQL_OK;
  if (!X || !Xt) return EQL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Xt)) return EQL_ERR_ALIGNMENT;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  if (f32) return from_cuda(eql::launch_group_dft_tf32(X, N, channels, Xt, (cudaStream_t)stream));
  if (eight)
    return from_cuda(
        eql::launch_group_dft8_tiled(X, N, channels, p->group, Xt, (cudaStream_t)stream));
  return from_cuda(eql::launch_group_dft_tiled(X, N, channels, Xt, (cudaStream_t)stream));
}

eqlinear_status_t eqlinear_forward_tiled(eqlinear_plan_t p, const void* Xt, int64_t N,
                                         const void* W_hat, const void* bias, eqlinear_act_t act,
                                         void* Y, void* stream) {
  EQL_TRACE();
  return pair_io(p, Xt, N, W_hat, bias, act, Y, 0, false, stream);
}

eqlinear_status_t eqlinear_forward_tiled_next(eqlinear_plan_t p, const void* Xt, int64_t N,
                                              const void* W_hat, const void* bias,
                                              eqlinear_act_t act, void* Yt_next, void* stream) {
  EQL_TRACE();
  return pair_io(p, Xt, N, W_hat, bias, act, Yt_next, 1, false, stream);
}

size_t eqlinear_chain_tiled_workspace_bytes(eqlinear_plan_t first, eqlinear_plan_t second,
                                            int64_t N) {
  if (!first || !second || N < 0) return 0;
  return eql::pair_chain_sync_bytes(N);
}

eqlinear_status_t eqlinear_forward_chain_tiled(eqlinear_plan_t a, eqlinear_plan_t b,
                                               const void* Xt, int64_t N, const void* W1_hat,
                                               const void* bias1, eqlinear_act_t act1,
                                               const void* W2_hat, const void* bias2, void* Ht,
                                               void* Y, void* workspace, size_t workspace_bytes,
                                               void* stream) {
  EQL_TRACE();
  if (!a || !b || N < 0) return EQL_ERR_INVALID_ARG;
  if (act1 != EQL_ACT_NONE && act1 != EQL_ACT_GELU) return EQL_ERR_INVALID_ARG;
  if (a->D != b->C || a->device != b->device) return EQL_ERR_INVALID_ARG;
  if (!has_pair_tiles(a) || !has_pair_tiles(b) || a->kernel == EQL_KERNEL_SIMT ||
      b->kernel == EQL_KERNEL_SIMT)
    return EQL_ERR_UNSUPPORTED;
  if (N == 0) return EQL_OK;
  if (!Xt || !W1_hat || !W2_hat || !Ht || !Y || !workspace) return EQL_ERR_INVALID_ARG;
  if (!aligned16(Xt) || !aligned16(W1_hat) || !aligned16(W2_hat) || !aligned16(Ht) ||
      !aligned16(Y) || (bias1 && !aligned16(bias1)) || (bias2 && !aligned16(bias2)) ||
      !aligned16(workspace))
    return EQL_ERR_ALIGNMENT;
  if (workspace_bytes < eql::pair_chain_sync_bytes(N)) return EQL_ERR_WORKSPACE;
  if (!eql::pair_tc_supported(N, a->C, a->D) || !eql::pair_tc_supported(N, b->C, b->D))
    return EQL_ERR_UNSUPPORTED;
  eqlinear_status_t s = check_plan_device(a);
  if (s != EQL_OK) return s;
  return from_cuda(eql::launch_pair_chain_tc(
      Xt, N, a->C, a->D, b->D, pair_fwd_tiles(a, W1_hat), bias1, pair_fwd_tiles(b, W2_hat), bias2,
      Ht, Y, static_cast<int*>(workspace), a->status, a->num_sms, (int)act1,
      (cudaStream_t)stream));
}

eqlinear_status_t eqlinear_backward_input_tiled(eqlinear_plan_t p, const void* dYt, int64_t N,
                                                const void* W_hat, void* dX, void* stream) {
  EQL_TRACE();
  return pair_io(p, dYt, N, W_hat, nullptr, EQL_ACT_NONE, dX, 0, true, stream);
}

// Both layers must be p4 FP16 plans with tensor-core tiles whose widths chain.
static eqlinear_status_t chain_check(eqlinear_plan_t a, eqlinear_plan_t b, int64_t N) {
  if (!a || !b || N < 0) return EQL_ERR_INVALID_ARG;
  if (a->D != b->C || a->device != b->device) return EQL_ERR_INVALID_ARG;
  const bool ok = a->T == 4 && b->T == 4 && a->dtype == EQL_F16 && b->dtype == EQL_F16 &&
                  a->kernel != EQL_KERNEL_SIMT && b->kernel != EQL_KERNEL_SIMT &&
                  has_tiles(a) && has_tiles(b);
  if (!ok) return EQL_ERR_UNSUPPORTED;
  if (N > 0 && (!eql::fwd_tc_supported(4, eql::DType::F16, N, a->C, a->D) ||
                !eql::fwd_tc_supported(4, eql::DType::F16, N, b->C, b->D)))
    return EQL_ERR_UNSUPPORTED;
  return EQL_OK;
}

size_t eqlinear_chain_workspace_bytes(eqlinear_plan_t first, eqlinear_plan_t second, int64_t N) {
  if (chain_check(first, second, N) != EQL_OK) return 0;
  return std::max<size_t>(eql::chain_tc_sync_bytes(N), 16);
}

eqlinear_status_t eqlinear_forward_chain(eqlinear_plan_t first, eqlinear_plan_t second,
                                         const void* X, int64_t N, const void* W1_hat,
                                         const void* bias1, eqlinear_act_t act1,
                                         const void* W2_hat, const void* bias2,
                                         int spectral_intermediate, void* H, void* Y,
                                         void* workspace, size_t workspace_bytes, void* stream) {
  EQL_TRACE();
  eqlinear_status_t s = chain_check(first, second, N);
  if (s != EQL_OK) return s;
  if (act1 != EQL_ACT_NONE && act1 != EQL_ACT_GELU) return EQL_ERR_INVALID_ARG;
  if (spectral_intermediate != 0 && spectral_intermediate != 1) return EQL_ERR_INVALID_ARG;
  if (N == 0) return EQL_OK;
  if (!X || !W1_hat || !W2_hat || !H || !Y) return EQL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(W1_hat) || !aligned16(W2_hat) || !aligned16(H) ||
      !aligned16(Y) || (bias1 && !aligned16(bias1)) || (bias2 && !aligned16(bias2)) ||
      (workspace && !aligned16(workspace)))
    return EQL_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < eqlinear_chain_workspace_bytes(first, second, N))
    return EQL_ERR_WORKSPACE;
  s = check_plan_device(first);
  if (s != EQL_OK) return s;
  return from_cuda(eql::launch_chain_tc(
      X, N, first->C, first->D, second->D, fwd_tiles(first, W1_hat), bias1,
      fwd_tiles(second, W2_hat), bias2, H, Y, static_cast<int*>(workspace), first->status,
      first->num_sms, (int)act1, spectral_intermediate, (cudaStream_t)stream));
}

// ---- group-circulant convolution ----------------------------------------------

static eqlinear_status_t backward_weight_impl(eqlinear_plan_t p, const void* X, const void* dY,
                                              int64_t N, void* dW, void* dbias, void* workspace,
                                              size_t workspace_bytes, eql::DType out_dt,
                                              void* stream, int spectra);

static bool conv_plan_ok(eqlinear_plan_t p) {
  return p && p->T == 4 && p->dtype == EQL_F16 && p->kernel != EQL_KERNEL_SIMT && has_tiles(p);
}
static size_t conv_tap_tiles(eqlinear_plan_t p) { return eql::tc_tile_bytes(4, p->C, p->D); }
static size_t conv_tap_planes(eqlinear_plan_t p) {
  return (size_t)eql::spec_planes(4) * plane_elems(p) * elem_size(p->dtype);
}
static size_t conv_tap_adj_tiles(eqlinear_plan_t p) { return eql::tc_tile_bytes(4, p->D, p->C); }
// Wc_hat: [taps x forward tiles][taps x (forward planes, adjoint planes)][taps x adjoint tiles]
static const char* conv_adj_tiles(eqlinear_plan_t p, int taps, const void* Wc_hat) {
  return static_cast<const char*>(Wc_hat) +
         (size_t)taps * (conv_tap_tiles(p) + 2 * conv_tap_planes(p));
}

size_t eqlinear_conv_prepared_weight_bytes(eqlinear_plan_t p, int KH, int KW) {
  if (!conv_plan_ok(p) || KH < 1 || KW < 1 || KH > 15 || KW > 15) return 0;
  // per tap: operand tiles (read by the kernel, all taps first), the forward
  // and adjoint planes they are made from, then the adjoint tiles of the flipped
  // taps (dX)
  return (size_t)KH * KW * (conv_tap_tiles(p) + 2 * conv_tap_planes(p) + conv_tap_adj_tiles(p));
}

eqlinear_status_t eqlinear_conv_prepare_weights(eqlinear_plan_t p, int KH, int KW,
                                                const void* Wc, void* Wc_hat, void* stream) {
  EQL_TRACE();
  if (!p || !Wc || !Wc_hat || KH < 1 || KW < 1 || KH > 15 || KW > 15)
    return EQL_ERR_INVALID_ARG;
  if (!conv_plan_ok(p)) return EQL_ERR_UNSUPPORTED;
  if (!aligned16(Wc) || !aligned16(Wc_hat)) return EQL_ERR_ALIGNMENT;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  const int taps = KH * KW;
  char* tiles = static_cast<char*>(Wc_hat);
  char* planes = tiles + (size_t)taps * conv_tap_tiles(p);
  const size_t w_tap = (size_t)p->D * p->C * 4 * elem_size(p->dtype);
  for (int tap = 0; tap < taps; ++tap) {
    char* fwd = planes + (size_t)tap * 2 * conv_tap_planes(p);
    char* adj = fwd + conv_tap_planes(p);
    s = from_cuda(eql::launch_prepare(4, to_dt(p->dtype), static_cast<const char*>(Wc) + tap * w_tap,
                                      p->C, p->D, fwd, adj, p->tw, st));
    if (s != EQL_OK) return s;
    s = from_cuda(eql::launch_tile_weights(4, fwd, p->C, p->D,
                                           tiles + (size_t)tap * conv_tap_tiles(p), st));
    if (s != EQL_OK) return s;
  }
  // dX is the convolution of dY with the flipped kernel of adjoint taps: tap (i, j)
  // of it holds the adjoint tiles of tap (KH-1-i, KW-1-j)
  char* adj_tiles = const_cast<char*>(conv_adj_tiles(p, taps, Wc_hat));
  for (int tap = 0; tap < taps; ++tap) {
    const int src = (KH - 1 - tap / KW) * KW + (KW - 1 - tap % KW);
    const char* adj = planes + (size_t)src * 2 * conv_tap_planes(p) + conv_tap_planes(p);
    s = from_cuda(eql::launch_tile_weights(4, adj, p->D, p->C,
                                           adj_tiles + (size_t)tap * conv_tap_adj_tiles(p), st));
    if (s != EQL_OK) return s;
  }
  return EQL_OK;
}

// The convolution's weight gradient multiplies the padded rows' group spectra
// (computed once) when the tensor-core kernel's planes variant takes the shape.
static bool conv_wgrad_on_planes(eqlinear_plan_t p) {
  return p->kernel != EQL_KERNEL_SIMT && p->C % 64 == 0 && p->D % 64 == 0;
}

size_t eqlinear_conv_backward_workspace_bytes(eqlinear_plan_t p, int64_t N, int H, int W, int KH,
                                              int KW, int pad_h, int pad_w) {
  if (!conv_plan_ok(p) || N < 0 || H < 1 || W < 1 || KH < 1 || KW < 1 || pad_h < 0 || pad_w < 0)
    return 0;
  const int64_t Ho = (int64_t)H + 2 * pad_h - KH + 1, Wo = (int64_t)W + 2 * pad_w - KW + 1;
  if (Ho < 1 || Wo < 1) return 0;
  // dX: the group DFT planes of dY; dW: X and dY on the padded pixel grid, then
  // the layer weight gradient's scratch for all of its rows
  const size_t dx = eql::conv_tc_planes_bytes(N, (int)Ho, (int)Wo, p->D);
  const int64_t rows = N * ((int64_t)H + 2 * pad_h) * ((int64_t)W + 2 * pad_w);
  const size_t xpad = ((size_t)rows * p->C * 4 * elem_size(p->dtype) + 255) / 256 * 256;
  const size_t gpad = ((size_t)rows * p->D * 4 * elem_size(p->dtype) + 255) / 256 * 256;
  // the taps' weight gradients run over rows - (i*Wp + j) rows each
  size_t wg = 0;
  for (int tap = 0; tap < KH * KW; ++tap) {
    const int64_t off = (int64_t)(tap / KW) * (W + 2 * pad_w) + tap % KW;
    wg = std::max(wg, eqlinear_backward_weight_workspace_bytes(p, rows - off));
  }
  // with C and D multiples of 64, the padded rows' group spectra too (as large as
  // the padded rows), and all taps' weight gradients in one launch
  const bool planes = conv_wgrad_on_planes(p);
  const size_t spectra = planes ? xpad + gpad : 0;
  if (planes)
    wg = std::max(wg, eql::wgrad_tc_conv_workspace(rows, p->C, p->D, KH * KW, p->num_sms));
  const size_t dw = xpad + gpad + spectra + wg;
  return std::max<size_t>(std::max(dx, dw), 16);
}

eqlinear_status_t eqlinear_conv_backward_input(eqlinear_plan_t p, const void* dY, int64_t N, int H,
                                               int W, int KH, int KW, int pad_h, int pad_w,
                                               const void* Wc_hat, void* dX, void* workspace,
                                               size_t workspace_bytes, void* stream) {
  EQL_TRACE();
  if (!p || N < 0 || H < 1 || W < 1 || KH < 1 || KW < 1 || pad_h < 0 || pad_w < 0)
    return EQL_ERR_INVALID_ARG;
  if (!conv_plan_ok(p)) return EQL_ERR_UNSUPPORTED;
  const int64_t Ho = (int64_t)H + 2 * pad_h - KH + 1, Wo = (int64_t)W + 2 * pad_w - KW + 1;
  if (Ho < 1 || Wo < 1) return EQL_ERR_INVALID_ARG;
  if (N == 0) return EQL_OK;
  const int qh = KH - 1 - pad_h, qw = KW - 1 - pad_w;
  if (qh < 0 || qw < 0 ||
      !eql::conv_tc_supported(4, to_dt(p->dtype), N, (int)Ho, (int)Wo, p->D, p->C, KH, KW, qh, qw))
    return EQL_ERR_UNSUPPORTED;
  if (!dY || !Wc_hat || !dX) return EQL_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(Wc_hat) || !aligned16(dX) || (workspace && !aligned16(workspace)))
    return EQL_ERR_ALIGNMENT;
  if (!workspace ||
      workspace_bytes < eqlinear_conv_backward_workspace_bytes(p, N, H, W, KH, KW, pad_h, pad_w))
    return EQL_ERR_WORKSPACE;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  return from_cuda(eql::launch_conv_tc(dY, N, (int)Ho, (int)Wo, p->D, p->C, KH, KW, qh, qw,
                                       conv_adj_tiles(p, KH * KW, Wc_hat), nullptr, dX, workspace,
                                       p->status, p->num_sms, 0, (cudaStream_t)stream));
}

eqlinear_status_t eqlinear_conv_backward_weight(eqlinear_plan_t p, const void* X, int64_t N, int H,
                                                int W, const void* dY, int KH, int KW, int pad_h,
                                                int pad_w, void* dWc, void* dbias, void* workspace,
                                                size_t workspace_bytes, void* stream) {
  EQL_TRACE();
  if (!p || N < 0 || H < 1 || W < 1 || KH < 1 || KW < 1 || pad_h < 0 || pad_w < 0)
    return EQL_ERR_INVALID_ARG;
  if (!conv_plan_ok(p)) return EQL_ERR_UNSUPPORTED;
  const int64_t Ho = (int64_t)H + 2 * pad_h - KH + 1, Wo = (int64_t)W + 2 * pad_w - KW + 1;
  if (Ho < 1 || Wo < 1) return EQL_ERR_INVALID_ARG;
  if (!dWc) return EQL_ERR_INVALID_ARG;
  if (N > 0 && (!X || !dY)) return EQL_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || (dY && !aligned16(dY)) || !aligned16(dWc) ||
      (dbias && !aligned16(dbias)) || (workspace && !aligned16(workspace)))
    return EQL_ERR_ALIGNMENT;
  if (!workspace ||
      workspace_bytes < eqlinear_conv_backward_workspace_bytes(p, N, H, W, KH, KW, pad_h, pad_w))
    return EQL_ERR_WORKSPACE;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  // On the padded grid (Hp x Wp per image) X_pad[n,y,x] = X[n, y-ph, x-pw] (zero
  // outside) and dY_pad[n,y,x] = dY[n,y,x] for y < Ho, x < Wo (zero elsewhere).
  // Output pixel (n,y,x) of tap (i,j) reads X_pad[n, y+i, x+j]: flattened, the
  // row i*Wp + j after dY_pad's row, with no wrap (x+j < Wp, y+i < Hp), so
  // dWc[i][j] is the layer's weight gradient of X_pad shifted by i*Wp + j rows
  // and dY_pad.  The rows it drops at the end are past the last valid pixel of
  // dY_pad, hence zero.
  const int Hp = H + 2 * pad_h, Wp = W + 2 * pad_w;
  const int64_t rows = N * (int64_t)Hp * Wp;
  const size_t es = elem_size(p->dtype);
  const size_t xpad = ((size_t)rows * p->C * 4 * es + 255) / 256 * 256;
  const size_t gpad = ((size_t)rows * p->D * 4 * es + 255) / 256 * 256;
  const bool on_planes = conv_wgrad_on_planes(p) && N > 0;
  char* xp = static_cast<char*>(workspace);
  char* gp = xp + xpad;
  char* xs = gp + gpad;  // (on_planes) spectra [4][rows][C] and [4][rows][D]
  char* gs = xs + xpad;
  char* ws = on_planes ? gs + gpad : gp + gpad;
  const size_t ws_bytes = workspace_bytes - (size_t)(ws - xp);
  if (N > 0) {
    s = from_cuda(eql::launch_conv_shift_rows(X, N, H, W, p->C * 4, 0, 0, pad_h, pad_w, Hp, Wp,
                                              xp, st));
    if (s != EQL_OK) return s;
    s = from_cuda(eql::launch_conv_shift_rows(dY, N, (int)Ho, (int)Wo, p->D * 4, 0, 0, 0, 0, Hp,
                                              Wp, gp, st));
    if (s != EQL_OK) return s;
  }
  const size_t w_tap = (size_t)p->D * p->C * 4 * es;
  if (on_planes) {
    // the padded rows' group spectra once; then one launch of the planes variant
    // with the taps as in-channel tiles, tap (i, j) reading X's spectra from row
    // i*Wp + j on
    if (ws_bytes < eql::wgrad_tc_conv_workspace(rows, p->C, p->D, KH * KW, p->num_sms))
      return EQL_ERR_WORKSPACE;
    s = from_cuda(eql::launch_conv_group_planes(xp, rows, p->C, xs, st));
    if (s != EQL_OK) return s;
    s = from_cuda(eql::launch_conv_group_planes(gp, rows, p->D, gs, st));
    if (s != EQL_OK) return s;
    return from_cuda(eql::launch_wgrad_tc_conv(xs, gs, rows, p->C, p->D, KH * KW, KW, Wp, ws,
                                               to_dt(p->dtype), dWc, dbias, p->status,
                                               p->num_sms, p->tw, st));
  }
  for (int tap = 0; tap < KH * KW; ++tap) {
    const int64_t off = (int64_t)(tap / KW) * Wp + tap % KW;
    const int64_t n_rows = N > 0 ? rows - off : 0;
    // dbias (the same for every tap) with the first tap only
    s = backward_weight_impl(p, N > 0 ? xp + (size_t)off * p->C * 4 * es : nullptr,
                             N > 0 ? gp : nullptr, n_rows,
                             static_cast<char*>(dWc) + (size_t)tap * w_tap,
                             tap == 0 ? dbias : nullptr, ws, ws_bytes, to_dt(p->dtype), stream,
                             0);
    if (s != EQL_OK) return s;
  }
  return EQL_OK;
}

size_t eqlinear_conv_workspace_bytes(eqlinear_plan_t p, int64_t N, int H, int W) {
  if (!conv_plan_ok(p) || N < 0 || H < 0 || W < 0) return 0;
  return std::max<size_t>(eql::conv_tc_planes_bytes(N, H, W, p->C), 16);
}

eqlinear_status_t eqlinear_conv_forward(eqlinear_plan_t p, const void* X, int64_t N, int H, int W,
                                        int KH, int KW, int pad_h, int pad_w,
                                        const void* Wc_hat, const void* bias, eqlinear_act_t act,
                                        void* Y, void* workspace, size_t workspace_bytes,
                                        void* stream) {
  EQL_TRACE();
  if (!p || N < 0 || H < 1 || W < 1 || KH < 1 || KW < 1 || pad_h < 0 || pad_w < 0)
    return EQL_ERR_INVALID_ARG;
  if (act != EQL_ACT_NONE && act != EQL_ACT_GELU) return EQL_ERR_INVALID_ARG;
  if (!conv_plan_ok(p)) return EQL_ERR_UNSUPPORTED;
  if ((int64_t)H + 2 * pad_h - KH + 1 < 1 || (int64_t)W + 2 * pad_w - KW + 1 < 1)
    return EQL_ERR_INVALID_ARG;
  if (N == 0) return EQL_OK;
  if (!eql::conv_tc_supported(4, to_dt(p->dtype), N, H, W, p->C, p->D, KH, KW, pad_h, pad_w))
    return EQL_ERR_UNSUPPORTED;
  if (!X || !Wc_hat || !Y) return EQL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(Wc_hat) || !aligned16(Y) || (bias && !aligned16(bias)) ||
      (workspace && !aligned16(workspace)))
    return EQL_ERR_ALIGNMENT;
  if (!workspace || workspace_bytes < eqlinear_conv_workspace_bytes(p, N, H, W))
    return EQL_ERR_WORKSPACE;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  return from_cuda(eql::launch_conv_tc(X, N, H, W, p->C, p->D, KH, KW, pad_h, pad_w, Wc_hat, bias,
                                       Y, workspace, p->status, p->num_sms, (int)act,
                                       (cudaStream_t)stream));
}

// The forward-shaped product (Cin -> Cout) with the input's group spectrum
// also written to `spectrum` [4][N][Cin]: tensor cores only (T = 4, FP16).
static eqlinear_status_t save_spectrum_io(eqlinear_plan_t p, const void* X, int64_t N, int Cin,
                                          int Cout, const void* tiles, const void* bias,
                                          eqlinear_act_t act, void* Y, void* spectrum,
                                          void* stream) {
  if (!p || N < 0) return EQL_ERR_INVALID_ARG;
  if (act != EQL_ACT_NONE && act != EQL_ACT_GELU) return EQL_ERR_INVALID_ARG;
  if (!(p->T == 4 && p->group == 0 && p->dtype == EQL_F16 && p->kernel != EQL_KERNEL_SIMT &&
        has_tiles(p)))
    return EQL_ERR_UNSUPPORTED;
  if (N == 0) return EQL_OK;
  if (!X || !tiles || !Y || !spectrum) return EQL_ERR_INVALID_ARG;
  if (!aligned16(X) || !aligned16(tiles) || !aligned16(Y) || !aligned16(spectrum) ||
      (bias && !aligned16(bias)))
    return EQL_ERR_ALIGNMENT;
  if (!eql::fwd_tc_supported(4, eql::DType::F16, N, Cin, Cout)) return EQL_ERR_UNSUPPORTED;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  return from_cuda(eql::launch_fwd_tc(4, X, N, Cin, Cout, tiles, bias, Y, p->status, p->num_sms,
                                      p->debug_drop_w_stage, (int)act, 3, (cudaStream_t)stream,
                                      0, spectrum));
}

eqlinear_status_t eqlinear_forward_save_spectrum(eqlinear_plan_t p, const void* X, int64_t N,
                                                 const void* W_hat, const void* bias,
                                                 eqlinear_act_t act, void* Y, void* Xhat,
                                                 void* stream) {
  EQL_TRACE();
  if (!p || !W_hat) return EQL_ERR_INVALID_ARG;
  return save_spectrum_io(p, X, N, p->C, p->D, fwd_tiles(p, W_hat), bias, act, Y, Xhat, stream);
}

eqlinear_status_t eqlinear_backward_input_save_spectrum(eqlinear_plan_t p, const void* dY,
                                                        int64_t N, const void* W_hat, void* dX,
                                                        void* dYhat, void* stream) {
  EQL_TRACE();
  if (!p || !W_hat) return EQL_ERR_INVALID_ARG;
  return save_spectrum_io(p, dY, N, p->D, p->C, adj_tiles(p, W_hat), nullptr, EQL_ACT_NONE, dX,
                          dYhat, stream);
}

eqlinear_status_t eqlinear_backward_input(eqlinear_plan_t p, const void* dY, int64_t N,
                                          const void* W_hat, void* dX, void* stream) {
  EQL_TRACE();
  if (!p || N < 0) return EQL_ERR_INVALID_ARG;
  if (p->group == 1) return EQL_ERR_UNSUPPORTED;
  if (N == 0) return EQL_OK;
  if (!dY || !W_hat || !dX) return EQL_ERR_INVALID_ARG;
  if (!aligned16(dY) || !aligned16(W_hat) || !aligned16(dX)) return EQL_ERR_ALIGNMENT;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  // dX is the forward-shaped product with the adjoint weights: input width D,
  // output width C; the CUDA-core path reads the forward block [P][D][C].
  return run_forward_like(p, dY, N, p->D, p->C, adj_tiles(p, W_hat), fwd_block(p, W_hat),
                          nullptr, dX, 0, (cudaStream_t)stream);
}

// Enough for either kernel, so the size does not depend on which one runs.
size_t eqlinear_backward_weight_workspace_bytes(eqlinear_plan_t p, int64_t N) {
  if (!p || N < 0) return 0;
  if (p->group == 1) return eql::d4_wgrad_workspace(N, p->C, p->D, p->num_sms);
  size_t need = eql::wgrad_simt_workspace(p->T, N, p->C, p->D, p->num_sms);
  const void* aligned = reinterpret_cast<const void*>(uintptr_t(256));
  if (wgrad_tc_ok(p, N, aligned, aligned))
    need = std::max(need, eql::wgrad_tc_workspace(N, p->C, p->D, p->num_sms));
  return need;
}

// spectra = 1: X and dY are the group spectra [4][N][C] and [4][N][D] that
// the save-spectrum calls wrote (tensor cores only; C and D multiples of 64);
// spectra = 2: the tiled planes eqlinear_group_dft writes (C, D multiples of 16).
static eqlinear_status_t backward_weight_impl(eqlinear_plan_t p, const void* X, const void* dY,
                                              int64_t N, void* dW, void* dbias, void* workspace,
                                              size_t workspace_bytes, eql::DType out_dt,
                                              void* stream, int spectra = 0) {
  if (!p || N < 0 || !dW) return EQL_ERR_INVALID_ARG;
  if (p->group == 1 && (spectra || p->kernel == EQL_KERNEL_TCGEN05)) return EQL_ERR_UNSUPPORTED;
  if (N > 0 && (!X || !dY)) return EQL_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || (dY && !aligned16(dY)) || !aligned16(dW) ||
      (dbias && !aligned16(dbias)) || (workspace && !aligned16(workspace)))
    return EQL_ERR_ALIGNMENT;
  if (spectra == 1 && !(p->T == 4 && p->dtype == EQL_F16 && p->kernel != EQL_KERNEL_SIMT &&
                        p->C % 64 == 0 && p->D % 64 == 0))
    return EQL_ERR_UNSUPPORTED;
  if (spectra == 2 && !(p->T == 4 && p->group == 0 && p->dtype == EQL_F16 &&
                        p->kernel != EQL_KERNEL_SIMT && has_tiles(p)))
    return EQL_ERR_UNSUPPORTED;
  if (!spectra && p->kernel == EQL_KERNEL_TCGEN05 && !wgrad_tc_ok(p, N, X, dY))
    return EQL_ERR_UNSUPPORTED;
  if (!workspace || workspace_bytes < eqlinear_backward_weight_workspace_bytes(p, N))
    return EQL_ERR_WORKSPACE;
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  cudaStream_t st = (cudaStream_t)stream;
  if (p->group == 1)  // D4: CUDA cores
    return from_cuda(eql::launch_d4_wgrad(X, dY, N, p->C, p->D, out_dt, dW, dbias,
                                          static_cast<float*>(workspace), p->num_sms, st));
  if (spectra == 1 && N > 0) {
    if (!eql::wgrad_tc_planes_supported(N, p->C, p->D, X, dY)) return EQL_ERR_UNSUPPORTED;
    return from_cuda(eql::launch_wgrad_tc(X, dY, N, p->C, p->D, workspace, out_dt, dW, dbias,
                                          p->status, p->num_sms, p->tw, st, 1));
  }
  if (spectra == 2 && N > 0) {
    if (!eql::wgrad_tc_supported(4, eql::DType::F16, N, p->C, p->D, X, dY))
      return EQL_ERR_UNSUPPORTED;
    return from_cuda(eql::launch_wgrad_tc(X, dY, N, p->C, p->D, workspace, out_dt, dW, dbias,
                                          p->status, p->num_sms, p->tw, st, 2));
  }
  if (!spectra && wgrad_use_tc(p, N, X, dY))
    return from_cuda(eql::launch_wgrad_tc(X, dY, N, p->C, p->D, workspace, out_dt, dW, dbias,
                                          p->status, p->num_sms, p->tw, st));
  const int splits = eql::wgrad_simt_splits(p->T, N, p->C, p->D, p->num_sms);
  return from_cuda(eql::launch_wgrad_simt(p->T, to_dt(p->dtype), out_dt, X, dY, N, p->C, p->D,
                                          dW, dbias, static_cast<float*>(workspace), splits,
                                          p->tw, st));
}

eqlinear_status_t eqlinear_backward_weight(eqlinear_plan_t p, const void* X, const void* dY,
                                           int64_t N, void* dW, void* dbias, void* workspace,
                                           size_t workspace_bytes, void* stream) {
  EQL_TRACE();
  if (!p) return EQL_ERR_INVALID_ARG;
  return backward_weight_impl(p, X, dY, N, dW, dbias, workspace, workspace_bytes,
                              to_dt(p->dtype), stream);
}

eqlinear_status_t eqlinear_backward_weight_f32(eqlinear_plan_t p, const void* X, const void* dY,
                                               int64_t N, float* dW, float* dbias,
                                               void* workspace, size_t workspace_bytes,
                                               void* stream) {
  EQL_TRACE();
  return backward_weight_impl(p, X, dY, N, dW, dbias, workspace, workspace_bytes,
                              eql::DType::F32, stream);
}

eqlinear_status_t eqlinear_backward_weight_from_spectra(eqlinear_plan_t p, const void* Xhat,
                                                        const void* dYhat, int64_t N, void* dW,
                                                        void* dbias, void* workspace,
                                                        size_t workspace_bytes, void* stream) {
  EQL_TRACE();
  if (!p) return EQL_ERR_INVALID_ARG;
  return backward_weight_impl(p, Xhat, dYhat, N, dW, dbias, workspace, workspace_bytes,
                              to_dt(p->dtype), stream, 1);
}

eqlinear_status_t eqlinear_backward_weight_from_spectra_f32(eqlinear_plan_t p, const void* Xhat,
                                                            const void* dYhat, int64_t N,
                                                            float* dW, float* dbias,
                                                            void* workspace,
                                                            size_t workspace_bytes, void* stream) {
  EQL_TRACE();
  return backward_weight_impl(p, Xhat, dYhat, N, dW, dbias, workspace, workspace_bytes,
                              eql::DType::F32, stream, 1);
}

eqlinear_status_t eqlinear_backward_weight_tiled(eqlinear_plan_t p, const void* Xt,
                                                  const void* dYt, int64_t N, void* dW,
                                                  void* dbias, void* workspace,
                                                  size_t workspace_bytes, void* stream) {
  EQL_TRACE();
  if (!p) return EQL_ERR_INVALID_ARG;
  return backward_weight_impl(p, Xt, dYt, N, dW, dbias, workspace, workspace_bytes,
                              to_dt(p->dtype), stream, 2);
}

eqlinear_status_t eqlinear_backward_weight_tiled_f32(eqlinear_plan_t p, const void* Xt,
                                                      const void* dYt, int64_t N, float* dW,
                                                      float* dbias, void* workspace,
                                                      size_t workspace_bytes, void* stream) {
  EQL_TRACE();
  return backward_weight_impl(p, Xt, dYt, N, dW, dbias, workspace, workspace_bytes,
                              eql::DType::F32, stream, 2);
}

eqlinear_status_t eqlinear_cast_from_f32(eqlinear_plan_t p, const float* src, int64_t count,
                                         void* dst, void* stream) {
  EQL_TRACE();
  if (!p || count < 0) return EQL_ERR_INVALID_ARG;
  if (count == 0) return EQL_OK;
  if (!src || !dst) return EQL_ERR_INVALID_ARG;
  const char* s0 = reinterpret_cast<const char*>(src);
  const char* d0 = static_cast<const char*>(dst);
  const size_t sb = (size_t)count * sizeof(float), db = (size_t)count * elem_size(p->dtype);
  const bool same_f32 = s0 == d0 && p->dtype == EQL_F32;  // a no-op
  if (!same_f32 && s0 < d0 + db && d0 < s0 + sb) return EQL_ERR_INVALID_ARG;  // overlap
  eqlinear_status_t s = check_plan_device(p);
  if (s != EQL_OK) return s;
  return from_cuda(eql::launch_cast_from_f32(to_dt(p->dtype), src, dst, count,
                                             (cudaStream_t)stream));
}

eqlinear_status_t eqlinear_get_status(eqlinear_plan_t p, void* stream) {
  EQL_TRACE();
  if (!p) return EQL_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return EQL_ERR_CUDA;
  int h = 0;
  if (cudaMemcpy(&h, p->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
    return EQL_ERR_CUDA;
  if (h != 0) {
    if (cudaMemset(p->status, 0, sizeof(int)) != cudaSuccess) return EQL_ERR_CUDA;
    return EQL_ERR_TIMEOUT;
  }
  return EQL_OK;
}

}  // extern "C"
