// Weight gradient for callers that cannot allocate device memory.
//
// eqlinear_backward_weight needs a caller-provided FP32 workspace for the
// partial spectra of its split reduction over rows.  Some callers cannot hand
// one over: a host program whose device memory is fully owned by another
// allocator or carved into a fixed arena at start-up, or a latency-critical
// loop that must not call cudaMalloc/cudaFree because those calls can
// synchronise the device and stall every other stream.  For them this file
// provides eqlinear_backward_weight_noalloc, which uses a scratch array that the
// library itself reserves as a file-scope __device__ variable.  The array exists
// on every GPU on which the library's module is loaded, for the lifetime of the
// process, and is shared by every call on that GPU.
#include <cstring>
#include <mutex>

#include "../../include/eqlinear.h"
#include "eql_kernels.h"
#include "eql_plan.h"

namespace {

// 16 MiB of FP32 partial spectra.  One row split needs T*C*D + D floats.
constexpr size_t kScratchFloats = size_t(4) << 20;
__device__ __align__(256) float g_wgrad_scratch[kScratchFloats];

// Device address of g_wgrad_scratch per device.  In host code the symbol name
// is only a host-side stand-in; the real address has to be asked for with the
// device current, once per device.
constexpr int kMaxDevices = 128;
float* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

cudaError_t scratch_address(int device, float** out) {
  if (device < 0 || device >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[device]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_wgrad_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[device] = static_cast<float*>(p);
  }
  *out = g_scratch_addr[device];
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" eqlinear_status_t eqlinear_backward_weight_noalloc(eqlinear_plan_t p, const void* X,
                                                              const void* dY, int64_t N,
                                                              void* dW, void* dbias,
                                                              void* stream) {
  if (!p || N < 0 || !dW) return EQL_ERR_INVALID_ARG;
  if (p->group == 1) return EQL_ERR_UNSUPPORTED;  // the D4 layer has no backward
  if (N > 0 && (!X || !dY)) return EQL_ERR_INVALID_ARG;
  if ((X && !aligned16(X)) || (dY && !aligned16(dY)) || !aligned16(dW) ||
      (dbias && !aligned16(dbias)))
    return EQL_ERR_ALIGNMENT;
  // one split of partial spectra must fit in the built-in scratch
  const size_t per_split = (size_t)p->T * p->C * p->D + (size_t)p->D;
  if (per_split > kScratchFloats) return EQL_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return EQL_ERR_CUDA;
  if (dev != p->device) return EQL_ERR_INVALID_ARG;
  float* scratch = nullptr;
  if (scratch_address(dev, &scratch) != cudaSuccess) return EQL_ERR_CUDA;
  // same split count as the allocating entry point, capped by the scratch size;
  // every partial the kernels later read is written first, so nothing needs
  // clearing between calls
  int splits = eql::wgrad_simt_splits(p->T, N, p->C, p->D, p->num_sms);
  const int fit = (int)(kScratchFloats / per_split);
  if (splits > fit) splits = fit;
  const eql::DType dt = p->dtype == EQL_F32 ? eql::DType::F32 : eql::DType::F16;
  const cudaError_t e = eql::launch_wgrad_simt(p->T, dt, dt, X, dY, N, p->C, p->D, dW,
                                               dbias, scratch, splits, p->tw,
                                               (cudaStream_t)stream);
  if (e == cudaSuccess) return EQL_OK;
  return e == cudaErrorNotSupported ? EQL_ERR_UNSUPPORTED : EQL_ERR_CUDA;
}
