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
#include <cuda.h>

#include <cstring>
#include <mutex>

#include "../../include/eqlinear.h"
#include "eql_kernels.h"
#include "eql_plan.h"

namespace {

// 16 MiB of FP32 partial spectra.  One row split needs T*C*D + D floats.
constexpr size_t kScratchFloats = size_t(4) << 20;
__device__ __align__(256) float g_wgrad_scratch[kScratchFloats];

// Device address of g_wgrad_scratch per CUDA context.  In host code the symbol
// name is only a host-side stand-in; the real address has to be asked for with
// the device current.  The module (and with it the array) is loaded once per
// context, so the address is cached per context, keyed by the driver's unique
// context id (never reused within a process): after cudaDeviceReset, or in a
// caller's own non-primary context, the lookup runs again instead of handing
// a stale address to the kernels.
constexpr int kMaxContexts = 64;
struct ScratchEntry {
  unsigned long long ctx_id;
  float* addr;
};
ScratchEntry g_scratch[kMaxContexts] = {};
int g_scratch_n = 0, g_scratch_next = 0;
std::mutex g_scratch_mu;

// Driver entry points, fetched through the runtime (the library does not link
// the driver library directly, so it loads on machines without a GPU driver).
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
template <typename Fn>
Fn driver_fn(const char* name) {
  void* f = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &f, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(f);
}

bool current_context_id(unsigned long long* id) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  CUcontext ctx = nullptr;
  return get_current && get_id && get_current(&ctx) == CUDA_SUCCESS && ctx != nullptr &&
         get_id(ctx, id) == CUDA_SUCCESS;
}

cudaError_t scratch_address(float** out) {
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  unsigned long long id = 0;
  bool have_id = current_context_id(&id);
  if (have_id)
    for (int i = 0; i < g_scratch_n; ++i)
      if (g_scratch[i].ctx_id == id) {
        *out = g_scratch[i].addr;
        return cudaSuccess;
      }
  // first call in this context (the lookup also makes the runtime's context
  // current on this thread if none was)
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, g_wgrad_scratch);
  if (e != cudaSuccess) return e;
  if (!have_id) have_id = current_context_id(&id);
  if (have_id) {
    g_scratch[g_scratch_next] = ScratchEntry{id, static_cast<float*>(p)};
    g_scratch_next = (g_scratch_next + 1) % kMaxContexts;
    if (g_scratch_n < kMaxContexts) ++g_scratch_n;
  }
  *out = static_cast<float*>(p);
  return cudaSuccess;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" eqlinear_status_t eqlinear_backward_weight_noalloc(eqlinear_plan_t p, const void* X,
                                                              const void* dY, int64_t N,
                                                              void* dW, void* dbias,
                                                              void* stream) {
  EQL_TRACE();
  if (!p || N < 0 || !dW) return EQL_ERR_INVALID_ARG;
  // the D4 weight gradient has its own kernel (eqlinear_backward_weight)
  if (p->group == 1) return EQL_ERR_UNSUPPORTED;
  // this call always runs the CUDA-core kernels; a plan forced to the tensor
  // cores asked for something it cannot give
  if (p->kernel == EQL_KERNEL_TCGEN05) return EQL_ERR_UNSUPPORTED;
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
  if (scratch_address(&scratch) != cudaSuccess) return EQL_ERR_CUDA;
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
