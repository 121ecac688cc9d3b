// Internal definition of the opaque plan handle of include/eqlinear.h.
#pragma once

#include <nvtx3/nvToolsExt.h>

#include "../../include/eqlinear.h"
#include "eql_common.cuh"

// One NVTX range per ABI call, named after the entry point (seen by Nsight
// tools and by ncu's --nvtx filters; header-only NVTX does nothing when no
// tool is attached).
struct EqlTraceRange {
  explicit EqlTraceRange(const char* name) { nvtxRangePushA(name); }
  ~EqlTraceRange() { nvtxRangePop(); }
  EqlTraceRange(const EqlTraceRange&) = delete;
  EqlTraceRange& operator=(const EqlTraceRange&) = delete;
};
#define EQL_TRACE() EqlTraceRange eql_trace_range_(__func__)

struct eqlinear_plan_s {
  int T, C, D;
  eqlinear_dtype_t dtype;
  eqlinear_kernel_t kernel;
  int device;
  int num_sms;
  int* status;  // device word written by kernels whose bounded waits give up
  int debug_drop_w_stage;  // test-only fault injection (EQL_DEBUG_DROP_W_STAGE), -1 = off
  int group;               // 0: cyclic group of order T; 1: dihedral group D4 (T = 8)
  eql::Twiddles tw;
};
