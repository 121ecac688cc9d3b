// Internal definition of the opaque plan handle of include/eqlinear.h.
#pragma once

#include "../../include/eqlinear.h"
#include "eql_common.cuh"

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
