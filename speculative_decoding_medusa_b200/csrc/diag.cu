// medusa_wait_flag: the library's bounded flag wait, run on a caller's flag.
//
// Every wait inside the library's kernels gives up after a budget of clock
// cycles, reports MEDUSA_ERR_TIMEOUT and returns.  This kernel runs the same
// wait (the one the heads' first GEMM uses for its stream-K partials) on a
// flag the caller owns, with a budget the caller chooses, so that the
// failure path can be exercised without anything being broken: a flag that
// nothing sets makes the wait run out.  Nothing asynchronous is outstanding
// in the kernel when it gives up.
#include <cuda_runtime.h>
#include <stdint.h>

#include "abi_internal.h"
#include "common.cuh"

namespace medusa {

__global__ void wait_flag_kernel(const int32_t* flag, int32_t value, long long budget,
                                 int32_t* status) {
  grid_dep_wait();
  grid_dep_launch();
  __shared__ int abort_flag;
  abort_flag = 0;
  wait_flag_bounded(flag, value, &abort_flag, status, budget);
}

medusa_status_t wait_flag(const int32_t* flag, int32_t value, long long budget_cycles,
                          int32_t* status, cudaStream_t stream) {
  const long long budget = budget_cycles > 0 ? budget_cycles : kSpinBudgetCycles;
  launch(wait_flag_kernel, 1, 1, 0, stream, flag, value, budget, status);
  return check_launch("wait_flag");
}

}  // namespace medusa

extern "C" medusa_status_t medusa_wait_flag(const int32_t* flag, int32_t value,
                                            long long budget_cycles, int32_t* dev_status,
                                            void* stream) {
  if (flag == nullptr || dev_status == nullptr)
    return medusa::fail(MEDUSA_ERR_INVALID_ARG, "wait_flag: null pointer");
  if ((reinterpret_cast<uintptr_t>(flag) & 3u) != 0)
    return medusa::fail(MEDUSA_ERR_ALIGNMENT, "wait_flag: flag must be 4-byte aligned");
  if (budget_cycles > medusa::kSpinBudgetCycles)
    return medusa::fail(MEDUSA_ERR_SHAPE, "wait_flag: budget above the library's bound");
  return medusa::wait_flag(flag, value, budget_cycles, dev_status,
                           static_cast<cudaStream_t>(stream));
}
