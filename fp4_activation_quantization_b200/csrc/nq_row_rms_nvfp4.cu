// nq_row_rms_nvfp4.cu — instantiates the row kernel for RMSNorm (+residual) + NVFP4
// (every built schedule, vector and scalar paths).  One file per operation so
// that the kernels compile in parallel.
#include "nq_row_kernel.cuh"

namespace nq {
const RowKernels& row_kernels_rms_nvfp4() {
  static const RowTable<kOpRmsNvfp4, 0> table;
  return table.k;
}
}  // namespace nq
