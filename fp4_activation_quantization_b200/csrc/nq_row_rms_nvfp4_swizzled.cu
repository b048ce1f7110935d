// nq_row_rms_nvfp4_swizzled.cu — instantiates the row kernel for RMSNorm
// (+residual) + NVFP4 with block scales in the swizzled 128 x 4-tile layout
// (every built schedule and variant).  One file per operation and output form
// so that the kernels compile in parallel.
#include "nq_row_kernel.cuh"

namespace nq {
const RowKernels& row_kernels_rms_nvfp4_swizzled() {
  static const RowTable<kOpRmsNvfp4, kOutAlt> table;
  return table.k;
}
}  // namespace nq
