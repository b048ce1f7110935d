// nq_row_rms_static.cu — instantiates the row kernel for RMSNorm (+residual) + static-scale
// e4m3 (every built schedule and variant).  One file per operation and FP8
// format so that the kernels compile in parallel.
#include "nq_row_kernel.cuh"

namespace nq {
const RowKernels& row_kernels_rms_static() {
  static const RowTable<kOpRmsStaticFp8, 0> table;
  return table.k;
}
}  // namespace nq
