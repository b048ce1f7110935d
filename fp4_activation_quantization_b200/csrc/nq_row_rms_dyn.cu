// nq_row_rms_dyn.cu — instantiates the row kernel for residual-add + RMSNorm + dynamic per-token
// e4m3 (every built schedule and variant).  One file per operation and FP8
// format so that the kernels compile in parallel.
#include "nq_row_kernel.cuh"

namespace nq {
const RowKernels& row_kernels_rms_dyn() {
  static const RowTable<kOpRmsDynFp8, 0> table;
  return table.k;
}
}  // namespace nq
