// nq_row_rms_dyn_e5m2.cu — instantiates the row kernel for residual-add + RMSNorm + dynamic per-token
// e5m2 (every built schedule and variant).  One file per operation and FP8
// format so that the kernels compile in parallel.
#include "nq_row_kernel.cuh"

namespace nq {
const RowKernels& row_kernels_rms_dyn_e5m2() {
  static const RowTable<kOpRmsDynFp8, kOutAlt> table;
  return table.k;
}
}  // namespace nq
