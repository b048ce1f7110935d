// nq_row_rms_group_e5m2_layout.cu — instantiates the row kernel for RMSNorm (+residual)
// + per-token-group e5m2 with column-major or packed-UE8M0 group scales (every
// built schedule and variant).  One file per operation and output form so
// that the kernels compile in parallel.
#include "nq_row_kernel.cuh"

namespace nq {
const RowKernels& row_kernels_rms_group_e5m2_layout() {
  static const RowTable<kOpRmsGroupFp8, kOutAlt | kOutScaleLayout> table;
  return table.k;
}
}  // namespace nq
