// nq_row_rms_dyn_scatter.cu — instantiates the row kernel for residual-add + RMSNorm + dynamic per-token e4m3
// with the rows stored to MoE destination rows (every built schedule of the
// register-row kernel).  One file per operation and output form so that the
// kernels compile in parallel.
#include "nq_row_kernel.cuh"

namespace nq {
const RowKernels& row_kernels_rms_dyn_scatter() {
  static const RowTable<kOpRmsDynFp8, kOutScatter> table;
  return table.k;
}
}  // namespace nq
