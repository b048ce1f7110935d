// nq_row_ln_static_e5m2.cu — instantiates the row kernel for LayerNorm + static-scale
// e5m2 (every built schedule and variant).  One file per operation and FP8
// format so that the kernels compile in parallel.
#include "nq_row_kernel.cuh"

namespace nq {
const RowKernels& row_kernels_ln_static_e5m2() {
  static const RowTable<kOpLnStaticFp8, kOutAlt> table;
  return table.k;
}
}  // namespace nq
