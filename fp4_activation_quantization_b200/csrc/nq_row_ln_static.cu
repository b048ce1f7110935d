// nq_row_ln_static.cu — instantiates the row kernel for LayerNorm + static-scale
// e4m3 (every built schedule and variant).  One file per operation and FP8
// format so that the kernels compile in parallel.
#include "nq_row_kernel.cuh"

namespace nq {
const RowKernels& row_kernels_ln_static() {
  static const RowTable<kOpLnStaticFp8, 0> table;
  return table.k;
}
}  // namespace nq
