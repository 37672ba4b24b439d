// k_gemm.cu -- batched dequantize-and-multiply on the sm_100a tensor cores (tcgen05).
//
// Placeholder until the tcgen05 kernel lands: no shape is eligible, so cq_dequant_gemm
// takes the GEMV kernels in slices of 8 batch columns.
#include "cq_internal.cuh"

namespace cq {

bool gemm_tc_eligible(const cq_qweight &, cq_dtype, int) { return false; }

size_t gemm_tc_workspace(int64_t, int64_t, int) { return 0; }

cq_status launch_gemm_tc(const cq_qweight &, const void *, int, float *, void *, size_t, cudaStream_t) {
  return fail(CQ_ERR_UNSUPPORTED, "cq_dequant_gemm: tensor-core path not built");
}

}  // namespace cq
