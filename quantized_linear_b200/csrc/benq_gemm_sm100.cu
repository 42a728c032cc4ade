// BenQ prefill GEMM on sm_100a tensor cores (tcgen05).  Placeholder until the kernel lands.
#include "ql_internal.cuh"

namespace {
__device__ int g_gemm_timeout = 0;
}

namespace ql {

ql_status benq_gemm_launch(const uint8_t *, const uint16_t *, const uint16_t *, void *, ql_out_dtype, int M, int, int,
                           cudaStream_t) {
  return fail(QL_ERR_UNSUPPORTED, "benq_linear: batch %d > 16 (tensor-core GEMM) not built yet", M);
}

ql_status benq_gemm_read_timeout(int *flag) {
  int zero = 0;
  if (cudaMemcpyFromSymbol(flag, g_gemm_timeout, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_gemm_timeout, &zero, sizeof(int)) != cudaSuccess)
    return fail(QL_ERR_CUDA, "ql_check: cannot read the device timeout flag");
  return QL_OK;
}

}  // namespace ql
