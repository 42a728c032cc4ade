// Internal helpers shared by the libqlinear translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "qlinear.h"

namespace ql {

// Records a message for ql_last_error() and returns `s`.
ql_status fail(ql_status s, const char *fmt, ...);
// Converts the launch state of the last kernel into a status (QL_ERR_CUDA on failure).
ql_status launch_status(const char *what);
// Multiprocessor count of the current device (cached per device).
int sm_count();
// cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes), skipped when the
// current device has already allowed `k` at least `bytes`.
cudaError_t set_max_smem(const void *k, int bytes);
template <typename... KArgs>
cudaError_t set_max_smem(void (*k)(KArgs...), int bytes) {
  return set_max_smem(reinterpret_cast<const void *>(k), bytes);
}
// Resident blocks of `k` per SM at this block size and dynamic shared memory on the current device
// (cudaOccupancyMaxActiveBlocksPerMultiprocessor, cached); 0 if the query fails.
int blocks_per_sm(const void *k, int threads, size_t smem);
template <typename... KArgs>
int blocks_per_sm(void (*k)(KArgs...), int threads, size_t smem) {
  return blocks_per_sm(reinterpret_cast<const void *>(k), threads, smem);
}

inline bool aligned(const void *p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Whether kernels are launched with programmatic dependent launch (ql_set_pdl).
bool pdl_enabled();

// Launches `k` on `s`, allowed to overlap the tail of the preceding kernel in the stream when
// overlap is enabled.  Every kernel launched this way calls qld::pdl_wait() before it reads
// anything but weights and before its first global store.
template <typename... KArgs, typename... Args>
cudaError_t launch(void (*k)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k, std::forward<Args>(args)...);
}

// ---- entry points implemented by the kernel translation units (arguments already validated) ----
ql_status benq_dequant_launch(const uint8_t *codes, const uint16_t *lut, uint16_t *W, int N, int K,
                              cudaStream_t s);
ql_status benq_gemv_launch(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y,
                           ql_out_dtype ydt, int B, int N, int K, cudaStream_t s);
ql_status benq_gemv_multi_launch(const benq_layer *layers, int S, const uint16_t *x, ql_out_dtype ydt, int B,
                                 int K, cudaStream_t s);
size_t benq_gemm_workspace_size(int M, int N, int K);
size_t benq_mlp_workspace_size(int B, int N, int K);
ql_status benq_encode_launch(const uint16_t *W, uint8_t *codes, uint16_t *lut, int N, int K, int iters,
                             cudaStream_t s);
ql_status benq_mlp_launch(const uint8_t *codes_g, const uint16_t *lut_g, const uint8_t *codes_u,
                          const uint16_t *lut_u, const uint16_t *x, void *h, ql_out_dtype ydt, int B, int N,
                          int K, void *ws, size_t ws_bytes, cudaStream_t s);
ql_status benq_gemm_launch(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y,
                           ql_out_dtype ydt, int M, int N, int K, void *ws, size_t ws_bytes, cudaStream_t s);
ql_status benq_gemm_read_timeout(int *flag);
ql_status selftest_timeout_launch(cudaStream_t s);  // reads and clears the GEMM's bounded-wait flag

size_t mdbf_workspace_size(int P, int n, int m, int r, int l, int B);
ql_status mdbf_linear_launch(const mdbf_path *paths, int P, int n, int m, int r, int l,
                             const uint16_t *x, void *y, ql_out_dtype ydt, int B, void *ws,
                             cudaStream_t s);
ql_status mdbf_linear_multi_launch(const mdbf_path *paths, int S, int P, int n, int m, int r, int l,
                                   const uint16_t *x, void *const *ys, ql_out_dtype ydt, int B, void *ws,
                                   cudaStream_t s);
ql_status mdbf_read_timeout(int *flag);   // reads and clears the MDBF kernels' bounded-wait flag
// batched MDBF (l * B above the decode kernels' limit) on the tensor cores, mdbf_gemm_sm100.cu:
// envelope ranks up to MDBF_GEMM_LMAX and layers whose n, m and r are all at least
// MDBF_GEMM_MIN.  Smaller layers would leave most of each 512 x 256 tile idle, and with only a
// handful of outputs or of rank terms per row a row's largest output can be a small remainder of
// cancelling terms, where fp16 factors are too coarse; those run through the decode kernels.
constexpr int MDBF_GEMM_LMAX = 32;
constexpr int MDBF_GEMM_MIN = 64;
inline bool mdbf_use_gemm(int n, int m, int r, int l, int B, int vlim) {
  return l * B > vlim && l <= MDBF_GEMM_LMAX && n >= MDBF_GEMM_MIN && m >= MDBF_GEMM_MIN && r >= MDBF_GEMM_MIN;
}
size_t mdbf_gemm_workspace_size(int P, int n, int m, int r, int l, int B);
ql_status mdbf_gemm_launch(const mdbf_path *paths, int P, int n, int m, int r, int l, const uint16_t *x,
                           void *y, ql_out_dtype ydt, int B, void *ws, cudaStream_t s);
ql_status mdbf_gemm_read_timeout(int *flag);
size_t mdbf_noalloc_scratch_limit();
ql_status mdbf_noalloc_scratch(void **ptr);
ql_status mdbf_dequant_launch(const mdbf_path *paths, int P, int n, int m, int r, int l, float *W,
                              float *F, float *G, cudaStream_t s);

}  // namespace ql

#include "ql_device.cuh"
