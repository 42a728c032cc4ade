// libqlinear C ABI: argument validation, dispatch, status reporting and host-only accounting.
// The kernels live in benq_gemv.cu, benq_gemm_sm100.cu and mdbf.cu.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "ql_internal.cuh"

namespace {
thread_local char g_msg[512] = "";

int pdl_default() {
  const char *e = std::getenv("QL_PDL");
  return (e && std::strcmp(e, "0") == 0) ? 0 : 1;
}
std::atomic<int> g_pdl{pdl_default()};
}  // namespace

namespace ql {

ql_status fail(ql_status s, const char *fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_msg, sizeof(g_msg), fmt, ap);
  va_end(ap);
  return s;
}

ql_status launch_status(const char *what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(QL_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  return QL_OK;
}

bool pdl_enabled() { return g_pdl.load(std::memory_order_relaxed) != 0; }

// Per-launch host work that depends only on the device, the kernel and its launch shape is done
// once: each of these runtime calls costs about a microsecond of host time per launch otherwise.
// (A cudaDeviceReset() on a device clears the function attributes but not these caches.)
cudaError_t set_max_smem(const void *k, int bytes) {
  static std::mutex mu;
  static std::map<std::pair<const void *, int>, int> done;   // (kernel, device) -> bytes already allowed
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  const auto key = std::make_pair(k, dev);
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto it = done.find(key);
    if (it != done.end() && it->second >= bytes) return cudaSuccess;
  }
  const cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) {
    std::lock_guard<std::mutex> lock(mu);
    int &v = done[key];
    v = std::max(v, bytes);
  }
  return e;
}

int blocks_per_sm(const void *k, int threads, size_t smem) {
  static std::mutex mu;
  static std::map<std::tuple<const void *, int, int, size_t>, int> cache;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const auto key = std::make_tuple(k, dev, threads, smem);
  {
    std::lock_guard<std::mutex> lock(mu);
    const auto it = cache.find(key);
    if (it != cache.end()) return it->second;
  }
  int n = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, threads, smem) != cudaSuccess || n < 0) return 0;
  std::lock_guard<std::mutex> lock(mu);
  cache[key] = n;
  return n;
}

int sm_count() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
    cache[dev] = v;
  }
  return cache[dev];
}

}  // namespace ql

using ql::aligned;
using ql::fail;

extern "C" {

const char *ql_last_error(void) { return g_msg; }

int ql_set_pdl(int enable) { return g_pdl.exchange(enable ? 1 : 0); }

size_t benq_linear_workspace_bytes(int B, int N, int K) {
  if (B <= 16) return 0;
  return ql::benq_gemm_workspace_size(B, N, K);
}

ql_status benq_linear(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y, ql_out_dtype y_dtype,
                      int B, int N, int K, ql_stream_t stream) {
  return benq_linear_ws(codes, lut, x, y, y_dtype, B, N, K, nullptr, 0, stream);
}

size_t benq_mlp_workspace_bytes(int B, int N, int K) { return ql::benq_mlp_workspace_size(B, N, K); }

ql_status benq_encode(const uint16_t *W, uint8_t *codes, uint16_t *lut, int N, int K, int lloyd_iters,
                      ql_stream_t stream) {
  g_msg[0] = 0;
  if (!W || !codes || !lut) return fail(QL_ERR_INVALID_ARG, "benq_encode: null pointer");
  if (N <= 0 || K <= 0 || K % 4) return fail(QL_ERR_INVALID_ARG, "benq_encode: N, K must be positive and K %% 4 == 0");
  if (lloyd_iters < 0 || lloyd_iters > 1000) return fail(QL_ERR_INVALID_ARG, "benq_encode: lloyd_iters must be in [0, 1000]");
  if (!aligned(W, 2) || !aligned(lut, 2)) return fail(QL_ERR_ALIGNMENT, "benq_encode: W and lut must be 2-byte aligned");
  return ql::benq_encode_launch(W, codes, lut, N, K, lloyd_iters, reinterpret_cast<cudaStream_t>(stream));
}

ql_status benq_mlp_gate_up(const uint8_t *codes_g, const uint16_t *lut_g, const uint8_t *codes_u, const uint16_t *lut_u,
                           const uint16_t *x, void *h, ql_out_dtype h_dtype, int B, int N, int K, void *workspace,
                           size_t ws_bytes, ql_stream_t stream) {
  g_msg[0] = 0;
  if (!codes_g || !lut_g || !codes_u || !lut_u || !x || !h) return fail(QL_ERR_INVALID_ARG, "benq_mlp_gate_up: null pointer");
  if ((workspace == nullptr) != (ws_bytes == 0))
    return fail(QL_ERR_INVALID_ARG, "benq_mlp_gate_up: workspace and ws_bytes must both be set or both be empty");
  if (workspace && !aligned(workspace, 256)) return fail(QL_ERR_ALIGNMENT, "benq_mlp_gate_up: workspace must be 256-byte aligned");
  if (B <= 0 || N <= 0 || K <= 0) return fail(QL_ERR_INVALID_ARG, "benq_mlp_gate_up: B, N, K must be positive");
  if (K % 4) return fail(QL_ERR_INVALID_ARG, "benq_mlp_gate_up: K = %d is not a multiple of 4", K);
  if (h_dtype != QL_OUT_F32 && h_dtype != QL_OUT_BF16) return fail(QL_ERR_INVALID_ARG, "benq_mlp_gate_up: bad h_dtype");
  if (!aligned(codes_g, 16) || !aligned(lut_g, 16) || !aligned(codes_u, 16) || !aligned(lut_u, 16) || !aligned(x, 16) ||
      !aligned(h, 16))
    return fail(QL_ERR_ALIGNMENT, "benq_mlp_gate_up: codes, tables, x and h must be 16-byte aligned");
  if (B > 16 && (K % 64 || N % 256))
    return fail(QL_ERR_UNSUPPORTED, "benq_mlp_gate_up: batch %d > 16 needs K %% 64 == 0 and N %% 256 == 0", B);
  const size_t need = ql::benq_mlp_workspace_size(B, N, K);
  if (ws_bytes < need) return fail(QL_ERR_INVALID_ARG, "benq_mlp_gate_up: workspace %zu < %zu bytes", ws_bytes, need);
  return ql::benq_mlp_launch(codes_g, lut_g, codes_u, lut_u, x, h, h_dtype, B, N, K, workspace, ws_bytes,
                             reinterpret_cast<cudaStream_t>(stream));
}

ql_status benq_linear_ws(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y, ql_out_dtype y_dtype,
                         int B, int N, int K, void *workspace, size_t ws_bytes, ql_stream_t stream) {
  g_msg[0] = 0;
  if (!codes || !lut || !x || !y) return fail(QL_ERR_INVALID_ARG, "benq_linear: null pointer");
  if ((workspace == nullptr) != (ws_bytes == 0))
    return fail(QL_ERR_INVALID_ARG, "benq_linear_ws: workspace and ws_bytes must both be set or both be empty");
  if (workspace && !aligned(workspace, 256)) return fail(QL_ERR_ALIGNMENT, "benq_linear_ws: workspace must be 256-byte aligned");
  if (B <= 0 || N <= 0 || K <= 0) return fail(QL_ERR_INVALID_ARG, "benq_linear: B, N, K must be positive");
  if (K % 4) return fail(QL_ERR_INVALID_ARG, "benq_linear: K = %d is not a multiple of 4", K);
  if (y_dtype != QL_OUT_F32 && y_dtype != QL_OUT_BF16) return fail(QL_ERR_INVALID_ARG, "benq_linear: bad y_dtype");
  if (!aligned(codes, 16) || !aligned(lut, 16) || !aligned(x, 16) || !aligned(y, 16))
    return fail(QL_ERR_ALIGNMENT, "benq_linear: codes, lut, x and y must be 16-byte aligned");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (B <= 16) return ql::benq_gemv_launch(codes, lut, x, y, y_dtype, B, N, K, s);
  if (K % 64 || N % 256)
    return fail(QL_ERR_UNSUPPORTED, "benq_linear: batch %d > 16 needs K %% 64 == 0 and N %% 256 == 0", B);
  return ql::benq_gemm_launch(codes, lut, x, y, y_dtype, B, N, K, workspace, ws_bytes, s);
}

ql_status benq_linear_multi(const benq_layer *layers, int S, const uint16_t *x, ql_out_dtype y_dtype, int B, int K,
                            ql_stream_t stream) {
  g_msg[0] = 0;
  if (!layers || !x) return fail(QL_ERR_INVALID_ARG, "benq_linear_multi: null pointer");
  if (S < 1 || S > 4) return fail(QL_ERR_INVALID_ARG, "benq_linear_multi: S = %d must be in [1, 4]", S);
  if (B <= 0 || K <= 0) return fail(QL_ERR_INVALID_ARG, "benq_linear_multi: B, K must be positive");
  if (K % 4) return fail(QL_ERR_INVALID_ARG, "benq_linear_multi: K = %d is not a multiple of 4", K);
  if (y_dtype != QL_OUT_F32 && y_dtype != QL_OUT_BF16) return fail(QL_ERR_INVALID_ARG, "benq_linear_multi: bad y_dtype");
  if (!aligned(x, 16)) return fail(QL_ERR_ALIGNMENT, "benq_linear_multi: x must be 16-byte aligned");
  for (int i = 0; i < S; ++i) {
    const benq_layer &L = layers[i];
    if (!L.codes || !L.lut || !L.y) return fail(QL_ERR_INVALID_ARG, "benq_linear_multi: null pointer in layer %d", i);
    if (L.N <= 0) return fail(QL_ERR_INVALID_ARG, "benq_linear_multi: layer %d has N = %d", i, L.N);
    if (!aligned(L.codes, 16) || !aligned(L.lut, 16) || !aligned(L.y, 16))
      return fail(QL_ERR_ALIGNMENT, "benq_linear_multi: codes, lut and y of layer %d must be 16-byte aligned", i);
    if (B > 16 && (K % 64 || L.N % 256))
      return fail(QL_ERR_UNSUPPORTED, "benq_linear_multi: batch %d > 16 needs K %% 64 == 0 and N %% 256 == 0", B);
  }
  return ql::benq_gemv_multi_launch(layers, S, x, y_dtype, B, K, reinterpret_cast<cudaStream_t>(stream));
}

ql_status benq_dequant_debug(const uint8_t *codes, const uint16_t *lut, uint16_t *W, int N, int K,
                             ql_stream_t stream) {
  g_msg[0] = 0;
  if (!codes || !lut || !W) return fail(QL_ERR_INVALID_ARG, "benq_dequant_debug: null pointer");
  if (N <= 0 || K <= 0) return fail(QL_ERR_INVALID_ARG, "benq_dequant_debug: N, K must be positive");
  if (K % 4) return fail(QL_ERR_INVALID_ARG, "benq_dequant_debug: K = %d is not a multiple of 4", K);
  if (!aligned(lut, 2) || !aligned(W, 2)) return fail(QL_ERR_ALIGNMENT, "benq_dequant_debug: lut and W must be 2-byte aligned");
  return ql::benq_dequant_launch(codes, lut, W, N, K, reinterpret_cast<cudaStream_t>(stream));
}

double benq_bits_per_weight(int K) { return K > 0 ? 6.0 + 64.0 * 16.0 / K : 0.0; }

static ql_status check_paths(const char *who, const mdbf_path *paths, int P, int n, int m, int r, int l) {
  if (!paths) return fail(QL_ERR_INVALID_ARG, "%s: null paths", who);
  if (P <= 0 || n <= 0 || m <= 0 || r <= 0 || l <= 0)
    return fail(QL_ERR_INVALID_ARG, "%s: P, n, m, r, l must be positive", who);
  if (r > (n < m ? n : m)) return fail(QL_ERR_INVALID_ARG, "%s: rank %d exceeds min(n, m)", who, r);
  for (int p = 0; p < P; ++p) {
    const mdbf_path &q = paths[p];
    if (!q.S_A || !q.S_B || !q.A_amp || !q.B_amp || !q.Q_U || !q.Q_V)
      return fail(QL_ERR_INVALID_ARG, "%s: path %d has a null pointer", who, p);
    if (q.ldSA < (size_t)(r + 7) / 8 || q.ldSB < (size_t)(m + 7) / 8)
      return fail(QL_ERR_INVALID_ARG, "%s: path %d row stride too small", who, p);
    if (q.ldSA % 4 || q.ldSB % 4 || !aligned(q.S_A, 4) || !aligned(q.S_B, 4))
      return fail(QL_ERR_ALIGNMENT, "%s: path %d sign rows must be 4-byte aligned (stride %% 4 == 0)", who, p);
    if (!aligned(q.A_amp, 2) || !aligned(q.B_amp, 2) || !aligned(q.Q_U, 2) || !aligned(q.Q_V, 2))
      return fail(QL_ERR_ALIGNMENT, "%s: path %d envelopes must be 2-byte aligned", who, p);
  }
  return QL_OK;
}

size_t mdbf_workspace_bytes(int P, int n, int m, int r, int l, int B) {
  if (P <= 0 || n <= 0 || m <= 0 || r <= 0 || l <= 0 || B <= 0) return 0;
  return ql::mdbf_workspace_size(P, n, m, r, l, B);
}

ql_status mdbf_linear(const mdbf_path *paths, int P, int n, int m, int r, int l, const uint16_t *x, void *y,
                      ql_out_dtype y_dtype, int B, void *workspace, size_t ws_bytes, ql_stream_t stream) {
  g_msg[0] = 0;
  ql_status st = check_paths("mdbf_linear", paths, P, n, m, r, l);
  if (st != QL_OK) return st;
  if (!x || !y || !workspace) return fail(QL_ERR_INVALID_ARG, "mdbf_linear: null x, y or workspace");
  if (B <= 0) return fail(QL_ERR_INVALID_ARG, "mdbf_linear: B must be positive");
  if (y_dtype != QL_OUT_F32 && y_dtype != QL_OUT_BF16) return fail(QL_ERR_INVALID_ARG, "mdbf_linear: bad y_dtype");
  if (!aligned(x, 2) || !aligned(y, 4) || !aligned(workspace, 256))
    return fail(QL_ERR_ALIGNMENT, "mdbf_linear: x 2-, y 4- and workspace 256-byte alignment required");
  const size_t need = ql::mdbf_workspace_size(P, n, m, r, l, B);
  if (ws_bytes < need) return fail(QL_ERR_INVALID_ARG, "mdbf_linear: workspace %zu < %zu bytes", ws_bytes, need);
  return ql::mdbf_linear_launch(paths, P, n, m, r, l, x, y, y_dtype, B, workspace,
                                reinterpret_cast<cudaStream_t>(stream));
}

ql_status mdbf_linear_multi(const mdbf_path *paths, int S, int P, int n, int m, int r, int l, const uint16_t *x,
                            void *const *ys, ql_out_dtype y_dtype, int B, void *workspace, size_t ws_bytes,
                            ql_stream_t stream) {
  g_msg[0] = 0;
  if (S < 1 || S > 4) return fail(QL_ERR_INVALID_ARG, "mdbf_linear_multi: S = %d must be in [1, 4]", S);
  if (P < 1 || S * P > 8) return fail(QL_ERR_INVALID_ARG, "mdbf_linear_multi: S * P = %d must be in [1, 8]", S * P);
  ql_status st = check_paths("mdbf_linear_multi", paths, S * P, n, m, r, l);
  if (st != QL_OK) return st;
  if (!x || !ys || !workspace) return fail(QL_ERR_INVALID_ARG, "mdbf_linear_multi: null x, ys or workspace");
  if (B <= 0) return fail(QL_ERR_INVALID_ARG, "mdbf_linear_multi: B must be positive");
  if (y_dtype != QL_OUT_F32 && y_dtype != QL_OUT_BF16)
    return fail(QL_ERR_INVALID_ARG, "mdbf_linear_multi: bad y_dtype");
  if (!aligned(x, 2) || !aligned(workspace, 256))
    return fail(QL_ERR_ALIGNMENT, "mdbf_linear_multi: x 2- and workspace 256-byte alignment required");
  for (int s = 0; s < S; ++s) {
    if (!ys[s]) return fail(QL_ERR_INVALID_ARG, "mdbf_linear_multi: null output %d", s);
    if (!aligned(ys[s], 4)) return fail(QL_ERR_ALIGNMENT, "mdbf_linear_multi: output %d must be 4-byte aligned", s);
  }
  const size_t need = ql::mdbf_workspace_size(S * P, n, m, r, l, B);
  if (ws_bytes < need)
    return fail(QL_ERR_INVALID_ARG, "mdbf_linear_multi: workspace %zu < %zu bytes", ws_bytes, need);
  return ql::mdbf_linear_multi_launch(paths, S, P, n, m, r, l, x, ys, y_dtype, B, workspace,
                                      reinterpret_cast<cudaStream_t>(stream));
}

ql_status mdbf_linear_noalloc(const mdbf_path *paths, int P, int n, int m, int r, int l, const uint16_t *x, void *y,
                              ql_out_dtype y_dtype, int B, ql_stream_t stream) {
  g_msg[0] = 0;
  ql_status st = check_paths("mdbf_linear_noalloc", paths, P, n, m, r, l);
  if (st != QL_OK) return st;
  if (!x || !y) return fail(QL_ERR_INVALID_ARG, "mdbf_linear_noalloc: null x or y");
  if (B <= 0) return fail(QL_ERR_INVALID_ARG, "mdbf_linear_noalloc: B must be positive");
  if (y_dtype != QL_OUT_F32 && y_dtype != QL_OUT_BF16)
    return fail(QL_ERR_INVALID_ARG, "mdbf_linear_noalloc: bad y_dtype");
  if (!aligned(x, 2) || !aligned(y, 4)) return fail(QL_ERR_ALIGNMENT, "mdbf_linear_noalloc: x 2- and y 4-byte alignment required");
  const size_t need = ql::mdbf_workspace_size(P, n, m, r, l, B);
  const size_t limit = ql::mdbf_noalloc_scratch_limit();
  if (need > limit)
    return fail(QL_ERR_UNSUPPORTED,
                "mdbf_linear_noalloc: these sizes need %zu bytes of scratch, more than the %zu-byte static array; "
                "use mdbf_linear with a caller workspace",
                need, limit);
  void *scratch = nullptr;
  st = ql::mdbf_noalloc_scratch(&scratch);
  if (st != QL_OK) return st;
  return ql::mdbf_linear_launch(paths, P, n, m, r, l, x, y, y_dtype, B, scratch,
                                reinterpret_cast<cudaStream_t>(stream));
}

size_t mdbf_noalloc_scratch_bytes(void) { return ql::mdbf_noalloc_scratch_limit(); }

ql_status mdbf_dequant_debug(const mdbf_path *paths, int P, int n, int m, int r, int l, float *W, float *F, float *G,
                             ql_stream_t stream) {
  g_msg[0] = 0;
  ql_status st = check_paths("mdbf_dequant_debug", paths, P, n, m, r, l);
  if (st != QL_OK) return st;
  if (!W) return fail(QL_ERR_INVALID_ARG, "mdbf_dequant_debug: null W");
  return ql::mdbf_dequant_launch(paths, P, n, m, r, l, W, F, G, reinterpret_cast<cudaStream_t>(stream));
}

double mdbf_effective_bits(int n, int m, int r, int P, int l, int scale_bits) {
  if (n <= 0 || m <= 0 || r <= 0 || P <= 0 || l <= 0 || scale_bits < 0) return 0.0;
  const double num = (double)P * ((double)r * (n + m) + (double)scale_bits * l * ((double)n + m + 2.0 * r));
  return num / ((double)n * m);
}

ql_status mdbf_select_rank(int n, int m, int P, int l, int scale_bits, double target_bits, int *r_out, int *clamped) {
  g_msg[0] = 0;
  if (!r_out || !clamped) return fail(QL_ERR_INVALID_ARG, "mdbf_select_rank: null output");
  if (n <= 0 || m <= 0 || P <= 0 || l <= 0 || scale_bits < 0 || !(target_bits > 0.0))
    return fail(QL_ERR_INVALID_ARG, "mdbf_select_rank: bad arguments");
  const int s = n < m ? n : m;
  // r = (b n m / P - sb l (n+m)) / ((n+m) + 2 sb l), exactly as a quotient of two products
  const long double num = (long double)target_bits * n * m / P - (long double)scale_bits * l * ((long double)n + m);
  const long double den = (long double)n + m + 2.0L * scale_bits * l;
  const long double rr = num / den;
  *clamped = 0;
  if (rr > (long double)s) {
    *r_out = s;
    *clamped = 1;
    return QL_OK;
  }
  const long double f = floorl(rr);
  if (f < 1.0L) return fail(QL_ERR_INVALID_ARG, "mdbf_select_rank: target %.6f bpw is below rank 1", target_bits);
  *r_out = (int)f;
  return QL_OK;
}

ql_status ql_selftest_timeout(ql_stream_t stream) {
  g_msg[0] = 0;
  return ql::selftest_timeout_launch(reinterpret_cast<cudaStream_t>(stream));
}

ql_status ql_check(ql_stream_t stream) {
  g_msg[0] = 0;
  cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(QL_ERR_CUDA, "ql_check: %s", cudaGetErrorString(e));
  int flag = 0, flag2 = 0, flag3 = 0;
  ql_status st = ql::benq_gemm_read_timeout(&flag);
  if (st != QL_OK) return st;
  st = ql::mdbf_read_timeout(&flag2);
  if (st != QL_OK) return st;
  st = ql::mdbf_gemm_read_timeout(&flag3);
  if (st != QL_OK) return st;
  if (flag) return fail(QL_ERR_TIMEOUT, "a bounded device-side wait of the GEMM ran out (code %d)", flag);
  if (flag2) return fail(QL_ERR_TIMEOUT, "a bounded device-side wait of the MDBF F stage ran out (code %d)", flag2);
  if (flag3) return fail(QL_ERR_TIMEOUT, "a bounded device-side wait of the MDBF GEMM ran out (code %d)", flag3);
  return QL_OK;
}

}  // extern "C"
