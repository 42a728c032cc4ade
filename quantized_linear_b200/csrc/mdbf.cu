// MDBF (multi-envelope double binary factorization) layer: forward pass and debug dequantizer.
//
// "MDBF (Multi-Envelope Double Binary Factorization)", section "Algorithm":
//   W ~= sum_p F_p G_p,  F = S_A (.) (A_amp Q_U^T),  G = S_B (.) (Q_V B_amp^T).
// The forward pass never forms W.  Writing the Hadamard products out,
//   (G x)_k = sum_i Q_V[k,i] * sum_j S_B[k,j] * (B_amp[j,i] x_j)
//   (F t)_a = sum_i A_amp[a,i] * sum_k S_A[a,k] * (Q_U[k,i] t_k)
// so each path is two products of a packed +-1 matrix with l*B dense vectors:
//   prologue  z[p][j][b*l+i] = B_amp[j,i] * x[b,j]                (exact in fp32)
//   G stage   u = S_B z;   t[k][b] = sum_i Q_V[k,i] u[k][b*l+i];
//             w[p][k][b*l+i] = Q_U[k,i] * t[k][b]                  (epilogue, fused)
//   F stage   v = S_A w;   y[b][a] = sum_p sum_i A_amp[a,i] v[a][b*l+i]   (epilogue, fused;
//             the path sum is taken inside one launch, in p order)
// Sign products: lane = matrix row, warps split the columns; each sign bit
// becomes +-1.0f (two integer ops) and multiplies the l*B vector values with
// FMAs; the vectors are read as warp-wide broadcasts.  Column-split partials
// are summed through shared memory in a fixed order.
#include <algorithm>
#include <mutex>

#include "ql_internal.cuh"

namespace {

constexpr int PMAX = 8;
constexpr int VLIM = 64;  // l * B limit

struct Paths {
  const uint8_t *SA[PMAX];
  const uint8_t *SB[PMAX];
  size_t ldSA[PMAX], ldSB[PMAX];
  const uint16_t *A[PMAX], *Bm[PMAX], *QU[PMAX], *QV[PMAX];
};

__host__ __device__ inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
__host__ __device__ inline int vpad(int vb) { return (vb + 3) & ~3; }

__device__ __forceinline__ uint32_t ldg_u32(const uint8_t *p) {
  uint32_t v;
  asm volatile("ld.global.nc.u32 %0, [%1];" : "=r"(v) : "l"(p));
  return v;
}
__device__ __forceinline__ float4 ldg_f4(const float *p) {
  float4 v;
  asm volatile("ld.global.nc.v4.f32 {%0, %1, %2, %3}, [%4];" : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w) : "l"(p));
  return v;
}

// z[p][j][v] = B_amp[j][i] * x[b][j] for v = b*l + i (zero padding up to a multiple of 4).
__global__ void mdbf_prologue_kernel(Paths ps, const uint16_t *__restrict__ x, float *__restrict__ Z, int m, int l,
                                     int B) {
  const int p = blockIdx.y;
  const int vb = l * B, vp = vpad(vb);
  const int64_t total = (int64_t)m * vp;
  float *zp = Z + (int64_t)p * total;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t j = e / vp;
    const int v = int(e - j * vp);
    float z = 0.f;
    if (v < vb) {
      const int b = v / l, i = v - b * l;
      z = qld::f16_to_f32(ps.Bm[p][j * l + i]) * qld::bf16_to_f32(x[(int64_t)b * m + j]);
    }
    zp[e] = z;
  }
}

// acc[v] += sum over this warp's columns of s[row][col] * vec[col][v]
template <int VMAX>
__device__ __forceinline__ void sign_dot(const uint8_t *row_bits, bool row_ok, const float *__restrict__ vec,
                                         int vp, int cols, int q0, int q1, float (&acc)[VMAX]) {
  for (int q = q0; q < q1; ++q) {
    const uint32_t bits = row_ok ? ldg_u32(row_bits + 4 * q) : 0u;
    const int jmax = min(32, cols - 32 * q);
    const float *vq = vec + (int64_t)32 * q * vp;
#pragma unroll 4
    for (int jj = 0; jj < 32; ++jj) {
      if (jj >= jmax) break;
      const float s = __uint_as_float(0xBF800000u ^ ((bits << (31 - jj)) & 0x80000000u));
      const float *vj = vq + (int64_t)jj * vp;
#pragma unroll
      for (int v4 = 0; v4 < VMAX / 4; ++v4) {
        if (4 * v4 < vp) {
          const float4 z = ldg_f4(vj + 4 * v4);
          acc[4 * v4 + 0] = fmaf(s, z.x, acc[4 * v4 + 0]);
          acc[4 * v4 + 1] = fmaf(s, z.y, acc[4 * v4 + 1]);
          acc[4 * v4 + 2] = fmaf(s, z.z, acc[4 * v4 + 2]);
          acc[4 * v4 + 3] = fmaf(s, z.w, acc[4 * v4 + 3]);
        }
      }
    }
  }
}

// Sums the per-warp partials (part[KS][VMAX][32]) into warp 0's acc, fixed order.
template <int VMAX>
__device__ __forceinline__ void reduce_warps(float *part, int vp, float (&acc)[VMAX]) {
  const int warp = threadIdx.y, lane = threadIdx.x, KS = blockDim.y;
#pragma unroll
  for (int v = 0; v < VMAX; ++v)
    if (v < vp) part[(warp * VMAX + v) * 32 + lane] = acc[v];
  __syncthreads();
  if (warp == 0) {
#pragma unroll
    for (int v = 0; v < VMAX; ++v) {
      if (v < vp) {
        float s = part[v * 32 + lane];
        for (int w = 1; w < KS; ++w) s += part[(w * VMAX + v) * 32 + lane];
        acc[v] = s;
      }
    }
  }
}

template <int VMAX>
__global__ void mdbf_g_stage_kernel(Paths ps, const float *__restrict__ Z, float *__restrict__ Wv, int m, int r,
                                    int l, int B) {
  extern __shared__ float part[];  // [KS][VMAX][32]
  const int p = blockIdx.y;
  const int lane = threadIdx.x, warp = threadIdx.y, KS = blockDim.y;
  const int k = blockIdx.x * 32 + lane;
  const bool ok = k < r;
  const int vb = l * B, vp = vpad(vb);
  const int nq = (m + 31) / 32;
  const int q0 = (int)((int64_t)nq * warp / KS), q1 = (int)((int64_t)nq * (warp + 1) / KS);
  float acc[VMAX];
#pragma unroll
  for (int v = 0; v < VMAX; ++v) acc[v] = 0.f;
  sign_dot<VMAX>(ps.SB[p] + (int64_t)(ok ? k : 0) * ps.ldSB[p], ok, Z + (int64_t)p * m * vp, vp, m, q0, q1, acc);
  reduce_warps<VMAX>(part, vp, acc);
  if (warp == 0 && ok) {
    float *out = Wv + ((int64_t)p * r + k) * vp;
    const uint16_t *qv = ps.QV[p] + (int64_t)k * l;
    const uint16_t *qu = ps.QU[p] + (int64_t)k * l;
#pragma unroll
    for (int v = 0; v < VMAX; ++v)
      if (v >= vb && v < vp) out[v] = 0.f;
    for (int b = 0; b < B; ++b) {
      float t = 0.f;
#pragma unroll
      for (int v = 0; v < VMAX; ++v)
        if (v >= b * l && v < (b + 1) * l) t = fmaf(qld::f16_to_f32(qv[v - b * l]), acc[v], t);
#pragma unroll
      for (int v = 0; v < VMAX; ++v)
        if (v >= b * l && v < (b + 1) * l) out[v] = qld::f16_to_f32(qu[v - b * l]) * t;
    }
  }
}

template <int VMAX>
__global__ void mdbf_f_stage_kernel(Paths ps, int P, const float *__restrict__ Wv, void *__restrict__ y, int ydt,
                                    int n, int r, int l, int B) {
  extern __shared__ float part[];  // [KS][VMAX][32]
  const int lane = threadIdx.x, warp = threadIdx.y, KS = blockDim.y;
  const int a = blockIdx.x * 32 + lane;
  const bool ok = a < n;
  const int vb = l * B, vp = vpad(vb);
  const int nq = (r + 31) / 32;
  const int q0 = (int)((int64_t)nq * warp / KS), q1 = (int)((int64_t)nq * (warp + 1) / KS);
  float yacc[VMAX];
#pragma unroll
  for (int v = 0; v < VMAX; ++v) yacc[v] = 0.f;
  for (int p = 0; p < P; ++p) {
    float acc[VMAX];
#pragma unroll
    for (int v = 0; v < VMAX; ++v) acc[v] = 0.f;
    sign_dot<VMAX>(ps.SA[p] + (int64_t)(ok ? a : 0) * ps.ldSA[p], ok, Wv + (int64_t)p * r * vp, vp, r, q0, q1, acc);
    if (p > 0) __syncthreads();  // previous path's reduction has finished reading `part`
    reduce_warps<VMAX>(part, vp, acc);
    if (warp == 0 && ok) {
      const uint16_t *am = ps.A[p] + (int64_t)a * l;
#pragma unroll
      for (int v = 0; v < VMAX; ++v) {
        if (v < vb) {
          const int b = v / l;
          const float av = qld::f16_to_f32(am[v - b * l]);
          // yacc[b] += A[a][i] * v[b*l+i], i ascending within each path
#pragma unroll
          for (int bb = 0; bb < VMAX; ++bb)
            if (bb == b) yacc[bb] = fmaf(av, acc[v], yacc[bb]);
        }
      }
    }
  }
  if (warp == 0 && ok) {
#pragma unroll
    for (int b = 0; b < VMAX; ++b) {
      if (b < B) {
        if (ydt == QL_OUT_F32)
          static_cast<float *>(y)[(int64_t)b * n + a] = yacc[b];
        else
          static_cast<uint16_t *>(y)[(int64_t)b * n + a] = qld::f32_to_bf16_rn(yacc[b]);
      }
    }
  }
}

// ---------------------------------------------------------------- debug dequantizer ----------
__device__ __forceinline__ float envelope(const uint16_t *L, const uint16_t *R, int l) {
  float e = qld::f16_to_f32(L[0]) * qld::f16_to_f32(R[0]);
  for (int i = 1; i < l; ++i) e = fmaf(qld::f16_to_f32(L[i]), qld::f16_to_f32(R[i]), e);
  return e;
}
__device__ __forceinline__ float sign_of(const uint8_t *row, int c) {
  return ((row[c >> 3] >> (c & 7)) & 1) ? 1.f : -1.f;
}

__global__ void mdbf_factors_kernel(Paths ps, float *__restrict__ F, float *__restrict__ G, int n, int m, int r,
                                    int l) {
  const int p = blockIdx.y;
  const int64_t nF = (int64_t)n * r, nG = (int64_t)r * m;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < nF + nG; e += (int64_t)gridDim.x * blockDim.x) {
    if (e < nF) {
      if (!F) continue;
      const int64_t a = e / r;
      const int k = int(e - a * r);
      F[(int64_t)p * nF + e] = sign_of(ps.SA[p] + a * ps.ldSA[p], k) * envelope(ps.A[p] + a * l, ps.QU[p] + (int64_t)k * l, l);
    } else {
      if (!G) continue;
      const int64_t f = e - nF;
      const int64_t k = f / m;
      const int j = int(f - k * m);
      G[(int64_t)p * nG + f] = sign_of(ps.SB[p] + k * ps.ldSB[p], j) * envelope(ps.QV[p] + k * l, ps.Bm[p] + (int64_t)j * l, l);
    }
  }
}

__global__ void mdbf_w_kernel(Paths ps, int P, float *__restrict__ W, int n, int m, int r, int l) {
  const int64_t total = (int64_t)n * m;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t a = e / m;
    const int j = int(e - a * m);
    double acc = 0.0;
    for (int p = 0; p < P; ++p) {
      const uint8_t *sa = ps.SA[p] + a * ps.ldSA[p];
      const uint16_t *am = ps.A[p] + a * l;
      const uint16_t *bm = ps.Bm[p] + (int64_t)j * l;
      for (int k = 0; k < r; ++k) {
        const float f = sign_of(sa, k) * envelope(am, ps.QU[p] + (int64_t)k * l, l);
        const float g = sign_of(ps.SB[p] + (int64_t)k * ps.ldSB[p], j) * envelope(ps.QV[p] + (int64_t)k * l, bm, l);
        acc = fma((double)f, (double)g, acc);
      }
    }
    W[e] = (float)acc;
  }
}

Paths pack_paths(const mdbf_path *paths, int P) {
  Paths ps = {};
  for (int p = 0; p < P; ++p) {
    ps.SA[p] = paths[p].S_A;
    ps.SB[p] = paths[p].S_B;
    ps.ldSA[p] = paths[p].ldSA;
    ps.ldSB[p] = paths[p].ldSB;
    ps.A[p] = paths[p].A_amp;
    ps.Bm[p] = paths[p].B_amp;
    ps.QU[p] = paths[p].Q_U;
    ps.QV[p] = paths[p].Q_V;
  }
  return ps;
}

template <int VMAX>
ql_status run_stages(const Paths &ps, int P, int n, int m, int r, int l, int B, float *Z, float *Wv,
                     void *y, ql_out_dtype ydt, cudaStream_t s) {
  constexpr int KSG = 8, KSF = 4;
  const size_t smg = (size_t)KSG * VMAX * 32 * sizeof(float), smf = (size_t)KSF * VMAX * 32 * sizeof(float);
  if (smg > 48 * 1024 &&
      cudaFuncSetAttribute(mdbf_g_stage_kernel<VMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smg) != cudaSuccess)
    return ql::fail(QL_ERR_CUDA, "mdbf_linear: cannot reserve shared memory");
  if (smf > 48 * 1024 &&
      cudaFuncSetAttribute(mdbf_f_stage_kernel<VMAX>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smf) != cudaSuccess)
    return ql::fail(QL_ERR_CUDA, "mdbf_linear: cannot reserve shared memory");
  {
    const dim3 block(32, KSG), grid((r + 31) / 32, P);
    mdbf_g_stage_kernel<VMAX><<<grid, block, smg, s>>>(ps, Z, Wv, m, r, l, B);
    ql_status st = ql::launch_status("mdbf_linear (G stage)");
    if (st != QL_OK) return st;
  }
  {
    const dim3 block(32, KSF), grid((n + 31) / 32);
    mdbf_f_stage_kernel<VMAX><<<grid, block, smf, s>>>(ps, P, Wv, y, (int)ydt, n, r, l, B);
    return ql::launch_status("mdbf_linear (F stage)");
  }
}

}  // namespace

namespace ql {

size_t mdbf_workspace_size(int P, int n, int m, int r, int l, int B) {
  (void)n;
  const size_t vp = (size_t)vpad(l * B);
  return align256((size_t)P * m * vp * sizeof(float)) + align256((size_t)P * r * vp * sizeof(float));
}

ql_status mdbf_linear_launch(const mdbf_path *paths, int P, int n, int m, int r, int l, const uint16_t *x,
                             void *y, ql_out_dtype ydt, int B, void *ws, cudaStream_t s) {
  if (P > PMAX) return fail(QL_ERR_UNSUPPORTED, "mdbf_linear: P = %d exceeds %d paths", P, PMAX);
  if (l * B > VLIM) return fail(QL_ERR_UNSUPPORTED, "mdbf_linear: l*B = %d exceeds %d", l * B, VLIM);
  const Paths ps = pack_paths(paths, P);
  const int vp = vpad(l * B);
  float *Z = static_cast<float *>(ws);
  float *Wv = reinterpret_cast<float *>(static_cast<char *>(ws) + align256((size_t)P * m * vp * sizeof(float)));
  {
    const int64_t total = (int64_t)m * vp;
    const int threads = 256;
    const int grid = (int)std::min<int64_t>((total + threads - 1) / threads, (int64_t)sm_count() * 4);
    mdbf_prologue_kernel<<<dim3(grid, P), threads, 0, s>>>(ps, x, Z, m, l, B);
    ql_status st = launch_status("mdbf_linear (prologue)");
    if (st != QL_OK) return st;
  }
  if (vp <= 4) return run_stages<4>(ps, P, n, m, r, l, B, Z, Wv, y, ydt, s);
  if (vp <= 8) return run_stages<8>(ps, P, n, m, r, l, B, Z, Wv, y, ydt, s);
  if (vp <= 16) return run_stages<16>(ps, P, n, m, r, l, B, Z, Wv, y, ydt, s);
  if (vp <= 32) return run_stages<32>(ps, P, n, m, r, l, B, Z, Wv, y, ydt, s);
  return run_stages<64>(ps, P, n, m, r, l, B, Z, Wv, y, ydt, s);
}

ql_status mdbf_dequant_launch(const mdbf_path *paths, int P, int n, int m, int r, int l, float *W, float *F,
                              float *G, cudaStream_t s) {
  if (P > PMAX) return fail(QL_ERR_UNSUPPORTED, "mdbf_dequant_debug: P = %d exceeds %d paths", P, PMAX);
  const Paths ps = pack_paths(paths, P);
  if (F || G) {
    const int64_t total = (int64_t)n * r + (int64_t)r * m;
    const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 8);
    mdbf_factors_kernel<<<dim3(grid, P), 256, 0, s>>>(ps, F, G, n, m, r, l);
    ql_status st = launch_status("mdbf_dequant_debug (factors)");
    if (st != QL_OK) return st;
  }
  const int64_t total = (int64_t)n * m;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 16);
  mdbf_w_kernel<<<grid, 256, 0, s>>>(ps, P, W, n, m, r, l);
  return launch_status("mdbf_dequant_debug (W)");
}

}  // namespace ql

// ------------------------------------------------------------------ no-allocation variant
// Some callers cannot call cudaMalloc at all: code running where the allocator is forbidden or
// unavailable (inside a custom allocator's own paths, in real-time threads that must never block
// in the driver, or in hosts whose memory budget is fixed before the first inference).  For them
// mdbf_linear_noalloc takes its scratch from this file-scope device array instead of a caller
// workspace.  Every GPU that loads the library holds it until the process exits.
constexpr size_t NOALLOC_SCRATCH_BYTES = size_t(4) << 20;   // 4 MiB
static __device__ __align__(256) unsigned char g_mdbf_scratch[NOALLOC_SCRATCH_BYTES];

namespace {
std::mutex g_scratch_mu;
void *g_scratch_ptr[64] = {nullptr};
}  // namespace

namespace ql {

size_t mdbf_noalloc_scratch_limit() { return NOALLOC_SCRATCH_BYTES; }

// Device address of the scratch array on the current device.  The host-side symbol is only a
// stand-in, so the address is looked up once per device (with that device current) and cached.
ql_status mdbf_noalloc_scratch(void **ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(QL_ERR_CUDA, "mdbf_linear_noalloc: no current CUDA device");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_ptr[dev]) {
    void *p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_mdbf_scratch);
    if (e != cudaSuccess || !p)
      return fail(QL_ERR_CUDA, "mdbf_linear_noalloc: cannot resolve the scratch array: %s", cudaGetErrorString(e));
    g_scratch_ptr[dev] = p;
  }
  *ptr = g_scratch_ptr[dev];
  return QL_OK;
}

}  // namespace ql
