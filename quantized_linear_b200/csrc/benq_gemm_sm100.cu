// BenQ prefill GEMM on sm_100a tensor cores: Y[M][N] = X[M][K] * W[N][K]^T, W decoded on the fly.
//
// W is never written to global memory ("Qwen3.8-27B -- BenQ 6-bit", "What BenQ stores": the
// gather lut[n][code] is fused into the GEMM).  One persistent CTA per SM walks 256 x 256 output
// tiles; per 64-wide K block:
//   * warp 0 loads the X tile (256 x 64 bf16, 128-byte swizzle) with tensor copies into a
//     3-stage ring released by the MMA; warp 2 loads the packed code tile (256 rows x 48 bytes)
//     into a 2-stage ring released as soon as the decoders have read it, plus the 256 row
//     tables of the tile (32 KB, once per tile) with a bulk copy;
//   * warps 3..18 (decoders) expand the code tile through the row tables into the bf16 W tile,
//     written directly in the K-major 128-byte-swizzled layout the tensor core reads, then fence
//     the writes for the async proxy;
//   * warp 1, one thread, issues tcgen05.mma (M=128, N=256, K=16, bf16 in, fp32 accumulate in
//     tensor memory): two M halves share each decoded W tile, so each decoded weight feeds 256
//     rows of X;
//   * after the last K block the decoder warps drain the 2 x 128 x 256 fp32 accumulators from
//     tensor memory (tcgen05.ld), round to bf16 (or keep fp32) and store Y.
// Stages are handed over with mbarriers; every wait gives up after a fixed clock budget, sets a
// device flag read by ql_check(), and the CTA winds down (tensor memory is freed on every path).
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "ql_internal.cuh"
#include "sm100_ptx.cuh"

namespace {

constexpr int BM = 256, BN = 256, BK = 64;        // CTA tile; BK = one 128-byte swizzle row of bf16
constexpr int SA = 3, SB = 2, SC = 2;             // stages: activations, decoded W, codes
constexpr int A_BYTES = BM * BK * 2;              // 32 KB
constexpr int B_BYTES = BN * BK * 2;              // 32 KB
constexpr int C_ROW = BK * 6 / 8;                 // 48 code bytes per row per K block
constexpr int C_BYTES = BN * C_ROW;               // 12 KB
constexpr int LUT_BYTES = BN * 128;               // 32 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + SA * A_BYTES;
constexpr int OFF_C = OFF_B + SB * B_BYTES;
constexpr int OFF_LUT = OFF_C + SC * C_BYTES + 128;   // 128 bytes of slack after the code tiles
constexpr int OFF_BAR = OFF_LUT + LUT_BYTES;
constexpr int NBAR = 2 * (SA + SB + SC) + 4;
constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;
constexpr int SMEM_BYTES = OFF_TMEM + 16 + 1024;          // + alignment slack
constexpr int NDEC = 16;                                 // decoder / epilogue warps (multiple of 8)
constexpr int THREADS = (3 + NDEC) * 32;   // A producer, MMA issuer, code producer, decoders
constexpr long long WAIT_BUDGET = 4000000000LL;           // clock cycles (~2 s)
constexpr uint32_t IDESC = sm100::idesc_bf16_f32(128, BN);

__device__ int g_gemm_timeout = 0;

struct Bars {
  uint32_t full_a, empty_a, full_b, empty_b, full_c, empty_c, lut_full, lut_empty, acc_full, acc_empty;
  __device__ Bars(uint32_t base)
      : full_a(base), empty_a(full_a + 8 * SA), full_b(empty_a + 8 * SA), empty_b(full_b + 8 * SB),
        full_c(empty_b + 8 * SB), empty_c(full_c + 8 * SC), lut_full(empty_c + 8 * SC), lut_empty(lut_full + 8),
        acc_full(lut_empty + 8), acc_empty(acc_full + 8) {}
};

__device__ __forceinline__ uint32_t lds32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds_u16(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts32(uint32_t a, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;" ::"r"(a), "r"(v) : "memory");
}

__global__ void __launch_bounds__(THREADS, 1)
    benq_gemm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_codes,
                     const uint16_t *__restrict__ lut, void *__restrict__ y, int ydt, int M, int N, int K) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const Bars bar(sbase + OFF_BAR);
  const uint32_t tmem_slot = sbase + OFF_TMEM;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int mt = (M + BM - 1) / BM, nt = N / BN, ntiles = mt * nt, nkb = K / BK;
  bool ok = true;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      sm100::mbar_init(bar.full_a + 8 * s, 1);
      sm100::mbar_init(bar.empty_a + 8 * s, 1);
    }
    for (int s = 0; s < SB; ++s) {
      sm100::mbar_init(bar.full_b + 8 * s, NDEC);
      sm100::mbar_init(bar.empty_b + 8 * s, 1);
    }
    for (int s = 0; s < SC; ++s) {
      sm100::mbar_init(bar.full_c + 8 * s, 1);
      sm100::mbar_init(bar.empty_c + 8 * s, NDEC);
    }
    sm100::mbar_init(bar.lut_full, 1);
    sm100::mbar_init(bar.lut_empty, NDEC);
    sm100::mbar_init(bar.acc_full, 1);
    sm100::mbar_init(bar.acc_empty, NDEC);
    sm100::fence_barrier_init();
    sm100::prefetch_tensormap(&map_x);
    sm100::prefetch_tensormap(&map_codes);
  }
  if (warp == 1) {
    sm100::tmem_alloc(tmem_slot, 512);
    sm100::tmem_relinquish();
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem_raw + (tmem_slot - raw));
  // codes and tables are weights: their producer starts at once; activations are read and y is
  // written only after the preceding kernel in the stream has completed
  qld::pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ activation producer (TMA)
    if (lane == 0) {
      qld::pdl_wait();
      int it = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
        const int m0 = (t % mt) * BM;
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % SA;
          if (it >= SA && !sm100::mbar_wait(bar.empty_a + 8 * s, ((it / SA) & 1) ^ 1, WAIT_BUDGET)) {
            ok = false;
            break;
          }
          sm100::mbar_arrive_expect_tx(bar.full_a + 8 * s, A_BYTES);
          sm100::tma_load_2d(sbase + OFF_A + s * A_BYTES, &map_x, kb * BK, m0, bar.full_a + 8 * s);
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ code and table producer (TMA)
    if (lane == 0) {
      int it = 0, tl = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tl) {
        const int n0 = (t / mt) * BN;
        if (tl > 0 && !sm100::mbar_wait(bar.lut_empty, (tl - 1) & 1, WAIT_BUDGET)) { ok = false; break; }
        sm100::mbar_arrive_expect_tx(bar.lut_full, LUT_BYTES);
        sm100::bulk_g2s(sbase + OFF_LUT, lut + (size_t)n0 * 64, LUT_BYTES, bar.lut_full);
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int s = it % SC;
          if (it >= SC && !sm100::mbar_wait(bar.empty_c + 8 * s, ((it / SC) & 1) ^ 1, WAIT_BUDGET)) {
            ok = false;
            break;
          }
          sm100::mbar_arrive_expect_tx(bar.full_c + 8 * s, C_BYTES);
          sm100::tma_load_2d(sbase + OFF_C + s * C_BYTES, &map_codes, kb * C_ROW, n0, bar.full_c + 8 * s);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int it = 0, tl = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tl) {
        if (tl > 0 && !sm100::mbar_wait(bar.acc_empty, (tl - 1) & 1, WAIT_BUDGET)) { ok = false; break; }
        sm100::tc_fence_after();
        for (int kb = 0; kb < nkb; ++kb, ++it) {
          const int sa = it % SA, sb = it % SB;
          if (!sm100::mbar_wait(bar.full_a + 8 * sa, (it / SA) & 1, WAIT_BUDGET) ||
              !sm100::mbar_wait(bar.full_b + 8 * sb, (it / SB) & 1, WAIT_BUDGET)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint32_t a = sbase + OFF_A + sa * A_BYTES, b = sbase + OFF_B + sb * B_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bdesc = sm100::sw128_kmajor_desc(b + kk * 32);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint64_t adesc = sm100::sw128_kmajor_desc(a + h * (A_BYTES / 2) + kk * 32);
              sm100::mma_bf16(tmem + h * BN, adesc, bdesc, IDESC, (kb | kk) ? 1u : 0u);
            }
          }
          sm100::mma_commit(bar.empty_a + 8 * sa);
          sm100::mma_commit(bar.empty_b + 8 * sb);
        }
        if (!ok) break;
        sm100::mma_commit(bar.acc_full);
      }
    }
  } else {
    // ------------------------------------------------------------ decoders, then epilogue
    const int dw = warp - 3;            // decoder index 0 .. NDEC-1
    const int q = warp & 3;             // tensor-memory lane quarter this warp may read
    const int ch = dw >> 2;             // which NDEC/4-th of the 256 accumulator columns it drains
    int it = 0, tl = 0;
    // lane l expands codes 2l, 2l+1 of a row's 64-code block: bits [12l, 12l+12) of its 48 bytes
    const int wq = (12 * lane) >> 5, wsh = (12 * lane) & 31;
    const int chunk = lane >> 2, inner = (lane & 3) * 4;
    // swizzled position of codes 2*lane, 2*lane+1 within row r = dw (mod 8) of a K block
    const uint32_t dst_lane = (dw >> 3) * 1024 + (dw & 7) * 128 + ((chunk ^ (dw & 7)) << 4) + inner;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++tl) {
      const int m0 = (t % mt) * BM, n0 = (t / mt) * BN;
      if (!sm100::mbar_wait(bar.lut_full, tl & 1, WAIT_BUDGET)) { ok = false; break; }
      for (int kb = 0; kb < nkb; ++kb, ++it) {
        const int sb = it % SB, sc = it % SC;
        if ((it >= SB && !sm100::mbar_wait(bar.empty_b + 8 * sb, ((it / SB) & 1) ^ 1, WAIT_BUDGET)) ||
            !sm100::mbar_wait(bar.full_c + 8 * sc, (it / SC) & 1, WAIT_BUDGET)) {
          ok = false;
          break;
        }
        // rows r = dw + NDEC*i: r & 7 == dw & 7 is fixed per warp, so every address below is
        // a per-warp base plus a compile-time multiple of the row step
        const uint32_t cb = sbase + OFF_C + sc * C_BYTES + dw * C_ROW + 4 * wq;
        const uint32_t bb = sbase + OFF_B + sb * B_BYTES + dst_lane;
        const uint32_t tb = sbase + OFF_LUT + dw * 128;
#pragma unroll 4
        for (int i = 0; i < BN / NDEC; ++i) {
          const uint32_t w0 = lds32(cb + i * NDEC * C_ROW);
          const uint32_t w1 = lds32(cb + i * NDEC * C_ROW + 4);   // may read the next row: unused bits
          const uint32_t v = __funnelshift_r(w0, w1, wsh);
          const uint32_t tbl = tb + i * NDEC * 128;
          const uint32_t e0 = lds_u16(((v << 1) & 0x7Eu) | tbl);
          const uint32_t e1 = lds_u16(((v >> 5) & 0x7Eu) | tbl);
          sts32(bb + i * (NDEC / 8) * 1024, __byte_perm(e0, e1, 0x5410));
        }
        sm100::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          sm100::mbar_arrive(bar.full_b + 8 * sb);
          sm100::mbar_arrive(bar.empty_c + 8 * sc);
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(bar.lut_empty);
      // epilogue: this warp drains lanes [32q, 32q+32) of both 128-row accumulators
      if (!sm100::mbar_wait(bar.acc_full, tl & 1, WAIT_BUDGET)) { ok = false; break; }
      qld::pdl_wait();
      sm100::tc_fence_after();
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int row = m0 + h * 128 + 32 * q + lane;
#pragma unroll 1
        for (int c = ch * (BN / 32) / (NDEC / 4); c < (ch + 1) * (BN / 32) / (NDEC / 4); ++c) {
          uint32_t v[32];
          sm100::tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + h * BN + c * 32, v);
          sm100::tmem_wait_ld();
          if (row < M) {
            if (ydt == QL_OUT_F32) {
              float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(y) + (size_t)row * N + n0 + c * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                     __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
            } else {
              uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(y) + (size_t)row * N + n0 + c * 32);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                uint32_t p[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  p[j] = uint32_t(qld::f32_to_bf16_rn(__uint_as_float(v[8 * i + 2 * j]))) |
                         (uint32_t(qld::f32_to_bf16_rn(__uint_as_float(v[8 * i + 2 * j + 1]))) << 16);
                dst[i] = make_uint4(p[0], p[1], p[2], p[3]);
              }
            }
          }
        }
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(bar.acc_empty);
    }
  }

  if (!ok) atomicExch(&g_gemm_timeout, 1);
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    sm100::tc_fence_after();
    sm100::tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static std::once_flag once;
  static EncodeTiledFn fn = nullptr;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

}  // namespace

namespace ql {

ql_status benq_gemm_launch(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y, ql_out_dtype ydt,
                           int M, int N, int K, cudaStream_t s) {
  if (N % BN || K % BK) return fail(QL_ERR_UNSUPPORTED, "benq_linear: batch > 16 needs N %% 256 == 0 and K %% 64 == 0");
  EncodeTiledFn enc = encode_fn();
  if (!enc) return fail(QL_ERR_CUDA, "benq_linear: cuTensorMapEncodeTiled is unavailable");
  CUtensorMap mx, mc;
  {
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {BK, BM};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t *>(x), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(QL_ERR_CUDA, "benq_linear: cannot encode the activation tensor map");
  }
  {
    const cuuint64_t rowbytes = (cuuint64_t)K * 3 / 4;
    const cuuint64_t dims[2] = {rowbytes, (cuuint64_t)N};
    const cuuint64_t strides[1] = {rowbytes};
    const cuuint32_t box[2] = {C_ROW, BN};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(codes), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(QL_ERR_CUDA, "benq_linear: cannot encode the code tensor map");
  }
  static std::once_flag attr_once;
  static cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once, [] {
    attr_err = cudaFuncSetAttribute(benq_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
  });
  if (attr_err != cudaSuccess) return fail(QL_ERR_CUDA, "benq_linear: cannot reserve GEMM shared memory");
  const int ntiles = ((M + BM - 1) / BM) * (N / BN);
  const int grid = std::min(ntiles, sm_count());
  launch(benq_gemm_kernel, grid, THREADS, SMEM_BYTES, s, mx, mc, lut, y, (int)ydt, M, N, K);
  return launch_status("benq_linear (tensor-core GEMM)");
}

ql_status benq_gemm_read_timeout(int *flag) {
  int zero = 0;
  if (cudaMemcpyFromSymbol(flag, g_gemm_timeout, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_gemm_timeout, &zero, sizeof(int)) != cudaSuccess)
    return fail(QL_ERR_CUDA, "ql_check: cannot read the device timeout flag");
  return QL_OK;
}

}  // namespace ql
