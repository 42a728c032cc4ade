// Scaffolding shared by the tensor-core GEMMs that run on CTA pairs (benq_gemm_sm100.cu and
// mdbf_gemm_sm100.cu): shared-memory accessors, the bounded wait, work items with a split last
// wave, and the host-side split plan.  Not part of the ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <mutex>

#include "sm100_ptx.cuh"

namespace pairgemm {

constexpr long long WAIT_BUDGET = 4000000000LL;   // clock cycles (~2 s)
constexpr int SPLIT_MAX = 8;                      // K ranges per tile of the last wave

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
__device__ __forceinline__ void sts64(uint32_t a, uint32_t lo, uint32_t hi) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(lo), "r"(hi) : "memory");
}
__device__ __forceinline__ uint32_t ld_volatile_u32(uint32_t a) {
  uint32_t v;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(v) : "r"(a) : "memory");
  return v;
}
__device__ __forceinline__ void st_cluster_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.relaxed.cluster.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// Bounded wait shared by all roles.  Gives up when the budget runs out or when the pair's abort
// flag is set; a thread that runs out sets the flag in both CTAs so that the others stop at once.
struct Waiter {
  uint32_t abort_local, abort_peer;
  long long budget = WAIT_BUDGET;
  __device__ bool wait(uint32_t bar, uint32_t parity, bool cluster_scope) const {
    auto probe = [&] {
      return cluster_scope ? sm100::mbar_try_wait_cluster(bar, parity) : sm100::mbar_try_wait(bar, parity);
    };
    if (probe()) return true;
    const long long t0 = clock64();
    while (!probe()) {
      if (ld_volatile_u32(abort_local) != 0) return false;
      if (clock64() - t0 > budget) {
        sts32(abort_local, 1);
        st_cluster_u32(abort_peer, 1);
        return false;
      }
    }
    return true;
  }
};

// ----------------------------------------------------------------------------------- epilogue
enum OutKind { OUT_F16 = 0, OUT_BF16 = 1, OUT_F32 = 2 };

__device__ __forceinline__ void sts128v(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z), "r"(w) : "memory");
}
__device__ __forceinline__ uint32_t pack2(float a, float b, int kind) {
  uint32_t r;
  if (kind == OUT_F16)
    asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  else
    asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(b), "f"(a));
  return r;
}

// Writes a CTA's 256 x 256 fp32 accumulator tile (rows m0 .. m0 + 255 of the output, two
// 128-lane halves at tmem and tmem + 256 columns) to columns n0 .. n0 + 255 through tensor
// stores.  The staging buffer `ring` is four 16 KB boxes of 128 rows x 128 bytes in the 128-byte
// swizzle of `map`; it holds one round: a 128-row half for 16-bit outputs, a quarter (32 columns
// per box) for fp32.  Epilogue warp (q, ch) = (its tensor-memory lane quarter, dw / 4) converts
// rows 32q .. 32q + 31 of box ch.  Each value is multiplied by row_scale[row] when row_scale is
// not null, then rounded to the output type (nearest even).  All ndec epilogue warps arrive on
// stg_full per round; warp 0's lane 0 issues the box stores (clipped at the output's edge),
// waits until the staging has been read and arrives on stg_free, which every warp waits on
// before reusing the buffer and before returning.  ep counts rounds across calls (phase parity).
// Returns false when a wait gave up.
__device__ __forceinline__ bool staged_tile_store(uint32_t tmem, uint32_t ring, const CUtensorMap *map, int kind,
                                                  const float *__restrict__ row_scale, int m0, int n0, int M,
                                                  int Nout, int q, int ch, int dw, int lane, const Waiter &wt,
                                                  uint32_t stg_full, uint32_t stg_free, int &ep) {
  const bool f32o = kind == OUT_F32;
  const int cpr = f32o ? 1 : 2, nround = f32o ? 4 : 2;
  const uint32_t rbase = ring + (uint32_t)ch * 16384u + (uint32_t)(32 * q + lane) * 128u;
  const uint32_t rsw = (uint32_t)(lane & 7);
#pragma unroll 1
  for (int rd = 0; rd < nround; ++rd) {
    const int h = f32o ? rd >> 1 : rd, cc = f32o ? rd & 1 : 0;
    const int row = m0 + h * 128 + 32 * q + lane;
    const float rs = (row_scale != nullptr && row < M) ? __ldg(row_scale + row) : 1.f;
    if (ep > 0 && !wt.wait(stg_free, (ep - 1) & 1, false)) return false;
#pragma unroll 1
    for (int k = 0; k < cpr; ++k) {
      const int c = 2 * ch + (f32o ? cc : k);   // accumulator chunk of 32 columns
      uint32_t v[32];
      sm100::tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + h * 256 + c * 32, v);
      sm100::tmem_wait_ld();
      if (f32o) {
#pragma unroll
        for (int j = 0; j < 8; ++j)
          sts128v(rbase + (((uint32_t)j ^ rsw) << 4), __float_as_uint(__uint_as_float(v[4 * j]) * rs),
                  __float_as_uint(__uint_as_float(v[4 * j + 1]) * rs), __float_as_uint(__uint_as_float(v[4 * j + 2]) * rs),
                  __float_as_uint(__uint_as_float(v[4 * j + 3]) * rs));
      } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            pk[e] = pack2(__uint_as_float(v[8 * j + 2 * e]) * rs, __uint_as_float(v[8 * j + 2 * e + 1]) * rs, kind);
          sts128v(rbase + (((uint32_t)(4 * k + j) ^ rsw) << 4), pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    sm100::fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) sm100::mbar_arrive(stg_full);
    if (dw == 0 && lane == 0) {
      if (!wt.wait(stg_full, ep & 1, false)) return false;
      const int y0 = m0 + h * 128;
      for (int b = 0; b < 4; ++b) {
        const int x0 = n0 + 64 * b + 32 * cc;
        if (x0 < Nout && y0 < M) sm100::tma_store_2d(map, x0, y0, ring + b * 16384u);
      }
      sm100::bulk_commit();
      sm100::bulk_wait_read0();
      sm100::mbar_arrive(stg_free);
    }
    ++ep;
  }
  // the staging buffer is written again by the caller: wait for the last round's stores to read it
  return wt.wait(stg_free, (ep - 1) & 1, false);
}

// M panel and N tile of pair tile t.  N-fastest (consecutive tiles, which run in the same wave, share
// an activation panel) when the activations outweigh the weight stream the decoders read, else
// M-fastest (they share a weight tile): the larger operand is then read from DRAM about once, and
// the split last wave re-reads what the previous wave has just brought into L2.
__device__ __forceinline__ void tile_mn(int t, int mt, int nt, int nfast, int &m, int &n) {
  if (nfast) {
    m = t / nt;
    n = t - m * nt;
  } else {
    n = t / mt;
    m = t - n * mt;
  }
}

// Work items: pair tiles 0 .. full-1 whole, then each of the remaining tiles (the last, partial
// wave) split into `parts` K ranges so that the otherwise idle pairs share it.  A split item
// writes an fp32 partial; the last CTA to finish a tile sums the partials in part order.
struct Item {
  int tile, kb0, kb1, part;   // part < 0: whole tile
};
__device__ __forceinline__ Item item_of(int i, int full, int parts, int nkb) {
  if (i < full) return {i, 0, nkb, -1};
  const int u = i - full, j = u / parts, q = u - j * parts;
  return {full + j, (int)((int64_t)q * nkb / parts), (int)((int64_t)(q + 1) * nkb / parts), q};
}

// Whole tiles run in full waves of `pairs` CTA pairs; when the last wave would leave at least
// half of the pairs idle, its L tiles are split into `parts` K ranges each (L * parts <= pairs).
// `pair_tile_bytes` is the size of one fp32 partial of a pair tile (both CTAs).
struct SplitPlan {
  int full, parts, leftover;
  size_t partial_bytes, counter_bytes;
};
inline SplitPlan split_plan(int ntiles, int nkb, int pairs, size_t pair_tile_bytes) {
  SplitPlan p{ntiles, 1, 0, 0, 0};
  if (pairs <= 0) return p;
  const int full = (ntiles / pairs) * pairs, left = ntiles - full;
  if (left > 0 && 2 * left <= pairs) {
    const int parts = std::min(std::min(pairs / left, SPLIT_MAX), nkb);
    if (parts >= 2) {
      p.full = full;
      p.parts = parts;
      p.leftover = left;
      p.partial_bytes = (size_t)left * parts * pair_tile_bytes;
      p.counter_bytes = ((size_t)left * 2 * sizeof(unsigned) + 255) / 256 * 256;
    }
  }
  return p;
}

// cuTensorMapEncodeTiled from the driver, looked up once through the runtime (no libcuda link).
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
inline EncodeTiledFn encode_tiled_fn() {
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

// Tensor map of a row-major 2-D array [rows][cols] of esize-byte elements (row stride ld
// elements) in boxes of box_rows rows x 128 bytes with the 128-byte swizzle (the tensor core's
// operand layout, and the staging layout of the tensor-store epilogue).
inline bool encode_rows_sw128(EncodeTiledFn enc, CUtensorMap *map, CUtensorMapDataType dt, const void *base,
                              uint64_t rows, uint64_t cols, uint64_t ld, uint32_t box_rows, uint32_t esize = 2) {
  const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)ld * esize};
  const cuuint32_t box[2] = {128 / esize, box_rows};
  const cuuint32_t es[2] = {1, 1};
  return enc(map, dt, 2, const_cast<void *>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace pairgemm
