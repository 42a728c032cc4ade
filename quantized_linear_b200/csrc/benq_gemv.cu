// BenQ 6-bit per-row LUT layer: debug dequantizer and the decode GEMV (batch <= 16).
//
// Format ("Qwen3.8-27B -- BenQ 6-bit", "What BenQ stores"): code k of row n is
// bits [6k, 6k+6) of the row's little-endian bitstream (4 codes per 3 bytes);
// its value is lut[n][code], a bf16 from the row's own 64-entry table.
//
// Decode GEMV design (bandwidth bound: 0.75 B of codes per weight):
//  * One CTA = C warps, C = ceil(K / 1024).  Lane l of warp w owns the same 32
//    consecutive codes [1024 w + 32 l, +32) of every row (24 bytes, read with
//    three 8-byte loads), so at batch 1 its 32 activations live in registers
//    for the whole kernel and the inner loop reads nothing but codes.
//  * The CTA walks blocks of R rows (grid-stride).  The R tables (128 B of
//    bf16 each) sit in shared memory, double-buffered; a lookup is a 16-bit
//    shared load at byte offset 2*code.  One table spans exactly the 32 banks
//    (two entries per 32-bit word) and all lanes read the same table, so a
//    lookup is never a bank conflict (lanes hitting one word are a broadcast).
//  * Per code: one shift (a funnel shift for codes straddling two words), one
//    AND to form 2*code, the lookup, and one mixed-precision FMA
//    (fma.rn.f32.bf16: bf16 x bf16 product, exact, added into fp32).
//  * Lane partial sums go to shared memory; after one barrier per row block
//    the C x 32 partials of each output are summed in a fixed order
//    (deterministic), and the next block's codes and tables are already in flight.
#include <algorithm>
#include <climits>

#include "ql_internal.cuh"

namespace {

constexpr int LANE_CODES = 32;
constexpr int WARP_CODES = 32 * LANE_CODES;
constexpr int MAX_WARPS = 20;  // K <= 20480 on the fast path (keeps ~100 registers per thread)

// ------------------------------------------------------------------------------------------
// Debug dequantizer: one thread per 3-byte group, 4 bf16 outputs.
// ------------------------------------------------------------------------------------------
__global__ void benq_dequant_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ lut,
                                    uint16_t *__restrict__ W, int N, int K) {
  const int64_t gpr = K / 4;
  const int64_t total = (int64_t)N * gpr;
  const int64_t rowbytes = 3LL * K / 4;
  qld::pdl_trigger();
  qld::pdl_wait();
  for (int64_t g = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; g < total;
       g += (int64_t)gridDim.x * blockDim.x) {
    const int64_t n = g / gpr;
    const int64_t q = g - n * gpr;
    const uint8_t *p = codes + n * rowbytes + 3 * q;
    const uint32_t v = uint32_t(p[0]) | (uint32_t(p[1]) << 8) | (uint32_t(p[2]) << 16);
    const uint16_t *t = lut + n * 64;
    uint16_t *w = W + n * (int64_t)K + 4 * q;
    w[0] = t[v & 63];
    w[1] = t[(v >> 6) & 63];
    w[2] = t[(v >> 12) & 63];
    w[3] = t[(v >> 18) & 63];
  }
}

__device__ __forceinline__ uint2 ldg_u2(const uint8_t *p) {
  uint2 v;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

__device__ __forceinline__ uint4 ldg_u4(const void *p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// 2*code of code j (0..31) of a lane's 6-word (192-bit) slice: the byte offset of its table entry.
template <int J>
__device__ __forceinline__ uint32_t entry_offset(const uint32_t (&w)[6]) {
  constexpr int s = 6 * J, q = s >> 5, h = s & 31;
  if constexpr (h == 0) {
    return (w[q] << 1) & 0x7Eu;
  } else if constexpr (h <= 26) {
    return (w[q] >> (h - 1)) & 0x7Eu;
  } else {
    return __funnelshift_r(w[q], w[q + 1], h - 1) & 0x7Eu;
  }
}

__device__ __forceinline__ uint16_t lds_u16(uint32_t saddr) {
  uint16_t v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(saddr));
  return v;
}

template <int J>
struct DecodeRow {
  template <int BM>
  static __device__ __forceinline__ void dot(const uint32_t (&w)[6], uint32_t tbl, const uint16_t (&xr)[32],
                                             float &acc) {
    DecodeRow<J - 1>::template dot<BM>(w, tbl, xr, acc);
    acc = qld::fma_bf16(lds_u16(tbl + entry_offset<J - 1>(w)), xr[J - 1], acc);
  }
  static __device__ __forceinline__ void decode(const uint32_t (&w)[6], uint32_t tbl, uint16_t (&out)[32]) {
    DecodeRow<J - 1>::decode(w, tbl, out);
    out[J - 1] = lds_u16(tbl + entry_offset<J - 1>(w));
  }
};
template <>
struct DecodeRow<0> {
  template <int BM>
  static __device__ __forceinline__ void dot(const uint32_t (&)[6], uint32_t, const uint16_t (&)[32], float &) {}
  static __device__ __forceinline__ void decode(const uint32_t (&)[6], uint32_t, uint16_t (&)[32]) {}
};

__device__ __forceinline__ void unpack_x(const uint4 (&v)[4], uint16_t (&xr)[32]) {
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint32_t u[4] = {v[t].x, v[t].y, v[t].z, v[t].w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      xr[8 * t + 2 * e] = uint16_t(u[e] & 0xFFFFu);
      xr[8 * t + 2 * e + 1] = uint16_t(u[e] >> 16);
    }
  }
}

template <int R, int BMAX>
__global__ void __launch_bounds__(MAX_WARPS * 32)
    benq_gemv_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ lut,
                     const uint16_t *__restrict__ x, void *__restrict__ y, int ydt, int B, int N, int K) {
  extern __shared__ __align__(16) unsigned char smem[];
  uint16_t *lut_s = reinterpret_cast<uint16_t *>(smem);             // [2][R][64]
  float *part = reinterpret_cast<float *>(smem + 2 * R * 128);      // [2][C][R*BMAX][32]
  const int C = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kc = warp * WARP_CODES + lane * LANE_CODES;
  const bool active = kc < K;
  const int64_t rowbytes = 3LL * K / 4;
  const uint8_t *cbase = codes + 3LL * kc / 4;
  const int nblk = (N + R - 1) / R;
  int blk = blockIdx.x;
  if (blk >= nblk) return;

  auto load_codes = [&](int b, uint32_t (&w)[R][6]) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int n = b * R + r;
      if (active && n < N) {
        const uint8_t *p = cbase + n * rowbytes;
        const uint2 a = ldg_u2(p), c = ldg_u2(p + 8), d = ldg_u2(p + 16);
        w[r][0] = a.x; w[r][1] = a.y; w[r][2] = c.x; w[r][3] = c.y; w[r][4] = d.x; w[r][5] = d.y;
      } else {
#pragma unroll
        for (int q = 0; q < 6; ++q) w[r][q] = 0;
      }
    }
  };
  // tables: threads 0 .. 8R-1 each move 16 bytes of the R x 128-byte block
  auto load_lut = [&](int b, uint4 &v) {
    v = make_uint4(0, 0, 0, 0);
    if (threadIdx.x < 8 * R) {
      const int n = b * R + (threadIdx.x >> 3);
      if (n < N) v = ldg_u4(lut + (int64_t)n * 64 + (threadIdx.x & 7) * 8);
    }
  };
  auto store_lut = [&](int buf, const uint4 &v) {
    if (threadIdx.x < 8 * R) reinterpret_cast<uint4 *>(lut_s + buf * R * 64)[threadIdx.x] = v;
  };

  // the first block's weights do not depend on the preceding kernel: fetch them before waiting
  uint32_t cur[R][6];
  {
    uint4 lv;
    load_lut(blk, lv);
    store_lut(0, lv);
    load_codes(blk, cur);
  }
  qld::pdl_trigger();
  qld::pdl_wait();

  uint16_t xr[32];
  if constexpr (BMAX == 1) {
    uint4 v[4] = {};
    if (active) {
#pragma unroll
      for (int t = 0; t < 4; ++t) v[t] = ldg_u4(x + kc + 8 * t);
    }
    unpack_x(v, xr);
  }
  __syncthreads();

  const uint32_t lut_saddr = static_cast<uint32_t>(__cvta_generic_to_shared(lut_s));
  for (int it = 0;; ++it) {
    const int buf = it & 1;
    const int nxt = blk + gridDim.x;
    const bool has_next = nxt < nblk;
    uint32_t nc[R][6];
    uint4 lv;
    if (has_next) {
      load_codes(nxt, nc);
      load_lut(nxt, lv);
    }

    float acc[R][BMAX];
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < BMAX; ++b) acc[r][b] = 0.f;

    if (active) {
      if constexpr (BMAX == 1) {
#pragma unroll
        for (int r = 0; r < R; ++r) {
          const uint32_t tbl = lut_saddr + (buf * R + r) * 128;
          DecodeRow<32>::dot<1>(cur[r], tbl, xr, acc[r][0]);
        }
      } else {
        uint16_t wv[R][32];
#pragma unroll
        for (int r = 0; r < R; ++r) DecodeRow<32>::decode(cur[r], lut_saddr + (buf * R + r) * 128, wv[r]);
#pragma unroll
        for (int b = 0; b < BMAX; ++b) {
          if (b < B) {
            uint4 v[4];
#pragma unroll
            for (int t = 0; t < 4; ++t) v[t] = ldg_u4(x + (int64_t)b * K + kc + 8 * t);
            unpack_x(v, xr);
#pragma unroll
            for (int r = 0; r < R; ++r) {
              float a = acc[r][b];
#pragma unroll
              for (int j = 0; j < 32; ++j) a = qld::fma_bf16(wv[r][j], xr[j], a);
              acc[r][b] = a;
            }
          }
        }
      }
    }

    float *pb = part + (size_t)buf * C * R * BMAX * 32;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int b = 0; b < BMAX; ++b) pb[((size_t)warp * R * BMAX + r * BMAX + b) * 32 + lane] = acc[r][b];
    if (has_next) store_lut(buf ^ 1, lv);
    __syncthreads();

    // sum the C x 32 partials of each output in a fixed order
    for (int o = warp; o < R * BMAX; o += C) {
      const int r = o / BMAX, b = o - r * BMAX;
      const int n = blk * R + r;
      if (b >= B || n >= N) continue;
      float s = 0.f;
      for (int c = 0; c < C; ++c) s += pb[((size_t)c * R * BMAX + o) * 32 + lane];
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
      if (lane == 0) {
        if (ydt == QL_OUT_F32)
          static_cast<float *>(y)[(int64_t)b * N + n] = s;
        else
          static_cast<uint16_t *>(y)[(int64_t)b * N + n] = qld::f32_to_bf16_rn(s);
      }
    }
    if (!has_next) break;
    blk = nxt;
#pragma unroll
    for (int r = 0; r < R; ++r)
#pragma unroll
      for (int q = 0; q < 6; ++q) cur[r][q] = nc[r][q];
  }
}

// Any K % 4 == 0: one warp per row, lanes over 3-byte groups, table read from global memory.
__global__ void benq_gemv_generic_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ lut,
                                         const uint16_t *__restrict__ x, void *__restrict__ y, int ydt, int B,
                                         int N, int K) {
  const int lane = threadIdx.x & 31;
  const int64_t rowbytes = 3LL * K / 4;
  qld::pdl_trigger();
  qld::pdl_wait();
  for (int64_t n = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5; n < N;
       n += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    float acc[16];
#pragma unroll
    for (int b = 0; b < 16; ++b) acc[b] = 0.f;
    const uint8_t *row = codes + n * rowbytes;
    const uint16_t *t = lut + n * 64;
    for (int q = lane; q < K / 4; q += 32) {
      const uint32_t v = uint32_t(row[3 * q]) | (uint32_t(row[3 * q + 1]) << 8) | (uint32_t(row[3 * q + 2]) << 16);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint16_t wv = t[(v >> (6 * e)) & 63];
#pragma unroll
        for (int b = 0; b < 16; ++b)
          if (b < B) acc[b] = qld::fma_bf16(wv, x[(int64_t)b * K + 4 * q + e], acc[b]);
      }
    }
#pragma unroll
    for (int b = 0; b < 16; ++b) {
      if (b >= B) break;
      float s = acc[b];
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
      if (lane == 0) {
        if (ydt == QL_OUT_F32)
          static_cast<float *>(y)[(int64_t)b * N + n] = s;
        else
          static_cast<uint16_t *>(y)[(int64_t)b * N + n] = qld::f32_to_bf16_rn(s);
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// Batch-1 kernel for whole tiles (K % 1024 == 0, N % B1_T == 0).  Same lane layout as above,
// with the work per code cut to: one shift, one AND|OR forming the 32-bit shared address of
// the table entry (tables are 128-byte aligned, so the OR is an add), one 16-bit shared load
// and one mixed-precision FMA of the raw bf16 entry with the raw bf16 activation.  Two
// accumulators per row halve the FMA dependency chain.  Two row groups of B1_R rows ping-pong
// in registers so the next group's codes are in flight while one is decoded; one barrier per
// tile of B1_T rows.  The table buffer index is a compile-time constant in each half of the
// tile loop, so every table address is a constant offset from one base.
// ------------------------------------------------------------------------------------------
constexpr int B1_R = 2, B1_T = 4;

struct B1Tables {
  uint16_t lut[2][B1_T][64];
};

// Byte offsets of the table entries of codes J and J + 1 (J even), as compile-time selections.
__device__ __forceinline__ void pair_offsets(const uint32_t (&w)[6], int j, uint32_t &o0, uint32_t &o1) {
  switch (j) {
#define QL_PAIR(J)                \
  case J:                         \
    o0 = entry_offset<J>(w);      \
    o1 = entry_offset<J + 1>(w);  \
    break;
    QL_PAIR(0) QL_PAIR(2) QL_PAIR(4) QL_PAIR(6) QL_PAIR(8) QL_PAIR(10) QL_PAIR(12) QL_PAIR(14)
    QL_PAIR(16) QL_PAIR(18) QL_PAIR(20) QL_PAIR(22) QL_PAIR(24) QL_PAIR(26) QL_PAIR(28) QL_PAIR(30)
#undef QL_PAIR
  }
}

template <int V>
struct IntC {
  static constexpr int value = V;
};

// Up to B1_MAXSEG layers of the same K read in one launch (MODE B1_MULTI): layer s owns the row
// tiles [tend[s - 1], tend[s]) of the launch (tend of unused entries is INT_MAX).
constexpr int B1_MAXSEG = 4;
struct B1Multi {
  const uint8_t *codes[B1_MAXSEG];
  const uint16_t *lut[B1_MAXSEG];
  void *y[B1_MAXSEG];
  int tend[B1_MAXSEG];
};
enum { B1_PLAIN = 0, B1_MLP = 1, B1_MULTI = 2 };

// MODE B1_MLP: the gated MLP h = silu(x W_g^T) * (x W_u^T) in the same launch: codes / lut are W_g
// and codes2 / lut2 W_u; a tile is two output features, its first row group the two gate rows and
// its second the two up rows, and the tile's sums leave as silu(g) * u.  MODE B1_MULTI: the layers
// of `ms` one after another, each tile taking its codes, tables and output from its own layer.
template <int MODE>
__global__ void __launch_bounds__(MAX_WARPS * 32, 1)
    benq_gemv_b1_kernel(const uint8_t *__restrict__ codes, const uint16_t *__restrict__ lut,
                        const uint8_t *__restrict__ codes2, const uint16_t *__restrict__ lut2,
                        const uint16_t *__restrict__ x, void *__restrict__ y, int ydt, int N, int K,
                        const __grid_constant__ B1Multi ms) {
  constexpr bool MLP = MODE == B1_MLP;
  __shared__ __align__(128) B1Tables tb;
  extern __shared__ __align__(16) float b1part[];  // [2][C][B1_T][32]
  const int C = blockDim.x >> 5;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kc = warp * WARP_CODES + lane * LANE_CODES;
  const uint32_t rowbytes = 3u * K / 4;
  const uint8_t *cbase = MODE == B1_MULTI ? nullptr : codes + 3u * kc / 4;
  const uint8_t *cbase2 = MLP ? codes2 + 3u * kc / 4 : nullptr;
  constexpr int TOUT = MLP ? B1_T / 2 : B1_T;   // output features per tile
  const int ntile = N / TOUT;
  int tile = blockIdx.x;
  if (tile >= ntile) return;
  // where tile t's rows live: this lane's code slice, the tables and the output, and the tile's index
  // within its layer
  struct Src {
    const uint8_t *c;
    const uint16_t *l;
    void *yy;
    int lt;
  };
  auto src_of = [&](int t) -> Src {
    if constexpr (MODE == B1_MULTI) {
      int sg = 0;
#pragma unroll
      for (int i = 1; i < B1_MAXSEG; ++i)
        if (t >= ms.tend[i - 1]) sg = i;
      return {ms.codes[sg] + 3u * kc / 4, ms.lut[sg], ms.y[sg], t - (sg ? ms.tend[sg - 1] : 0)};
    } else {
      return {cbase, lut, y, t};
    }
  };
  // Before waiting on the preceding kernel, pull this CTA's first tile of weights (codes and
  // tables) toward L2; prefetches hold no registers, so the loop below is compiled as if they
  // were absent.  Activations are loaded first after the wait: loading them after the codes
  // made the compiler schedule the decode loop far worse.
  if constexpr (MLP) {
    const uint8_t *p = cbase + (size_t)tile * TOUT * rowbytes, *p2 = cbase2 + (size_t)tile * TOUT * rowbytes;
#pragma unroll
    for (int r = 0; r < TOUT; ++r) {
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p + (size_t)r * rowbytes));
      asm volatile("prefetch.global.L2 [%0];" ::"l"(p2 + (size_t)r * rowbytes));
    }
    if (threadIdx.x < B1_T)
      asm volatile("prefetch.global.L2 [%0];" ::"l"((threadIdx.x < TOUT ? lut : lut2) +
                                                      ((size_t)tile * TOUT + (threadIdx.x % TOUT)) * 64));
  } else {
    const Src sr = src_of(tile);
    const uint8_t *p = sr.c + (size_t)sr.lt * B1_T * rowbytes;
#pragma unroll
    for (int r = 0; r < B1_T; ++r) asm volatile("prefetch.global.L2 [%0];" ::"l"(p + (size_t)r * rowbytes));
    if (threadIdx.x < B1_T)
      asm volatile("prefetch.global.L2 [%0];" ::"l"(sr.l + ((size_t)sr.lt * B1_T + threadIdx.x) * 64));
  }
  qld::pdl_trigger();
  qld::pdl_wait();
  uint16_t xh[32];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    const uint4 v = ldg_u4(x + kc + 8 * t);
    const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      xh[8 * t + 2 * e] = u[e] & 0xFFFF;
      xh[8 * t + 2 * e + 1] = u[e] >> 16;
    }
  }
  // rows of tile t's row group grp (grp = 0, 1): B1_R consecutive rows of W, or for MLP the
  // tile's two gate rows (grp 0) and its two up rows (grp 1)
  auto load_rows = [&](int t, int grp, uint32_t (&w)[B1_R][6]) {
    const Src sr = src_of(t);
    const uint8_t *p = MLP ? (grp == 0 ? cbase : cbase2) + (size_t)t * TOUT * rowbytes
                           : sr.c + (size_t)(sr.lt * B1_T + grp * B1_R) * rowbytes;
#pragma unroll
    for (int r = 0; r < B1_R; ++r) {
      const uint2 a = ldg_u2(p + r * rowbytes), c = ldg_u2(p + r * rowbytes + 8), d = ldg_u2(p + r * rowbytes + 16);
      w[r][0] = a.x; w[r][1] = a.y; w[r][2] = c.x; w[r][3] = c.y; w[r][4] = d.x; w[r][5] = d.y;
    }
  };
  auto load_lut = [&](int t, uint4 &v) {
    if (threadIdx.x < 8 * B1_T) {
      const int i = threadIdx.x >> 3;   // table row of the tile
      const Src sr = src_of(t);
      const uint16_t *src = MLP ? (i < TOUT ? lut : lut2) + ((size_t)t * TOUT + (i % TOUT)) * 64
                                : sr.l + ((size_t)sr.lt * B1_T + i) * 64;
      v = ldg_u4(src + (threadIdx.x & 7) * 8);
    }
  };
  auto store_lut = [&](int buf, const uint4 &v) {
    if (threadIdx.x < 8 * B1_T) reinterpret_cast<uint4 *>(&tb.lut[buf][0][0])[threadIdx.x] = v;
  };
  auto dot = [&](const uint32_t (&w)[6], const uint16_t *tp) -> float {
    const uint32_t tbs = (uint32_t)__cvta_generic_to_shared(tp);
    float a0 = 0.f, a1 = 0.f;
#pragma unroll
    for (int j = 0; j < 32; j += 2) {
      uint32_t o0, o1;
      pair_offsets(w, j, o0, o1);
      a0 = qld::fma_bf16(lds_u16(o0 | tbs), xh[j], a0);
      a1 = qld::fma_bf16(lds_u16(o1 | tbs), xh[j + 1], a1);
    }
    return a0 + a1;
  };
  uint4 lv = make_uint4(0, 0, 0, 0);
  load_lut(tile, lv);
  store_lut(0, lv);
  uint32_t ga[B1_R][6], gb[B1_R][6];
  load_rows(tile, 0, ga);
  __syncthreads();
  float *mypart = b1part + (warp * B1_T) * 32 + lane;
  constexpr int GP = B1_T / B1_R;  // even

  // One tile with table buffer BUF.  On entry ga holds the tile's first row group; on exit it
  // holds the next tile's first group.  Returns whether there is a next tile.
  auto do_tile = [&](auto bufc, int nxt) {
    constexpr int BUF = decltype(bufc)::value;
    const bool has_next = nxt < ntile;
    if (has_next) load_lut(nxt, lv);
    float *pb = mypart + BUF * C * B1_T * 32;
#pragma unroll
    for (int g = 0; g < GP; g += 2) {
      load_rows(tile, g + 1, gb);
#pragma unroll
      for (int r = 0; r < B1_R; ++r) pb[(g * B1_R + r) * 32] = dot(ga[r], &tb.lut[BUF][g * B1_R + r][0]);
      if (g + 2 < GP)
        load_rows(tile, g + 2, ga);
      else if (has_next)
        load_rows(nxt, 0, ga);
#pragma unroll
      for (int r = 0; r < B1_R; ++r)
        pb[((g + 1) * B1_R + r) * 32] = dot(gb[r], &tb.lut[BUF][(g + 1) * B1_R + r][0]);
    }
    if (has_next) store_lut(BUF ^ 1, lv);
    __syncthreads();
    const float *pr = b1part + BUF * C * B1_T * 32;
    if constexpr (MLP) {
      for (int o = warp; o < TOUT; o += C) {
        float g = 0.f, u = 0.f;
        for (int c = 0; c < C; ++c) {
          g += pr[(c * B1_T + o) * 32 + lane];
          u += pr[(c * B1_T + TOUT + o) * 32 + lane];
        }
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) {
          g += __shfl_xor_sync(0xffffffffu, g, d);
          u += __shfl_xor_sync(0xffffffffu, u, d);
        }
        if (lane == 0) {
          const float h = qld::silu_mul(g, u);
          const int n = tile * TOUT + o;
          if (ydt == QL_OUT_F32)
            static_cast<float *>(y)[n] = h;
          else
            static_cast<uint16_t *>(y)[n] = qld::f32_to_bf16_rn(h);
        }
      }
    } else {
      const Src sr = src_of(tile);
      for (int o = warp; o < B1_T; o += C) {
        float s = 0.f;
        for (int c = 0; c < C; ++c) s += pr[(c * B1_T + o) * 32 + lane];
#pragma unroll
        for (int d = 16; d > 0; d >>= 1) s += __shfl_xor_sync(0xffffffffu, s, d);
        if (lane == 0) {
          const int n = sr.lt * B1_T + o;
          if (ydt == QL_OUT_F32)
            static_cast<float *>(sr.yy)[n] = s;
          else
            static_cast<uint16_t *>(sr.yy)[n] = qld::f32_to_bf16_rn(s);
        }
      }
    }
    tile = nxt;
    return has_next;
  };
  while (true) {
    if (!do_tile(IntC<0>{}, tile + gridDim.x)) break;
    if (!do_tile(IntC<1>{}, tile + gridDim.x)) break;
  }
}

template <int MODE>
ql_status launch_b1(const uint8_t *codes, const uint16_t *lut, const uint8_t *codes2, const uint16_t *lut2,
                    const uint16_t *x, void *y, ql_out_dtype ydt, int N, int K, cudaStream_t s,
                    const B1Multi &ms = B1Multi{}) {
  constexpr bool MLP = MODE == B1_MLP;
  const int C = K / WARP_CODES;
  const int threads = C * 32;
  const size_t smem = (size_t)2 * C * B1_T * 32 * sizeof(float);
  const int per_sm = ql::blocks_per_sm(benq_gemv_b1_kernel<MODE>, threads, smem);
  if (per_sm < 1) return ql::fail(QL_ERR_CUDA, "benq_linear: occupancy query failed");
  const int grid = std::min(N / (MLP ? B1_T / 2 : B1_T), per_sm * ql::sm_count());
  ql::launch(benq_gemv_b1_kernel<MODE>, grid, threads, smem, s, codes, lut, codes2, lut2, x, y, (int)ydt, N, K, ms);
  return ql::launch_status(MODE == B1_MLP     ? "benq_mlp_gate_up (batch-1 GEMV)"
                           : MODE == B1_MULTI ? "benq_linear_multi (batch-1 GEMV)"
                                              : "benq_linear (batch-1 GEMV)");
}

template <int R, int BMAX>
ql_status launch_fast(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y, ql_out_dtype ydt,
                      int B, int N, int K, cudaStream_t s) {
  const int C = (K + WARP_CODES - 1) / WARP_CODES;
  const int threads = C * 32;
  const size_t smem = 2 * R * 128 + (size_t)2 * C * R * BMAX * 32 * sizeof(float);
  auto kern = benq_gemv_kernel<R, BMAX>;
  if (smem > 48 * 1024) {
    if (ql::set_max_smem(kern, (int)smem) != cudaSuccess)
      return ql::fail(QL_ERR_CUDA, "benq_linear: cannot reserve %zu bytes of shared memory", smem);
  }
  const int per_sm = ql::blocks_per_sm(kern, threads, smem);
  if (per_sm < 1) return ql::fail(QL_ERR_CUDA, "benq_linear: occupancy query failed");
  const int nblk = (N + R - 1) / R;
  const int grid = std::min(nblk, per_sm * ql::sm_count());
  ql::launch(kern, grid, threads, smem, s, codes, lut, x, y, (int)ydt, B, N, K);
  return ql::launch_status("benq_linear (decode GEMV)");
}

}  // namespace

namespace ql {

ql_status benq_dequant_launch(const uint8_t *codes, const uint16_t *lut, uint16_t *W, int N, int K,
                              cudaStream_t s) {
  const int64_t total = (int64_t)N * (K / 4);
  const int threads = 256;
  const int64_t want = (total + threads - 1) / threads;
  const int grid = (int)std::min<int64_t>(want, (int64_t)sm_count() * 8);
  launch(benq_dequant_kernel, grid, threads, 0, s, codes, lut, W, N, K);
  return launch_status("benq_dequant_debug");
}

ql_status benq_gemv_launch(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y,
                           ql_out_dtype ydt, int B, int N, int K, cudaStream_t s) {
  const bool fast = (K % LANE_CODES == 0) && K <= MAX_WARPS * WARP_CODES && aligned(codes, 16) &&
                    aligned(x, 16);
  if (fast) {
    if (B == 1 && K % WARP_CODES == 0 && N % B1_T == 0)
      return launch_b1<B1_PLAIN>(codes, lut, nullptr, nullptr, x, y, ydt, N, K, s);
    if (B == 1) return launch_fast<4, 1>(codes, lut, x, y, ydt, B, N, K, s);
    if (B <= 2) return launch_fast<2, 2>(codes, lut, x, y, ydt, B, N, K, s);
    if (B <= 4) return launch_fast<2, 4>(codes, lut, x, y, ydt, B, N, K, s);
    if (B <= 8) return launch_fast<2, 8>(codes, lut, x, y, ydt, B, N, K, s);
    return launch_fast<1, 16>(codes, lut, x, y, ydt, B, N, K, s);
  }
  const int threads = 256;
  const int64_t want = ((int64_t)N * 32 + threads - 1) / threads;
  const int grid = (int)std::min<int64_t>(want, (int64_t)sm_count() * 8);
  launch(benq_gemv_generic_kernel, grid, threads, 0, s, codes, lut, x, y, (int)ydt, B, N, K);
  return launch_status("benq_linear (generic GEMV)");
}

// Several layers of the same K that read the same x: one batch-1 launch over all their row tiles
// when every layer takes the batch-1 kernel, else one call per layer.
ql_status benq_gemv_multi_launch(const benq_layer *layers, int S, const uint16_t *x, ql_out_dtype ydt, int B, int K,
                                 cudaStream_t s) {
  bool one = B == 1 && S <= B1_MAXSEG && K % WARP_CODES == 0 && K <= MAX_WARPS * WARP_CODES && aligned(x, 16);
  for (int i = 0; i < S && one; ++i) one = layers[i].N % B1_T == 0 && aligned(layers[i].codes, 16);
  if (!one) {
    for (int i = 0; i < S; ++i) {
      const ql_status st = B <= 16 ? benq_gemv_launch(layers[i].codes, layers[i].lut, x, layers[i].y, ydt, B, layers[i].N, K, s)
                                   : benq_gemm_launch(layers[i].codes, layers[i].lut, x, layers[i].y, ydt, B, layers[i].N, K,
                                                      nullptr, 0, s);
      if (st != QL_OK) return st;
    }
    return QL_OK;
  }
  B1Multi ms{};
  int rows = 0;
  for (int i = 0; i < B1_MAXSEG; ++i) {
    if (i < S) {
      ms.codes[i] = layers[i].codes;
      ms.lut[i] = layers[i].lut;
      ms.y[i] = layers[i].y;
      rows += layers[i].N;
      ms.tend[i] = rows / B1_T;
    } else {
      ms.tend[i] = INT_MAX;
    }
  }
  return launch_b1<B1_MULTI>(nullptr, nullptr, nullptr, nullptr, x, nullptr, ydt, rows, K, s, ms);
}

// ------------------------------------------------------------------------------- gated MLP
// h = silu(g) * u elementwise from the two projections' fp32 outputs (batches the fused batch-1
// kernel does not take).
__global__ void __launch_bounds__(256) mlp_silu_mul_kernel(const float *__restrict__ g, const float *__restrict__ u,
                                                           void *__restrict__ h, int ydt, size_t count) {
  qld::pdl_trigger();
  qld::pdl_wait();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (size_t)gridDim.x * blockDim.x) {
    const float v = qld::silu_mul(g[i], u[i]);
    if (ydt == QL_OUT_F32)
      static_cast<float *>(h)[i] = v;
    else
      static_cast<uint16_t *>(h)[i] = qld::f32_to_bf16_rn(v);
  }
}

bool mlp_fused_shape(int B, int N, int K) {
  return B == 1 && K % WARP_CODES == 0 && K <= MAX_WARPS * WARP_CODES && N % (B1_T / 2) == 0;
}

size_t benq_mlp_workspace_size(int B, int N, int K) {
  if (B <= 0 || N <= 0 || K <= 0) return 0;
  if (mlp_fused_shape(B, N, K)) return 0;
  return ((size_t)2 * B * N * sizeof(float) + 255) / 256 * 256;
}

ql_status benq_mlp_launch(const uint8_t *codes_g, const uint16_t *lut_g, const uint8_t *codes_u, const uint16_t *lut_u,
                          const uint16_t *x, void *h, ql_out_dtype ydt, int B, int N, int K, void *ws, size_t ws_bytes,
                          cudaStream_t s) {
  // arguments validated by the caller (pointers 16-byte aligned, workspace large enough)
  if (mlp_fused_shape(B, N, K)) return launch_b1<B1_MLP>(codes_g, lut_g, codes_u, lut_u, x, h, ydt, N, K, s);
  (void)ws_bytes;
  float *g = static_cast<float *>(ws), *u = g + (size_t)B * N;
  ql_status st = B <= 16 ? benq_gemv_launch(codes_g, lut_g, x, g, QL_OUT_F32, B, N, K, s)
                         : benq_gemm_launch(codes_g, lut_g, x, g, QL_OUT_F32, B, N, K, nullptr, 0, s);
  if (st != QL_OK) return st;
  st = B <= 16 ? benq_gemv_launch(codes_u, lut_u, x, u, QL_OUT_F32, B, N, K, s)
               : benq_gemm_launch(codes_u, lut_u, x, u, QL_OUT_F32, B, N, K, nullptr, 0, s);
  if (st != QL_OK) return st;
  const size_t count = (size_t)B * N;
  const int grid = (int)std::min<size_t>((count + 255) / 256, (size_t)sm_count() * 8);
  launch(mlp_silu_mul_kernel, grid, 256, 0, s, static_cast<const float *>(g), static_cast<const float *>(u), h,
         (int)ydt, count);
  return launch_status("benq_mlp_gate_up (silu * up)");
}

}  // namespace ql
