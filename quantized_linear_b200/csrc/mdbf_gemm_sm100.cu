// MDBF prefill on sm_100a tensor cores: Y[B][n] = X W^T with W = sum_p F_p G_p, W never formed.
//
// "MDBF (Multi-Envelope Double Binary Factorization)", section "Algorithm":
//   F = S_A (.) (A_amp Q_U^T)   (n x r),     G = S_B (.) (Q_V B_amp^T)   (r x m).
// For a batch of token rows the product is two dense contractions, both on the tensor cores:
//   T = X [G_1; ..; G_P]^T            (B x P r: the paths side by side along N),
//   Y = T [F_1 .. F_P]^T              (the paths concatenated along K, so their sum is free).
// Neither factor is ever written to memory.  Inside the GEMM that consumes it, each factor element
// is rebuilt from its packed sign bit and its envelope entry sum_i L[row][i] R[col][i]: the
// envelope of a 16 x 8 block is one warp MMA (mma.sync m16n8k16, fp16 in, fp32 out; the fp16 x
// fp16 products are exact), the sign flips the fp16 sign bit, and the element is rounded to fp16
// straight into the tensor core's shared-memory operand tile.
//
// Numerics.  The tensor-core operands are fp16 (both operands of kind::f16 must share one type,
// and fp16's 11-bit significand keeps the result well inside the parity tolerance where bf16's
// 8 bits would not).  Activations arrive as bf16, whose range is wider than fp16's, so each token
// row is first scaled by a power of two (exact) into X' with max|X'| in [2^-e, 2^(1-e)); e >= 0 is
// the smallest exponent for which the envelope bound
//   |T'[b][k]| <= m * max|X'| * beta,   beta = max_p sum_i max_k|Q_V[k][i]| * max_j|B_amp[j][i]|,
// stays below half the fp16 maximum, so the intermediate T' = X' G^T is stored in fp16 without
// overflow.  The factors get the same treatment: every element of G obeys
// |G[k][j]| <= sum_i |Q_V[k][i]| |B_amp[j][i]| <= beta, and every element of F likewise
// |F[a][k]| <= alpha = max_p sum_i max_a|A_amp[a][i]| * max_k|Q_U[k][i]|, so G is rebuilt as
// G 2^-eg and F as F 2^-ef with eg, ef >= 0 the smallest exponents that put the bounds at or below
// 2^15 (beta in the bound above is then beta 2^-eg).  A power of two commutes with every fp32
// rounding of the envelope sum, so each rebuilt element is the oracle's envelope times 2^-e
// exactly before its rounding to fp16, and no factor element can leave fp16's range whatever the
// envelopes' magnitudes.  The last epilogue multiplies each row by 2^(eg + ef - s_b), the inverse
// of all three powers of two.
//
// Launches per call: envelope column maxima, activation prep (scale, convert, pad), GEMM 1
// (decodes G), GEMM 2 (decodes F).  The GEMMs share the CTA-pair structure of the BenQ GEMM: CTA
// r of a pair owns rows [256 r, 256 r + 256) of a 512 x 256 output tile and decodes operand rows
// [128 r, 128 r + 128); pair MMAs (M = 256 over two CTAs, N = 256, K = 16) read A from each CTA and
// B from both.  Per CTA: warp 0 loads A tiles (256 x 64 fp16, 128-byte swizzle) with tensor
// copies, warp 1 issues the pair MMAs (even CTA) or relays the odd CTA's decoded blocks to them,
// warps 2..17 decode the factor operand and then drain the accumulators.  No tensor or bulk load is multicast.  Every wait is bounded (see
// pair_gemm.cuh); a wait that runs out sets a flag read by ql_check().
#include <cuda.h>

#include <algorithm>
#include <mutex>
#include <type_traits>

#include "pair_gemm.cuh"
#include "ql_internal.cuh"
#include "sm100_ptx.cuh"

namespace {

using namespace pairgemm;

constexpr int PMAX = 8;                           // paths per call (the ABI's limit)
constexpr int LMAX = ql::MDBF_GEMM_LMAX;            // envelope rank handled by these kernels
constexpr int BM = 256;                           // A rows per CTA (two 128-row MMA halves)
constexpr int PM = 2 * BM;                        // A rows per pair tile
constexpr int BN = 256;                           // operand rows per pair tile (the MMA's N)
constexpr int BNH = BN / 2;                       // operand rows decoded by each CTA
constexpr int BK = 64;                            // one 128-byte swizzle row of fp16
constexpr int SA = 4, SB = 4;                     // stages: A tiles, decoded operand tiles
constexpr int A_BYTES = BM * BK * 2;              // 32 KB
constexpr int B_BYTES = BNH * BK * 2;             // 16 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + SA * A_BYTES;
constexpr int CW_BYTES = 256;                     // l <= 4: one warp's fp32 column pairs of a K block
constexpr int OFF_CW = OFF_B + SB * B_BYTES;      // two of them per decoder warp
constexpr int OFF_BAR = OFF_CW + 16 * 2 * CW_BYTES;
constexpr int NBAR = 2 * SA + 3 * SB + 6;
constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;      // tensor-memory address, abort flag, last-part flag
constexpr int SMEM_BYTES = OFF_TMEM + 16 + 1024;  // + alignment slack
constexpr int NDEC = 16;                          // decoder / epilogue warps: 8 row groups x 2 column halves
constexpr int THREADS = (2 + NDEC) * 32;          // A producer, MMA issuer, decoders
constexpr uint32_t IDESC = sm100::idesc_f16_f32(2 * 128, BN);   // pair MMA: M = 256 over two CTAs
constexpr uint16_t PAIR = 0x3;
// Bound the intermediate T' is kept under: half the fp16 maximum, which leaves room for the fp16
// rounding of the decoded G and for the fp32 accumulation order.
constexpr float T_BOUND = 32768.0f;
// Bound each rebuilt factor element is kept under (the same margin below the fp16 maximum).
constexpr float F_BOUND = 32768.0f;
static_assert(OFF_B % 1024 == 0 && A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms");
static_assert(SMEM_BYTES <= 232448, "shared memory");
static_assert(SB * B_BYTES == 4 * 16384, "the B ring stages one epilogue round: four 16 KB boxes");

__device__ int g_mgemm_timeout = 0;

// One factor operand, as the GEMM that decodes it sees it: element (row, col) of path p is
//   sign(bit col of S[p] row `row`) * sum_i Lrow[p][row][i] * Lcol[p][col][i].
// For G: rows are k (r of them), columns j (m), Lrow = Q_V, Lcol = B_amp, S = S_B; the paths sit
// side by side along the GEMM's N (path p owns rows [p seg, p seg + r)).  For F: rows are a (n),
// columns k (r), Lrow = A_amp, Lcol = Q_U, S = S_A; the paths follow one another along K (path p
// owns K columns [p seg, p seg + r)).  seg = r rounded up to the K block.
struct Factor {
  const uint8_t *S[PMAX];
  size_t ld[PMAX];
  const uint16_t *Lrow[PMAX];
  const uint16_t *Lcol[PMAX];
  int rows, cols, seg, P, l;
  int l_vec2;   // l even and every envelope base 4-byte aligned
  // l <= 4: the column envelopes once more, as fp32 [P][cpad / 2][4 terms][2 columns] (column pair
  // q holds columns 2q, 2q + 1), zero past l and past cols; cpad = the padded column count.
  const float *cpair;
  int cpad;
  // the power of two 2^-e the rebuilt elements are scaled by (written by the activation prep)
  const float *scale;
};

using qld::f2;
using qld::f2split;
using qld::f2u;
using qld::ffma2;

struct Bars {
  // full_a, peer_b and acc_empty are used in the even CTA only (both CTAs arrive on full_a and
  // acc_empty; the odd CTA's forwarder on peer_b).  dec_done collects this CTA's decoder warps.
  // stg_full / stg_free hand each epilogue round's staging buffer to the tensor stores and back.
  uint32_t full_a, empty_a, dec_done, peer_b, empty_b, acc_full, acc_empty, split_done, split_go, stg_full, stg_free;
  __device__ Bars(uint32_t base)
      : full_a(base), empty_a(full_a + 8 * SA), dec_done(empty_a + 8 * SA), peer_b(dec_done + 8 * SB),
        empty_b(peer_b + 8 * SB), acc_full(empty_b + 8 * SB), acc_empty(acc_full + 8), split_done(acc_empty + 8),
        split_go(split_done + 8), stg_full(split_go + 8), stg_free(stg_full + 8) {}
};

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts64(uint32_t a, uint32_t x, uint32_t y) {
  asm volatile("st.shared.v2.u32 [%0], {%1, %2};" ::"r"(a), "r"(x), "r"(y) : "memory");
}

// {fp16(lo), fp16(hi)} rounded to nearest even, lo in the low half
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint16_t f16_rn(float f) {
  uint16_t h;
  asm("cvt.rn.f16.f32 %0, %1;" : "=h"(h) : "f"(f));
  return h;
}

// Sign-flip mask of an fp16 pair from two adjacent sign bits: bit 1 keeps the value (+1), bit 0
// flips it (-1).  JL = 0 takes bits 0 and 1 of e, JL = 1 bits 8 and 9; the multiply copies the
// pair to bits 15/16 and 30/31 at once, and the mask keeps 15 and 31.
template <int JL>
__device__ __forceinline__ uint32_t sign_flip(uint32_t e) {
  constexpr uint32_t keep = JL == 0 ? 0x3u : 0x300u;
  constexpr uint32_t spread = JL == 0 ? 0x40008000u : 0x00400080u;   // 2^30 + 2^15, 2^22 + 2^7
  uint32_t t;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(t) : "r"(e & keep), "r"(spread));
  return ~t & 0x80008000u;
}

// Two consecutive fp16 envelope entries v[i], v[i + 1] of one row (zero past l).
__device__ __forceinline__ uint32_t env_pair(const uint16_t *__restrict__ v, int l, int i, bool vec2) {
  if (i >= l) return 0u;
  if (vec2) return __ldg(reinterpret_cast<const unsigned int *>(v + i));
  const uint32_t lo = __ldg(reinterpret_cast<const unsigned short *>(v + i));
  const uint32_t hi = i + 1 < l ? __ldg(reinterpret_cast<const unsigned short *>(v + i + 1)) : 0u;
  return lo | (hi << 16);
}

// ------------------------------------------------------------------ envelope column maxima
// emax[p][w][z][i] = max |E_w[.][i]| over row slice z of NSL for the four envelopes E_0 = Q_V,
// E_1 = B_amp (G), E_2 = A_amp, E_3 = Q_U (F) (grid P x 4 x NSL, plus the column pairs).
// Weights are read before the wait on the preceding kernel; the store comes after it.
constexpr int NSL = 16;
// Column-pair copy for the l <= 4 decoders: thread q of slice z writes the fp32 pair block of
// columns 2q, 2q + 1 of path p (grid P x 1 x NSL, one launch per factor).
__device__ __forceinline__ void write_colpairs(const Factor &f, int p, int z, float *__restrict__ out) {
  const int npair = f.cpad / 2, per = (npair + NSL - 1) / NSL;
  const unsigned short *v = reinterpret_cast<const unsigned short *>(f.Lcol[p]);
  float *o = out + (size_t)p * npair * 8;
  for (int q = z * per + (int)threadIdx.x; q < min(npair, (z + 1) * per); q += blockDim.x) {
    float e[8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int col = 2 * q + h;
        e[2 * i + h] = (i < f.l && col < f.cols) ? qld::f16_to_f32(__ldg(v + (size_t)col * f.l + i)) : 0.f;
      }
    reinterpret_cast<float4 *>(o + (size_t)q * 8)[0] = make_float4(e[0], e[1], e[2], e[3]);
    reinterpret_cast<float4 *>(o + (size_t)q * 8)[1] = make_float4(e[4], e[5], e[6], e[7]);
  }
}

// blockIdx.y 0 .. 3: the maxima below; 4: column pairs of g (into g.cpair); 5: of f.
__global__ void __launch_bounds__(256) mdbf_envmax_kernel(Factor g, Factor f, float *__restrict__ emax,
                                                          float *__restrict__ gpair, float *__restrict__ fpair) {
  qld::pdl_trigger();
  const int p = blockIdx.x, which = blockIdx.y, z = blockIdx.z;
  if (which >= 4) {
    qld::pdl_wait();
    if (which == 4) write_colpairs(g, p, z, gpair);
    else write_colpairs(f, p, z, fpair);
    return;
  }
  const Factor &fc = which < 2 ? g : f;
  const unsigned short *v = reinterpret_cast<const unsigned short *>((which & 1) == 0 ? fc.Lrow[p] : fc.Lcol[p]);
  const int nrow = (which & 1) == 0 ? fc.rows : fc.cols, l = g.l;
  const int per = (nrow + NSL - 1) / NSL, r0 = z * per, r1 = min(nrow, r0 + per);
  __shared__ float red[8][LMAX];
  float mx[LMAX];
#pragma unroll
  for (int i = 0; i < LMAX; ++i) mx[i] = 0.f;
  for (int rr = r0 + (int)threadIdx.x; rr < r1; rr += blockDim.x) {
#pragma unroll
    for (int i = 0; i < LMAX; ++i)
      if (i < l) mx[i] = fmaxf(mx[i], fabsf(qld::f16_to_f32(__ldg(v + (size_t)rr * l + i))));
  }
#pragma unroll
  for (int i = 0; i < LMAX; ++i) {
    float a = mx[i];
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5][i] = a;
  }
  __syncthreads();
  qld::pdl_wait();
  if ((int)threadIdx.x < l) {
    float a = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) a = fmaxf(a, red[w][threadIdx.x]);
    emax[((p * 4 + which) * NSL + z) * LMAX + threadIdx.x] = a;
  }
}

// ------------------------------------------------------------------ activation prep
// The bound (max over paths) of sum_i max|E_w0[.][i]| * max|E_w1[.][i]| from the slice maxima.
__device__ float envelope_bound(const float *__restrict__ emax, int P, int l, int w0) {
  float bound = 0.f;
  for (int p = 0; p < P; ++p) {
    float sp = 0.f;
    for (int i = 0; i < l; ++i) {
      float a = 0.f, b = 0.f;
      for (int z = 0; z < NSL; ++z) {
        a = fmaxf(a, emax[((p * 4 + w0) * NSL + z) * LMAX + i]);
        b = fmaxf(b, emax[((p * 4 + w0 + 1) * NSL + z) * LMAX + i]);
      }
      sp += a * b;
    }
    bound = fmaxf(bound, sp);
  }
  return bound;
}
// Smallest e >= 0 with v 2^-e <= lim (v finite and >= 0).
__device__ int down_exponent(float v, float lim) {
  const float need = v / lim;
  if (!(need > 1.0f)) return 0;
  int ex;
  const float f = frexpf(need, &ex);   // need = f 2^ex, f in [0.5, 1)
  return f == 0.5f ? ex - 1 : ex;
}
// One CTA per token row b: X'[b][j] = fp16(x[b][j] * 2^s_b) for j < m, 0 for m <= j < mp, and
// inv_s[b] = 2^(eg + ef - s_b), with s_b, eg and ef chosen as described at the top of this file.
// CTA 0 also writes the factor scales fsc = {2^-eg, 2^-ef} and clears the split-tile counters of
// both GEMMs.
__global__ void __launch_bounds__(256) mdbf_xprep_kernel(const uint16_t *__restrict__ x, int m, int mp,
                                                         const float *__restrict__ emax, int P, int l,
                                                         uint16_t *__restrict__ xs, float *__restrict__ inv_s,
                                                         float *__restrict__ fsc,
                                                         unsigned *__restrict__ counters, int ncounters, int vec8) {
  qld::pdl_trigger();
  qld::pdl_wait();
  const int b = blockIdx.x, tid = threadIdx.x;
  const uint16_t *xr = x + (size_t)b * m;
  __shared__ float red[8];
  __shared__ int s_exp;
  if (b == 0)
    for (int i = tid; i < ncounters; i += blockDim.x) counters[i] = 0u;
  float mx = 0.f;
  if (vec8) {
    for (int j = tid * 8; j < m; j += blockDim.x * 8) {
      const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + j));
      const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
        mx = fmaxf(mx, fmaxf(fabsf(qld::bf16_to_f32(w[i] & 0xFFFFu)), fabsf(qld::bf16_to_f32(w[i] >> 16))));
    }
  } else {
    for (int j = tid; j < m; j += blockDim.x) mx = fmaxf(mx, fabsf(qld::bf16_to_f32(xr[j])));
  }
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if ((tid & 31) == 0) red[tid >> 5] = mx;
  __syncthreads();
  if (tid == 0) {
    float rmax = 0.f;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) rmax = fmaxf(rmax, red[w]);
    // factor scales: |G| <= beta 2^-eg and |F| <= alpha 2^-ef stay at or below F_BOUND
    const float beta0 = envelope_bound(emax, P, l, 0), alpha = envelope_bound(emax, P, l, 2);
    const int eg = down_exponent(beta0, F_BOUND), ef = down_exponent(alpha, F_BOUND);
    const float beta = ldexpf(beta0, -eg);
    if (b == 0) {
      fsc[0] = ldexpf(1.0f, -eg);
      fsc[1] = ldexpf(1.0f, -ef);
    }
    // e: smallest e >= 0 with m * 2^(1-e) * beta <= T_BOUND
    const int e = down_exponent(2.0f * (float)m * beta, T_BOUND);
    int se = 0;   // scale exponent: max|x'| = rmax 2^se in [2^-e, 2^(1-e))
    if (rmax > 0.f) {
      int ex;
      (void)frexpf(rmax, &ex);   // rmax in [2^(ex-1), 2^ex)
      se = 1 - ex - e;
    }
    se = max(-126, min(127, se));
    s_exp = se;
    inv_s[b] = ldexpf(1.0f, eg + ef - se);
  }
  __syncthreads();
  const float s = ldexpf(1.0f, s_exp);
  uint16_t *xo = xs + (size_t)b * mp;
  if (vec8) {
    for (int j = tid * 8; j < mp; j += blockDim.x * 8) {
      uint32_t o[4] = {0u, 0u, 0u, 0u};
      if (j < m) {
        const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr + j));
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          o[i] = pack_f16x2(qld::bf16_to_f32(w[i] & 0xFFFFu) * s, qld::bf16_to_f32(w[i] >> 16) * s);
      }
      *reinterpret_cast<uint4 *>(xo + j) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  } else {
    for (int j = tid; j < mp; j += blockDim.x) xo[j] = j < m ? f16_rn(qld::bf16_to_f32(xr[j]) * s) : (uint16_t)0;
  }
}

// ------------------------------------------------------------------ output stores
// NV consecutive accumulator values of one output row, starting at column col0.
//   G stage (FST false): T' in fp16, unscaled; Nout is a multiple of 64, so a span is either
//   wholly inside or wholly past it, and T' rows are 16-byte aligned.
//   F stage: y in bf16 (round to nearest even) or fp32, each value times the row's inverse scale
//   rs (a power of two, so the product is exact); spans past n or rows that are not vector-aligned
//   are stored element by element.
template <bool FST, int NV>
__device__ __forceinline__ void put_span(void *out, int ldo, bool ovec, int ydt, int row, int col0, int Nout,
                                         const float (&v)[NV], float rs) {
  static_assert(NV % 4 == 0, "spans of 4");
  if (!FST) {
    if (col0 >= Nout) return;
    uint16_t *o = static_cast<uint16_t *>(out) + (size_t)row * ldo + col0;
#pragma unroll
    for (int i = 0; i < NV / 4; ++i)
      *reinterpret_cast<uint2 *>(o + 4 * i) = make_uint2(pack_f16x2(v[4 * i], v[4 * i + 1]), pack_f16x2(v[4 * i + 2], v[4 * i + 3]));
    return;
  }
  const bool whole = ovec && col0 + NV <= Nout;
  if (ydt == QL_OUT_F32) {
    float *o = static_cast<float *>(out) + (size_t)row * ldo + col0;
    if (whole) {
#pragma unroll
      for (int i = 0; i < NV / 4; ++i)
        *reinterpret_cast<float4 *>(o + 4 * i) = make_float4(v[4 * i] * rs, v[4 * i + 1] * rs, v[4 * i + 2] * rs, v[4 * i + 3] * rs);
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if (col0 + i < Nout) o[i] = v[i] * rs;
    }
  } else {
    uint16_t *o = static_cast<uint16_t *>(out) + (size_t)row * ldo + col0;
    if (whole) {
#pragma unroll
      for (int i = 0; i < NV / 4; ++i) {
        const uint32_t lo = uint32_t(qld::f32_to_bf16_rn(v[4 * i] * rs)) | (uint32_t(qld::f32_to_bf16_rn(v[4 * i + 1] * rs)) << 16);
        const uint32_t hi = uint32_t(qld::f32_to_bf16_rn(v[4 * i + 2] * rs)) | (uint32_t(qld::f32_to_bf16_rn(v[4 * i + 3] * rs)) << 16);
        *reinterpret_cast<uint2 *>(o + 4 * i) = make_uint2(lo, hi);
      }
    } else {
#pragma unroll
      for (int i = 0; i < NV; ++i)
        if (col0 + i < Nout) o[i] = qld::f32_to_bf16_rn(v[i] * rs);
    }
  }
}

// ------------------------------------------------------------------ the GEMM
// C[M][Nout] = A[M][K] D[Nout][K]^T with A an fp16 array read by tensor copies (map_a) and D the
// factor operand decoded on the fly.  FST false: D = [G_1; ..; G_P] (N = P seg), C = T' in fp16.
// FST true: D = [F_1 .. F_P] (K = P seg), C = y scaled by row_scale.  LK: envelope terms
// covered (l <= LK).  LK = 4: packed fp32 FMAs, four terms per element pair; LK = 8, 16, 32: warp
// MMAs in LC chunks of 16 terms.
template <bool FST, int LK, int LC = (LK + 15) / 16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    mdbf_gemm_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ Factor fac,
                     const __grid_constant__ CUtensorMap map_out, int tstore,
                     void *__restrict__ out, int ldo, int ovec, int ydt, const float *__restrict__ row_scale, int M,
                     int Nout, int nkb, float *__restrict__ part_ws, unsigned *__restrict__ part_cnt, int full,
                     int parts, int nfast) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(smem_raw));
  const uint32_t sbase = (raw + 1023u) & ~1023u;
  const Bars bar(sbase + OFF_BAR);
  const uint32_t tmem_slot = sbase + OFF_TMEM;
  const uint32_t rank = sm100::cluster_ctarank();        // 0: the even CTA, which issues the MMAs
  const bool lead = rank == 0;
  const Waiter wt{tmem_slot + 4, sm100::mapa_shared(tmem_slot + 4, rank ^ 1u)};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const int mt = (M + PM - 1) / PM, nt = (Nout + BN - 1) / BN, ntiles = mt * nt;
  const int nitems = full + (ntiles - full) * parts;
  bool ok = true;

  if (threadIdx.x == 0) {
    for (int s = 0; s < SA; ++s) {
      sm100::mbar_init(bar.full_a + 8 * s, 1);
      sm100::mbar_init(bar.empty_a + 8 * s, 1);
    }
    for (int s = 0; s < SB; ++s) {
      sm100::mbar_init(bar.dec_done + 8 * s, NDEC);
      sm100::mbar_init(bar.peer_b + 8 * s, 1);
      sm100::mbar_init(bar.empty_b + 8 * s, 1);
    }
    sm100::mbar_init(bar.acc_full, 1);
    sm100::mbar_init(bar.acc_empty, 2 * NDEC);
    sm100::mbar_init(bar.split_done, NDEC);
    sm100::mbar_init(bar.split_go, 1);
    sm100::mbar_init(bar.stg_full, NDEC);
    sm100::mbar_init(bar.stg_free, 1);
    sts32(tmem_slot + 4, 0);
    sm100::fence_barrier_init();
    sm100::prefetch_tensormap(&map_a);
    if (tstore) sm100::prefetch_tensormap(&map_out);
  }
  if (warp == 1) {
    __syncwarp();
    sm100::tmem_alloc_pair(tmem_slot, 512);
    sm100::tmem_relinquish_pair();
  }
  sm100::tc_fence_before();
  sm100::cluster_sync();   // both CTAs' barriers initialised and tensor memory allocated
  sm100::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(smem_raw + (tmem_slot - raw));
  // the factor operand comes from weights (its decoders may start at once, except that l <= 4
  // reads column pairs from the workspace); A is read and C written only after the preceding
  // kernel in the stream has completed
  qld::pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ A producer (tensor copies)
    if (lane == 0) {
      qld::pdl_wait();
      const uint32_t lead_full_a = sm100::mapa_shared(bar.full_a, 0);
      int it = 0;
      for (int wi = pair; wi < nitems && ok; wi += npairs) {
        const Item w = item_of(wi, full, parts, nkb);
        int mi, ni;
        tile_mn(w.tile, mt, nt, nfast, mi, ni);
        const int m0 = mi * PM + (int)rank * BM;
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int s = it % SA;
          if (it >= SA && !wt.wait(bar.empty_a + 8 * s, ((it / SA) & 1) ^ 1, true)) {
            ok = false;
            break;
          }
          if (lead) sm100::mbar_arrive_expect_tx(bar.full_a + 8 * s, 2 * A_BYTES);
          sm100::tma_load_2d_pair(sbase + OFF_A + s * A_BYTES, &map_a, kb * BK, m0, lead_full_a + 8 * s);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ pair MMA issuer (even CTA)
    if (lead && lane == 0) {
      int it = 0, tl = 0;
      for (int wi = pair; wi < nitems && ok; wi += npairs, ++tl) {
        const Item w = item_of(wi, full, parts, nkb);
        if (tl > 0 && !wt.wait(bar.acc_empty, (tl - 1) & 1, true)) { ok = false; break; }
        sm100::tc_fence_after();
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int sa = it % SA, sb = it % SB;
          if (!wt.wait(bar.full_a + 8 * sa, (it / SA) & 1, true) ||
              !wt.wait(bar.dec_done + 8 * sb, (it / SB) & 1, false) ||
              !wt.wait(bar.peer_b + 8 * sb, (it / SB) & 1, true)) {
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
              sm100::mma_f16kind_pair(tmem + h * BN, adesc, bdesc, IDESC, (kb > w.kb0 || kk > 0) ? 1u : 0u);
            }
          }
          sm100::mma_commit_pair(bar.empty_a + 8 * sa, PAIR);
          sm100::mma_commit_pair(bar.empty_b + 8 * sb, PAIR);
        }
        if (!ok) break;
        sm100::mma_commit_pair(bar.acc_full, PAIR);
      }
    } else if (!lead && lane == 0) {
      // ---------------------------------------------------------- forwarder (odd CTA)
      // relays each decoded block of this CTA to the even CTA's MMA thread: one cluster-scope
      // release per block instead of one per decoder warp
      const uint32_t lead_peer_b = sm100::mapa_shared(bar.peer_b, 0);
      int it = 0;
      for (int wi = pair; wi < nitems && ok; wi += npairs) {
        const Item w = item_of(wi, full, parts, nkb);
        for (int kb = w.kb0; kb < w.kb1; ++kb, ++it) {
          const int sb = it % SB;
          if (!wt.wait(bar.dec_done + 8 * sb, (it / SB) & 1, false)) {
            ok = false;
            break;
          }
          sm100::mbar_arrive_cluster(lead_peer_b + 8 * sb);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ decoders, then epilogue
    // Decoder warp dw rebuilds rows [16 rg, 16 rg + 16) x columns [32 hh, 32 hh + 32) of this
    // CTA's 128 x 64 operand block per K block: four m16n8k16 envelope MMAs (one per 8 columns,
    // one per 16 envelope terms), then per element pair a sign flip and one 32-bit shared store
    // in the 128-byte-swizzled K-major layout.  Lane (g, t) = (lane / 4, lane % 4) owns rows g and
    // g + 8 of the group and columns 8 jj + 2t, 8 jj + 2t + 1.  The sign words and column
    // envelopes of the next K block are loaded while this one is decoded; pointers advance by a
    // fixed stride per block, and only a block that reaches past the last column tests columns.
    const int dw = warp - 2;            // decoder index 0 .. NDEC-1
    const int q = warp & 3;             // tensor-memory lane quarter this warp may read
    const int ch = dw >> 2;             // which quarter of the 256 accumulator columns it drains
    const int rg = dw & 7, hh = dw >> 3;
    const int g = lane >> 2, t = lane & 3;
    const uint32_t st_off = (uint32_t)(2 * rg) * 1024u + (uint32_t)g * 128u + 4u * (uint32_t)t;
    const uint32_t xsw = (uint32_t)((4 * hh) ^ g);
    const uint32_t lead_acc_empty = sm100::mapa_shared(bar.acc_empty, 0);
    const int kbp = fac.seg / BK;                      // K blocks per path (F stage)
    const int l = fac.l, cols = fac.cols;
    const bool lvec = fac.l_vec2 != 0;
    // The factor scale (and for l <= 4 the fp32 column pairs) is workspace written by this call's
    // first kernels, not weights, so the decoders wait for the preceding kernel (and with it for
    // every earlier one) first.
    qld::pdl_wait();
    const float fsc = __ldcg(fac.scale);
    const size_t lblk = (size_t)BK * l;                // column-envelope elements per K block
    const int l8 = 8 * l;
    // this lane's envelope terms: 16c + 2t, +1 (k0) and 16c + 2t + 8, +1 (k1) of chunk c
    bool k0v[LC], k1v[LC];
#pragma unroll
    for (int c = 0; c < LC; ++c) {
      k0v[c] = 16 * c + 2 * t < l;
      k1v[c] = LK > 8 && 16 * c + 2 * t + 8 < l;
    }
    int it = 0, tl = 0, ns = 0, ep = 0;
    for (int wi = pair; wi < nitems && ok; wi += npairs, ++tl) {
      const Item w = item_of(wi, full, parts, nkb);
      int mi, ni;
      tile_mn(w.tile, mt, nt, nfast, mi, ni);
      const int m0 = mi * PM + (int)rank * BM, n0 = ni * BN;
      if constexpr (LK == 4) {
        // l <= 4, packed fp32 FMAs: warp dw rebuilds rows [32 rq, 32 rq + 32) x columns
        // [16 cq, 16 cq + 16) of this CTA's 128 x 64 block (rq = dw % 4, cq = dw / 4); lane (g, t)
        // owns rows g + 8k (k < 4) and the column pairs 8u + 2t, +1 (u < 2).  Four rows per lane
        // halve the column-envelope reads per element against two; each 32-bit store of a warp
        // covers 8 rows of one swizzle atom, conflict-free.
        const int rq = dw & 3, cq = dw >> 2;
        const int grow = n0 + BNH * (int)rank + 32 * rq;
        const int prow = FST ? 0 : grow / fac.seg;
        const bool pv = FST || prow < fac.P;
        const int r0 = (FST ? grow : grow - prow * fac.seg) + g;   // path-local row of k = 0
        bool vr[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) vr[k] = pv && r0 + 8 * k < fac.rows;
        // row envelope terms of row pairs (k = 2j, 2j + 1), [j][term]: each packed FMA computes
        // one column for two rows
        uint64_t rr2[2][4];
        auto load_rows = [&](int p) {
          const uint16_t *L = fac.Lrow[p];
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int ka = 2 * j, kb2 = 2 * j + 1;
              // times the factor's power-of-two scale: exact, and exact through every FMA below
              const float a = (vr[ka] && i < l) ? qld::f16_to_f32(L[(size_t)(r0 + 8 * ka) * l + i]) * fsc : 0.f;
              const float b = (vr[kb2] && i < l) ? qld::f16_to_f32(L[(size_t)(r0 + 8 * kb2) * l + i]) * fsc : 0.f;
              rr2[j][i] = f2(a, b);
            }
        };
        int fp = FST ? w.kb0 / kbp : prow, fkl = FST ? w.kb0 - fp * kbp : w.kb0;
        const uint8_t *sg = nullptr;   // sign row r0 of path fp from the warp's 16 columns; row k at + 8k ld
        size_t sld8 = 0;
        const float *cpp = nullptr;    // fp32 pair block of the warp's 16 columns
        auto set_path = [&](int p) {
          const size_t ld = fac.ld[p];
          sg = fac.S[p] + (size_t)r0 * ld + 2 * cq;
          sld8 = 8 * ld;
          cpp = fac.cpair + ((size_t)p * (fac.cpad / 2) + 8 * cq) * 8;
        };
        if (pv) set_path(fp);
        struct Pre {
          uint32_t w[4];   // 16 sign bits per row
          uint2 c;         // this lane's 8 bytes of the warp's 256-byte pair block
        };
        auto fetch = [&](Pre &o) {
          // A 16-bit sign load that starts inside the row's ceil(cols / 8) bytes ends inside its
          // stride (rows 4-byte aligned, strides multiples of 4, checked by the ABI); bits past
          // the last column meet a zero column envelope.  Pair blocks are zero-padded to cpad.
          const int kc = fkl * BK + 16 * cq;
          const bool win = pv && kc < cols;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            o.w[k] = (vr[k] && win) ? (uint32_t)__ldg(reinterpret_cast<const unsigned short *>(sg + k * sld8 + 8 * fkl)) : 0u;
          o.c = pv ? __ldg(reinterpret_cast<const uint2 *>(cpp + (size_t)fkl * (BK / 2) * 8) + lane) : make_uint2(0u, 0u);
          if (FST && ++fkl == kbp) {
            fkl = 0;
            if (++fp < fac.P) set_path(fp);
          } else if (!FST) {
            ++fkl;
          }
        };
        int pc = FST ? w.kb0 / kbp : prow, kcl = FST ? w.kb0 - pc * kbp : 0;
        if (FST || pv) {
          load_rows(pc);
        } else {
#pragma unroll
          for (int j = 0; j < 2; ++j)
#pragma unroll
            for (int i = 0; i < 4; ++i) rr2[j][i] = f2(0.f, 0.f);
        }
        // per-lane store offsets in a B stage: row 32 rq + g + 8k is row g of atom 4 rq + k
        const uint32_t so0 = (uint32_t)(4 * rq) * 1024u + (uint32_t)g * 128u + 4u * (uint32_t)t;
        const uint32_t sx0 = ((uint32_t)(2 * cq) ^ (uint32_t)g) << 4, sx1 = ((uint32_t)(2 * cq + 1) ^ (uint32_t)g) << 4;
        const uint32_t cwb = sbase + OFF_CW + dw * 2 * CW_BYTES;   // this warp's two pair blocks
        Pre p0, p1;
        fetch(p0);
        sts64(cwb + (it & 1) * CW_BYTES + 8 * lane, p0.c.x, p0.c.y);
        __syncwarp();
        // two block buffers, the loop unrolled by two so that each keeps fixed registers; the
        // loads for block kb + 1 are issued before block kb is decoded
        auto step = [&](int kb, const Pre &cur, Pre &next) -> bool {
          if (kb + 1 < w.kb1) fetch(next);
          if (FST && kcl == kbp) {
            kcl = 0;
            load_rows(++pc);
          }
          const int sb = it % SB;
          if (it >= SB && !wt.wait(bar.empty_b + 8 * sb, ((it / SB) & 1) ^ 1, true)) return false;
          const uint32_t base = sbase + OFF_B + sb * B_BYTES + so0;
          const uint32_t cb = cwb + (it & 1) * CW_BYTES;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            // pair block 4u + t: {C[c][i], C[c + 1][i]} for terms i = 0, 1 then 2, 3
            const uint4 c0 = lds128(cb + (4 * u + t) * 32), c1 = lds128(cb + (4 * u + t) * 32 + 16);
            const uint32_t cv[2][4] = {{c0.x, c0.z, c1.x, c1.z}, {c0.y, c0.w, c1.y, c1.w}};   // [column][term]
            float e[2][4];   // [column][row k]
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                // envelope terms in ascending order, one rounding per term, as the oracle sums them
                uint64_t acc = f2(0.f, 0.f);
#pragma unroll
                for (int i = 0; i < 4; ++i) acc = ffma2(rr2[j][i], f2u(cv[h][i], cv[h][i]), acc);
                f2split(acc, e[h][2 * j], e[h][2 * j + 1]);
              }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint32_t sgn = cur.w[k] >> (2 * t);
              const uint32_t flip = u ? sign_flip<1>(sgn) : sign_flip<0>(sgn);
              sts32(base + (uint32_t)k * 1024u + (u ? sx1 : sx0), pack_f16x2(e[0][k], e[1][k]) ^ flip);
            }
          }
          // handed to this CTA's MMA side through a CTA-scope barrier: the even CTA's MMA thread
          // waits on it directly, the odd CTA's forwarder relays it at cluster scope
          sm100::fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) sm100::mbar_arrive(bar.dec_done + 8 * sb);
          if (FST) ++kcl;
          if (kb + 1 < w.kb1) {
            // every lane has read this block's pairs (the arrive above follows a __syncwarp)
            sts64(cwb + ((it + 1) & 1) * CW_BYTES + 8 * lane, next.c.x, next.c.y);
            __syncwarp();
          }
          ++it;
          return true;
        };
        for (int kb = w.kb0; kb < w.kb1;) {
          if (!step(kb, p0, p1)) { ok = false; break; }
          if (++kb >= w.kb1) break;
          if (!step(kb, p1, p0)) { ok = false; break; }
          ++kb;
        }
      } else {
      // first operand row of this warp's group (along the GEMM's N); in the G stage it fixes the
      // path, in the F stage the path follows the K block
      const int grow = n0 + BNH * (int)rank + 16 * rg;
      const int prow = FST ? 0 : grow / fac.seg;
      const bool pv = FST || prow < fac.P;
      const int ra = (FST ? grow : grow - prow * fac.seg) + g, rb = ra + 8;
      const bool va = pv && ra < fac.rows, vb = pv && rb < fac.rows;
      uint32_t afr[LC][4];
      uint64_t ra2[4], rb2[4];   // l <= 4: row envelope terms as {v, v} pairs
      auto load_rows = [&](int p) {
        const uint16_t *L = fac.Lrow[p];
        if constexpr (LK == 4) {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float a = (va && i < l) ? qld::f16_to_f32(L[(size_t)ra * l + i]) : 0.f;
            const float b = (vb && i < l) ? qld::f16_to_f32(L[(size_t)rb * l + i]) : 0.f;
            ra2[i] = f2(a, a);
            rb2[i] = f2(b, b);
          }
        } else {
#pragma unroll
          for (int c = 0; c < LC; ++c) {
            const int k0 = 16 * c + 2 * t;
            afr[c][0] = va ? env_pair(L + (size_t)ra * l, l, k0, lvec) : 0u;
            afr[c][1] = vb ? env_pair(L + (size_t)rb * l, l, k0, lvec) : 0u;
            afr[c][2] = (LK > 8 && va) ? env_pair(L + (size_t)ra * l, l, k0 + 8, lvec) : 0u;
            afr[c][3] = (LK > 8 && vb) ? env_pair(L + (size_t)rb * l, l, k0 + 8, lvec) : 0u;
          }
        }
      };
      // fetch state: path fp and path-local K block fkl of the next block to load
      int fp = FST ? w.kb0 / kbp : prow;
      int fkl = FST ? w.kb0 - fp * kbp : w.kb0;
      const uint8_t *sga = nullptr, *sgb = nullptr;   // sign rows ra, rb from the warp's column half
      const uint16_t *lcp = nullptr;                 // column envelope of column 32 hh + g
      const float *cpp = nullptr;                    // l <= 4: fp32 pair block of columns 32 hh + 2t, +1
      auto set_path = [&](int p) {
        const size_t ld = fac.ld[p];
        sga = fac.S[p] + (size_t)ra * ld + 4 * hh;
        sgb = sga + 8 * ld;
        lcp = fac.Lcol[p] + (size_t)(32 * hh + g) * l;
        cpp = fac.cpair + ((size_t)p * (fac.cpad / 2) + 16 * hh) * 8;
      };
      if (pv) set_path(fp);
      struct PreM {
        uint32_t wa, wb, b[4][LC][2];
      };
      struct PreF {
        uint32_t wa, wb;
        uint4 c;   // this lane's 16 bytes of the warp's 512-byte column-pair block
      };
      using Pre = std::conditional_t<LK == 4, PreF, PreM>;
      auto fetch = [&](Pre &o) {
        const int kc = fkl * BK + 32 * hh;           // first column of the warp's half in the path
        // The 32 sign bits of the half's columns: rows are 4-byte aligned with strides that are
        // multiples of 4 (checked by the ABI), so a word that starts inside the row's
        // ceil(cols / 8) bytes ends inside its stride; bits past the last column are padding and
        // meet a zero column envelope.
        const bool win = pv && kc < cols;            // the half starts inside the row
        const int lim = win ? cols - kc - g : 0;     // column 8 jj + g of the half is in range iff 8 jj < lim
        o.wa = (va && win) ? __ldg(reinterpret_cast<const unsigned int *>(sga + 8 * fkl)) : 0u;
        o.wb = (vb && win) ? __ldg(reinterpret_cast<const unsigned int *>(sgb + 8 * fkl)) : 0u;
        if constexpr (LK == 4) {
          // the warp's 16 column pairs (padded with zeros to cpad columns: no column test), 16
          // bytes per lane; parked in shared memory before the block is decoded
          o.c = pv ? __ldg(reinterpret_cast<const uint4 *>(cpp + (size_t)fkl * (BK / 2) * 8) + lane)
                   : make_uint4(0u, 0u, 0u, 0u);
        } else {
        const uint16_t *cp = lcp + (size_t)fkl * lblk;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const bool okc = 8 * jj < lim;
#pragma unroll
          for (int c = 0; c < LC; ++c) {
            if (lvec) {
              const unsigned int *v = reinterpret_cast<const unsigned int *>(cp + jj * l8 + 16 * c + 2 * t);
              o.b[jj][c][0] = (okc && k0v[c]) ? __ldg(v) : 0u;
              o.b[jj][c][1] = (okc && k1v[c]) ? __ldg(v + 4) : 0u;
            } else {
              o.b[jj][c][0] = okc ? env_pair(cp + jj * l8, l, 16 * c + 2 * t, false) : 0u;
              o.b[jj][c][1] = (LK > 8 && okc) ? env_pair(cp + jj * l8, l, 16 * c + 2 * t + 8, false) : 0u;
            }
          }
        }
        }
        if (FST && ++fkl == kbp) {
          fkl = 0;
          if (++fp < fac.P) set_path(fp);
        } else if (!FST) {
          ++fkl;
        }
      };
      // path and path-local K block of the block being decoded (F stage)
      int pc = FST ? w.kb0 / kbp : prow, kcl = FST ? w.kb0 - pc * kbp : 0;
      if (FST || pv) {
        load_rows(pc);
      } else {
#pragma unroll
        for (int c = 0; c < LC; ++c) afr[c][0] = afr[c][1] = afr[c][2] = afr[c][3] = 0u;
      }
      // Block buffers in a ring, the loop unrolled by the ring's length so that each buffer keeps
      // fixed registers.  l <= 4 (three buffers): the loads for block kb + 2 are issued while block
      // kb is decoded and first needed two blocks later, so the decoders are not paced by the
      // memory latency.  The larger warp-MMA fragments fit two buffers (one block ahead).
      constexpr int RING = LK == 4 ? 3 : 2;
      Pre p0, p1, p2;
      fetch(p0);
      if (RING == 3 && w.kb0 + 1 < w.kb1) fetch(p1);
      const uint32_t cwb = sbase + OFF_CW + dw * 2 * CW_BYTES;   // this warp's two column-pair blocks
      if constexpr (LK == 4) {
        sts128(cwb + (it & 1) * CW_BYTES + 16 * lane, p0.c);
        __syncwarp();
      }
      auto step = [&](int kb, const Pre &cur, const Pre &next, Pre &fill) -> bool {
        if (kb + RING - 1 < w.kb1) fetch(fill);
        if (FST && kcl == kbp) {
          kcl = 0;
          load_rows(++pc);
        }
        const int sb = it % SB;
        if (it >= SB && !wt.wait(bar.empty_b + 8 * sb, ((it / SB) & 1) ^ 1, true)) return false;
        const uint32_t base = sbase + OFF_B + sb * B_BYTES + st_off;
        const uint32_t ea = cur.wa >> (2 * t), eb = cur.wb >> (2 * t);
        const uint32_t ea2 = ea >> 16, eb2 = eb >> 16;
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          float d[4] = {0.f, 0.f, 0.f, 0.f};
          if constexpr (LK == 4) {
            // envelope terms in ascending order, one rounding per term, as the oracle sums them
            const uint32_t cb = cwb + (it & 1) * CW_BYTES + (4 * jj + t) * 32;
            const uint4 c0 = lds128(cb), c1 = lds128(cb + 16);
            const uint64_t b[4] = {f2u(c0.x, c0.y), f2u(c0.z, c0.w), f2u(c1.x, c1.y), f2u(c1.z, c1.w)};
            uint64_t ea = f2(0.f, 0.f), eb = f2(0.f, 0.f);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              ea = ffma2(ra2[i], b[i], ea);
              eb = ffma2(rb2[i], b[i], eb);
            }
            f2split(ea, d[0], d[1]);
            f2split(eb, d[2], d[3]);
          } else {
#pragma unroll
            for (int c = 0; c < LC; ++c) mma_f16_16816(d, afr[c], cur.b[jj][c][0], cur.b[jj][c][1]);
#pragma unroll
            for (int c = 0; c < 4; ++c) d[c] *= fsc;
          }
          const uint32_t sa_ = jj < 2 ? ea : ea2, sb_ = jj < 2 ? eb : eb2;
          const uint32_t fa = (jj & 1) ? sign_flip<1>(sa_) : sign_flip<0>(sa_);
          const uint32_t fb = (jj & 1) ? sign_flip<1>(sb_) : sign_flip<0>(sb_);
          const uint32_t off = (xsw ^ (uint32_t)jj) << 4;
          sts32(base + off, pack_f16x2(d[0], d[1]) ^ fa);
          sts32(base + 1024u + off, pack_f16x2(d[2], d[3]) ^ fb);
        }
        // the block is handed to this CTA's MMA side through a CTA-scope barrier: the even CTA's
        // MMA thread waits on it directly, the odd CTA's forwarder relays it at cluster scope
        sm100::fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(bar.dec_done + 8 * sb);
        if (FST) ++kcl;
        if constexpr (LK == 4) {
          if (kb + 1 < w.kb1) {
            // every lane has read this block's pairs (the arrive above follows a __syncwarp)
            sts128(cwb + ((it + 1) & 1) * CW_BYTES + 16 * lane, next.c);
            __syncwarp();
          }
        }
        ++it;
        return true;
      };
      if constexpr (RING == 3) {
        for (int kb = w.kb0; kb < w.kb1;) {
          if (!step(kb, p0, p1, p2)) { ok = false; break; }
          if (++kb >= w.kb1) break;
          if (!step(kb, p1, p2, p0)) { ok = false; break; }
          if (++kb >= w.kb1) break;
          if (!step(kb, p2, p0, p1)) { ok = false; break; }
          ++kb;
        }
      } else {
        for (int kb = w.kb0; kb < w.kb1;) {
          if (!step(kb, p0, p1, p1)) { ok = false; break; }
          if (++kb >= w.kb1) break;
          if (!step(kb, p1, p0, p0)) { ok = false; break; }
          ++kb;
        }
      }
      }
      if (!ok) break;
      // epilogue: this warp drains lanes [32q, 32q+32) of both 128-row accumulators
      if (!wt.wait(bar.acc_full, tl & 1, true)) { ok = false; break; }
      qld::pdl_wait();
      sm100::tc_fence_after();
      const bool split = w.part >= 0;
      if (!split && tstore) {
        // Whole tile through tensor stores: once acc_full has fired every block of the tile has
        // been consumed, so the B ring (4 x 16 KB) is free to stage the output.
        if (!staged_tile_store(tmem, sbase + OFF_B, &map_out, FST ? (ydt == QL_OUT_F32 ? OUT_F32 : OUT_BF16) : OUT_F16,
                               FST ? row_scale : nullptr, m0, n0, M, Nout, q, ch, dw, lane, wt, bar.stg_full,
                               bar.stg_free, ep)) {
          ok = false;
          break;
        }
        sm100::tc_fence_before();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive_cluster(lead_acc_empty);
        continue;
      }
      // fp32 partials of a split tile: [tile - full][part][rank][BM rows][BN columns]

      float *const slot =
          split ? part_ws + ((size_t)((w.tile - full) * parts + w.part) * 2 + rank) * (size_t)(BM * BN) : nullptr;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        const int lr = h * 128 + 32 * q + lane, row = m0 + lr;
        const float rs = (FST && !split && row < M) ? __ldg(row_scale + row) : 1.f;
#pragma unroll 1
        for (int c = ch * (BN / 32) / (NDEC / 4); c < (ch + 1) * (BN / 32) / (NDEC / 4); ++c) {
          uint32_t v[32];
          sm100::tmem_ld_32x32b_x32(tmem + ((uint32_t)(32 * q) << 16) + h * BN + c * 32, v);
          sm100::tmem_wait_ld();
          if (split) {
            float4 *dst = reinterpret_cast<float4 *>(slot + (size_t)lr * BN + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                   __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
          } else if (row < M) {
            float f[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) f[i] = __uint_as_float(v[i]);
            put_span<FST, 32>(out, ldo, ovec != 0, ydt, row, n0 + c * 32, Nout, f, rs);
          }
        }
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive_cluster(lead_acc_empty);
      if (split) {
        // The last of the tile's parts to finish (per CTA half) sums all parts in part order.
        __threadfence();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(bar.split_done);
        const uint32_t last_flag = tmem_slot + 8;
        if (dw == 0) {
          if (!wt.wait(bar.split_done, ns & 1, false)) { ok = false; break; }
          if (lane == 0) {
            __threadfence();
            unsigned *cnt = part_cnt + (w.tile - full) * 2 + rank;
            const bool last = atomicAdd(cnt, 1u) == (unsigned)parts - 1;
            if (last) {
              atomicExch(cnt, 0u);
              __threadfence();
            }
            sts32(last_flag, last ? 1u : 0u);
            sm100::mbar_arrive(bar.split_go);
          }
          __syncwarp();
        }
        if (!wt.wait(bar.split_go, ns & 1, false)) { ok = false; break; }
        ++ns;
        if (lds32(last_flag)) {
          const float *p0 = part_ws + ((size_t)(w.tile - full) * parts * 2 + rank) * (size_t)(BM * BN);
          const size_t pstride = (size_t)2 * BM * BN;
          for (int e = (dw * 32 + lane) * 4; e < BM * BN; e += NDEC * 32 * 4) {
            const int row = m0 + e / BN, col = n0 + e % BN;
            float4 a = __ldcg(reinterpret_cast<const float4 *>(p0 + e));
            for (int pq = 1; pq < parts; ++pq) {
              const float4 b = __ldcg(reinterpret_cast<const float4 *>(p0 + pq * pstride + e));
              a.x += b.x; a.y += b.y; a.z += b.z; a.w += b.w;
            }
            if (row >= M) continue;
            const float f[4] = {a.x, a.y, a.z, a.w};
            put_span<FST, 4>(out, ldo, ovec != 0, ydt, row, col, Nout, f, FST ? __ldg(row_scale + row) : 1.f);
          }
        }
      }
    }
  }

  if (warp == 2 && lane == 0) sm100::bulk_wait0();   // the tensor stores issued by decoder 0
  if (!ok) atomicExch(&g_mgemm_timeout, 1);
  // neither CTA leaves while its peer may still arrive on its barriers, read its shared memory
  // through a pair MMA or write its tensor memory
  sm100::tc_fence_before();
  sm100::cluster_sync();
  if (warp == 1) {
    __syncwarp();
    sm100::tc_fence_after();
    sm100::tmem_dealloc_pair(tmem, 512);
  }
}

// ---------------------------------------------------------------------------- host side
// Opts each GEMM instance into its dynamic shared memory (once per device).
template <bool FST, int LK>
cudaError_t smem_attr_one() {
  return ql::set_max_smem(mdbf_gemm_kernel<FST, LK>, SMEM_BYTES);
}
cudaError_t smem_attr() {
  cudaError_t e = cudaSuccess;
  for (cudaError_t r : {smem_attr_one<false, 4>(), smem_attr_one<true, 4>(), smem_attr_one<false, 8>(),
                        smem_attr_one<true, 8>(), smem_attr_one<false, 16>(), smem_attr_one<true, 16>(),
                        smem_attr_one<false, 32>(), smem_attr_one<true, 32>()})
    if (e == cudaSuccess) e = r;
  return e;
}

// CTA pairs that can be resident at once on the current device (cached per device); 0 when no
// device is usable (the split of the last wave is then not planned).
int resident_pairs() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    (void)cudaGetLastError();
    return 0;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (smem_attr() == cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(2 * (ql::sm_count() / 2));
      cfg.blockDim = dim3(THREADS);
      cfg.dynamicSmemBytes = SMEM_BYTES;
      if (cudaOccupancyMaxActiveClusters(&n, mdbf_gemm_kernel<false, 8>, &cfg) != cudaSuccess || n <= 0) n = 0;
    }
    if (n <= 0) {
      (void)cudaGetLastError();
      n = ql::sm_count() / 2;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

inline size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

// Workspace of one call: envelope maxima, the fp32 column pairs of both factors (l <= 4),
// inverse row scales, the two factor scales, X' [B][mp] fp16, T' [B][P seg] fp16, the split
// counters of both GEMMs, and one region of fp32 partials that GEMM 1 and then GEMM 2 use in turn.
struct GemmWs {
  int mp, seg;
  SplitPlan g1, g2;
  size_t emax, gpair, fpair, inv_s, fsc, xs, ts, cnt, part, total;
};
GemmWs gemm_ws(int P, int n, int m, int r, int B, int pairs) {
  GemmWs L;
  L.mp = (m + BK - 1) / BK * BK;
  L.seg = (r + BK - 1) / BK * BK;
  const int mt = (B + PM - 1) / PM;
  const size_t tile_bytes = (size_t)2 * BM * BN * sizeof(float);
  L.g1 = split_plan(mt * ((P * L.seg + BN - 1) / BN), L.mp / BK, pairs, tile_bytes);
  L.g2 = split_plan(mt * ((n + BN - 1) / BN), P * L.seg / BK, pairs, tile_bytes);
  L.emax = 0;
  L.gpair = L.emax + align256((size_t)P * 4 * NSL * LMAX * sizeof(float));
  L.fpair = L.gpair + align256((size_t)P * L.mp * 16);
  L.inv_s = L.fpair + align256((size_t)P * L.seg * 16);
  L.fsc = L.inv_s + align256((size_t)B * sizeof(float));
  L.xs = L.fsc + 256;
  L.ts = L.xs + align256((size_t)B * L.mp * 2);
  L.cnt = L.ts + align256((size_t)B * P * L.seg * 2);
  L.part = L.cnt + L.g1.counter_bytes + L.g2.counter_bytes;
  L.total = L.part + std::max(L.g1.partial_bytes, L.g2.partial_bytes);
  return L;
}

Factor make_factor(const mdbf_path *paths, int P, bool f_stage, int n, int m, int r, int l, const GemmWs &L,
                   const char *base) {
  Factor f = {};
  bool l2 = l % 2 == 0;
  for (int p = 0; p < P; ++p) {
    const mdbf_path &q = paths[p];
    f.S[p] = f_stage ? q.S_A : q.S_B;
    f.ld[p] = f_stage ? q.ldSA : q.ldSB;
    f.Lrow[p] = f_stage ? q.A_amp : q.Q_V;
    f.Lcol[p] = f_stage ? q.Q_U : q.B_amp;
    l2 = l2 && ql::aligned(f.Lrow[p], 4) && ql::aligned(f.Lcol[p], 4);
  }
  f.rows = f_stage ? n : r;
  f.cols = f_stage ? r : m;
  f.seg = L.seg;
  f.cpad = f_stage ? L.seg : L.mp;
  f.cpair = reinterpret_cast<const float *>(base + (f_stage ? L.fpair : L.gpair));
  f.scale = reinterpret_cast<const float *>(base + L.fsc) + (f_stage ? 1 : 0);
  f.P = P;
  f.l = l;
  f.l_vec2 = l2 ? 1 : 0;
  return f;
}

// Outputs: T' through tensor stores (mto, always); y through tensor stores when my is valid
// (ystore), else with direct stores.
struct OutMaps {
  CUtensorMap mto, my;
  bool ystore;
};

template <int LK>
void launch_gemms(const CUtensorMap &mx, const CUtensorMap &mt_, const OutMaps &om, const Factor &fg, const Factor &ff,
                  const GemmWs &L, char *base, void *y, int ydt, bool yvec, int B, int P, int n, int resident,
                  cudaStream_t s) {
  float *part = reinterpret_cast<float *>(base + L.part);
  unsigned *cnt1 = reinterpret_cast<unsigned *>(base + L.cnt);
  unsigned *cnt2 = reinterpret_cast<unsigned *>(base + L.cnt + L.g1.counter_bytes);
  const int items1 = L.g1.full + L.g1.leftover * L.g1.parts, items2 = L.g2.full + L.g2.leftover * L.g2.parts;
  // N-fastest tiles when the activations (2 bytes per element) outweigh the sign bits (1/8 byte)
  const int nfast1 = 16.0 * B > (double)P * L.seg ? 1 : 0, nfast2 = 16.0 * B > (double)n ? 1 : 0;
  ql::launch(mdbf_gemm_kernel<false, LK>, 2 * std::min(items1, resident), THREADS, SMEM_BYTES, s, mx, fg, om.mto, 1,
             static_cast<void *>(base + L.ts), P * L.seg, 1, 0, static_cast<const float *>(nullptr), B, P * L.seg,
             L.mp / BK, part, cnt1, L.g1.full, L.g1.parts, nfast1);
  ql::launch(mdbf_gemm_kernel<true, LK>, 2 * std::min(items2, resident), THREADS, SMEM_BYTES, s, mt_, ff, om.my,
             om.ystore ? 1 : 0, y, n,
             yvec ? 1 : 0, ydt, reinterpret_cast<const float *>(base + L.inv_s), B, n, P * L.seg / BK, part, cnt2,
             L.g2.full, L.g2.parts, nfast2);
}

}  // namespace

namespace ql {

size_t mdbf_gemm_workspace_size(int P, int n, int m, int r, int l, int B) {
  if (P <= 0 || n <= 0 || m <= 0 || r <= 0 || l <= 0 || l > LMAX || B <= 0) return 0;
  return gemm_ws(P, n, m, r, B, resident_pairs()).total;
}

ql_status mdbf_gemm_launch(const mdbf_path *paths, int P, int n, int m, int r, int l, const uint16_t *x, void *y,
                           ql_out_dtype ydt, int B, void *ws, cudaStream_t s) {
  if (P > PMAX) return fail(QL_ERR_UNSUPPORTED, "mdbf_linear: P = %d exceeds %d paths", P, PMAX);
  if (l > LMAX) return fail(QL_ERR_UNSUPPORTED, "mdbf_linear: the batched path takes l <= %d (got %d)", LMAX, l);
  EncodeTiledFn enc = encode_tiled_fn();
  if (!enc) return fail(QL_ERR_CUDA, "mdbf_linear: cuTensorMapEncodeTiled is unavailable");
  if (smem_attr() != cudaSuccess) return fail(QL_ERR_CUDA, "mdbf_linear: cannot reserve GEMM shared memory");
  const int resident = std::max(1, resident_pairs());
  const GemmWs L = gemm_ws(P, n, m, r, B, resident);
  char *base = static_cast<char *>(ws);
  CUtensorMap mx, mtm;
  if (!encode_rows_sw128(enc, &mx, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base + L.xs, B, L.mp, L.mp, BM) ||
      !encode_rows_sw128(enc, &mtm, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base + L.ts, B, (uint64_t)P * L.seg,
                         (uint64_t)P * L.seg, BM))
    return fail(QL_ERR_CUDA, "mdbf_linear: cannot encode the activation tensor maps");
  const bool yvec = aligned(y, 16) && (ydt == QL_OUT_F32 ? n % 4 == 0 : n % 8 == 0);
  OutMaps om = {};
  if (!encode_rows_sw128(enc, &om.mto, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, base + L.ts, B, (uint64_t)P * L.seg,
                         (uint64_t)P * L.seg, 128))
    return fail(QL_ERR_CUDA, "mdbf_linear: cannot encode the intermediate's tensor map");
  om.ystore = yvec && encode_rows_sw128(enc, &om.my,
                                        ydt == QL_OUT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                                        y, B, n, n, 128, ydt == QL_OUT_F32 ? 4 : 2);
  const Factor fg = make_factor(paths, P, false, n, m, r, l, L, base);
  const Factor ff = make_factor(paths, P, true, n, m, r, l, L, base);
  float *emax = reinterpret_cast<float *>(base + L.emax);
  launch(mdbf_envmax_kernel, dim3(P, l <= 4 ? 6 : 4, NSL), 256, 0, s, fg, ff, emax,
         reinterpret_cast<float *>(base + L.gpair), reinterpret_cast<float *>(base + L.fpair));
  ql_status st = launch_status("mdbf_linear (envelope maxima)");
  if (st != QL_OK) return st;
  const bool xvec = m % 8 == 0 && aligned(x, 16);
  const int ncnt = (int)((L.g1.counter_bytes + L.g2.counter_bytes) / sizeof(unsigned));
  launch(mdbf_xprep_kernel, B, 256, 0, s, x, m, L.mp, static_cast<const float *>(emax), P, l,
         reinterpret_cast<uint16_t *>(base + L.xs), reinterpret_cast<float *>(base + L.inv_s),
         reinterpret_cast<float *>(base + L.fsc), reinterpret_cast<unsigned *>(base + L.cnt), ncnt, xvec ? 1 : 0);
  st = launch_status("mdbf_linear (activation prep)");
  if (st != QL_OK) return st;
  if (l <= 4)
    launch_gemms<4>(mx, mtm, om, fg, ff, L, base, y, (int)ydt, yvec, B, P, n, resident, s);
  else if (l <= 8)
    launch_gemms<8>(mx, mtm, om, fg, ff, L, base, y, (int)ydt, yvec, B, P, n, resident, s);
  else if (l <= 16)
    launch_gemms<16>(mx, mtm, om, fg, ff, L, base, y, (int)ydt, yvec, B, P, n, resident, s);
  else
    launch_gemms<32>(mx, mtm, om, fg, ff, L, base, y, (int)ydt, yvec, B, P, n, resident, s);
  return launch_status("mdbf_linear (tensor-core GEMMs)");
}

ql_status mdbf_gemm_read_timeout(int *flag) {
  int zero = 0;
  if (cudaMemcpyFromSymbol(flag, g_mgemm_timeout, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_mgemm_timeout, &zero, sizeof(int)) != cudaSuccess)
    return fail(QL_ERR_CUDA, "ql_check: cannot read the device timeout flag");
  return QL_OK;
}

}  // namespace ql
