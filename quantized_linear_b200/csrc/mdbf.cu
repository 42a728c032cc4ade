// MDBF (multi-envelope double binary factorization) layer: forward pass and debug dequantizer.
//
// "MDBF (Multi-Envelope Double Binary Factorization)", section "Algorithm":
//   W ~= sum_p F_p G_p,  F = S_A (.) (A_amp Q_U^T),  G = S_B (.) (Q_V B_amp^T).
// The forward pass never forms W.  Writing the Hadamard products out,
//   (G x)_k = sum_i Q_V[k,i] * sum_j S_B[k,j] * (B_amp[j,i] x_j)
//   (F t)_a = sum_i A_amp[a,i] * sum_k S_A[a,k] * (Q_U[k,i] t_k)
// so each path is two products of a packed +-1 matrix with l*B dense vectors:
//   prologue  z[p][j][b*l+i] = B_amp[j,i] * x[b,j]                (exact in fp32, packed as
//             bf16 high + low MMA fragments, or for the split G stage quantised per
//             128-column group to two signed bytes: "Sign products on the s8 warp MMA")
//   G stage   u = S_B z;   t[k][b] = sum_i Q_V[k,i] u[k][b*l+i];
//             w[p][k][b*l+i] = Q_U[k,i] * t[k][b]                  (epilogue, fused)
//   F stage   v = S_A w;   y[b][a] = sum_p sum_i A_amp[a,i] v[a][b*l+i]   (epilogue, fused;
//             the path sum is taken inside one launch, in p order)
// The sign products run on the warp MMA (see "Sign products on the warp MMA"
// below); column-split partials are summed through shared memory in a fixed
// order, so results are deterministic.  Launches per call: pack z, G stage
// (which also packs w for the F stage), F stage.
#include <algorithm>
#include <mutex>

#include "ql_internal.cuh"
#include "sm100_ptx.cuh"

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

// ------------------------------------------------------------------------------------------
// Sign products on the warp MMA.
//
// OUT[rows][v] = sum_c s[row][c] * VEC[c][v] is an (rows x cols) x (cols x V) product with a +-1
// left operand.  Each sign bit becomes a bf16 +-1 (exact) straight in the A fragment of
// mma.m16n8k16 (bf16 in, fp32 accumulate); the dense right operand VEC (fp32) is split into a
// bf16 high part and a bf16 low part (relative error ~2^-16) and laid out once, in a prologue,
// as ready-made B fragments.  The K ordering inside one 32-column sign word is permuted so that
// the two bits of every A register sit 16 bit positions apart: one shift and one masked XOR
// build a register, i.e. one integer op per sign bit.  Logical K pairs of MMA h (h = 0, 1) map
// to physical columns (c, c + 16) with c = 8h + q (pair 2q, 2q+1) and c = 8h + 4 + q (pair
// 2q+8, 2q+9), q = lane % 4; the B fragments are packed with the same map.
// B fragment columns: n < V hold the high parts of vector n, V <= n < 2V the low parts, the
// rest zero; NB = ceil(2V / 8) MMAs cover them.  Columns past `cols` pack as zero, so the
// padding bits of the last sign word contribute nothing.
// ------------------------------------------------------------------------------------------
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// bf16 pair {+-1 from bit (15 - s) of w, +-1 from bit (31 - s)}: bit 1 -> +1.0, bit 0 -> -1.0
__device__ __forceinline__ uint32_t sign_pair(uint32_t w, int s) {
  return ((w << s) & 0x80008000u) ^ 0xBF80BF80u;
}
// The same with the shift given as the multiplier 2^s: the multiply runs on the FMA pipe, which
// the sign products leave idle, instead of the integer pipe that the mask-and-flip also needs.
__device__ __forceinline__ uint32_t sign_pair_mul(uint32_t w, uint32_t pow2s) {
  uint32_t t;
  asm("mul.lo.u32 %0, %1, %2;" : "=r"(t) : "r"(w), "r"(pow2s));
  return (t & 0x80008000u) ^ 0xBF80BF80u;
}

__device__ __forceinline__ uint32_t bf16_rn_bits(float f) { return qld::f32_to_bf16_rn(f); }

// value of B-fragment column n at physical column c: high / low bf16 part of VEC[c][v]
template <typename Get>
__device__ __forceinline__ uint32_t frag_value(Get get, int c, int n, int cols, int V) {
  if (c >= cols || n >= 2 * V) return 0u;
  const float v = get(c, n < V ? n : n - V);
  const uint32_t hi = bf16_rn_bits(v);
  if (n < V) return hi;
  return bf16_rn_bits(v - __uint_as_float(hi << 16));
}

// packed B fragments of one 32-column word, VB[qw][nb][lane] as uint4 = {MMA 0 regs, MMA 1 regs}
template <typename Get>
__device__ __forceinline__ uint4 pack_fragment(Get get, int qw, int nb, int lane, int cols, int V) {
  const int g = lane >> 2, q = lane & 3, n = 8 * nb + g;
  uint32_t o[4];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int ca = 32 * qw + 8 * h + q, cb = ca + 4;
    o[2 * h] = frag_value(get, ca, n, cols, V) | (frag_value(get, ca + 16, n, cols, V) << 16);
    o[2 * h + 1] = frag_value(get, cb, n, cols, V) | (frag_value(get, cb + 16, n, cols, V) << 16);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// G-stage B fragments from z[j][b*l+i] = B_amp[j][i] * x[b][j] (exact in fp32).  One thread per
// fragment register set (word qw, n block nb, lane): its 8 columns' B_amp and x values are all
// loaded before any is used, and the weights (B_amp) are pulled toward L2 before the wait on
// the preceding kernel.
__global__ void mdbf_pack_z_kernel(Paths ps, const uint16_t *__restrict__ x, uint4 *__restrict__ out, int m, int l,
                                   int B, int NB, unsigned *__restrict__ cnt, int ncnt) {
  const int p = blockIdx.y;
  const int QW = (m + 31) / 32, V = l * B;
  const int64_t total = (int64_t)QW * NB * 32;
  const uint16_t *bm = ps.Bm[p];
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x)
    if ((e & 31) == 0) {
      const int64_t c0 = std::min<int64_t>(32 * ((e >> 5) / NB), m - 1);   // first column of the word, in bounds
      asm volatile("prefetch.global.L2 [%0];" ::"l"(bm + c0 * l));
    }
  qld::pdl_trigger();
  qld::pdl_wait();
  // the arrival counts of the split G stage that follows (the launch before this one has completed)
  if (p == 0)
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < ncnt; e += gridDim.x * blockDim.x) cnt[e] = 0u;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
    const int lane = int(e & 31), g = lane >> 2, q = lane & 3;
    const int64_t f = e >> 5;
    const int qw = int(f / NB), nb = int(f % NB), nn = 8 * nb + g;
    // the 8 physical columns of this lane's registers (see "Sign products on the warp MMA")
    int col[8];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int ca = 32 * qw + 8 * h + q, cb = ca + 4;
      col[4 * h] = ca; col[4 * h + 1] = ca + 16; col[4 * h + 2] = cb; col[4 * h + 3] = cb + 16;
    }
    const bool live = nn < 2 * V;
    const int v = nn < V ? nn : nn - V, b = live ? v / l : 0, i = live ? v - b * l : 0;
    float z[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const bool in = live && col[t] < m;
      const int c = in ? col[t] : 0;
      const float bv = qld::f16_to_f32(bm[(int64_t)c * l + i]);
      const float xv = qld::bf16_to_f32(x[(int64_t)b * m + c]);
      z[t] = in ? bv * xv : 0.f;
    }
    uint32_t o[8];
#pragma unroll
    for (int t = 0; t < 8; ++t) {
      const uint32_t hi = bf16_rn_bits(z[t]);
      o[t] = nn < V ? hi : bf16_rn_bits(z[t] - __uint_as_float(hi << 16));
      if (!live) o[t] = 0u;
    }
    out[(int64_t)p * total + e] = make_uint4(o[0] | (o[1] << 16), o[2] | (o[3] << 16), o[4] | (o[5] << 16), o[6] | (o[7] << 16));
  }
}

// ------------------------------------------------------------------------------------------
// Sign products on the s8 warp MMA (the split G stage, NB = 1: l * B <= 4 vectors).
//
// z is quantised once, by the pack kernel below, per group of 4 words (128 columns) and vector v:
//   q[j][v] = rint(z[j][v] / s[v]),  s[v] the smallest power of two >= max_j |z[j][v]| / Z8_QMAX
// over the group's columns (so z / s and s q are exact scalings),
// and q = 256 h + lo is split into two signed bytes (lo in [-128, 127]; |q| <= Z8_QMAX keeps h in
// [-128, 127]).  The sign operand enters as 0/1 bytes b = (sign + 1) / 2, so with the group's byte
// sums H = sum_j h_j and L = sum_j lo_j,
//   sum_j sign_j q_j = 256 (2 sum_j b_j h_j - H) + (2 sum_j b_j lo_j - L),
// exact integers; each group's two int32 sums are scaled into fp32 once.  One quantised z is
// within 2^-16 of its group's largest |z|, i.e. a relative error of ~1e-4 at most on u = S_B z
// where the bf16 high + low split of the other G kernels gives ~1e-6; both are far inside the
// forward pass's tolerance.  mma.m16n8k32 (s8 in, s32 accumulate) takes one 32-column word per
// instruction, with the K order inside a word permuted so that an A register is one shift and one
// mask of a sign word: byte e of register a0 (a2) of lane q holds physical column q + 8e
// (q + 4 + 8e), i.e. logical k = 4q + e (16 + 4q + e) is physical column q + 8e (q + 4 + 8e).  B
// column n (n < V: the high bytes of vector n; V <= n < 2V: the low bytes of vector n - V; else
// zero) is packed with the same map: register b0 (b1) of lane (n, q) holds the bytes of columns
// q + 8e (q + 4 + 8e), e = 0 .. 3, of the word.  Columns past m pack as zero.
// ------------------------------------------------------------------------------------------
constexpr int Z8_QMAX = 32639;   // 32767 - 128
// per path and 4-word group: the scales and byte sums of its vectors (zero past V)
struct __align__(16) Z8Meta {
  float s[4];
  int hs[4];
  int ls[4];
};
__device__ __forceinline__ void mma_s8_16832(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                             uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One CTA per (path, group), warp u on word u of the group: z of the group's 128 columns, its
// scales and byte sums (meta) and its 4 words of B fragments (out[p][qw][lane] = {b0, b1}).  The
// B_amp values (weights) are loaded before the wait on the preceding kernel.  A group holding a
// non-finite z gets a NaN scale, so the outputs it reaches are NaN.  Also clears the split G
// stage's arrival counts.
__global__ void __launch_bounds__(128)
    mdbf_pack_z8_kernel(Paths ps, const uint16_t *__restrict__ x, uint2 *__restrict__ out, Z8Meta *__restrict__ meta,
                        int m, int l, int B, unsigned *__restrict__ cnt, int ncnt) {
  __shared__ int8_t qs[8][128];     // [B column n][column of the group]
  __shared__ float wmax[4][4];      // [warp][vector]
  __shared__ int wsum[4][2][4];     // [warp][high, low][vector]
  __shared__ int nonfinite;
  const int p = blockIdx.y, grp = blockIdx.x, u = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int QW = (m + 31) / 32, G4 = (QW + 3) / 4, V = l * B;
  const int j = 128 * grp + 32 * u + lane;
  const bool in = j < m;
  const uint16_t *bm = ps.Bm[p];
  float bv[4];
#pragma unroll
  for (int v = 0; v < 4; ++v) bv[v] = (v < V && in) ? qld::f16_to_f32(bm[(int64_t)j * l + (v % l)]) : 0.f;
  if (threadIdx.x == 0) nonfinite = 0;
  qld::pdl_trigger();
  qld::pdl_wait();
  if (p == 0)
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < ncnt; e += gridDim.x * blockDim.x) cnt[e] = 0u;
  float z[4];
  bool finite = true;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    z[v] = (v < V && in) ? bv[v] * qld::bf16_to_f32(x[(int64_t)(v / l) * m + j]) : 0.f;
    finite = finite && isfinite(z[v]);
  }
#pragma unroll
  for (int v = 0; v < 4; ++v) {   // |z| as bits: non-negative floats order as unsigned integers
    const unsigned mx = __reduce_max_sync(0xffffffffu, __float_as_uint(fabsf(z[v])));
    if (lane == 0) wmax[u][v] = __uint_as_float(mx);
  }
  __syncthreads();   // also orders nonfinite = 0 before the flags below
  if (!finite) nonfinite = 1;
  int hq[4], lq[4];
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const float mx = fmaxf(fmaxf(wmax[0][v], wmax[1][v]), fmaxf(wmax[2][v], wmax[3][v]));
    // s = 2^e, the smallest power of two with max|z| / s <= Z8_QMAX: z / s is exact, and so is s q
    int ex;
    const float fr = frexpf(mx, &ex);   // mx = fr 2^ex, fr in [0.5, 1) (0 for mx = 0)
    const int e = ex - 15 + (fr * 32768.f > (float)Z8_QMAX ? 1 : 0);
    const int qv = isfinite(mx) ? min(Z8_QMAX, max(-Z8_QMAX, __float2int_rn(ldexpf(z[v], -e)))) : 0;
    lq[v] = ((qv + 128) & 255) - 128;
    hq[v] = (qv - lq[v]) >> 8;
    const int hs = __reduce_add_sync(0xffffffffu, hq[v]), ls = __reduce_add_sync(0xffffffffu, lq[v]);
    if (lane == 0) {
      wsum[u][0][v] = hs;
      wsum[u][1][v] = ls;
    }
    if (threadIdx.x == 0) meta[(size_t)p * G4 + grp].s[v] = ldexpf(1.f, e);   // NaN scales below if not finite
  }
#pragma unroll
  for (int n = 0; n < 8; ++n) {
    int val = 0;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      if (v < V && n == v) val = hq[v];
      if (v < V && n == V + v) val = lq[v];
    }
    qs[n][32 * u + lane] = (int8_t)val;
  }
  __syncthreads();
  if (threadIdx.x < 4) {
    const int v = threadIdx.x;
    Z8Meta *const mt = meta + (size_t)p * G4 + grp;
    const bool live = v < V;
    mt->hs[v] = live ? wsum[0][0][v] + wsum[1][0][v] + wsum[2][0][v] + wsum[3][0][v] : 0;
    mt->ls[v] = live ? wsum[0][1][v] + wsum[1][1][v] + wsum[2][1][v] + wsum[3][1][v] : 0;
    if (!live) mt->s[v] = 0.f;
    else if (nonfinite) mt->s[v] = __int_as_float(0x7fc00000);
  }
  const int qw = 4 * grp + u;
  if (qw < QW) {
    const int g = lane >> 2, q = lane & 3;
    uint32_t b0 = 0, b1 = 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      b0 |= (uint32_t)(uint8_t)qs[g][32 * u + q + 8 * e] << (8 * e);
      b1 |= (uint32_t)(uint8_t)qs[g][32 * u + q + 4 + 8 * e] << (8 * e);
    }
    out[((size_t)p * QW + qw) * 32 + lane] = make_uint2(b0, b1);
  }
}

// Pulls rows [row0, row0 + nrows) of a sign matrix toward L2.  Sign bits are weights, so this
// may run before the wait on the preceding kernel; every address stays inside its row.
__device__ __forceinline__ void prefetch_sign_rows(const uint8_t *S, size_t ld, int row0, int nrows, int rows) {
  const int lines = (int)((ld + 127) / 128);
  for (int e = threadIdx.x; e < nrows * lines; e += blockDim.x) {
    const int rr = e / lines, c = e - rr * lines;
    if (row0 + rr < rows) asm volatile("prefetch.global.L2 [%0];" ::"l"(S + (size_t)(row0 + rr) * ld + 128 * c));
  }
}

constexpr int SP_WARPS = 8;
constexpr int SP_U = 4;   // sign words per load group (one 16-byte load per row when rows are 16-byte aligned)

// Accumulates one warp's share of words [w0, w1) into acc for RT row tiles of 16 rows at row0.
// w0 is a multiple of SP_U.  VEC16: sign rows are 16-byte aligned, so SP_U words load at once.
template <int NB, int RT, bool VEC16>
__device__ __forceinline__ void sign_mma_rows(const uint8_t *__restrict__ S, size_t ld, int rows, int row0,
                                              const uint4 *__restrict__ vb, int w0, int w1,
                                              float (&acc)[RT][NB][4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const uint32_t *rp[RT][2];
  bool ok[RT][2];
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int row = row0 + 16 * rt + g + 8 * hh;
      ok[rt][hh] = row < rows;
      rp[rt][hh] = reinterpret_cast<const uint32_t *>(S + (size_t)(ok[rt][hh] ? row : 0) * ld);
    }
  for (int qw0 = w0; qw0 < w1; qw0 += SP_U) {
    uint32_t sw[SP_U][RT][2];
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        if constexpr (VEC16) {
          const uint4 v = ok[rt][hh] ? __ldg(reinterpret_cast<const uint4 *>(rp[rt][hh] + qw0)) : make_uint4(0, 0, 0, 0);
          sw[0][rt][hh] = v.x; sw[1][rt][hh] = v.y; sw[2][rt][hh] = v.z; sw[3][rt][hh] = v.w;
        } else {
#pragma unroll
          for (int u = 0; u < SP_U; ++u)
            sw[u][rt][hh] = (ok[rt][hh] && qw0 + u < w1) ? __ldg(rp[rt][hh] + qw0 + u) : 0u;
        }
      }
    // fragments: all SP_U words up front when they are few registers, else one word at a time
    constexpr int UB = NB <= 2 ? SP_U : 1;
    uint4 bf[UB][NB];
    auto load_frags = [&](int slot, int qw) {
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
        bf[slot][nb] = (qw < w1) ? __ldg(vb + ((size_t)qw * NB + nb) * 32 + lane) : make_uint4(0, 0, 0, 0);
    };
    if constexpr (UB == SP_U) {
#pragma unroll
      for (int u = 0; u < SP_U; ++u) load_frags(u, qw0 + u);
    }
#pragma unroll
    for (int u = 0; u < SP_U; ++u) {
      const int slot = UB == SP_U ? u : 0;
      if constexpr (UB != SP_U) load_frags(0, qw0 + u);
#pragma unroll
      for (int rt = 0; rt < RT; ++rt) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int sa = 15 - 8 * h - q, sb = 11 - 8 * h - q;
          const uint32_t a0 = sign_pair(sw[u][rt][0], sa), a1 = sign_pair(sw[u][rt][1], sa);
          const uint32_t a2 = sign_pair(sw[u][rt][0], sb), a3 = sign_pair(sw[u][rt][1], sb);
#pragma unroll
          for (int nb = 0; nb < NB; ++nb) {
            const uint32_t b0 = h ? bf[slot][nb].z : bf[slot][nb].x, b1 = h ? bf[slot][nb].w : bf[slot][nb].y;
            mma16816(acc[rt][nb], a0, a1, a2, a3, b0, b1);
          }
        }
      }
    }
  }
}

__device__ __forceinline__ void warp_words(int QW, int warp, int &w0, int &w1) {
  const int groups = (QW + SP_U - 1) / SP_U;
  w0 = SP_U * (int)((int64_t)groups * warp / SP_WARPS);
  w1 = min(QW, SP_U * (int)((int64_t)groups * (warp + 1) / SP_WARPS));
}

// Sums the warps' fragments into D[rt][16][8 NB] (fp32, shared), fixed order.
template <int NB, int RT>
__device__ __forceinline__ void reduce_fragments(float *red, float *D, const float (&acc)[RT][NB][4]) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int PER = RT * NB * 4 * 32;
#pragma unroll
  for (int rt = 0; rt < RT; ++rt)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int i = 0; i < 4; ++i) red[warp * PER + ((rt * NB + nb) * 4 + i) * 32 + lane] = acc[rt][nb][i];
  __syncthreads();
  for (int e = threadIdx.x; e < PER; e += blockDim.x) {
    float s = red[e];
    for (int w = 1; w < SP_WARPS; ++w) s += red[w * PER + e];
    const int ln = e & 31, i = (e >> 5) & 3, nb = (e >> 7) % NB, rt = (e >> 7) / NB;
    const int row = (ln >> 2) + 8 * (i >> 1), n = 8 * nb + 2 * (ln & 3) + (i & 1);
    D[(rt * 16 + row) * (8 * NB) + n] = s;
  }
  __syncthreads();
}

// G stage over 32 rows k (one word of the F stage):
//   t[k][b] = sum_i Q_V[k][i] u[k][b*l+i],  w[k][b*l+i] = Q_U[k][i] t[k][b],
// and w is written straight out as the F stage's packed B fragments for that word.
template <int NB, bool VEC16>
__global__ void __launch_bounds__(SP_WARPS * 32) mdbf_g_mma_kernel(Paths ps, const uint4 *__restrict__ zpk,
                                                                     uint4 *__restrict__ wpk, int m, int r, int l,
                                                                     int B) {
  extern __shared__ float sm[];
  float *red = sm, *D = sm + SP_WARPS * 2 * NB * 128, *Ws = D + 32 * 8 * NB;
  const int p = blockIdx.y, warp = threadIdx.x >> 5;
  const int QW = (m + 31) / 32, V = l * B;
  const int row0 = blockIdx.x * 32;
  prefetch_sign_rows(ps.SB[p], ps.ldSB[p], row0, 32, r);
  qld::pdl_trigger();
  qld::pdl_wait();
  float acc[2][NB][4];
#pragma unroll
  for (int rt = 0; rt < 2; ++rt)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[rt][nb][i] = 0.f;
  int w0, w1;
  warp_words(QW, warp, w0, w1);
  sign_mma_rows<NB, 2, VEC16>(ps.SB[p], ps.ldSB[p], r, row0, zpk + (size_t)p * QW * NB * 32, w0, w1, acc);
  reduce_fragments<NB, 2>(red, D, acc);
  for (int e = threadIdx.x; e < 32 * B; e += blockDim.x) {
    const int rr = e / B, b = e - rr * B, k = row0 + rr;
    float *wo = Ws + rr * V + b * l;
    if (k >= r) {
      for (int i = 0; i < l; ++i) wo[i] = 0.f;
      continue;
    }
    const float *Dr = D + rr * (8 * NB);
    const uint16_t *qv = ps.QV[p] + (int64_t)k * l, *qu = ps.QU[p] + (int64_t)k * l;
    float t = 0.f;
    for (int i = 0; i < l; ++i) t = fmaf(qld::f16_to_f32(qv[i]), Dr[b * l + i] + Dr[V + b * l + i], t);
    for (int i = 0; i < l; ++i) wo[i] = qld::f16_to_f32(qu[i]) * t;
  }
  __syncthreads();
  const int qw = blockIdx.x, QWr = (r + 31) / 32;
  auto get = [&](int c, int v) { return Ws[(c - 32 * qw) * V + v]; };
  for (int e = threadIdx.x; e < NB * 32; e += blockDim.x)
    wpk[((size_t)p * QWr + qw) * NB * 32 + e] = pack_fragment(get, qw, e >> 5, e & 31, r, V);
}

// G stage as above, with each warp streaming its word groups through a private STG-stage ring in
// shared memory filled by cp.async: per group of SP_U words, lane (g, q) copies 16 bytes of sign
// row g + 8q (the 32 rows of the block) and its own 16-byte fragment register sets, STG - 1 groups
// ahead of the one being multiplied.  The first groups' signs are requested before the wait on
// the preceding kernel.  Needs 16-byte aligned sign rows.  Four stages fit two CTAs per SM, three
// stages three (NB = 1); the host takes three when the blocks would otherwise need a second round.
constexpr int GR_STAGES = 4;

// set when a bounded wait of an MDBF kernel runs out; read and cleared by ql_check()
__device__ int g_mdbf_timeout = 0;

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ uint32_t lds32s(uint32_t a) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];" : "=r"(v) : "r"(a));
  return v;
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async4(uint32_t dst, const void *src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <int NB>
__host__ __device__ constexpr int g_ring_stage_bytes() { return 32 * 16 + SP_U * NB * 32 * 16; }

template <int NB, int STG>
__global__ void __launch_bounds__(SP_WARPS * 32) mdbf_g_tile_kernel(Paths ps, const uint4 *__restrict__ zpk,
                                                                      uint4 *__restrict__ wpk, int m, int r, int l,
                                                                      int B) {
  constexpr int STAGE = g_ring_stage_bytes<NB>();
  extern __shared__ __align__(128) unsigned char gsm[];
  const uint32_t sbase = static_cast<uint32_t>(__cvta_generic_to_shared(gsm));
  float *red = reinterpret_cast<float *>(gsm + SP_WARPS * STG * STAGE), *D = red + SP_WARPS * 2 * NB * 128,
        *Ws = D + 32 * 8 * NB;
  const int p = blockIdx.y, warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int QW = (m + 31) / 32, V = l * B;
  const int row0 = blockIdx.x * 32;
  const size_t ld = ps.ldSB[p];
  const uint32_t ring = sbase + warp * STG * STAGE;
  const uint4 *vb = zpk + (size_t)p * QW * NB * 32;
  // this lane's sign row (rows past r repeat the last row; their results are dropped)
  const uint8_t *srow = ps.SB[p] + (size_t)min(row0 + g + 8 * q, r - 1) * ld;
  int w0, w1;
  warp_words(QW, warp, w0, w1);
  const int ngroups = (w1 - w0 + SP_U - 1) / SP_U;
  auto issue_signs = [&](int grp) {
    const uint32_t st = ring + (grp % STG) * STAGE;
    cp_async16(st + (g + 8 * q) * 16, srow + 4 * (w0 + SP_U * grp));   // 16 bytes: SP_U sign words
  };
  auto issue_frags = [&](int grp) {
    const uint32_t st = ring + (grp % STG) * STAGE + 32 * 16;
#pragma unroll
    for (int u = 0; u < SP_U; ++u) {
      const int qw = min(w0 + SP_U * grp + u, QW - 1);   // words past the range are loaded but multiply zero-padding... see below
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) cp_async16(st + ((u * NB + nb) * 32 + lane) * 16, vb + ((size_t)qw * NB + nb) * 32 + lane);
    }
  };
  for (int grp = 0; grp < STG - 1 && grp < ngroups; ++grp) issue_signs(grp);
  // The epilogue's Q_V and Q_U rows (weights) travel to shared memory with the first copy group
  // when both blocks start on 4-byte boundaries and hold whole 4-byte words; else the epilogue
  // reads them from global memory.
  const int rows_b = min(32, r - row0);
  const uint16_t *const qv0 = ps.QV[p] + (size_t)row0 * l, *const qu0 = ps.QU[p] + (size_t)row0 * l;
  const bool q_smem = ((reinterpret_cast<uintptr_t>(qv0) | reinterpret_cast<uintptr_t>(qu0)) & 3) == 0 &&
                      (rows_b * l) % 2 == 0;
  uint16_t *const qs = reinterpret_cast<uint16_t *>(Ws + 32 * V);   // [2][32 l]: Q_V rows, Q_U rows
  if (q_smem) {
    const uint32_t qsa = static_cast<uint32_t>(__cvta_generic_to_shared(qs));
    const int words = rows_b * l / 2;
    for (int e = threadIdx.x; e < 2 * words; e += blockDim.x) {
      const int which = e / words, j = e - which * words;
      cp_async4(qsa + 4 * (which * 16 * l + j), (which ? qu0 : qv0) + 2 * j);
    }
  }
  qld::pdl_trigger();
  qld::pdl_wait();
  for (int grp = 0; grp < STG - 1; ++grp) {
    if (grp < ngroups) issue_frags(grp);
    cp_async_commit();
  }

  float acc[2][NB][4];
#pragma unroll
  for (int rt = 0; rt < 2; ++rt)
#pragma unroll
    for (int nb = 0; nb < NB; ++nb)
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[rt][nb][i] = 0.f;
  for (int grp = 0; grp < ngroups; ++grp) {
    cp_async_wait<STG - 2>();
    __syncwarp();   // sign rows were copied by other lanes of the warp
    const uint32_t st = ring + (grp % STG) * STAGE;
    uint32_t sw[SP_U][2][2];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const uint4 v = lds128(st + (16 * rt + g + 8 * hh) * 16);
        sw[0][rt][hh] = v.x; sw[1][rt][hh] = v.y; sw[2][rt][hh] = v.z; sw[3][rt][hh] = v.w;
      }
    uint4 bf[SP_U][NB];
#pragma unroll
    for (int u = 0; u < SP_U; ++u)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb) bf[u][nb] = lds128(st + 32 * 16 + ((u * NB + nb) * 32 + lane) * 16);
    __syncwarp();   // every lane has read this stage before it is refilled
    const int nxt = grp + STG - 1;
    if (nxt < ngroups) {
      issue_signs(nxt);
      issue_frags(nxt);
    }
    cp_async_commit();
    const int valid = min(SP_U, w1 - (w0 + SP_U * grp));   // words of this group inside the warp's range
#pragma unroll
    for (int u = 0; u < SP_U; ++u) {
      if (u >= valid) break;
#pragma unroll
      for (int rt = 0; rt < 2; ++rt) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t ma = 1u << (15 - 8 * h - q), mb = 1u << (11 - 8 * h - q);
          const uint32_t a0 = sign_pair_mul(sw[u][rt][0], ma), a1 = sign_pair_mul(sw[u][rt][1], ma);
          const uint32_t a2 = sign_pair_mul(sw[u][rt][0], mb), a3 = sign_pair_mul(sw[u][rt][1], mb);
#pragma unroll
          for (int nb = 0; nb < NB; ++nb)
            mma16816(acc[rt][nb], a0, a1, a2, a3, h ? bf[u][nb].z : bf[u][nb].x, h ? bf[u][nb].w : bf[u][nb].y);
        }
      }
    }
  }
  cp_async_wait<0>();
  reduce_fragments<NB, 2>(red, D, acc);
  for (int e = threadIdx.x; e < 32 * B; e += blockDim.x) {
    const int rr = e / B, b = e - rr * B, k = row0 + rr;
    float *wo = Ws + rr * V + b * l;
    if (k >= r) {
      for (int i = 0; i < l; ++i) wo[i] = 0.f;
      continue;
    }
    const float *Dr = D + rr * (8 * NB);
    const uint16_t *qv = q_smem ? qs + rr * l : ps.QV[p] + (int64_t)k * l;
    const uint16_t *qu = q_smem ? qs + 32 * l + rr * l : ps.QU[p] + (int64_t)k * l;
    float t = 0.f;
    for (int i = 0; i < l; ++i) t = fmaf(qld::f16_to_f32(qv[i]), Dr[b * l + i] + Dr[V + b * l + i], t);
    for (int i = 0; i < l; ++i) wo[i] = qld::f16_to_f32(qu[i]) * t;
  }
  __syncthreads();
  const int qw = blockIdx.x, QWr = (r + 31) / 32;
  auto get = [&](int c, int v) { return Ws[(c - 32 * qw) * V + v]; };
  for (int e = threadIdx.x; e < NB * 32; e += blockDim.x)
    wpk[((size_t)p * QWr + qw) * NB * 32 + e] = pack_fragment(get, qw, e >> 5, e & 31, r, V);
}

__device__ __forceinline__ uint2 lds64(uint32_t a) {
  uint2 v;
  asm volatile("ld.shared.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "r"(a));
  return v;
}

// fp32 scale and byte-sum correction of B column n for one group, from its Z8Meta at `mt`
// (shared memory): high bytes weigh 256 s, low bytes s; columns past 2V are zero.
__device__ __forceinline__ void z8_column(uint32_t mt, int n, int V, float &fac, int &corr) {
  fac = 0.f;
  corr = 0;
  if (n < 2 * V) {
    const int v = n < V ? n : n - V;
    fac = __uint_as_float(lds32s(mt + 4 * v)) * (n < V ? 256.f : 1.f);
    corr = (int)lds32s(mt + (n < V ? 16 : 32) + 4 * v);
  }
}


// F stage: y[b][a] = sum_p sum_i A_amp[a][i] v_p[a][b*l+i], paths summed in p order
template <int NB, int RT, bool VEC16>
__global__ void __launch_bounds__(SP_WARPS * 32) mdbf_f_mma_kernel(Paths ps, int P, const uint4 *__restrict__ wpk,
                                                                     void *__restrict__ y, int ydt, int n, int r, int l,
                                                                     int B) {
  extern __shared__ float sm[];
  float *red = sm, *D = sm + SP_WARPS * RT * NB * 128, *yacc = D + RT * 16 * 8 * NB;
  const int warp = threadIdx.x >> 5;
  const int QW = (r + 31) / 32, V = l * B;
  const int row0 = blockIdx.x * 16 * RT;
  prefetch_sign_rows(ps.SA[0], ps.ldSA[0], row0, 16 * RT, n);
  qld::pdl_trigger();
  qld::pdl_wait();
  for (int e = threadIdx.x; e < 16 * RT * B; e += blockDim.x) yacc[e] = 0.f;
  int w0, w1;
  warp_words(QW, warp, w0, w1);
  for (int p = 0; p < P; ++p) {
    float acc[RT][NB][4];
#pragma unroll
    for (int rt = 0; rt < RT; ++rt)
#pragma unroll
      for (int nb = 0; nb < NB; ++nb)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[rt][nb][i] = 0.f;
    sign_mma_rows<NB, RT, VEC16>(ps.SA[p], ps.ldSA[p], n, row0, wpk + (size_t)p * QW * NB * 32, w0, w1, acc);
    reduce_fragments<NB, RT>(red, D, acc);
    for (int e = threadIdx.x; e < 16 * RT * B; e += blockDim.x) {
      const int rr = e / B, b = e - rr * B, a = row0 + rr;
      if (a >= n) continue;
      const float *Dr = D + rr * (8 * NB);
      const uint16_t *am = ps.A[p] + (int64_t)a * l;
      float s = yacc[e];
      for (int i = 0; i < l; ++i) s = fmaf(qld::f16_to_f32(am[i]), Dr[b * l + i] + Dr[V + b * l + i], s);
      yacc[e] = s;
    }
    __syncthreads();
  }
  for (int e = threadIdx.x; e < 16 * RT * B; e += blockDim.x) {
    const int rr = e / B, b = e - rr * B, a = row0 + rr;
    if (a >= n) continue;
    if (ydt == QL_OUT_F32)
      static_cast<float *>(y)[(int64_t)b * n + a] = yacc[e];
    else
      static_cast<uint16_t *>(y)[(int64_t)b * n + a] = qld::f32_to_bf16_rn(yacc[e]);
  }
}

// ---------------------------------------------------------------- F stage, staged tiles ------
// One CTA per 128 rows of S_A.  Each path's 128-row sign block is contiguous in memory (rows are
// ldSA apart), so one bulk copy brings it into shared memory, issued before the wait on the G
// stage (signs are weights); the path's packed w fragments follow after the wait.  Two stages
// let path p + 1 (or p + 2) arrive while path p is multiplied.  Warp w owns rows
// [16 (w % 8), +16) of the block over the K-word group w / 8 (KG groups of consecutive words);
// the groups' partial sums are added in group order.  Paths are summed in p order.
constexpr int FT_TILES = 8;   // 16-row tiles of a full-size (128-row) F block
constexpr long long FT_WAIT_BUDGET = 4000000000LL;   // clock cycles (~2 s)


struct FTileLayout {
  uint32_t sign_bytes, frag_bytes, stage_bytes, nstage, off_bars, off_d, off_y, off_a, a_stride, total;
};
constexpr uint32_t FT_A_STAGE_MAX = 16 * 1024;   // shared-memory bytes for the CTA's A_amp rows
__host__ __device__ inline FTileLayout ftile_layout(size_t ld_max, int r, int NB, int B, int P, int l, int nstage, int KG,
                                                    int tiles) {
  FTileLayout L;
  L.sign_bytes = (uint32_t)((16 * tiles * ld_max + 127) / 128 * 128);
  L.frag_bytes = (uint32_t)((r + 31) / 32) * NB * 32 * 16;
  L.stage_bytes = L.sign_bytes + L.frag_bytes;
  L.nstage = (uint32_t)nstage;
  L.off_bars = L.nstage * L.stage_bytes;
  L.off_d = L.off_bars + 128;                                   // per-warp D scratch [16][8 NB] fp32
  L.off_y = L.off_d + KG * tiles * 16 * 8 * NB * 4;              // per-row-tile y accumulators [16][B] fp32
  L.off_a = L.off_y + tiles * 16 * B * 4;                        // A_amp rows of every path [P][16 tiles][l]
  const uint32_t a_bytes = (uint32_t)(P * 16 * tiles * l * 2 + 15) / 16 * 16;
  L.a_stride = a_bytes <= FT_A_STAGE_MAX ? (uint32_t)(16 * tiles * l) : 0u;   // 0: read A_amp from global
  L.total = L.off_a + (L.a_stride ? a_bytes : 0u);
  return L;
}


template <int NB, int KG, int RT, int NRG>
__global__ void __launch_bounds__(NRG * 32 * KG)
    mdbf_f_tile_kernel(Paths ps, int P, const uint4 *__restrict__ wpk, void *__restrict__ y, int ydt, int n, int r,
                       int l, int B, FTileLayout L) {
  constexpr int TILES = RT * NRG;      // 16-row tiles per CTA: NRG row groups of RT tiles
  extern __shared__ __align__(128) unsigned char fsm[];
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(fsm));
  const int QW = (r + 31) / 32, V = l * B;
  const int row0 = blockIdx.x * 16 * TILES, rows = min(16 * TILES, n - row0);
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int rg = wid % NRG, kg = wid / NRG;   // row group, K-word group
  const int qw0 = kg * QW / KG, qw1 = (kg + 1) * QW / KG;
  const int rbase = 16 * RT * rg;             // first row of this warp's tiles within the block
  const uint32_t bars = base + L.off_bars;
  float *const dsc_all = reinterpret_cast<float *>(fsm + L.off_d);    // [KG][8 tiles][16][8 NB]
  float *const yacc_all = reinterpret_cast<float *>(fsm + L.off_y);   // [8 tiles][16][B]
  auto dsc_of = [&](int k, int tile) { return dsc_all + ((size_t)k * TILES + tile) * 16 * 8 * NB; };
  if (kg == 0)
    for (int e = lane; e < RT * 16 * B; e += 32) yacc_all[RT * rg * 16 * B + e] = 0.f;

  // stage s receives path p's signs (weights) and w fragments (made by the G stage)
  int issued[2] = {0, 0};   // copies issued per stage (thread 0), for the drain after a timeout
  auto issue = [&](int p, int st, bool after_wait) {
    const uint32_t bar = bars + 8 * st, dst = base + st * L.stage_bytes;
    const uint32_t sbytes = (uint32_t)(rows * ps.ldSA[p]);
    if (!after_wait) {
      ++issued[st];
      sm100::mbar_arrive_expect_tx(bar, sbytes + L.frag_bytes);
      sm100::bulk_g2s(dst, ps.SA[p] + (size_t)row0 * ps.ldSA[p], sbytes, bar);
    } else {
      sm100::bulk_g2s(dst + L.sign_bytes, wpk + (size_t)p * QW * NB * 32, L.frag_bytes, bar);
    }
  };
  if (threadIdx.x == 0) {
    for (int st = 0; st < (int)L.nstage; ++st) sm100::mbar_init(bars + 8 * st, 1);
    sm100::fence_barrier_init();
    for (int p = 0; p < P && p < (int)L.nstage; ++p) issue(p, p, false);
    qld::pdl_trigger();
    qld::pdl_wait();
    for (int p = 0; p < P && p < (int)L.nstage; ++p) issue(p, p, true);
  }
  // the epilogue's A_amp rows (weights) to shared memory while the G stage is still running; warp
  // 0 (whose thread 0 has already waited for the G stage above) takes no share
  uint16_t *const a_sm = reinterpret_cast<uint16_t *>(fsm + L.off_a);
  if (L.a_stride && threadIdx.x >= 32)
    for (int e = threadIdx.x - 32; e < P * rows * l; e += blockDim.x - 32) {
      const int pp = e / (rows * l), j = e - pp * rows * l;
      a_sm[pp * L.a_stride + j] = ps.A[pp][(int64_t)row0 * l + j];
    }
  qld::pdl_wait();
  __syncthreads();

  bool ok = true;
  const bool live = rbase < rows;   // rows past `rows` read stale bytes and are never stored
  for (int p = 0; p < P; ++p) {
    const int st = p % (int)L.nstage;
    if (!sm100::mbar_wait(bars + 8 * st, (p / (int)L.nstage) & 1, FT_WAIT_BUDGET)) ok = false;
    if (ok && live) {
      const uint32_t sb = base + st * L.stage_bytes;
      const uint32_t ldp = (uint32_t)ps.ldSA[p];
      uint32_t r0[RT];
#pragma unroll
      for (int t = 0; t < RT; ++t) r0[t] = sb + (rbase + 16 * t + g) * ldp;
      const uint32_t fb = sb + L.sign_bytes + lane * 16;
      float acc[RT][NB][4];
#pragma unroll
      for (int t = 0; t < RT; ++t)
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) acc[t][nb][0] = acc[t][nb][1] = acc[t][nb][2] = acc[t][nb][3] = 0.f;
#pragma unroll 2
      for (int qw = qw0; qw < qw1; ++qw) {
        uint32_t s0[RT], s1[RT];
#pragma unroll
        for (int t = 0; t < RT; ++t) {
          s0[t] = lds32s(r0[t] + 4 * qw);
          s1[t] = lds32s(r0[t] + 8 * ldp + 4 * qw);
        }
        uint4 bf[NB];
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) bf[nb] = lds128(fb + (qw * NB + nb) * 512);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t ma = 1u << (15 - 8 * h - q), mb = 1u << (11 - 8 * h - q);
#pragma unroll
          for (int t = 0; t < RT; ++t) {
            const uint32_t a0 = sign_pair_mul(s0[t], ma), a1 = sign_pair_mul(s1[t], ma),
                           a2 = sign_pair_mul(s0[t], mb), a3 = sign_pair_mul(s1[t], mb);
#pragma unroll
            for (int nb = 0; nb < NB; ++nb)
              mma16816(acc[t][nb], a0, a1, a2, a3, h ? bf[nb].z : bf[nb].x, h ? bf[nb].w : bf[nb].y);
          }
        }
      }
      // D fragments -> this K group's scratch [tile][16 rows][8 NB columns]
#pragma unroll
      for (int t = 0; t < RT; ++t) {
        float *dsc = dsc_of(kg, RT * rg + t);
#pragma unroll
        for (int nb = 0; nb < NB; ++nb) {
          const int c = 8 * nb + 2 * q;
          dsc[g * 8 * NB + c] = acc[t][nb][0];
          dsc[g * 8 * NB + c + 1] = acc[t][nb][1];
          dsc[(g + 8) * 8 * NB + c] = acc[t][nb][2];
          dsc[(g + 8) * 8 * NB + c + 1] = acc[t][nb][3];
        }
      }
    }
    __syncthreads();   // every warp is done with stage st and has written its partial D
    if (ok && kg == 0 && live) {
      // sum the K groups' partials in group order, then the A_amp epilogue
      for (int t = 0; t < RT; ++t) {
        const int tile = RT * rg + t;
        float *dsc = dsc_of(0, tile);
        for (int e = lane; e < 16 * 8 * NB; e += 32) {
          float d = dsc[e];
          for (int k = 1; k < KG; ++k) d += dsc_of(k, tile)[e];
          dsc[e] = d;
        }
        __syncwarp();
        float *yacc = yacc_all + tile * 16 * B;
        for (int e = lane; e < 16 * B; e += 32) {
          const int rr = e / B, b = e - rr * B, a = row0 + 16 * tile + rr;
          if (a >= n) continue;
          const float *Dr = dsc + rr * 8 * NB;
          const uint16_t *am = L.a_stride ? a_sm + p * L.a_stride + (16 * tile + rr) * l : ps.A[p] + (int64_t)a * l;
          float sacc = yacc[e];
          for (int i = 0; i < l; ++i) sacc = fmaf(qld::f16_to_f32(am[i]), Dr[b * l + i] + Dr[V + b * l + i], sacc);
          yacc[e] = sacc;
        }
      }
    }
    __syncthreads();   // partials consumed; stage st free
    if (threadIdx.x == 0 && p + (int)L.nstage < P && ok) {
      issue(p + L.nstage, st, false);
      issue(p + L.nstage, st, true);
    }
  }
  if (!ok) {
    if (threadIdx.x == 0) {
      atomicExch(&g_mdbf_timeout, 1);
      // leave no copy in flight: wait (bounded) for the last phase of every stage
      for (int st = 0; st < (int)L.nstage; ++st)
        if (issued[st] > 0) (void)sm100::mbar_wait(bars + 8 * st, (issued[st] - 1) & 1, FT_WAIT_BUDGET);
    }
    __syncthreads();
    return;
  }
  if (kg != 0 || !live) return;
  for (int t = 0; t < RT; ++t) {
    const int tile = RT * rg + t;
    const float *yacc = yacc_all + tile * 16 * B;
    for (int e = lane; e < 16 * B; e += 32) {
      const int rr = e / B, b = e - rr * B, a = row0 + 16 * tile + rr;
      if (a >= n) continue;
      if (ydt == QL_OUT_F32)
        static_cast<float *>(y)[(int64_t)b * n + a] = yacc[e];
      else
        static_cast<uint16_t *>(y)[(int64_t)b * n + a] = qld::f32_to_bf16_rn(yacc[e]);
    }
  }
}

// ------------------------------------------------ F stage, one fragment block per word ----------
// For NB == 1 (l * B <= 4, the decode batches) and at most two paths.  One CTA per 16 * RT * NRG
// rows holds both paths in shared memory: each path's sign block arrives by bulk copy before the
// wait on the G stage (weights) and its w fragments by a bulk copy right after it, both counted on
// the path's mbarrier.  Every warp then runs both paths in one pass over its K-word group, one
// accumulator set per path, with no barrier between the paths.  The A_amp epilogue runs in
// registers: lane (g, q) holds columns 2q, 2q + 1 of rows g and g + 8 of each 16-row tile, i.e. the
// high or low part of vector (b, i), so it adds A_amp[row][i] times its values into the row's sum
// for b and the four lanes of a row combine them by shuffles; the K-word groups' sums are then
// added in group order.  Paths are summed inside each lane in p order.  One barrier per CTA,
// before the group sums.  Several layers of one x (mdbf_linear_multi) share a launch: CTA i works on
// layer i / (row blocks per layer), whose paths are P consecutive entries of the path list and
// whose w fragments are those paths' entries of the workspace.
constexpr int F1_PMAX = 2;
constexpr int LAYERS_MAX = 4;
// outputs of the layers of one launch (mdbf_linear_multi); one entry for a single layer
struct LayerOuts {
  void *y[LAYERS_MAX];
};

template <int RT, int NRG>
__global__ void __launch_bounds__(NRG * 32 * 8)
    mdbf_f_nb1_kernel(Paths ps, int P, const uint4 *__restrict__ wpk, const __grid_constant__ LayerOuts outs, int ydt,
                      int n, int r, int l, int B, uint32_t sign_stride, uint32_t frag_bytes) {
  constexpr int KG = 8, TILES = RT * NRG, ROWS = 16 * TILES;
  extern __shared__ __align__(128) unsigned char fsm[];
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(fsm));
  const int QW = (r + 31) / 32, V = l * B;
  // layer of this CTA (several layers of one x in one launch): its paths are [p0, p0 + P)
  const int nfb = (n + ROWS - 1) / ROWS, layer = blockIdx.x / nfb, p0 = layer * P;
  void *const y = outs.y[layer];
  const int row0 = (blockIdx.x - layer * nfb) * ROWS, rows = min(ROWS, n - row0);
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const int rg = wid % NRG, kg = wid / NRG;
  const int qw0 = kg * QW / KG, qw1 = (kg + 1) * QW / KG;
  const int rbase = 16 * RT * rg;
  const uint32_t frag_base = base + F1_PMAX * sign_stride;                  // [P][frag_bytes]
  const uint32_t bars = frag_base + F1_PMAX * frag_bytes;                   // one mbarrier per path
  const uint32_t abort_a = bars + 64;                                        // set when a wait ran out
  uint16_t *const a_sm = reinterpret_cast<uint16_t *>(fsm + F1_PMAX * (sign_stride + frag_bytes) + 128);   // [P][ROWS][l]
  float *const ypart = reinterpret_cast<float *>(fsm + F1_PMAX * (sign_stride + frag_bytes) + 128 +
                                                 ((F1_PMAX * ROWS * l * 2 + 15) / 16) * 16);   // [KG][ROWS][B]
  if (threadIdx.x == 0) {
    for (int p = 0; p < P; ++p) sm100::mbar_init(bars + 8 * p, 1);
    asm volatile("st.shared.u32 [%0], %1;" ::"r"(abort_a), "r"(0u) : "memory");
    sm100::fence_barrier_init();
    for (int p = 0; p < P; ++p) {
      const uint32_t sbytes = (uint32_t)(rows * ps.ldSA[p0 + p]);
      sm100::mbar_arrive_expect_tx(bars + 8 * p, sbytes + frag_bytes);
      sm100::bulk_g2s(base + p * sign_stride, ps.SA[p0 + p] + (size_t)row0 * ps.ldSA[p0 + p], sbytes, bars + 8 * p);
    }
  }
  for (int e = threadIdx.x; e < P * rows * l; e += blockDim.x) {
    const int pp = e / (rows * l), j = e - pp * (rows * l);
    a_sm[pp * ROWS * l + j] = ps.A[p0 + pp][(int64_t)row0 * l + j];
  }
  qld::pdl_trigger();
  qld::pdl_wait();
  // the w fragments are made by the G stage: copied after the wait
  if (threadIdx.x == 0)
    for (int p = 0; p < P; ++p) sm100::bulk_g2s(frag_base + p * frag_bytes, wpk + (size_t)(p0 + p) * QW * 32, frag_bytes, bars + 8 * p);
  __syncthreads();

  bool ok = true;
  const bool live = rbase < rows;   // rows past `rows` read stale bytes and are never stored
  float acc[F1_PMAX][RT][4];
#pragma unroll
  for (int p = 0; p < F1_PMAX; ++p)
#pragma unroll
    for (int t = 0; t < RT; ++t) acc[p][t][0] = acc[p][t][1] = acc[p][t][2] = acc[p][t][3] = 0.f;
#pragma unroll
  for (int p = 0; p < F1_PMAX; ++p) {
    if (p >= P) break;
    if (!sm100::mbar_wait(bars + 8 * p, 0, FT_WAIT_BUDGET)) ok = false;
    if (!ok || !live || qw0 >= qw1) continue;
    const uint32_t sb = base + p * sign_stride;
    const uint32_t ldp = (uint32_t)ps.ldSA[p0 + p];
    uint32_t r0[RT];
#pragma unroll
    for (int t = 0; t < RT; ++t) r0[t] = sb + (rbase + 16 * t + g) * ldp;
    const uint32_t fb = frag_base + p * frag_bytes + lane * 16;
#pragma unroll 2
    for (int qw = qw0; qw < qw1; ++qw) {
      const uint4 bf = lds128(fb + qw * 512);
      uint32_t s0[RT], s1[RT];
#pragma unroll
      for (int t = 0; t < RT; ++t) {
        s0[t] = lds32s(r0[t] + 4 * qw);
        s1[t] = lds32s(r0[t] + 8 * ldp + 4 * qw);
      }
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint32_t ma = 1u << (15 - 8 * h - q), mb = 1u << (11 - 8 * h - q);
#pragma unroll
        for (int t = 0; t < RT; ++t) {
          const uint32_t a0 = sign_pair_mul(s0[t], ma), a1 = sign_pair_mul(s1[t], ma),
                         a2 = sign_pair_mul(s0[t], mb), a3 = sign_pair_mul(s1[t], mb);
          mma16816(acc[p][t], a0, a1, a2, a3, h ? bf.z : bf.x, h ? bf.w : bf.y);
        }
      }
    }
  }
  // register epilogue: this lane's columns c = 2q + j (j = 0, 1) are the high (c < V) or low
  // (V <= c < 2V) part of vector v = b * l + i; add A_amp[row][i] times them into the row's sum for b
  float yb[2 * RT][4];   // [tile t, half hh][b]
#pragma unroll
  for (int k = 0; k < 2 * RT; ++k) yb[k][0] = yb[k][1] = yb[k][2] = yb[k][3] = 0.f;
  if (live) {
#pragma unroll
    for (int p = 0; p < F1_PMAX; ++p) {
      if (p >= P) break;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int c = 2 * q + j;
        if (c >= 2 * V) continue;
        const int v = c < V ? c : c - V, b = v / l, i = v - b * l;
#pragma unroll
        for (int t = 0; t < RT; ++t)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int rl = rbase + 16 * t + g + 8 * hh;   // block-local row
            const float a = qld::f16_to_f32(a_sm[(p * ROWS + rl) * l + i]);
#pragma unroll
            for (int bb = 0; bb < 4; ++bb)
              if (bb == b) yb[2 * t + hh][bb] = fmaf(a, acc[p][t][2 * hh + j], yb[2 * t + hh][bb]);
          }
      }
    }
  }
#pragma unroll
  for (int k = 0; k < 2 * RT; ++k)
#pragma unroll
    for (int bb = 0; bb < 4; ++bb) {
      float v = yb[k][bb];
      v += __shfl_xor_sync(0xffffffffu, v, 1);
      v += __shfl_xor_sync(0xffffffffu, v, 2);
      yb[k][bb] = v;
    }
  if (live && q == 0) {
#pragma unroll
    for (int t = 0; t < RT; ++t)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int rl = rbase + 16 * t + g + 8 * hh;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb)
          if (bb < B) ypart[((size_t)kg * ROWS + rl) * B + bb] = yb[2 * t + hh][bb];
      }
  }
  if (!ok) asm volatile("st.shared.u32 [%0], %1;" ::"r"(abort_a), "r"(1u) : "memory");
  __syncthreads();   // every thread arrives here exactly once, whether its waits ran out or not
  uint32_t aborted;
  asm volatile("ld.volatile.shared.u32 %0, [%1];" : "=r"(aborted) : "r"(abort_a) : "memory");
  if (aborted) {
    if (threadIdx.x == 0) {
      atomicExch(&g_mdbf_timeout, 1);
      // leave no copy in flight: wait (bounded) for every path's sign block
      for (int p = 0; p < P; ++p) (void)sm100::mbar_wait(bars + 8 * p, 0, FT_WAIT_BUDGET);
    }
    return;
  }
  for (int e = threadIdx.x; e < rows * B; e += blockDim.x) {
    const int rl = e / B, b = e - rl * B, a = row0 + rl;
    float sacc = 0.f;
#pragma unroll
    for (int k = 0; k < KG; ++k) sacc += ypart[((size_t)k * ROWS + rl) * B + b];
    if (ydt == QL_OUT_F32)
      static_cast<float *>(y)[(int64_t)b * n + a] = sacc;
    else
      static_cast<uint16_t *>(y)[(int64_t)b * n + a] = qld::f32_to_bf16_rn(sacc);
  }
}

inline size_t f_nb1_smem(uint32_t sign_stride, uint32_t frag_bytes, int rows, int l, int B) {
  return (size_t)F1_PMAX * (sign_stride + frag_bytes) + 128 + ((F1_PMAX * rows * l * 2 + 15) / 16) * 16 +
         (size_t)8 * rows * B * 4;
}

// Rows per CTA of mdbf_f_nb1_kernel for S layers of n rows: 32 or 64 when the CTAs then run in one
// round on the SMs (each holds both paths' w fragments, so one CTA per SM is the norm), else 128.
// The 27B-class down shape (n = 5120) takes 64: 80 CTAs, where 32-row ones ran 160 CTAs in two rounds.
inline int nb1_rows(int S, int n) {
  const int sms = ql::sm_count();
  if (S * ((n + 31) / 32) <= sms) return 32;
  if (S * ((n + 63) / 64) <= sms) return 64;
  return 128;
}

// ------------------------------------------------------ G stage in split-K units (NB == 1) ----------
// A unit is GS_ROWS = 128 rows of S_B of one path over one K slice, a run of 4-word groups.  Its
// sign segments (one bulk copy per row, requested before the wait on pack z: signs are weights) and
// the slice's z fragments and Z8Meta entries (bulk copies after the wait) sit in shared memory,
// where 16 warps (4 row groups of 32 rows x 4 runs of 4-word groups) multiply them on the s8 MMA
// (see "Sign products on the s8 warp MMA"), scaling each group's int32 sums into fp32 once.  The
// runs' sums are added in run order.  With several slices per row block every unit writes its 128 x 8 partial
// sums to the workspace and counts itself in; the last unit of the row block to arrive adds the
// slices' partials in slice order (so the result does not depend on which unit that is) and runs
// the epilogue
//   t[k][b] = sum_i Q_V[k][i] u[k][b*l+i],  w[k][b*l+i] = Q_U[k][i] t[k][b],
// writing the block's w as the F stage's packed fragments (4 words).  It also clears the count
// for the next call; pack z clears the counts as well, so a fresh workspace needs no preparation.
// Slices are sized so that the units fill the SMs: a row block of S_B per SM is too little work
// for the 27B-class layers (r = 2886: 23 row blocks per path).  Used for long sign rows, where
// each unit's shared-memory staging replaces many small ring copies per warp.
constexpr int GS_RT = 2, GS_NRG = 4, GS_KG = 4, GS_ROWS = 16 * GS_RT * GS_NRG;
constexpr int GS_SMAX = 16;   // slices per row block at most (sizes the workspace)

struct GsLayout {
  int S;              // K slices per row block
  uint32_t sstride;   // bytes per sign row in shared memory (word count = 4 mod 8: conflict-free rows)
  uint32_t frag_off;  // z fragments (s8) and their groups' Z8Meta, then (after the products) the K groups'
                      // partial sums
  uint32_t meta_rel;  // the Z8Meta entries, relative to frag_off
  uint32_t bar_off;   // mbarriers and the last-unit flag (32 bytes)
  uint32_t q_off;     // the block's Q_V rows, then its Q_U rows: [2][GS_ROWS][l] fp16
  uint32_t total;
};

inline GsLayout gs_layout(int S, int m, int l, int B) {
  const int QWm = (m + 31) / 32, G4 = (QWm + 3) / 4;
  const int gps = (G4 + S - 1) / S;   // 4-word groups of the largest slice
  int words = 4 * gps;
  while (words % 8 != 4) words += 4;
  GsLayout L;
  L.S = S;
  L.sstride = 4u * (uint32_t)words;
  const uint32_t sign_bytes = (uint32_t)GS_ROWS * L.sstride;
  // after the products the sign region holds the row sums D [128][8] and the w rows [128][V]
  const uint32_t sign_region = std::max(sign_bytes, (uint32_t)(GS_ROWS * 8 + GS_ROWS * l * B) * 4);
  L.frag_off = (sign_region + 127) / 128 * 128;
  L.meta_rel = (uint32_t)(4 * gps) * 256;
  const uint32_t frag_region =
      std::max(L.meta_rel + (uint32_t)gps * (uint32_t)sizeof(Z8Meta), (uint32_t)(GS_KG * GS_ROWS * 8) * 4);
  L.bar_off = L.frag_off + frag_region;
  L.q_off = L.bar_off + 32;
  L.total = L.q_off + 2u * GS_ROWS * (uint32_t)l * 2u;
  return L;
}

__global__ void __launch_bounds__(GS_KG * GS_NRG * 32, 1)
    mdbf_g_split_kernel(Paths ps, const uint2 *__restrict__ zq, const Z8Meta *__restrict__ zmeta,
                        uint4 *__restrict__ wpk, float *__restrict__ part, unsigned *__restrict__ cnt, int m, int r,
                        int l, int B, GsLayout L) {
  constexpr int RT = GS_RT, NRG = GS_NRG, KG = GS_KG, ROWS = GS_ROWS;
  extern __shared__ __align__(128) unsigned char gsm[];
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(gsm));
  const int QWm = (m + 31) / 32, QWr = (r + 31) / 32, G4 = (QWm + 3) / 4, V = l * B;
  const int nrb = (r + ROWS - 1) / ROWS, S = L.S;
  const int unit = blockIdx.x, ks = unit % S, pr = unit / S, rb = pr % nrb, p = pr / nrb;
  const int g0 = ks * G4 / S, g1 = (ks + 1) * G4 / S;
  const int w0 = 4 * g0, wn = min(4 * g1, QWm) - w0;   // the slice's words of z
  const int k0 = rb * ROWS, rows = min(ROWS, r - k0);
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, q = lane & 3;
  const uint32_t sign_bar = base + L.bar_off, frag_bar = sign_bar + 8, flag_a = sign_bar + 16;
  const size_t ld = ps.ldSB[p];
  const uint32_t seg = 16u * (uint32_t)(g1 - g0);   // sign bytes of one row in the slice
  if (threadIdx.x == 0) {
    sm100::mbar_init(sign_bar, 1);
    sm100::mbar_init(frag_bar, 1);
    sm100::fence_barrier_init();
    sm100::mbar_arrive_expect_tx(sign_bar, (uint32_t)rows * seg);
  }
  __syncthreads();
  if ((int)threadIdx.x < rows)
    sm100::bulk_g2s(base + threadIdx.x * L.sstride, ps.SB[p] + (size_t)(k0 + threadIdx.x) * ld + 16 * g0, seg,
                    sign_bar);
  // the epilogue's Q_V and Q_U rows (weights) into shared memory, before the wait: only the last
  // unit of the row block uses them, and reading them there from global memory put a chain of
  // dependent loads on the block's critical path
  uint16_t *const qs = reinterpret_cast<uint16_t *>(gsm + L.q_off);
  for (int e = threadIdx.x; e < 2 * rows * l; e += blockDim.x) {
    const int which = e / (rows * l), j = e - which * (rows * l);
    qs[which * ROWS * l + j] = (which ? ps.QU[p] : ps.QV[p])[(size_t)k0 * l + j];
  }
  qld::pdl_trigger();
  qld::pdl_wait();
  const int ng = g1 - g0;   // the slice's 4-word groups
  if (threadIdx.x == 0) {
    sm100::mbar_arrive_expect_tx(frag_bar, (uint32_t)wn * 256 + (uint32_t)ng * (uint32_t)sizeof(Z8Meta));
    sm100::bulk_g2s(base + L.frag_off, zq + ((size_t)p * QWm + w0) * 32, (uint32_t)wn * 256, frag_bar);
    sm100::bulk_g2s(base + L.frag_off + L.meta_rel, zmeta + (size_t)p * G4 + g0, (uint32_t)ng * (uint32_t)sizeof(Z8Meta),
                    frag_bar);
  }

  bool ok = true;
  const int rg = wid % NRG, kg = wid / NRG;
  const int gq0 = kg * ng / KG, gq1 = (kg + 1) * ng / KG;   // this warp's groups of the slice
  const int rbase = 16 * RT * rg;
  float acc[RT][4];
#pragma unroll
  for (int t = 0; t < RT; ++t) acc[t][0] = acc[t][1] = acc[t][2] = acc[t][3] = 0.f;
  if (!sm100::mbar_wait(sign_bar, 0, FT_WAIT_BUDGET) || !sm100::mbar_wait(frag_bar, 0, FT_WAIT_BUDGET)) ok = false;
  // rows past `rows` hold stale bytes: +-1 signs all the same, whose sums are never used
  if (ok && rbase < rows) {
    uint32_t r0[RT];
#pragma unroll
    for (int t = 0; t < RT; ++t) r0[t] = base + (rbase + 16 * t + g) * L.sstride;
    const uint32_t fb = base + L.frag_off + lane * 8;
    const uint32_t l8 = 8 * L.sstride;
    for (int gq = gq0; gq < gq1; ++gq) {
      float fac[2];
      int corr[2];
#pragma unroll
      for (int j = 0; j < 2; ++j)
        z8_column(base + L.frag_off + L.meta_rel + gq * (uint32_t)sizeof(Z8Meta), 2 * q + j, V, fac[j], corr[j]);
      int ia[RT][4];
#pragma unroll
      for (int t = 0; t < RT; ++t) ia[t][0] = ia[t][1] = ia[t][2] = ia[t][3] = 0;
      const int nw = min(4, wn - 4 * gq);   // the last group of m may hold fewer words
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (u >= nw) break;
        const int qw = 4 * gq + u;
        const uint2 bz = lds64(fb + qw * 256);
#pragma unroll
        for (int t = 0; t < RT; ++t) {
          const uint32_t s0 = lds32s(r0[t] + 4 * qw), s1 = lds32s(r0[t] + l8 + 4 * qw);
          mma_s8_16832(ia[t], (s0 >> q) & 0x01010101u, (s1 >> q) & 0x01010101u, (s0 >> (q + 4)) & 0x01010101u,
                       (s1 >> (q + 4)) & 0x01010101u, bz.x, bz.y);
        }
      }
#pragma unroll
      for (int t = 0; t < RT; ++t)
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[t][i] = fmaf(fac[i & 1], (float)(2 * ia[t][i] - corr[i & 1]), acc[t][i]);
    }
  }
  if (!ok) atomicExch(&g_mdbf_timeout, 1);
  // A wait that ran out leaves its copy in flight: wait again (bounded) before the region is reused.
  if (!ok && threadIdx.x == 0) {
    (void)sm100::mbar_wait(sign_bar, 0, FT_WAIT_BUDGET);
    (void)sm100::mbar_wait(frag_bar, 0, FT_WAIT_BUDGET);
  }
  __syncthreads();   // every warp is done with the fragments: their region takes the partial sums
  float *const red = reinterpret_cast<float *>(gsm + L.frag_off);   // [KG][ROWS][8]
#pragma unroll
  for (int t = 0; t < RT; ++t)
#pragma unroll
    for (int i = 0; i < 4; ++i)
      red[(kg * ROWS + rbase + 16 * t + g + 8 * (i >> 1)) * 8 + 2 * q + (i & 1)] = acc[t][i];
  __syncthreads();
  float *const D = reinterpret_cast<float *>(gsm);   // [ROWS][8], over the sign rows
  float *const Ws = D + ROWS * 8;                     // [ROWS][V]
  for (int e = threadIdx.x; e < ROWS * 8; e += blockDim.x) {
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < KG; ++k) sum += red[k * ROWS * 8 + e];
    if (S == 1)
      D[e] = sum;
    else
      part[(size_t)unit * ROWS * 8 + e] = sum;
  }
  if (S > 1) {
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
      const bool last = atomicAdd(cnt + pr, 1u) == (unsigned)S - 1;
      if (last) atomicExch(cnt + pr, 0u);
      asm volatile("st.shared.u32 [%0], %1;" ::"r"(flag_a), "r"(last ? 1u : 0u) : "memory");
    }
    __syncthreads();
    uint32_t last;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(last) : "r"(flag_a) : "memory");
    if (!last) return;
    __threadfence();
    const float *pb = part + (size_t)pr * S * ROWS * 8;
    for (int e = threadIdx.x; e < ROWS * 8; e += blockDim.x) {
      float v[GS_SMAX];   // every slice's load issued before the first add
#pragma unroll
      for (int s2 = 0; s2 < GS_SMAX; ++s2) v[s2] = s2 < S ? __ldcg(pb + (size_t)s2 * ROWS * 8 + e) : 0.f;
      float sum = 0.f;
#pragma unroll
      for (int s2 = 0; s2 < GS_SMAX; ++s2)
        if (s2 < S) sum += v[s2];
      D[e] = sum;
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < ROWS * B; e += blockDim.x) {
    const int rr = e / B, b = e - rr * B, k = k0 + rr;
    float *wo = Ws + rr * V + b * l;
    if (k >= r) {
      for (int i = 0; i < l; ++i) wo[i] = 0.f;
      continue;
    }
    const float *Dr = D + rr * 8;
    const uint16_t *qv = qs + rr * l, *qu = qs + ROWS * l + rr * l;
    float t = 0.f;
    for (int i = 0; i < l; ++i) t = fmaf(qld::f16_to_f32(qv[i]), Dr[b * l + i] + Dr[V + b * l + i], t);
    for (int i = 0; i < l; ++i) wo[i] = qld::f16_to_f32(qu[i]) * t;
  }
  __syncthreads();
  if (threadIdx.x < ROWS) {
    const int qw = k0 / 32 + (threadIdx.x >> 5);
    if (qw < QWr) {
      auto get = [&](int c, int v) { return Ws[(c - k0) * V + v]; };
      wpk[((size_t)p * QWr + qw) * 32 + lane] = pack_fragment(get, qw, 0, lane, r, V);
    }
  }
}

// The split G stage for a layer, if its shared memory fits: slices enough to fill the SMs, more
// if a slice would not fit.
struct GsPlan {
  bool ok;
  int units;
  GsLayout L;
};
inline GsPlan gs_plan(int P, int m, int r, int l, int B) {
  GsPlan gp{};
  const int nrb = (r + GS_ROWS - 1) / GS_ROWS, G4 = ((m + 31) / 32 + 3) / 4;
  const int smax = std::min(GS_SMAX, G4);
  for (int S = std::max(1, std::min(smax, ql::sm_count() / (P * nrb))); S <= smax; ++S) {
    const GsLayout L = gs_layout(S, m, l, B);
    if (L.total <= 227 * 1024) {
      gp.ok = true;
      gp.units = P * nrb * S;
      gp.L = L;
      return gp;
    }
  }
  return gp;
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
  qld::pdl_trigger();
  qld::pdl_wait();
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
  qld::pdl_trigger();
  qld::pdl_wait();
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

int nb_for(int V) {
  const int need = (2 * V + 7) / 8;
  int nb = 1;
  while (nb < need) nb *= 2;
  return nb;
}

// workspace: packed z fragments, packed w fragments, and for NB == 1 the split G stage's partial
// sums and arrival counts
struct WsLayout {
  size_t zpk, wpk, part, cnt, total;
};
WsLayout ws_layout(int P, int m, int r, int l, int B) {
  const int NB = nb_for(l * B), nrb = (r + GS_ROWS - 1) / GS_ROWS;
  WsLayout L;
  L.zpk = 0;
  L.wpk = align256((size_t)P * ((m + 31) / 32) * NB * 32 * sizeof(uint4));
  L.part = L.wpk + align256((size_t)P * ((r + 31) / 32) * NB * 32 * sizeof(uint4));
  const int smax = std::min(GS_SMAX, ((m + 31) / 32 + 3) / 4);   // as gs_plan: at most one slice per 4-word group
  const size_t part_bytes = NB == 1 && smax > 1 ? (size_t)P * nrb * smax * GS_ROWS * 8 * sizeof(float) : 0;
  L.cnt = L.part + align256(part_bytes);
  L.total = L.cnt + (NB == 1 ? align256((size_t)P * nrb * sizeof(unsigned)) : 0);
  return L;
}

// The three launches of a decode call.  S layers of P paths each (S > 1 only where the F stage is
// mdbf_f_nb1_kernel, see nb1_fits): pack z and the G stage run over all S * P paths, whose
// workspace entries are laid out path by path; the F stage sums each layer's paths into its output.
// the ring G kernel with three stages (NB = 1 only, where that fits three CTAs per SM) or four
template <int NB>
auto ring_g_kernel(bool three) {
  if constexpr (NB == 1)
    return three ? mdbf_g_tile_kernel<1, 3> : mdbf_g_tile_kernel<1, GR_STAGES>;
  else
    return mdbf_g_tile_kernel<NB, GR_STAGES>;
}

template <int NB, int RTF, bool VEC16>
ql_status run_mma_stages(const Paths &ps, int S, int P, int n, int m, int r, int l, int B, const uint16_t *x,
                         uint4 *zpk, uint4 *wpk, float *part, unsigned *cnt, const LayerOuts &outs, ql_out_dtype ydt,
                         cudaStream_t s) {
  const int PT = S * P;
  void *const y = outs.y[0];
  const size_t smg = (size_t)(SP_WARPS * 2 * NB * 128 + 32 * 8 * NB + 32 * l * B) * sizeof(float);
  const size_t smf = (size_t)(SP_WARPS * RTF * NB * 128 + RTF * 16 * 8 * NB + RTF * 16 * B) * sizeof(float);
  auto kg = mdbf_g_mma_kernel<NB, VEC16>;
  auto kf = mdbf_f_mma_kernel<NB, RTF, VEC16>;
  if (ql::set_max_smem(kg, (int)smg) != cudaSuccess ||
      ql::set_max_smem(kf, (int)smf) != cudaSuccess)
    return ql::fail(QL_ERR_CUDA, "mdbf_linear: cannot reserve shared memory");
  // G stage through per-warp cp.async rings when sign rows are 16-byte aligned and the vectors
  // are narrow (decode batches); wider ones keep mdbf_g_mma_kernel.
  constexpr bool g_ring = VEC16 && NB <= 2;
  // the split G stage for NB == 1 on long sign rows (m >= 8192: 256 words or more), when its shared
  // memory fits; shorter rows keep the ring kernel, which is faster there (27B-class gate/up,
  // m = 5120: 26.5 against 28.1 us per call; down, m = 17408: 33.4 against 35.4 us)
  GsPlan gsp{};
  if constexpr (VEC16 && NB == 1)
    if (m >= 8192) gsp = gs_plan(P, m, r, l, B);
  // The split G stage runs on the s8 MMA over z quantised by mdbf_pack_z8_kernel (27B-class down
  // call: 28.9 -> 27.4 us).  The ring kernel keeps the bf16 form: an s8 ring measured slower on a
  // single 27B-class gate or up call (27.4 against 26.8 us), its longer pack launch costing what
  // its products saved.  Whether a layer takes the s8 form depends on its own sizes only, so
  // mdbf_linear_multi gives each layer what mdbf_linear gives it, bit for bit.
  const bool z8 = gsp.ok;
  // three ring stages fit three CTAs per SM (NB = 1), four fit two: three when a launch has more
  // blocks than two per SM (the gate and up projections in one multi call: 364 blocks)
  const bool g_ring3 = NB == 1 && (int64_t)((r + 31) / 32) * PT > 2LL * ql::sm_count();
  const size_t smg_t = (size_t)SP_WARPS * (g_ring3 ? 3 : GR_STAGES) * g_ring_stage_bytes<NB>() + smg +
                       (size_t)2 * 32 * l * 2;
  if constexpr (g_ring) {
    if (ql::set_max_smem(ring_g_kernel<NB>(g_ring3), (int)smg_t) != cudaSuccess)
      return ql::fail(QL_ERR_CUDA, "mdbf_linear: cannot reserve shared memory");
  }
  const int QW = (m + 31) / 32;
  uint2 *const zq = reinterpret_cast<uint2 *>(zpk);   // z8: [PT][QW][32] fragments, then [PT][G4] Z8Meta
  Z8Meta *const zmeta = reinterpret_cast<Z8Meta *>(reinterpret_cast<char *>(zpk) + (size_t)PT * QW * 256);
  const int ncnt = gsp.ok && gsp.L.S > 1 ? PT * ((r + GS_ROWS - 1) / GS_ROWS) : 0;
  if (z8) {
    const int G4 = (QW + 3) / 4;
    ql::launch(mdbf_pack_z8_kernel, dim3(G4, PT), 128, 0, s, ps, x, zq, zmeta, m, l, B, cnt, ncnt);
  } else {
    const int64_t total = (int64_t)QW * NB * 32;
    const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)ql::sm_count() * 4);
    ql::launch(mdbf_pack_z_kernel, dim3(grid, PT), 256, 0, s, ps, x, zpk, m, l, B, NB, cnt, ncnt);
  }
  {
    ql_status st = ql::launch_status("mdbf_linear (pack z)");
    if (st != QL_OK) return st;
  }
  if (gsp.ok) {
    if (ql::set_max_smem(mdbf_g_split_kernel, (int)gsp.L.total) != cudaSuccess)
      return ql::fail(QL_ERR_CUDA, "mdbf_linear: cannot reserve shared memory");
    ql::launch(mdbf_g_split_kernel, S * gsp.units, GS_KG * GS_NRG * 32, gsp.L.total, s, ps, (const uint2 *)zq,
               (const Z8Meta *)zmeta, wpk, part, cnt, m, r, l, B, gsp.L);
  } else if constexpr (g_ring) {
    ql::launch(ring_g_kernel<NB>(g_ring3), dim3((r + 31) / 32, PT), SP_WARPS * 32, smg_t, s, ps, (const uint4 *)zpk,
               wpk, m, r, l, B);
  } else
    ql::launch(kg, dim3((r + 31) / 32, PT), SP_WARPS * 32, smg, s, ps, (const uint4 *)zpk, wpk, m, r, l, B);
  ql_status st = ql::launch_status("mdbf_linear (G stage)");
  if (st != QL_OK) return st;
  if constexpr (VEC16 && NB == 1) {
    if (P <= F1_PMAX) {
      // both paths in one pass
      size_t ld_max = 0;
      for (int p = 0; p < PT; ++p) ld_max = std::max(ld_max, ps.ldSA[p]);
      const int rows = nb1_rows(S, n);
      const uint32_t sign_stride = (uint32_t)((rows * ld_max + 127) / 128 * 128);
      const uint32_t frag_bytes = (uint32_t)((r + 31) / 32) * 32 * 16;
      const size_t sm = f_nb1_smem(sign_stride, frag_bytes, rows, l, B);
      if (sm <= 227 * 1024) {
        auto kt = rows == 128 ? mdbf_f_nb1_kernel<2, 4> : rows == 64 ? mdbf_f_nb1_kernel<2, 2> : mdbf_f_nb1_kernel<2, 1>;
        if (ql::set_max_smem(kt, (int)sm) != cudaSuccess)
          return ql::fail(QL_ERR_CUDA, "mdbf_linear: cannot reserve shared memory");
        ql::launch(kt, S * ((n + rows - 1) / rows), rows / 32 * 32 * 8, sm, s, ps, P, (const uint4 *)wpk, outs,
                   (int)ydt, n, r, l, B, sign_stride, frag_bytes);
        return ql::launch_status("mdbf_linear (F stage)");
      }
    }
  }
  if (S > 1) return ql::fail(QL_ERR_UNSUPPORTED, "mdbf_linear_multi: layers in one launch need the one-pass F stage");
  if constexpr (VEC16) {
    // staged-tile F stage when two (else one) path stages fit in shared memory
    size_t ld_max = 0;
    for (int p = 0; p < P; ++p) ld_max = std::max(ld_max, ps.ldSA[p]);
    constexpr int RT = NB <= 2 ? 2 : 1;                   // row tiles per warp, sharing each fragment load
    constexpr int KG = NB <= 2 ? 8 : NB == 4 ? 4 : NB == 8 ? 2 : 1;   // K-word groups: as many warps as registers allow
    // 32-row CTAs (RT == 2, one stage, three per SM) when 128-row ones would leave SMs idle and the
    // 32-row ones still fit in one round; else 128-row CTAs
    const bool small = RT == 2 && (n + 127) / 128 < ql::sm_count() && (n + 31) / 32 <= 3 * ql::sm_count();
    const int tiles = small ? RT : FT_TILES;
    FTileLayout L = ftile_layout(ld_max, r, NB, B, P, l, small ? 1 : 2, KG, tiles);
    if (L.total > 227 * 1024) L = ftile_layout(ld_max, r, NB, B, P, l, 1, KG, tiles);
    if (L.total <= 227 * 1024) {
      auto kt = small ? mdbf_f_tile_kernel<NB, KG, RT, 1> : mdbf_f_tile_kernel<NB, KG, RT, FT_TILES / RT>;
      if (ql::set_max_smem(kt, (int)L.total) != cudaSuccess)
        return ql::fail(QL_ERR_CUDA, "mdbf_linear: cannot reserve shared memory");
      const int threads = (small ? 1 : FT_TILES / RT) * 32 * KG;
      ql::launch(kt, (n + 16 * tiles - 1) / (16 * tiles), threads, L.total, s, ps, P, (const uint4 *)wpk, y,
                 (int)ydt, n, r, l, B, L);
      return ql::launch_status("mdbf_linear (F stage)");
    }
  }
  ql::launch(kf, (n + 16 * RTF - 1) / (16 * RTF), SP_WARPS * 32, smf, s, ps, P, (const uint4 *)wpk, y, (int)ydt, n,
             r, l, B);
  return ql::launch_status("mdbf_linear (F stage)");
}

template <int NB, bool VEC16>
ql_status run_nb(const Paths &ps, int S, int P, int n, int m, int r, int l, int B, const uint16_t *x, uint4 *zpk,
                 uint4 *wpk, float *part, unsigned *cnt, const LayerOuts &outs, ql_out_dtype ydt, cudaStream_t s) {
  // two 16-row tiles per F block once there are enough rows to fill the machine twice over
  if (NB == 1 && n >= 16 * 2 * 4 * ql::sm_count())
    return run_mma_stages<NB, 2, VEC16>(ps, S, P, n, m, r, l, B, x, zpk, wpk, part, cnt, outs, ydt, s);
  return run_mma_stages<NB, 1, VEC16>(ps, S, P, n, m, r, l, B, x, zpk, wpk, part, cnt, outs, ydt, s);
}

template <bool VEC16>
ql_status run_vec(const Paths &ps, int S, int P, int n, int m, int r, int l, int B, const uint16_t *x, uint4 *zpk,
                  uint4 *wpk, float *part, unsigned *cnt, const LayerOuts &outs, ql_out_dtype ydt, cudaStream_t s) {
  switch (nb_for(l * B)) {
    case 1: return run_nb<1, VEC16>(ps, S, P, n, m, r, l, B, x, zpk, wpk, part, cnt, outs, ydt, s);
    case 2: return run_nb<2, VEC16>(ps, S, P, n, m, r, l, B, x, zpk, wpk, part, cnt, outs, ydt, s);
    case 4: return run_nb<4, VEC16>(ps, S, P, n, m, r, l, B, x, zpk, wpk, part, cnt, outs, ydt, s);
    case 8: return run_nb<8, VEC16>(ps, S, P, n, m, r, l, B, x, zpk, wpk, part, cnt, outs, ydt, s);
    default: return run_nb<16, VEC16>(ps, S, P, n, m, r, l, B, x, zpk, wpk, part, cnt, outs, ydt, s);
  }
}

// Whether S > 1 layers can share the decode launches: their F stage must be the one-pass kernel
// (NB == 1, at most two paths per layer, 16-byte aligned sign rows, its shared memory within the
// limit); the same test run_mma_stages makes before it picks that kernel.
bool nb1_fits(const mdbf_path *paths, int PT, int P, int n, int r, int l, int B) {
  if (l * B > 4 || P > F1_PMAX) return false;
  size_t ld_max = 0;
  for (int p = 0; p < PT; ++p) {
    if (paths[p].ldSA % 16 || paths[p].ldSB % 16 || !ql::aligned(paths[p].S_A, 16) || !ql::aligned(paths[p].S_B, 16))
      return false;
    ld_max = std::max(ld_max, paths[p].ldSA);
  }
  const int rows = nb1_rows(PT / P, n);
  const uint32_t sign_stride = (uint32_t)((rows * ld_max + 127) / 128 * 128);
  const uint32_t frag_bytes = (uint32_t)((r + 31) / 32) * 32 * 16;
  return f_nb1_smem(sign_stride, frag_bytes, rows, l, B) <= 227 * 1024;
}

}  // namespace

namespace ql {

ql_status mdbf_read_timeout(int *flag) {
  int zero = 0;
  if (cudaMemcpyFromSymbol(flag, g_mdbf_timeout, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_mdbf_timeout, &zero, sizeof(int)) != cudaSuccess)
    return fail(QL_ERR_CUDA, "ql_check: cannot read the device timeout flag");
  return QL_OK;
}

// Batches with l * B above VLIM run on the tensor cores (mdbf_gemm_sm100.cu) when the layer
// qualifies (mdbf_use_gemm), otherwise through the decode kernels VLIM / l rows at a time.
size_t mdbf_workspace_size(int P, int n, int m, int r, int l, int B) {
  if (mdbf_use_gemm(n, m, r, l, B, VLIM)) return mdbf_gemm_workspace_size(P, n, m, r, l, B);
  if (l * B > VLIM && l <= VLIM) B = VLIM / l;
  return ws_layout(P, m, r, l, B).total;
}

ql_status mdbf_decode_launch(const mdbf_path *paths, int S, int P, int n, int m, int r, int l, const uint16_t *x,
                             const LayerOuts &outs, ql_out_dtype ydt, int B, void *ws, cudaStream_t s);

ql_status mdbf_linear_launch(const mdbf_path *paths, int P, int n, int m, int r, int l, const uint16_t *x,
                             void *y, ql_out_dtype ydt, int B, void *ws, cudaStream_t s) {
  if (P > PMAX) return fail(QL_ERR_UNSUPPORTED, "mdbf_linear: P = %d exceeds %d paths", P, PMAX);
  LayerOuts outs{};
  outs.y[0] = y;
  if (l * B <= VLIM) return mdbf_decode_launch(paths, 1, P, n, m, r, l, x, outs, ydt, B, ws, s);
  if (mdbf_use_gemm(n, m, r, l, B, VLIM)) return mdbf_gemm_launch(paths, P, n, m, r, l, x, y, ydt, B, ws, s);
  if (l > VLIM) return fail(QL_ERR_UNSUPPORTED, "mdbf_linear: l = %d exceeds %d", l, VLIM);
  const int bc = VLIM / l;
  const size_t ysz = ydt == QL_OUT_F32 ? 4 : 2;
  for (int b0 = 0; b0 < B; b0 += bc) {
    outs.y[0] = static_cast<char *>(y) + (size_t)b0 * n * ysz;
    const ql_status st = mdbf_decode_launch(paths, 1, P, n, m, r, l, x + (size_t)b0 * m, outs, ydt,
                                            std::min(bc, B - b0), ws, s);
    if (st != QL_OK) return st;
  }
  return QL_OK;
}

// S layers of one x: one set of decode launches for all of them where their F stage is the one-pass
// kernel, else the layers one after another (the workspace, sized for S * P paths, serves each).
ql_status mdbf_linear_multi_launch(const mdbf_path *paths, int S, int P, int n, int m, int r, int l, const uint16_t *x,
                                   void *const *ys, ql_out_dtype ydt, int B, void *ws, cudaStream_t s) {
  if (S < 1 || S > LAYERS_MAX || S * P > PMAX)
    return fail(QL_ERR_UNSUPPORTED, "mdbf_linear_multi: %d layers of %d paths (at most %d layers and %d paths)", S, P,
                LAYERS_MAX, PMAX);
  if (S > 1 && l * B <= VLIM && nb1_fits(paths, S * P, P, n, r, l, B)) {
    LayerOuts outs{};
    for (int i = 0; i < S; ++i) outs.y[i] = ys[i];
    return mdbf_decode_launch(paths, S, P, n, m, r, l, x, outs, ydt, B, ws, s);
  }
  for (int i = 0; i < S; ++i) {
    const ql_status st = mdbf_linear_launch(paths + (size_t)i * P, P, n, m, r, l, x, ys[i], ydt, B, ws, s);
    if (st != QL_OK) return st;
  }
  return QL_OK;
}

// The decode kernels: one pass for l * B <= VLIM token rows, S layers of P paths.
ql_status mdbf_decode_launch(const mdbf_path *paths, int S, int P, int n, int m, int r, int l, const uint16_t *x,
                             const LayerOuts &outs, ql_out_dtype ydt, int B, void *ws, cudaStream_t s) {
  const int PT = S * P;
  const Paths ps = pack_paths(paths, PT);
  const WsLayout L = ws_layout(PT, m, r, l, B);
  char *base = static_cast<char *>(ws);
  uint4 *zpk = reinterpret_cast<uint4 *>(base + L.zpk);
  uint4 *wpk = reinterpret_cast<uint4 *>(base + L.wpk);
  float *part = reinterpret_cast<float *>(base + L.part);
  unsigned *cnt = reinterpret_cast<unsigned *>(base + L.cnt);
  bool vec16 = true;
  for (int p = 0; p < PT; ++p)
    vec16 = vec16 && paths[p].ldSA % 16 == 0 && paths[p].ldSB % 16 == 0 && aligned(paths[p].S_A, 16) &&
            aligned(paths[p].S_B, 16);
  if (vec16) return run_vec<true>(ps, S, P, n, m, r, l, B, x, zpk, wpk, part, cnt, outs, ydt, s);
  return run_vec<false>(ps, S, P, n, m, r, l, B, x, zpk, wpk, part, cnt, outs, ydt, s);
}

ql_status mdbf_dequant_launch(const mdbf_path *paths, int P, int n, int m, int r, int l, float *W, float *F,
                              float *G, cudaStream_t s) {
  if (P > PMAX) return fail(QL_ERR_UNSUPPORTED, "mdbf_dequant_debug: P = %d exceeds %d paths", P, PMAX);
  const Paths ps = pack_paths(paths, P);
  if (F || G) {
    const int64_t total = (int64_t)n * r + (int64_t)r * m;
    const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 8);
    launch(mdbf_factors_kernel, dim3(grid, P), 256, 0, s, ps, F, G, n, m, r, l);
    ql_status st = launch_status("mdbf_dequant_debug (factors)");
    if (st != QL_OK) return st;
  }
  const int64_t total = (int64_t)n * m;
  const int grid = (int)std::min<int64_t>((total + 255) / 256, (int64_t)sm_count() * 16);
  launch(mdbf_w_kernel, grid, 256, 0, s, ps, P, W, n, m, r, l);
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
// The array's device address, per device, with the unique id of the context it was looked up in.
struct ScratchAddr {
  bool valid;
  unsigned long long ctx_id;
  void *ptr;
};
ScratchAddr g_scratch_addr[64] = {};

using CtxGetCurrentFn = int (*)(void **);                     // cuCtxGetCurrent
using CtxGetIdFn = int (*)(void *, unsigned long long *);     // cuCtxGetId
template <typename F>
F driver_fn(const char *name) {
  void *p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess && q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<F>(p);
  return nullptr;
}
// Id of the calling thread's current context.  The driver never hands the same id to two
// contexts of one process, so a context torn down and created again (cudaDeviceReset, a host
// that resets its device) gets a new id even where its handle is reused.
bool current_ctx_id(unsigned long long *id) {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  void *ctx = nullptr;
  return get_current && get_id && get_current(&ctx) == 0 && ctx && get_id(ctx, id) == 0;
}
}  // namespace

namespace ql {

size_t mdbf_noalloc_scratch_limit() { return NOALLOC_SCRATCH_BYTES; }

// Device address of the scratch array on the current device.  The host-side symbol is only a
// stand-in, so the address is looked up with the device current and cached with the context it
// belongs to; a new context on the device (the module then loads at another address) is looked
// up again, and where the context cannot be identified the lookup runs on every call.
ql_status mdbf_noalloc_scratch(void **ptr) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64)
    return fail(QL_ERR_CUDA, "mdbf_linear_noalloc: no current CUDA device");
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  ScratchAddr &e = g_scratch_addr[dev];
  unsigned long long id = 0;
  if (e.valid && current_ctx_id(&id) && id == e.ctx_id) {
    *ptr = e.ptr;
    return QL_OK;
  }
  void *p = nullptr;
  const cudaError_t err = cudaGetSymbolAddress(&p, g_mdbf_scratch);
  if (err != cudaSuccess || !p)
    return fail(QL_ERR_CUDA, "mdbf_linear_noalloc: cannot resolve the scratch array: %s", cudaGetErrorString(err));
  // the lookup made the device's primary context current if the thread had none
  e.valid = current_ctx_id(&id);
  e.ctx_id = id;
  e.ptr = p;
  *ptr = p;
  return QL_OK;
}

}  // namespace ql
