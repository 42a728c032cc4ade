// BenQ encoder on the GPU: a bf16 matrix W [N][K] to BenQ storage (packed 6-bit codes and per-row
// bf16 tables), the step before the linear path.
//
// "Qwen3.8-27B -- BenQ 6-bit", sections "Why equal-width shells" and the calibration notes: the 32
// magnitude tiers of a row are equal-width shells of its range, each tier's level is the mean of
// the magnitudes in it, the table is refined Lloyd-style, and weights take their nearest level
// (the uncalibrated path).  Per row:
//   D = max|w| / 32;  tier t = min(floor(|w| / D), 31)              (fp64, exact division by 32)
//   level t = mean of the magnitudes in tier t (fp64), the shell midpoint (t + 1/2) D when empty,
//             rounded fp64 -> fp32 -> bf16 (nearest even both times)
//   lloyd_iters rounds: every magnitude to its nearest level (lower tier on an exact tie), then the
//             member means as above (a level without members keeps its value)
//   code = 32 + t for w >= 0 (zero and -0 included), 31 - t for w < 0, t the nearest level;
//   table [-L31 .. -L0, L0 .. L31]; an all-zero row gets zero levels and codes 32.
// The tier sums are exact in fp64 whenever a row's nonzero magnitudes span less than 2^30 (bf16
// values carry 8 significant bits and a row has at most 2^15 of them), so the order in which the
// atomics add them does not change the result.
//
// One CTA of 256 threads per row; per-warp tier histograms (count, fp64 sum) in shared memory.
#include <cuda_bf16.h>

#include <algorithm>

#include "ql_internal.cuh"

namespace {

constexpr int ENC_THREADS = 256;
constexpr int ENC_WARPS = ENC_THREADS / 32;

__device__ __forceinline__ double bf16_abs(uint16_t b) { return (double)__uint_as_float((uint32_t)(b & 0x7FFFu) << 16); }

// fp64 -> fp32 -> bf16, each rounded to nearest even; returned as the bf16 bits
__device__ __forceinline__ uint16_t level_bits(double v) {
  const float f = __double2float_rn(v);
  return __bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// index of the level nearest to a (lower index on an exact tie); distances are exact in fp64.
// lv: the 32 levels in shared memory (every lane reads the same entry: broadcast loads).
__device__ __forceinline__ int nearest_level(double a, const double *lv) {
  int best = 0;
  double bd = fabs(a - lv[0]);
#pragma unroll
  for (int t = 1; t < 32; ++t) {
    const double d = fabs(a - lv[t]);
    if (d < bd) {
      bd = d;
      best = t;
    }
  }
  return best;
}

__global__ void __launch_bounds__(ENC_THREADS) benq_encode_kernel(const uint16_t *__restrict__ W,
                                                                  uint8_t *__restrict__ codes,
                                                                  uint16_t *__restrict__ lut, int K, int iters) {
  qld::pdl_trigger();
  qld::pdl_wait();
  const int n = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint16_t *wr = W + (size_t)n * K;
  __shared__ double s_sum[ENC_WARPS][32];
  __shared__ unsigned s_cnt[ENC_WARPS][32];
  __shared__ double s_lv[32];
  __shared__ float s_red[ENC_WARPS];
  // 1. row maximum of |w| (bf16 -> fp32 is exact)
  float mx = 0.f;
  for (int k = tid; k < K; k += ENC_THREADS) mx = fmaxf(mx, (float)bf16_abs(wr[k]));
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) s_red[warp] = mx;
  __syncthreads();
  float amax = 0.f;
  for (int i = 0; i < ENC_WARPS; ++i) amax = fmaxf(amax, s_red[i]);
  const double D = (double)amax / 32.0;

  auto clear = [&] {
    for (int i = tid; i < ENC_WARPS * 32; i += ENC_THREADS) {
      (&s_sum[0][0])[i] = 0.0;
      (&s_cnt[0][0])[i] = 0u;
    }
  };
  // levels from the per-warp histograms: member mean, else `fallback(t)`
  auto finish_levels = [&](auto fallback) {
    if (tid < 32) {
      double sum = 0.0;
      unsigned cnt = 0;
      for (int i = 0; i < ENC_WARPS; ++i) {
        sum += s_sum[i][tid];
        cnt += s_cnt[i][tid];
      }
      const double mean = cnt ? sum / (double)cnt : fallback(tid);
      s_lv[tid] = (double)__uint_as_float((uint32_t)level_bits(mean) << 16);
    }
  };

  if (amax == 0.f) {
    if (tid < 32) s_lv[tid] = 0.0;
  } else {
    // 2. equal-width shells
    clear();
    __syncthreads();
    for (int k = tid; k < K; k += ENC_THREADS) {
      const double a = bf16_abs(wr[k]);
      // clamped to [0, 31] so that a non-finite weight (outside the contract) cannot index out of
      // the histogram: (int) of a NaN quotient is INT_MIN
      const int t = max(0, min((int)floor(a / D), 31));
      atomicAdd(&s_sum[warp][t], a);
      atomicAdd(&s_cnt[warp][t], 1u);
    }
    __syncthreads();
    finish_levels([&](int t) { return ((double)t + 0.5) * D; });
    __syncthreads();
    // 3. Lloyd rounds
    for (int it = 0; it < iters; ++it) {
      // s_lv is only read until finish_levels, where thread t reads and then rewrites entry t
      clear();
      __syncthreads();
      for (int k = tid; k < K; k += ENC_THREADS) {
        const double a = bf16_abs(wr[k]);
        const int t = nearest_level(a, s_lv);
        atomicAdd(&s_sum[warp][t], a);
        atomicAdd(&s_cnt[warp][t], 1u);
      }
      __syncthreads();
      finish_levels([&](int t) { return s_lv[t]; });
      __syncthreads();
    }
  }
  __syncthreads();
  // 4. table
  if (tid < 32) {
    const uint16_t b = __bfloat16_as_ushort(__float2bfloat16_rn((float)s_lv[tid]));
    lut[(size_t)n * 64 + 32 + tid] = b;
    lut[(size_t)n * 64 + 31 - tid] = (uint16_t)(b | 0x8000u);
  }
  // 5. codes, packed 4 per 3 bytes (little-endian bitstream)
  uint8_t *cr = codes + (size_t)n * (3 * K / 4);
  for (int g = tid; g < K / 4; g += ENC_THREADS) {
    uint32_t v = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint16_t b = wr[4 * g + j];
      const int t = amax == 0.f ? 0 : nearest_level(bf16_abs(b), s_lv);
      const bool neg = (b & 0x8000u) && (b & 0x7FFFu);
      v |= (uint32_t)(neg ? 31 - t : 32 + t) << (6 * j);
    }
    cr[3 * g] = (uint8_t)v;
    cr[3 * g + 1] = (uint8_t)(v >> 8);
    cr[3 * g + 2] = (uint8_t)(v >> 16);
  }
}

}  // namespace

namespace ql {

ql_status benq_encode_launch(const uint16_t *W, uint8_t *codes, uint16_t *lut, int N, int K, int iters,
                             cudaStream_t s) {
  launch(benq_encode_kernel, N, ENC_THREADS, 0, s, W, codes, lut, K, iters);
  return launch_status("benq_encode");
}

}  // namespace ql
