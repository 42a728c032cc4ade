// BenQ prefill GEMM on sm_100a tensor cores: Y[M][N] = X[M][K] * W[N][K]^T, W decoded on the fly.
//
// W is never written to global memory ("Qwen3.8-27B -- BenQ 6-bit", "What BenQ stores": the
// gather lut[n][code] is fused into the GEMM).  The work unit is a CTA pair (a cluster of two
// CTAs on two SMs) and a 512 x 256 output tile: CTA r of the pair owns X rows [256 r, 256 r + 256)
// of the tile and decodes W rows [128 r, 128 r + 128) of it.  Pair MMAs (tcgen05.mma.cta_group::2,
// M = 256, N = 256, K = 16) read A from each CTA's own shared memory and B from both, so every
// decoded weight feeds all 512 rows of X while each SM decodes only half of the W tile and each
// SM's tensor core reads only its half of B.  Per 64-wide K block, in each CTA:
//   * warp 0 loads its X tile (256 x 64 bf16, 128-byte swizzle) with tensor copies into a 3-stage
//     ring; completion is counted on the even CTA's barrier, whose MMA thread consumes both;
//   * warp 2 loads its packed codes for 4 K blocks at a time (128 rows x 192 bytes: narrow rows
//     make slow tensor copies) into a 2-stage ring, plus the 128 row tables of the tile (16 KB,
//     once per tile) with a bulk copy;
//   * warps 3..18 (decoders) expand the code tile through the row tables into the bf16 W half
//     tile, two K blocks per pass, written directly in the K-major 128-byte-swizzled layout the
//     tensor core reads, fence the writes for the async proxy and arrive on a barrier of their
//     own CTA;
//   * in the even CTA, warp 1 (one thread) waits for both CTAs' decoded halves and issues the
//     pair MMAs (two M halves share each decoded W tile) into both CTAs' tensor memory
//     (2 x 128 x 256 fp32 per CTA), signalling stage release to both CTAs with a multicast
//     commit; in the odd CTA one thread of warp 1 relays each decoded block to it at cluster
//     scope (one release per block instead of one per decoder warp);
//   * after the last K block the decoder warps of each CTA drain their own accumulators
//     (tcgen05.ld), round to bf16 (or keep fp32) and store Y, through tensor stores staged in the
//     decoded-W ring when Y's rows are 16-byte aligned.
// No tensor or bulk load is multicast.  Every wait gives up after a fixed clock budget or as soon
// as another wait of the pair has given up, sets a device flag read by ql_check(), and the CTA
// winds down; both CTAs meet at a cluster barrier before tensor memory is freed and they exit.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "ql_internal.cuh"
#include "pair_gemm.cuh"
#include "sm100_ptx.cuh"

namespace {

using namespace pairgemm;

constexpr int BM = 256;                           // X rows per CTA (two 128-row MMA halves)
constexpr int PM = 2 * BM;                        // X rows per pair tile
constexpr int BN = 256;                           // W rows per pair tile (the MMA's N)
constexpr int BNH = BN / 2;                       // W rows decoded by each CTA
constexpr int BK = 64;                            // one 128-byte swizzle row of bf16
constexpr int SA = 3, SB = 4, SC = 2;             // stages: activations, decoded W, codes
constexpr int A_BYTES = BM * BK * 2;              // 32 KB
constexpr int B_BYTES = BNH * BK * 2;             // 16 KB
constexpr int C_ROW = BK * 6 / 8;                 // 48 code bytes per row per K block
constexpr int CKB = 4;                            // K blocks per code stage (one copy of 192-byte rows)
constexpr int C_SROW = CKB * C_ROW;               // 192 code bytes per row per code stage
constexpr int C_BYTES = BNH * C_SROW;             // 24 KB
constexpr int LUT_BYTES = BNH * 128;              // 16 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + SA * A_BYTES;
constexpr int OFF_C = OFF_B + SB * B_BYTES;
constexpr int OFF_LUT = OFF_C + SC * C_BYTES + 128;   // 128 bytes of slack: the last row's second code word
constexpr int OFF_BAR = OFF_LUT + LUT_BYTES;
constexpr int NBAR = 2 * (SA + SB + SC) + SB + 8;
constexpr int OFF_TMEM = OFF_BAR + NBAR * 8;          // tensor-memory address, abort flag, last-part flag
constexpr int SMEM_BYTES = OFF_TMEM + 16 + 1024;      // + alignment slack
constexpr int NDEC = 16;                              // decoder / epilogue warps (multiple of 8)
constexpr int THREADS = (3 + NDEC) * 32;              // A producer, MMA issuer, code producer, decoders
constexpr uint32_t IDESC = sm100::idesc_bf16_f32(2 * 128, BN);   // pair MMA: M = 256 over two CTAs
constexpr uint16_t PAIR = 0x3;                        // both CTAs of the cluster
static_assert(OFF_B % 1024 == 0 && A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms");
static_assert(OFF_LUT % 128 == 0 && OFF_BAR % 8 == 0, "alignment");
static_assert(SB * B_BYTES == 4 * 16384, "the decoded-W ring stages one epilogue round: four 16 KB boxes");
static_assert(SMEM_BYTES <= 232448, "shared memory");

__device__ int g_gemm_timeout = 0;

struct Bars {
  // full_a, peer_b and acc_empty are used in the even CTA only (both CTAs arrive on full_a and
  // acc_empty, the odd CTA's forwarder on peer_b); dec_done collects this CTA's decoder warps;
  // the others are local to each CTA.
  uint32_t full_a, empty_a, dec_done, empty_b, full_c, empty_c, lut_full, lut_empty, acc_full, acc_empty, split_done,
      split_go, stg_full, stg_free, peer_b;
  __device__ Bars(uint32_t base)
      : full_a(base), empty_a(full_a + 8 * SA), dec_done(empty_a + 8 * SA), empty_b(dec_done + 8 * SB),
        full_c(empty_b + 8 * SB), empty_c(full_c + 8 * SC), lut_full(empty_c + 8 * SC), lut_empty(lut_full + 8),
        acc_full(lut_empty + 8), acc_empty(acc_full + 8), split_done(acc_empty + 8), split_go(split_done + 8),
        stg_full(split_go + 8), stg_free(stg_full + 8), peer_b(stg_free + 8) {}
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(THREADS, 1)
    benq_gemm_kernel(const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_codes,
                     const __grid_constant__ CUtensorMap map_y, int tstore, const uint16_t *__restrict__ lut, void *__restrict__ y, int ydt, int M, int N, int K,
                     float *__restrict__ part_ws, unsigned *__restrict__ part_cnt, int full, int parts, int nfast) {
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
  const int mt = (M + PM - 1) / PM, nt = N / BN, ntiles = mt * nt, nkb = K / BK;
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
    for (int s = 0; s < SC; ++s) {
      sm100::mbar_init(bar.full_c + 8 * s, 1);
      sm100::mbar_init(bar.empty_c + 8 * s, NDEC);
    }
    sm100::mbar_init(bar.lut_full, 1);
    sm100::mbar_init(bar.lut_empty, NDEC);
    sm100::mbar_init(bar.acc_full, 1);
    sm100::mbar_init(bar.acc_empty, 2 * NDEC);
    sm100::mbar_init(bar.split_done, NDEC);
    sm100::mbar_init(bar.split_go, 1);
    sm100::mbar_init(bar.stg_full, NDEC);
    sm100::mbar_init(bar.stg_free, 1);
    sts32(tmem_slot + 4, 0);
    sm100::fence_barrier_init();
    sm100::prefetch_tensormap(&map_x);
    sm100::prefetch_tensormap(&map_codes);
    if (tstore) sm100::prefetch_tensormap(&map_y);
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
  // codes and tables are weights: their producer starts at once; activations are read and y is
  // written only after the preceding kernel in the stream has completed
  qld::pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ activation producer (tensor copies)
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
          sm100::tma_load_2d_pair(sbase + OFF_A + s * A_BYTES, &map_x, kb * BK, m0, lead_full_a + 8 * s);
        }
      }
    }
  } else if (warp == 2) {
    // ------------------------------------------------------------ code and table producer (local)
    if (lane == 0) {
      int ic = 0, tl = 0;
      for (int wi = pair; wi < nitems && ok; wi += npairs, ++tl) {
        const Item w = item_of(wi, full, parts, nkb);
        int mi, ni;
        tile_mn(w.tile, mt, nt, nfast, mi, ni);
        const int n0 = ni * BN + (int)rank * BNH;
        const int ncs = (w.kb1 - w.kb0 + CKB - 1) / CKB;   // code stages; a ragged last one reads zeros
        if (tl > 0 && !wt.wait(bar.lut_empty, (tl - 1) & 1, false)) { ok = false; break; }
        sm100::mbar_arrive_expect_tx(bar.lut_full, LUT_BYTES);
        sm100::bulk_g2s(sbase + OFF_LUT, lut + (size_t)n0 * 64, LUT_BYTES, bar.lut_full);
        for (int cs = 0; cs < ncs; ++cs, ++ic) {
          const int s = ic % SC;
          if (ic >= SC && !wt.wait(bar.empty_c + 8 * s, ((ic / SC) & 1) ^ 1, false)) {
            ok = false;
            break;
          }
          sm100::mbar_arrive_expect_tx(bar.full_c + 8 * s, C_BYTES);
          sm100::tma_load_2d(sbase + OFF_C + s * C_BYTES, &map_codes, (w.kb0 + cs * CKB) * C_ROW, n0,
                             bar.full_c + 8 * s);
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
    const int dw = warp - 3;            // decoder index 0 .. NDEC-1
    const int q = warp & 3;             // tensor-memory lane quarter this warp may read
    const int ch = dw >> 2;             // which NDEC/4-th of the 256 accumulator columns it drains
    const uint32_t lead_acc_empty = sm100::mapa_shared(bar.acc_empty, 0);
    int it = 0, tl = 0, ic = 0, ns = 0, ep = 0;
    // A pass decodes two K blocks: lanes 0-15 the first, 16-31 the second.  Lane l expands the 4
    // codes in bytes [3l, 3l + 3) of the two blocks' 96 code bytes of a row (codes 4(l&15) ..
    // 4(l&15)+3 of its block), so two 32-bit loads serve 4 codes and its output is 8 bytes.
    const int half = lane >> 4;
    const int cwo = 4 * ((3 * lane) >> 2), csh = 8 * ((3 * lane) & 3);
    // swizzled position of those 4 codes within row r = dw (mod 8) of a K block
    const uint32_t dst_lane =
        (dw >> 3) * 1024 + (dw & 7) * 128 + ((((lane & 15) >> 1) ^ (dw & 7)) << 4) + (lane & 1) * 8;
    for (int wi = pair; wi < nitems && ok; wi += npairs, ++tl) {
      const Item w = item_of(wi, full, parts, nkb);
      int mi, ni;
      tile_mn(w.tile, mt, nt, nfast, mi, ni);
      const int m0 = mi * PM + (int)rank * BM, n0 = ni * BN;
      if (!wt.wait(bar.lut_full, tl & 1, false)) { ok = false; break; }
      for (int kb = w.kb0; kb < w.kb1;) {
        const bool two = kb + 1 < w.kb1;
        const int sb0 = it % SB, sb1 = (it + 1) % SB, sc = ic % SC, sub = (kb - w.kb0) % CKB;   // sub is 0 or 2
        if ((it >= SB && !wt.wait(bar.empty_b + 8 * sb0, ((it / SB) & 1) ^ 1, true)) ||
            (two && it + 1 >= SB && !wt.wait(bar.empty_b + 8 * sb1, (((it + 1) / SB) & 1) ^ 1, true)) ||
            (sub == 0 && !wt.wait(bar.full_c + 8 * sc, (ic / SC) & 1, false))) {
          ok = false;
          break;
        }
        // rows r = dw + NDEC*i: r & 7 == dw & 7 is fixed per warp, so every address below is
        // a per-warp base plus a compile-time multiple of the row step.  All code words of the
        // warp's rows are loaded before the first lookup.
        const uint32_t cb = sbase + OFF_C + sc * C_BYTES + dw * C_SROW + sub * C_ROW + cwo;
        const uint32_t bb = sbase + OFF_B + (half ? sb1 : sb0) * B_BYTES + dst_lane;
        const uint32_t tb = sbase + OFF_LUT + dw * 128;
        constexpr int RPW = BNH / NDEC;   // rows per decoder warp per K block
        uint32_t v[RPW];
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
          const uint32_t w0 = lds32(cb + i * NDEC * C_SROW);
          const uint32_t w1 = lds32(cb + i * NDEC * C_SROW + 4);   // may read past the row: unused bits
          v[i] = __funnelshift_r(w0, w1, csh);
        }
        const bool store = half == 0 || two;
#pragma unroll
        for (int i = 0; i < RPW; ++i) {
          const uint32_t tbl = tb + i * NDEC * 128;
          const uint32_t e0 = lds_u16(((v[i] << 1) & 0x7Eu) | tbl);
          const uint32_t e1 = lds_u16(((v[i] >> 5) & 0x7Eu) | tbl);
          const uint32_t e2 = lds_u16(((v[i] >> 11) & 0x7Eu) | tbl);
          const uint32_t e3 = lds_u16(((v[i] >> 17) & 0x7Eu) | tbl);
          if (store) sts64(bb + i * (NDEC / 8) * 1024, __byte_perm(e0, e1, 0x5410), __byte_perm(e2, e3, 0x5410));
        }
        sm100::fence_proxy_async_smem();
        __syncwarp();
        const int step = two ? 2 : 1;
        const bool stage_done = sub + step >= CKB || kb + step == w.kb1;
        if (lane == 0) {
          // this CTA's MMA side takes the blocks through a CTA-scope barrier: the even CTA's MMA
          // thread waits on it directly, the odd CTA's forwarder relays it at cluster scope
          sm100::mbar_arrive(bar.dec_done + 8 * sb0);
          if (two) sm100::mbar_arrive(bar.dec_done + 8 * sb1);
          if (stage_done) sm100::mbar_arrive(bar.empty_c + 8 * sc);
        }
        if (stage_done) ++ic;
        kb += step;
        it += step;
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(bar.lut_empty);
      // epilogue: this warp drains lanes [32q, 32q+32) of both 128-row accumulators
      if (!wt.wait(bar.acc_full, tl & 1, true)) { ok = false; break; }
      qld::pdl_wait();
      sm100::tc_fence_after();
      const bool split = w.part >= 0;
      if (!split && tstore) {
        // Whole tile through tensor stores: once acc_full has fired every decoded block of the
        // tile has been consumed, so the decoded-W ring (4 x 16 KB) is free to stage the output.
        if (!staged_tile_store(tmem, sbase + OFF_B, &map_y, ydt == QL_OUT_F32 ? OUT_F32 : OUT_BF16, nullptr, m0, n0, M,
                               N, q, ch, dw, lane, wt, bar.stg_full, bar.stg_free, ep)) {
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
              atomicExch(cnt, 0u);   // ready for the next call
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
            if (ydt == QL_OUT_F32) {
              *reinterpret_cast<float4 *>(static_cast<float *>(y) + (size_t)row * N + col) = a;
            } else {
              const uint32_t lo = uint32_t(qld::f32_to_bf16_rn(a.x)) | (uint32_t(qld::f32_to_bf16_rn(a.y)) << 16);
              const uint32_t hi = uint32_t(qld::f32_to_bf16_rn(a.z)) | (uint32_t(qld::f32_to_bf16_rn(a.w)) << 16);
              *reinterpret_cast<uint2 *>(static_cast<uint16_t *>(y) + (size_t)row * N + col) = make_uint2(lo, hi);
            }
          }
        }
      }
    }
  }

  if (warp == 3 && lane == 0) sm100::bulk_wait0();   // the tensor stores issued by decoder 0
  if (!ok) atomicExch(&g_gemm_timeout, 1);
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

// Self-test of the bounded waits: a CTA pair where the even CTA waits on an mbarrier nothing ever
// arrives on, with a short budget.  Its wait runs out, raises the abort flag in both CTAs (the odd
// CTA's own wait on an equally idle barrier ends through that flag), and both record the timeout in
// the flag ql_check() reads; the kernel then returns normally.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(32, 1) selftest_timeout_kernel(long long budget) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ uint32_t abort_flag;
  const uint32_t b = static_cast<uint32_t>(__cvta_generic_to_shared(&bar));
  const uint32_t f = static_cast<uint32_t>(__cvta_generic_to_shared(&abort_flag));
  const uint32_t rank = sm100::cluster_ctarank();
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    sts32(f, 0);
    sm100::fence_barrier_init();
  }
  sm100::cluster_sync();
  const Waiter wt{f, sm100::mapa_shared(f, rank ^ 1u), rank == 0 ? budget : WAIT_BUDGET};
  bool ok = true;
  if (threadIdx.x == 0) ok = wt.wait(b, 0, false);
  if (!ok) atomicExch(&g_gemm_timeout, 2);
  sm100::cluster_sync();   // neither CTA leaves while the other may still write its abort flag
}

// ---------------------------------------------------------------------------- host side
// Opts the GEMM kernel into its dynamic shared memory (once per device).
cudaError_t smem_attr() { return ql::set_max_smem(benq_gemm_kernel, SMEM_BYTES); }

// CTA pairs that can be resident at once on the current device (cached per device).
int resident_pairs() {
  static std::mutex mu;
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) dev = 0;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    (void)smem_attr();   // the occupancy query needs the kernel's shared-memory opt-in
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (ql::sm_count() / 2));
    cfg.blockDim = dim3(THREADS);
    cfg.dynamicSmemBytes = SMEM_BYTES;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, benq_gemm_kernel, &cfg) != cudaSuccess || n <= 0) {
      (void)cudaGetLastError();
      n = ql::sm_count() / 2;
    }
    cache[dev] = n;
  }
  return cache[dev];
}

SplitPlan split_plan(int M, int N, int K, int pairs) {
  return pairgemm::split_plan(((M + PM - 1) / PM) * (N / BN), K / BK, pairs, (size_t)2 * BM * BN * sizeof(float));
}

}  // namespace

namespace ql {

size_t benq_gemm_workspace_size(int M, int N, int K) {
  if (M <= 0 || N <= 0 || K <= 0 || N % BN || K % BK) return 0;
  const SplitPlan p = split_plan(M, N, K, resident_pairs());
  return p.partial_bytes + p.counter_bytes;
}

ql_status benq_gemm_launch(const uint8_t *codes, const uint16_t *lut, const uint16_t *x, void *y, ql_out_dtype ydt,
                           int M, int N, int K, void *ws, size_t ws_bytes, cudaStream_t s) {
  if (N % BN || K % BK) return fail(QL_ERR_UNSUPPORTED, "benq_linear: batch > 16 needs N %% 256 == 0 and K %% 64 == 0");
  EncodeTiledFn enc = encode_tiled_fn();
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
    const cuuint32_t box[2] = {C_SROW, BNH};
    const cuuint32_t es[2] = {1, 1};
    if (enc(&mc, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(codes), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return fail(QL_ERR_CUDA, "benq_linear: cannot encode the code tensor map");
  }
  // y through tensor stores when its rows are 16-byte aligned (N % 256 == 0 here), else direct stores
  CUtensorMap my = {};
  const bool tstore = aligned(y, 16) && encode_rows_sw128(enc, &my, ydt == QL_OUT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32
                                                                                    : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                                                          y, M, N, N, 128, ydt == QL_OUT_F32 ? 4 : 2);
  if (smem_attr() != cudaSuccess) return fail(QL_ERR_CUDA, "benq_linear: cannot reserve GEMM shared memory");
  const int ntiles = ((M + PM - 1) / PM) * (N / BN);
  const int resident = resident_pairs();
  SplitPlan plan = split_plan(M, N, K, resident);
  float *part_ws = nullptr;
  unsigned *part_cnt = nullptr;
  if (plan.parts > 1 && ws != nullptr && ws_bytes >= plan.partial_bytes + plan.counter_bytes) {
    part_ws = static_cast<float *>(ws);
    part_cnt = reinterpret_cast<unsigned *>(static_cast<char *>(ws) + plan.partial_bytes);
    if (cudaMemsetAsync(part_cnt, 0, plan.counter_bytes, s) != cudaSuccess)
      return fail(QL_ERR_CUDA, "benq_linear: cannot clear the split-tile counters");
  } else {
    plan = SplitPlan{ntiles, 1, 0, 0, 0};   // no (or too small a) workspace: whole tiles only
  }
  const int nitems = plan.full + plan.leftover * plan.parts;
  const int pairs = std::min(nitems, resident);
  // N-fastest tiles when the activations (2 bytes per element) outweigh the packed codes (0.75)
  const int nfast = 2.0 * M > 0.75 * N ? 1 : 0;
  launch(benq_gemm_kernel, 2 * pairs, THREADS, SMEM_BYTES, s, mx, mc, my, tstore ? 1 : 0, lut, y, (int)ydt, M, N, K, part_ws, part_cnt,
         plan.full, plan.parts, nfast);
  return launch_status("benq_linear (tensor-core GEMM)");
}

ql_status selftest_timeout_launch(cudaStream_t s) {
  launch(selftest_timeout_kernel, 2, 32, 0, s, 20000000LL);   // ~10 ms at 2 GHz
  return launch_status("ql_selftest_timeout");
}

ql_status benq_gemm_read_timeout(int *flag) {
  int zero = 0;
  if (cudaMemcpyFromSymbol(flag, g_gemm_timeout, sizeof(int)) != cudaSuccess ||
      cudaMemcpyToSymbol(g_gemm_timeout, &zero, sizeof(int)) != cudaSuccess)
    return fail(QL_ERR_CUDA, "ql_check: cannot read the device timeout flag");
  return QL_OK;
}

}  // namespace ql
