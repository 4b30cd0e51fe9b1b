// The MLP's block-scaled FP4 GEMMs with their fused epilogues (FourTune §3.3
// "MLP Fusion": the first fully connected GEMM is fused with the quantization
// that the second one needs, so the hidden activation is never materialized).
//
//   epi 1, FC1 forward:  acc = Q(X) Q(R1)^T + L1 U1;  h = bf16(acc + b1) (saved
//                        for the backward);  a = GELU_tanh(h) in fp32;
//                        Q(a) (FC2's 4-bit input);  L2 = bf16(bf16(a) D2)
//   epi 2, FC2 dX:       acc = Q(G) Q(R2) + P2 D2^T  (= d_a);
//                        d_h = bf16(acc GELU'(h)) (saved for dB1);  Q(d_h)
//                        (FC1's 4-bit gradient);  P1 = bf16(d_h U1^T)
//
// The main loop is the single-CTA FP4 GEMM's (gemm_fp4.cu): 128 x 256 output
// tiles, TMA code boxes per 256-wide K-block, scale warps writing the block
// scales into TMEM, the low-rank blocks accumulated by bf16 MMAs.  What is new
// is the epilogue's low-rank projection T Wp (T = bf16(a) or d_h) -- a
// reduction over the N columns of the GEMM, i.e. across output tiles:
//   * a CTA walks units: N tiles [sp*per, +per) of one 128-row tile, so that
//     the projection of a unit's tiles accumulates in a TMEM accumulator;
//   * per tile the epilogue writes T [128 x 256] into shared memory (four
//     128-byte-swizzled [128 x 64] chunks) and the MMA warp multiplies it with
//     Wp's 256 rows (two pipeline stages of the TMA ring) on the bf16 tensor
//     cores -- issued after the next tile's main loop, so that the epilogue of
//     one tile overlaps the MMAs of the next;
//   * at the end of a unit its fp32 partial [128, RP] goes to global memory;
//     the last unit of a 128-row tile (a counter) sums the partials in split
//     order (deterministic) and rounds once to bf16.
// Shared memory: three 48 KB stages + the 64 KB T buffer.  TMEM: the 256-column
// accumulator, two 48-column scale slots (a stage uses slot g % 2, rewritten
// once the MMAs of stage g - 2 are done) and the projection accumulator.
//
// Warp roles: warp 0 lane 0 producer; warp 1 TMEM owner, lane 0 issues the
// MMAs; warps 4..11 epilogue (warp w: TMEM lanes 32 (w % 4).., columns
// 128 ((w - 4) / 4).. of the tile); warps 12..15 scale warps.
#include "common.cuh"
#include "kernels.h"

namespace ft {

namespace {

constexpr int kMlStages = 3;
constexpr int kMlThreads = 512;
constexpr int kMlBN = 256;
constexpr uint32_t kMlA = 128 * 128;                  // A codes / A2 bf16 tile
constexpr uint32_t kMlB = kMlBN * 128;                // B codes / B2 bf16 tile / projection weight
constexpr uint32_t kMlStage = kMlA + kMlB;            // 48 KB
constexpr uint32_t kMlT = 4 * 128 * 128;              // T: four [128 x 64] bf16 chunks
constexpr uint32_t kMlTail = 512;
constexpr uint32_t kMlSmem = 1024 + kMlStages * kMlStage + kMlT + kMlTail;
constexpr int kMlSfSlots = 2;
constexpr uint32_t kMlSfCols = 16 + 32;               // A's 4 k-steps x 4, B's 4 k-steps x 2 chunks x 4
constexpr uint32_t kMlProjCol = kMlBN + kMlSfSlots * kMlSfCols;
constexpr int kMlProjStages = 2;                      // Wp's 256 rows: two stages of two 64-row chunks
static_assert(kMlSmem <= 232448, "shared memory budget");
static_assert(kMlProjCol + 128 <= 512, "TMEM budget");

__device__ __forceinline__ uint32_t ml_pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// Maximum of a non-negative float over the 16 lanes of this lane's half-warp.
__device__ __forceinline__ float max16_half(float a, int lane) {
  const unsigned mask = lane < 16 ? 0x0000FFFFu : 0xFFFF0000u;
  return __uint_as_float(__reduce_max_sync(mask, __float_as_uint(a)));
}

}  // namespace

template <int EPI>
__global__ void __launch_bounds__(kMlThreads, 1)
    gemm_mlp_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                    const __grid_constant__ CUtensorMap tmW, const MlpGemmParams mp) {
  const GemmParams& p = mp.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* tbuf = smem + kMlStages * kMlStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(tbuf + kMlT);
  uint64_t* empty = full + kMlStages;
  uint64_t* sf_full = empty + kMlStages;        // [kMlSfSlots] scale warps -> MMA
  uint64_t* sf_empty = sf_full + kMlSfSlots;    // [kMlSfSlots] MMAs that read the slot are done
  uint64_t* acc_full = sf_empty + kMlSfSlots;   // MMA -> epilogue: tile accumulated
  uint64_t* acc_empty = acc_full + 1;           // epilogue -> MMA: accumulator read out
  uint64_t* t_full = acc_empty + 1;             // epilogue -> MMA: T written
  uint64_t* t_empty = t_full + 1;               // MMA -> epilogue: T's projection done
  uint64_t* mma_done = t_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* s_last = abort_flag + 1;
  volatile int* abortp = abort_flag;
  static_assert((2 * kMlStages + 2 * kMlSfSlots + 5) * 8 + 16 <= kMlTail, "barriers and flags fit the tail");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int KB = (p.K + 255) / 256;       // FP4 K-blocks
  const int KS = (p.K + 63) / 64;         // 64-wide k-steps: scale blocks per 128-row chunk
  const int EB = (p.R2 + 63) / 64;        // bf16 low-rank blocks
  const int TM = KB + EB;                 // main stages per tile
  const int tiles_n = (p.N + kMlBN - 1) / kMlBN;
  const int units = ((p.M + 127) / 128) * mp.nsplit;
  const int nchunk_b = (p.N + 127) / 128;
  const int RP = mp.RP;
  const int NB = (RP + 63) / 64;          // 64-column boxes of an MN-major Wp row block
  const int NP = mp.wp_mn_major ? 64 * NB : RP;   // N of the projection MMA (padded columns are zero)
  const int KSo = (p.N + 63) / 64;        // k-steps of Q(T)'s MMA-ready scale layout (cols = N)

  if (threadIdx.x == 0) {
    for (int s = 0; s < kMlStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int s = 0; s < kMlSfSlots; ++s) {
      mbar_init(&sf_full[s], 4);
      mbar_init(&sf_empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);
    mbar_init(t_full, 8);
    mbar_init(t_empty, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    tma_prefetch(&tmW);
    if (EB) {
      tma_prefetch(&tmA2);
      tma_prefetch(&tmB2);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait_prior();

  if (warp == 0) {
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      int prev_n0 = -1;
      // one ring stage: wait for the slot, then issue `issue(st, bar)`
      auto stage = [&](auto&& issue) -> bool {
        const int s = g % kMlStages;
        if (!mbar_wait(&empty[s], ((g / kMlStages) & 1) ^ 1, p.status, abortp)) return false;
        issue(smem + s * kMlStage, &full[s]);
        ++g;
        return true;
      };
      // the projection weight's rows n0 .. n0 + 255, chunks 2 ps, 2 ps + 1
      auto proj_stages = [&](int n0) -> bool {
        for (int ps = 0; ps < kMlProjStages; ++ps) {
          const bool okp = stage([&](uint8_t* st, uint64_t* bar) {
            if (mp.wp_mn_major) {   // D2 [N, RP]: boxes of 64 rows x 64 columns
              mbar_arrive_expect_tx(bar, 2u * NB * 8192u);
              for (int kc = 0; kc < 2; ++kc)
                for (int nb = 0; nb < NB; ++nb)
                  tma_load_2d(st + (kc * NB + nb) * 8192, &tmW, bar, 64 * nb, n0 + 64 * (2 * ps + kc));
            } else {                // U1 [RP, N]: boxes of RP rows x 64 columns
              mbar_arrive_expect_tx(bar, 2u * static_cast<uint32_t>(RP) * 128u);
              for (int kc = 0; kc < 2; ++kc)
                tma_load_2d(st + kc * RP * 128, &tmW, bar, n0 + 64 * (2 * ps + kc), 0);
            }
          });
          if (!okp) return false;
        }
        return true;
      };
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int m0 = (u / mp.nsplit) * 128, sp = u % mp.nsplit;
        const int nhi = min(tiles_n, (sp + 1) * mp.per);
        for (int nt = sp * mp.per; nt < nhi && ok; ++nt) {
          const int n0 = nt * kMlBN;
          for (int i = 0; i < TM && ok; ++i) {
            ok = stage([&](uint8_t* st, uint64_t* bar) {
              if (i < KB) {
                mbar_arrive_expect_tx(bar, kMlA + kMlB);
                tma_load_2d(st, &tmA, bar, i * 128, m0);
                tma_load_2d(st + kMlA, &tmB, bar, i * 128, n0);
              } else {
                const int e = i - KB;
                mbar_arrive_expect_tx(bar, kMlA + kMlB);
                tma_load_2d(st, &tmA2, bar, e * 64, m0);
                if (p.b2_mn_major) {
                  for (int c = 0; c < kMlBN / 64; ++c) tma_load_2d(st + kMlA + 8192 * c, &tmB2, bar, n0 + 64 * c, e * 64);
                } else {
                  tma_load_2d(st + kMlA, &tmB2, bar, e * 64, n0);
                }
              }
            });
          }
          if (ok && prev_n0 >= 0) ok = proj_stages(prev_n0);
          prev_n0 = n0;
        }
      }
      if (ok && prev_n0 >= 0) ok = proj_stages(prev_n0);
      if (*abortp) {  // let copies already in flight land before the CTA exits
        for (int j = max(0, g - kMlStages); j < g; ++j)
          mbar_wait_drain(&full[j % kMlStages], (j / kMlStages) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc4 = idesc_fp4_block16(128, kMlBN);
      const uint32_t idesc16 = idesc_bf16(128, kMlBN, false, p.b2_mn_major != 0);
      const uint32_t idescP = idesc_bf16(128, NP, false, mp.wp_mn_major != 0);
      const uint32_t tb = smem_u32(tbuf);
      int g = 0, j = 0;
      bool ok = true, have_prev = false, prev_first = false;
      // wait for ring stage g and its scale slot
      auto take = [&](int& s, int& sl) -> bool {
        s = g % kMlStages;
        sl = g % kMlSfSlots;
        return mbar_wait(&full[s], (g / kMlStages) & 1, p.status, abortp) &&
               mbar_wait(&sf_full[sl], (g / kMlSfSlots) & 1, p.status, abortp);
      };
      auto release = [&](int s, int sl) {
        tc_commit(&empty[s]);
        tc_commit(&sf_empty[sl]);
        ++g;
      };
      // projection of the previous tile: T (written by the epilogue) times Wp
      auto project = [&](int jt, bool first_of_unit) -> bool {
        if (!mbar_wait(t_full, jt & 1, p.status, abortp)) return false;
        for (int ps = 0; ps < kMlProjStages; ++ps) {
          int s, sl;
          if (!take(s, sl)) return false;
          tc_fence_after();
          const uint32_t w_addr = smem_u32(smem + s * kMlStage);
          for (int kc = 0; kc < 2; ++kc) {
            const uint32_t t_addr = tb + (2 * ps + kc) * 16384;
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const uint64_t bdesc = mp.wp_mn_major
                                         ? desc_mnmajor_sw128(w_addr + kc * NB * 8192 + 2048 * t, 8192)
                                         : desc_kmajor_sw128(w_addr + kc * RP * 128 + 32 * t);
              const bool fresh = first_of_unit && ps == 0 && kc == 0 && t == 0;
              mma_bf16(tmem + kMlProjCol, desc_kmajor_sw128(t_addr + 32 * t), bdesc, idescP, fresh ? 0u : 1u);
            }
          }
          release(s, sl);
        }
        tc_commit(t_empty);
        return true;
      };
      for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
        const int sp = u % mp.nsplit;
        const int nlo = sp * mp.per, nhi = min(tiles_n, (sp + 1) * mp.per);
        for (int nt = nlo; nt < nhi && ok; ++nt, ++j) {
          if (j > 0 && !mbar_wait(acc_empty, (j - 1) & 1, p.status, abortp)) {
            ok = false;
            break;
          }
          tc_fence_after();
          for (int i = 0; i < TM; ++i) {
            int s, sl;
            if (!take(s, sl)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(smem + s * kMlStage);
            const uint32_t b_addr = a_addr + kMlA;
            if (i < KB) {
              const int nks = min(4, KS - 4 * i);
              const uint32_t sf_col = kMlBN + sl * kMlSfCols;
              for (int t = 0; t < nks; ++t)
                mma_fp4_block16(tmem, desc_kmajor_sw128(a_addr + 32 * t), desc_kmajor_sw128(b_addr + 32 * t), idesc4,
                                tmem + sf_col + 4 * t, tmem + sf_col + 16 + 8 * t, (i | t) != 0 ? 1u : 0u);
            } else {
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                const uint64_t bdesc =
                    p.b2_mn_major ? desc_mnmajor_sw128(b_addr + 2048 * t, 8192) : desc_kmajor_sw128(b_addr + 32 * t);
                mma_bf16(tmem, desc_kmajor_sw128(a_addr + 32 * t), bdesc, idesc16, 1u);
              }
            }
            release(s, sl);
          }
          if (!ok) break;
          tc_commit(acc_full);
          if (have_prev && !project(j - 1, prev_first)) {
            ok = false;
            break;
          }
          have_prev = true;
          prev_first = nt == nlo;
        }
      }
      if (ok && have_prev) project(j - 1, prev_first);
      tc_commit(mma_done);
      mbar_wait_drain(mma_done, 0, kWaitLimitNs);  // every MMA done before TMEM can be freed
    }
  } else if (warp >= 12) {
    // Scale warp of TMEM lane quadrant q: for an FP4 stage, A's k-step t at
    // columns 4t..4t+3 of the slot (the MMA reads 4t+q here), B's k-step t,
    // chunk c at 16+8t+4c..+3; stages without scales only pass the slot on.
    const int q = warp & 3;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
    int g = 0;
    bool ok = true;
    auto fetch = [&](int mt, int nt, int i, uint32_t (&a)[4], uint32_t (&b)[32]) {
      const int nks = min(4, KS - 4 * i);
      const int nc = nt * 2;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        a[t] = 0u;
        if (t < nks)
          a[t] = __ldg(reinterpret_cast<const uint32_t*>(p.sfa + (static_cast<size_t>(mt) * KS + 4 * i + t) * 512 +
                                                         16 * lane + 4 * q));
      }
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          uint4 x = make_uint4(0u, 0u, 0u, 0u);   // zero scales past N (their codes are zero)
          if (t < nks && nc + c < nchunk_b)
            x = __ldg(reinterpret_cast<const uint4*>(p.sfb + (static_cast<size_t>(nc + c) * KS + 4 * i + t) * 512 +
                                                     16 * lane));
          b[4 * (2 * t + c)] = x.x;
          b[4 * (2 * t + c) + 1] = x.y;
          b[4 * (2 * t + c) + 2] = x.z;
          b[4 * (2 * t + c) + 3] = x.w;
        }
      }
    };
    // pass ring stage g: wait for its scale slot, write the scales (if any), hand it to the MMA
    auto put = [&](const uint32_t* a, const uint32_t* b) -> bool {
      const int sl = g % kMlSfSlots;
      bool okw = true;
      if (lane == 0) okw = mbar_wait(&sf_empty[sl], ((g / kMlSfSlots) & 1) ^ 1, p.status, abortp);
      okw = __shfl_sync(0xFFFFFFFFu, okw ? 1 : 0, 0) != 0;
      if (!okw) return false;
      tc_fence_after();
      if (a) {
        const uint32_t sf_col = kMlBN + sl * kMlSfCols;
        uint32_t a16[16], b32[32];
#pragma unroll
        for (int e = 0; e < 16; ++e) a16[e] = a[e >> 2];
#pragma unroll
        for (int e = 0; e < 32; ++e) b32[e] = b[e];
        tmem_st_32x32b_x16(trow + sf_col, a16);
        tmem_st_32x32b_x32(trow + sf_col + 16, b32);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_full[sl]);
      ++g;
      return true;
    };
    bool have_prev = false;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int mt = u / mp.nsplit, sp = u % mp.nsplit;
      const int nhi = min(tiles_n, (sp + 1) * mp.per);
      for (int nt = sp * mp.per; nt < nhi && ok; ++nt) {
        // the tile's FP4 stages, the next one's loads in flight while one is stored
        uint32_t a0[4], b0[32], a1[4], b1[32];
        if (KB > 0) fetch(mt, nt, 0, a0, b0);
        for (int i = 0; i < KB && ok; i += 2) {
          if (i + 1 < KB) fetch(mt, nt, i + 1, a1, b1);
          ok = put(a0, b0);
          if (!ok || i + 1 >= KB) break;
          if (i + 2 < KB) fetch(mt, nt, i + 2, a0, b0);
          ok = put(a1, b1);
        }
        for (int i = 0; i < EB && ok; ++i) ok = put(nullptr, nullptr);
        for (int i = 0; have_prev && i < kMlProjStages && ok; ++i) ok = put(nullptr, nullptr);
        have_prev = true;
      }
    }
    for (int i = 0; have_prev && i < kMlProjStages && ok; ++i) ok = put(nullptr, nullptr);
  } else if (warp >= 4) {
    // ---- epilogue: 8 warps; warp w owns rows 32 q.. (q = w % 4) of the tile and
    // columns c_lo .. c_lo + 127.  The eight warps leave together (named_bar_or).
    const int q = warp & 3;
    const int c_lo = ((warp - 4) >> 2) * 128;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c_lo);
    const uint32_t paddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + kMlProjCol;
    const int r_loc = 32 * q + lane;                        // this lane's row of the tile
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(p.bias);
    const int half = RP / 2;                                // projection columns of this warp's half
    const int pc0 = ((warp - 4) >> 2) * half;
    int j = 0;
    int prev_m0 = 0, prev_sp = 0;
    bool have_prev = false, prev_last = false;

    // The unit's projection accumulator -> fp32 partial; the last unit of the
    // 128-row tile sums all partials in split order and rounds to bf16.
    auto finish_unit = [&](int m0, int sp) {
      const int row = m0 + r_loc;
      for (int c = 0; c < half; c += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(paddr + pc0 + c, v);
        tmem_ld_wait();
        if (row < p.M) {
          float4* dst = reinterpret_cast<float4*>(mp.part + (static_cast<long long>(sp) * p.M + row) * RP + pc0 + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)   // this warp's columns only (half is a multiple of 8)
            if (c + 4 * e < half)
              dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                   __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
      // one thread publishes this unit's partial (ordered before it by the
      // barrier) with a gpu-scope fence before its counter increment; the last
      // unit's fence after the increment orders its reads after all others
      named_bar_sync(1, 256);
      if (threadIdx.x == 128) {
        __threadfence();
        const int prev = atomicAdd(&mp.counters[m0 / 128], 1);
        __threadfence();
        *s_last = (prev == mp.nsplit - 1);
      }
      named_bar_sync(1, 256);
      if (*s_last) {
        const int c4 = RP / 4;
        for (int idx = static_cast<int>(threadIdx.x) - 128; idx < 128 * c4; idx += 256) {
          const int rr = m0 + idx / c4, cc = 4 * (idx % c4);
          if (rr >= p.M) continue;
          float4 acc = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
          for (int s2 = 0; s2 < mp.nsplit; ++s2) {
            const float4 x = __ldcg(reinterpret_cast<const float4*>(mp.part + (static_cast<long long>(s2) * p.M + rr) * RP + cc));
            acc.x += x.x;
            acc.y += x.y;
            acc.z += x.z;
            acc.w += x.w;
          }
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(mp.proj_out) + static_cast<long long>(rr) * RP + cc) =
              make_uint2(ml_pack_bf16x2(acc.x, acc.y), ml_pack_bf16x2(acc.z, acc.w));
        }
        if (threadIdx.x == 128) mp.counters[m0 / 128] = 0;
      }
    };

    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int m0 = (u / mp.nsplit) * 128, sp = u % mp.nsplit;
      const int nhi = min(tiles_n, (sp + 1) * mp.per);
      for (int nt = sp * mp.per; nt < nhi; ++nt, ++j) {
        const int n0 = nt * kMlBN + c_lo;                   // this warp's first column
        const int row = m0 + r_loc;
        const bool row_ok = row < p.M;
        uint32_t hw[64];                                    // the warp's 128 columns of h / d_h (bf16 pairs)
        if (EPI == 2) {                                     // h, loaded while the tile's MMAs run
          const uint4* hp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(mp.h) +
                                                           static_cast<long long>(row) * p.N + n0);
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            const uint4 x = (row_ok && n0 + 8 * k < p.N) ? hp[k] : make_uint4(0u, 0u, 0u, 0u);
            hw[4 * k] = x.x;
            hw[4 * k + 1] = x.y;
            hw[4 * k + 2] = x.z;
            hw[4 * k + 3] = x.w;
          }
        }
        const bool got = mbar_wait(acc_full, j & 1, p.status, abortp);
        if (named_bar_or(1, 256, !got || *abortp)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (EPI == 1) {
          // h = bf16(acc + b1), 32 columns per round
#pragma unroll
          for (int rd = 0; rd < 4; ++rd) {
            uint32_t v[2][16];
            tmem_ld_32x32b_x16(taddr + 32 * rd, v[0]);
            tmem_ld_32x32b_x16(taddr + 32 * rd + 16, v[1]);
            uint4 bw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              bw[k] = make_uint4(0u, 0u, 0u, 0u);
              if (bias && n0 + 32 * rd + 8 * k < p.N) bw[k] = __ldg(reinterpret_cast<const uint4*>(bias + n0 + 32 * rd) + k);
            }
            tmem_ld_wait();
#pragma unroll
            for (int k = 0; k < 2; ++k) {
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                const uint4 b4 = bw[2 * k + e / 4];
                const uint32_t bb = (e & 3) == 0 ? b4.x : (e & 3) == 1 ? b4.y : (e & 3) == 2 ? b4.z : b4.w;
                hw[16 * rd + 8 * k + e] = ml_pack_bf16x2(__uint_as_float(v[k][2 * e]) + bf16_bits_to_f32(bb & 0xFFFFu),
                                                         __uint_as_float(v[k][2 * e + 1]) + bf16_bits_to_f32(bb >> 16));
              }
            }
          }
        } else {
          // d_h = bf16(acc * GELU'(h)), 16 columns per round, in place of h
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint32_t v[16];
            tmem_ld_32x32b_x16(taddr + 16 * c, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float g0, d0, g1, d1;
              gelu_tanh_and_grad(bf16_bits_to_f32(hw[8 * c + e] & 0xFFFFu), &g0, &d0);
              gelu_tanh_and_grad(bf16_bits_to_f32(hw[8 * c + e] >> 16), &g1, &d1);
              hw[8 * c + e] = ml_pack_bf16x2(__uint_as_float(v[2 * e]) * d0, __uint_as_float(v[2 * e + 1]) * d1);
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        // h (FC1) or d_h (FC2 dX): each lane stores its row, 32-byte pieces
        if (row_ok) {
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(mp.out_h) + static_cast<long long>(row) * p.N + n0);
#pragma unroll
          for (int k = 0; k < 16; ++k)
            if (n0 + 8 * k < p.N) dst[k] = make_uint4(hw[4 * k], hw[4 * k + 1], hw[4 * k + 2], hw[4 * k + 3]);
        }
        // T is free once the previous tile's projection is done; a unit that
        // ended with the previous tile hands its accumulator on first
        if (have_prev) {
          const bool freed = mbar_wait(t_empty, (j - 1) & 1, p.status, abortp);
          if (named_bar_or(1, 256, !freed || *abortp)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (prev_last) finish_unit(prev_m0, prev_sp);
        }
        // per 16-column block: Q(.) codes and scales, T = the projection's input
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const int col = n0 + 16 * c;
          float v[16];
          uint32_t tw[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            v[2 * e] = bf16_bits_to_f32(hw[8 * c + e] & 0xFFFFu);
            v[2 * e + 1] = bf16_bits_to_f32(hw[8 * c + e] >> 16);
          }
          if (EPI == 1) {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = gelu_tanh(v[e]);
#pragma unroll
            for (int e = 0; e < 8; ++e) tw[e] = ml_pack_bf16x2(v[2 * e], v[2 * e + 1]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) tw[e] = hw[8 * c + e];
          }
          const bool inside = row_ok && col < p.N;
          if (!inside) {
#pragma unroll
            for (int e = 0; e < 16; ++e) v[e] = 0.0f;
#pragma unroll
            for (int e = 0; e < 8; ++e) tw[e] = 0u;
          }
          float m = 0.0f;
#pragma unroll
          for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(v[e]));
          const float amax = max16_half(m, lane);           // the 16x16 block: 16 rows = 16 lanes
          uint32_t packed[2], sc;
          if (EPI == 1)
            quantize_block_row_f32<16>(v, amax, packed, &sc);
          else
            quantize_block_row<16>(v, amax, packed, &sc);
          if (inside) {
            *reinterpret_cast<uint2*>(mp.q_codes + static_cast<long long>(row) * (p.N / 2) + col / 2) =
                make_uint2(packed[0], packed[1]);
            if ((lane & 15) == 0)
              mp.q_scales[static_cast<long long>(row / 16) * (p.N / 16) + col / 16] = static_cast<uint8_t>(sc);
            if (EPI == 1 && mp.dbg) {
              float4* dst = reinterpret_cast<float4*>(mp.dbg + static_cast<long long>(row) * p.N + col);
#pragma unroll
              for (int e = 0; e < 4; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
            }
          }
          // MMA-ready copy: every row of the block; groups past N inside the last
          // 64-column step and rows past M hold 0
          if (mp.q_sf && col / 16 < 4 * KSo)
            mp.q_sf[sf_mma_offset(row, col / 16, KSo)] = static_cast<uint8_t>(inside ? sc : 0u);
          // T chunk (c_lo + 16 c) / 64, 16-byte units u, u + 1 of row r_loc, 128-byte swizzle
          const int cl = c_lo + 16 * c;
          uint8_t* trow = tbuf + (cl / 64) * 16384 + r_loc * 128;
          const int u0 = (cl % 64) / 8;
          *reinterpret_cast<uint4*>(trow + ((u0 ^ (r_loc & 7)) << 4)) = make_uint4(tw[0], tw[1], tw[2], tw[3]);
          *reinterpret_cast<uint4*>(trow + (((u0 + 1) ^ (r_loc & 7)) << 4)) = make_uint4(tw[4], tw[5], tw[6], tw[7]);
        }
        fence_proxy_async_smem();   // T's generic stores -> the tensor cores' reads
        tc_fence_before();          // the projection accumulator was read out before
        __syncwarp();
        if (lane == 0) mbar_arrive(t_full);
        have_prev = true;
        prev_last = nt == nhi - 1;
        prev_m0 = m0;
        prev_sp = sp;
      }
    }
    if (ok && have_prev) {
      const bool freed = mbar_wait(t_empty, (j - 1) & 1, p.status, abortp);
      if (!named_bar_or(1, 256, !freed || *abortp)) {
        tc_fence_after();
        finish_unit(prev_m0, prev_sp);
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

cudaError_t launch_gemm_mlp(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmA2,
                            const CUtensorMap& tmB2, const CUtensorMap& tmW, const MlpGemmParams& p, int num_sms,
                            cudaStream_t stream) {
  if ((p.epi != 1 && p.epi != 2) || p.RP < 16 || p.RP > 128 || p.RP % 16 || p.nsplit < 1 || p.per < 1)
    return cudaErrorInvalidValue;
  auto kernel = p.epi == 1 ? gemm_mlp_kernel<1> : gemm_mlp_kernel<2>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kMlSmem));
  if (e != cudaSuccess) return e;
  const int units = ((p.g.M + 127) / 128) * p.nsplit;
  const int grid = units < num_sms ? units : num_sms;
  return launch_pdl(kernel, dim3(grid), dim3(kMlThreads), kMlSmem, stream, tmA, tmB, tmA2, tmB2, tmW, p);
}

}  // namespace ft
