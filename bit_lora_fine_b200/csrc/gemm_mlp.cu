// The MLP's block-scaled FP4 GEMMs with their fused epilogues (FourTune §3.3
// "MLP Fusion": the first fully connected GEMM is fused with the quantization
// that the second one needs, so the hidden activation is never materialized).
//
//   epi 1, FC1 forward:  acc = Q(X) Q(R1)^T + L1 U1;  h = bf16(acc + b1) (saved
//                        for the backward);  a = GELU_tanh(h) in fp32;  FC2's
//                        input bf16(a) for all three of its branches:
//                        Q(bf16(a)) and L2 = bf16(bf16(a) D2)
//   epi 2, FC2 dX:       acc = Q(G) Q(R2) + P2 D2^T  (= d_a);
//                        d_h = bf16(acc GELU'(h)) (saved for dB1);  Q(d_h)
//                        (FC1's 4-bit gradient);  P1 = bf16(d_h U1^T)
//
// The main loop is the single-CTA FP4 GEMM's (gemm_fp4.cu): 128 x 256 output
// tiles, TMA code boxes per 256-wide K-block, scale warps writing the block
// scales into TMEM (from shared memory here: each K-block's scale blocks come
// into its stage by bulk copies), the low-rank blocks accumulated by bf16 MMAs.  What is new
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
//     launch_proj_reduce then sums the partials in split order
//     (deterministic) and rounds once to bf16, over all row tiles at once (a
//     last-unit sum inside this kernel fell on a few CTAs: in rounds of
//     lockstep units the same CTA finishes last for many row tiles).
// Shared memory: three 54 KB stages (codes or bf16 tiles, and the K-block's
// MMA-ready scale blocks: the scale warps read them from there, so that large
// K keeps three stages of scales in flight without registers) and the 64 KB T
// buffer (which also stages h / d_h for whole-row stores).  TMEM: the
// 256-column accumulator, two 48-column scale slots (a stage uses slot g % 2,
// rewritten once the MMAs of stage g - 2 are done) and the projection
// accumulator.
//
// Warp roles: warp 0 lane 0 producer; warp 1 TMEM owner, lane 0 issues the
// MMAs; warps 2..17 epilogue (warp w: TMEM lanes 32 (w % 4).., columns
// 64 ((w - 2) / 4).. of the tile -- sixteen warps, so that the GELU and
// quantizer arithmetic of one tile hides its latencies while the next tile's
// MMAs run); warps 18..21 scale warps.  704 threads leave 80 registers per
// thread.
#include "common.cuh"
#include "kernels.h"

namespace ft {

namespace {

constexpr int kMlStages = 3;
constexpr int kMlEpiWarps = 16;
constexpr int kMlEpiThreads = 32 * kMlEpiWarps;
constexpr int kMlEpi0 = 2;                            // first epilogue warp
constexpr int kMlScale0 = kMlEpi0 + kMlEpiWarps;      // first scale warp
constexpr int kMlThreads = 32 * (kMlScale0 + 4);      // 704
// Registers are allocated per warp from the register file quarter of the SM
// sub-partition the warp runs on (16384 each): 22 warps put 6 on a quarter.
constexpr int kMlMaxReg = 80;
static_assert(((kMlThreads / 32 + 3) / 4) * 32 * kMlMaxReg <= 16384, "registers fit each sub-partition");
constexpr int kMlBN = 256;
constexpr uint32_t kMlA = 128 * 128;                  // A codes / A2 bf16 tile
constexpr uint32_t kMlB = kMlBN * 128;                // B codes / B2 bf16 tile / projection weight
constexpr uint32_t kMlSfA = 4 * 512;                  // A's scale blocks of a K-block (4 k-steps)
constexpr uint32_t kMlSfB = 2 * 4 * 512;              // B's: [128-row chunk][k-step][512 B]
constexpr uint32_t kMlStage = kMlA + kMlB + kMlSfA + kMlSfB;   // 54 KB
constexpr uint32_t kMlT = 4 * 128 * 128;              // T: four [128 x 64] bf16 chunks
constexpr uint32_t kMlTail = 512;
// no alignment slack: the dynamic shared memory starts 1024-byte aligned (the
// kernel checks it and refuses to run otherwise)
constexpr uint32_t kMlSmem = kMlStages * kMlStage + kMlT + kMlTail;
constexpr int kMlSfSlots = 2;
constexpr uint32_t kMlSfCols = 16 + 32;               // A's 4 k-steps x 4, B's 4 k-steps x 2 chunks x 4
constexpr uint32_t kMlProjCol = kMlBN + kMlSfSlots * kMlSfCols;
constexpr int kMlProjStages = 2;                      // Wp's 256 rows: two stages of two 64-row chunks
static_assert(kMlSmem <= 232448, "shared memory budget");
static_assert(kMlStage % 1024 == 0, "stages keep the 1024-byte alignment of the swizzled tiles");
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
__global__ void __maxnreg__(kMlMaxReg)
    gemm_mlp_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                    const __grid_constant__ CUtensorMap tmW, const MlpGemmParams mp) {
  const GemmParams& p = mp.g;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {   // uniform: every thread leaves before any barrier or TMEM use
    if (threadIdx.x == 0 && blockIdx.x == 0 && mp.g.status) atomicCAS(mp.g.status, 0, kDevUnsupported);
    return;
  }
  uint8_t* smem = smem_raw;
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
    mbar_init(acc_empty, kMlEpiWarps);
    mbar_init(t_full, kMlEpiWarps);
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
                // codes by TMA, the K-block's MMA-ready scale blocks by bulk copies
                // (nks 512-byte blocks each for A and for B's 128-row chunks)
                const int nks = min(4, KS - 4 * i);
                const uint32_t sfbytes = static_cast<uint32_t>(nks) * 512u;
                const int nb = (n0 / 128 + 1 < nchunk_b) ? 2 : 1;
                mbar_arrive_expect_tx(bar, kMlA + kMlB + sfbytes * static_cast<uint32_t>(1 + nb));
                tma_load_2d(st, &tmA, bar, i * 128, m0);
                tma_load_2d(st + kMlA, &tmB, bar, i * 128, n0);
                bulk_load(st + kMlA + kMlB, p.sfa + (static_cast<size_t>(m0 / 128) * KS + 4 * i) * 512, sfbytes, bar);
                for (int c = 0; c < nb; ++c)
                  bulk_load(st + kMlA + kMlB + kMlSfA + c * 2048,
                            p.sfb + (static_cast<size_t>(n0 / 128 + c) * KS + 4 * i) * 512, sfbytes, bar);
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
  } else if (warp >= kMlScale0) {
    // Scale warp of TMEM lane quadrant q: for an FP4 stage, A's k-step t at
    // columns 4t..4t+3 of the slot (the MMA reads 4t+q here), B's k-step t,
    // chunk c at 16+8t+4c..+3; stages without scales only pass the slot on.
    const int q = warp & 3;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
    int g = 0;
    bool ok = true;
    // stage g's scale blocks, from the stage once its copies have landed
    auto fetch = [&](int nt, int i, uint32_t (&a)[4], uint32_t (&b)[32]) -> bool {
      const int s = g % kMlStages;
      bool okw = true;
      if (lane == 0) okw = mbar_wait(&full[s], (g / kMlStages) & 1, p.status, abortp);
      if (__shfl_sync(0xFFFFFFFFu, okw ? 1 : 0, 0) == 0) return false;
      const uint8_t* sf = smem + s * kMlStage + kMlA + kMlB;
      const int nks = min(4, KS - 4 * i);
      const int nc = nt * 2;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        a[t] = t < nks ? *reinterpret_cast<const uint32_t*>(sf + t * 512 + 16 * lane + 4 * q) : 0u;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          uint4 x = make_uint4(0u, 0u, 0u, 0u);   // zero scales past N (their codes are zero)
          if (t < nks && nc + c < nchunk_b)
            x = *reinterpret_cast<const uint4*>(sf + kMlSfA + c * 2048 + t * 512 + 16 * lane);
          b[4 * (2 * t + c)] = x.x;
          b[4 * (2 * t + c) + 1] = x.y;
          b[4 * (2 * t + c) + 2] = x.z;
          b[4 * (2 * t + c) + 3] = x.w;
        }
      }
      return true;
    };
    // pass ring stage g: wait for its scale slot, write the scales (if any), hand it to the MMA
    auto put = [&](bool has, const uint32_t (&a)[4], const uint32_t (&b)[32]) -> bool {
      const int sl = g % kMlSfSlots;
      bool okw = true;
      if (lane == 0) okw = mbar_wait(&sf_empty[sl], ((g / kMlSfSlots) & 1) ^ 1, p.status, abortp);
      okw = __shfl_sync(0xFFFFFFFFu, okw ? 1 : 0, 0) != 0;
      if (!okw) return false;
      tc_fence_after();
      if (has) {
        const uint32_t sf_col = kMlBN + sl * kMlSfCols;
#pragma unroll
        for (int t = 0; t < 4; ++t) tmem_st_32x32b_x4_rep(trow + sf_col + 4 * t, a[t]);
        tmem_st_32x32b_x32(trow + sf_col + 16, b);
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
      const int sp = u % mp.nsplit;
      const int nhi = min(tiles_n, (sp + 1) * mp.per);
      for (int nt = sp * mp.per; nt < nhi && ok; ++nt) {
        // the tile's FP4 stages: each stage's scale blocks arrive with its codes
        uint32_t a0[4], b0[32];
        for (int i = 0; i < KB && ok; ++i) ok = fetch(nt, i, a0, b0) && put(true, a0, b0);
        for (int i = 0; i < EB && ok; ++i) ok = put(false, a0, b0);
        for (int i = 0; have_prev && i < kMlProjStages && ok; ++i) ok = put(false, a0, b0);
        have_prev = true;
      }
    }
    {
      uint32_t a0[4] = {0u, 0u, 0u, 0u}, b0[32];
      for (int i = 0; have_prev && i < kMlProjStages && ok; ++i) ok = put(false, a0, b0);
    }
  } else if (warp >= kMlEpi0) {
    // ---- epilogue: 16 warps; warp w owns rows 32 q.. (q = w % 4: the TMEM lane
    // quadrant a warp may access) of the tile and columns c_lo .. c_lo + 63.  The
    // sixteen warps leave together (named_bar_or).
    const int q = warp & 3;
    const int cq = (warp - kMlEpi0) >> 2;
    const int c_lo = 64 * cq;
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c_lo);
    const uint32_t paddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + kMlProjCol;
    const int r_loc = 32 * q + lane;                        // this lane's row of the tile
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(p.bias);
    const int quarter = RP / 4;                             // projection columns of this warp (a multiple of 4)
    const int pc0 = cq * quarter;
    int j = 0;
    int prev_m0 = 0, prev_sp = 0;
    bool have_prev = false, prev_last = false;

    // The unit's projection accumulator -> its fp32 partial (the split-order
    // sum of all units' partials is launch_proj_reduce's)
    auto finish_unit = [&](int m0, int sp) {
      const int row = m0 + r_loc;
      for (int c = 0; c < quarter; c += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(paddr + pc0 + c, v);
        tmem_ld_wait();
        if (row < p.M) {
          float4* dst = reinterpret_cast<float4*>(mp.part + (static_cast<long long>(sp) * p.M + row) * RP + pc0 + c);
#pragma unroll
          for (int e = 0; e < 4; ++e)   // this warp's columns only
            if (c + 4 * e < quarter)
              dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                   __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
    };

    // this lane's row of T: chunk cq (the warp's 64 columns), 128-byte swizzled
    uint8_t* const t_row = tbuf + cq * 16384 + r_loc * 128;
    const int sw = r_loc & 7;
    bool ok = true;
    for (int u = blockIdx.x; u < units && ok; u += gridDim.x) {
      const int m0 = (u / mp.nsplit) * 128, sp = u % mp.nsplit;
      const int nhi = min(tiles_n, (sp + 1) * mp.per);
      for (int nt = sp * mp.per; nt < nhi; ++nt, ++j) {
        const int n0 = nt * kMlBN + c_lo;                   // this warp's first column
        const int row = m0 + r_loc;
        const bool row_ok = row < p.M;
        // loaded while the tile's MMAs run: EPI 1 the bias of the warp's 64
        // columns (lane l < 8 holds columns n0 + 8 l .. + 7; shuffled out
        // below), EPI 2 the lane's row of h
        uint4 bq = make_uint4(0u, 0u, 0u, 0u);
        uint32_t hw[32];
        if (EPI == 1) {
          if (bias && n0 + 8 * (lane & 7) < p.N) bq = __ldg(reinterpret_cast<const uint4*>(bias + n0) + (lane & 7));
        } else {
          const uint4* hp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(mp.h) +
                                                           static_cast<long long>(row) * p.N + n0);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            const uint4 x = (row_ok && n0 + 8 * k < p.N) ? hp[k] : make_uint4(0u, 0u, 0u, 0u);
            hw[4 * k] = x.x;
            hw[4 * k + 1] = x.y;
            hw[4 * k + 2] = x.z;
            hw[4 * k + 3] = x.w;
          }
        }
        const bool got = mbar_wait(acc_full, j & 1, p.status, abortp);
        if (named_bar_or(1, kMlEpiThreads, !got || *abortp)) {
          ok = false;
          break;
        }
        // T is free once the previous tile's projection is done (it runs right
        // after this tile's main loop); a unit that ended with the previous
        // tile hands its projection accumulator on first
        if (have_prev) {
          const bool freed = mbar_wait(t_empty, (j - 1) & 1, p.status, abortp);
          if (named_bar_or(1, kMlEpiThreads, !freed || *abortp)) {
            ok = false;
            break;
          }
          if (prev_last) {
            tc_fence_after();
            finish_unit(prev_m0, prev_sp);
          }
        }
        tc_fence_after();
        // ---- phase 1, 16 columns at a time: the accumulator -> h = bf16(acc + b1)
        // (EPI 1) or d_h = bf16(acc GELU'(h)) (EPI 2), to global memory and to T
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {   // rolled: the epilogue's code stays small
          const int col = n0 + 16 * c;
          uint32_t v[16], w[8];
          tmem_ld_32x32b_x16(taddr + 16 * c, v);
          tmem_ld_wait();
          if (EPI == 1) {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const uint32_t part = (e & 3) == 0 ? bq.x : (e & 3) == 1 ? bq.y : (e & 3) == 2 ? bq.z : bq.w;
              const uint32_t bb = __shfl_sync(0xFFFFFFFFu, part, 2 * c + (e >> 2));
              w[e] = ml_pack_bf16x2(__uint_as_float(v[2 * e]) + bf16_bits_to_f32(bb & 0xFFFFu),
                                    __uint_as_float(v[2 * e + 1]) + bf16_bits_to_f32(bb >> 16));
            }
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              float g0, d0, g1, d1;
              const uint32_t hh = hw[e];
              gelu_tanh_and_grad(bf16_bits_to_f32(hh & 0xFFFFu), &g0, &d0);
              gelu_tanh_and_grad(bf16_bits_to_f32(hh >> 16), &g1, &d1);
              w[e] = ml_pack_bf16x2(__uint_as_float(v[2 * e]) * d0, __uint_as_float(v[2 * e + 1]) * d1);
            }
#pragma unroll
            for (int e = 0; e < 24; ++e) hw[e] = hw[e + 8];   // the next 16 columns to the front
          }
          if (EPI == 2 && !(row_ok && col < p.N)) {
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = 0u;   // T: zero outside the matrix
          }
          *reinterpret_cast<uint4*>(t_row + (((2 * c) ^ sw) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
          *reinterpret_cast<uint4*>(t_row + (((2 * c + 1) ^ sw) << 4)) = make_uint4(w[4], w[5], w[6], w[7]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);   // the next tile's MMAs may start
        // EPI 2: the next tile of the unit reads this lane's row of h 256 columns
        // on; pull its line into L2 now, so that the prefetch into registers at
        // the top of the next tile does not wait on HBM
        if (EPI == 2 && nt + 1 < nhi && row_ok && n0 + kMlBN < p.N)
          prefetch_l2(static_cast<const __nv_bfloat16*>(mp.h) + static_cast<long long>(row) * p.N + n0 + kMlBN);
        // h / d_h to global memory from T: the warp's 32 rows x 128 bytes, four
        // whole rows (512 contiguous-by-row bytes) per store
#pragma unroll 2
        for (int i = 0; i < 8; ++i) {
          const int rr = 32 * q + 4 * i + (lane >> 3), un = lane & 7;
          const uint4 x = *reinterpret_cast<const uint4*>(tbuf + cq * 16384 + rr * 128 + ((un ^ (rr & 7)) << 4));
          if (m0 + rr < p.M && n0 + 8 * un < p.N)
            *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(mp.out_h) + static_cast<long long>(m0 + rr) * p.N +
                                      n0 + 8 * un) = x;
        }
        // ---- phase 2, per 16-column block of T: (EPI 1: T = bf16(GELU(h)) in
        // place) the block's Q(T) codes and scale, T being the shared bf16 input
        // of the next layer's branches (bf16(a) or d_h)
        uint32_t sfw = 0u;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          const int col = n0 + 16 * c;
          const bool inside = row_ok && col < p.N;
          uint4* const tp0 = reinterpret_cast<uint4*>(t_row + (((2 * c) ^ sw) << 4));
          uint4* const tp1 = reinterpret_cast<uint4*>(t_row + (((2 * c + 1) ^ sw) << 4));
          const uint4 x0 = *tp0, x1 = *tp1;
          uint32_t tw[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
          if (EPI == 1) {
            float2* dbg = (mp.dbg && inside) ? reinterpret_cast<float2*>(mp.dbg + static_cast<long long>(row) * p.N + col)
                                             : nullptr;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const float a0 = gelu_tanh(bf16_bits_to_f32(tw[e] & 0xFFFFu));
              const float a1 = gelu_tanh(bf16_bits_to_f32(tw[e] >> 16));
              tw[e] = inside ? ml_pack_bf16x2(a0, a1) : 0u;
              if (dbg) dbg[e] = make_float2(a0, a1);
            }
            *tp0 = make_uint4(tw[0], tw[1], tw[2], tw[3]);
            *tp1 = make_uint4(tw[4], tw[5], tw[6], tw[7]);
          }
          float v[16];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            v[2 * e] = bf16_bits_to_f32(tw[e] & 0xFFFFu);
            v[2 * e + 1] = bf16_bits_to_f32(tw[e] >> 16);
          }
          float m = 0.0f;
#pragma unroll
          for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(v[e]));
          const float amax = max16_half(m, lane);           // the 16x16 block: 16 rows = 16 lanes
          uint32_t packed[2], sc;
          quantize_block_row<16>(v, amax, packed, &sc);      // bf16 values: the exact division-free path
          if (!inside) sc = 0u;
          sfw |= sc << (8 * c);
          if (inside) {
            *reinterpret_cast<uint2*>(mp.q_codes + static_cast<long long>(row) * (p.N / 2) + col / 2) =
                make_uint2(packed[0], packed[1]);
            if ((lane & 15) == 0)
              mp.q_scales[static_cast<long long>(row / 16) * (p.N / 16) + col / 16] = static_cast<uint8_t>(sc);
          }
        }
        // the MMA-ready copy of the scales: the warp's k-step, four scales of
        // this row in one word (rows past M and groups past N hold 0)
        if (mp.q_sf && n0 < 64 * KSo)
          *reinterpret_cast<uint32_t*>(mp.q_sf + sf_mma_offset(row, n0 / 16, KSo)) = sfw;
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
      if (!named_bar_or(1, kMlEpiThreads, !freed || *abortp)) {
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

namespace {
// out [M, RP] = bf16(sum over s in split order of part[s, M, RP]), one float4 a thread
__global__ void __launch_bounds__(256) proj_reduce_kernel(const float4* __restrict__ part, int nsplit, long long n4,
                                                          uint2* __restrict__ out) {
  pdl_launch_dependents();
  pdl_wait_prior();
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    float4 acc = __ldcs(part + i);
    for (int sp = 1; sp < nsplit; ++sp) {
      const float4 x = __ldcs(part + sp * n4 + i);
      acc.x += x.x;
      acc.y += x.y;
      acc.z += x.z;
      acc.w += x.w;
    }
    out[i] = make_uint2(ml_pack_bf16x2(acc.x, acc.y), ml_pack_bf16x2(acc.z, acc.w));
  }
}
}  // namespace

cudaError_t launch_proj_reduce(const float* part, int nsplit, int M, int RP, void* out, int num_sms,
                               cudaStream_t stream) {
  if (nsplit < 1 || M < 1 || RP % 4) return cudaErrorInvalidValue;
  const long long n4 = static_cast<long long>(M) * RP / 4;
  const long long want = (n4 + 255) / 256;
  const int grid = static_cast<int>(want < 4LL * num_sms ? want : 4LL * num_sms);
  return launch_pdl(proj_reduce_kernel, dim3(grid), dim3(256), 0, stream, reinterpret_cast<const float4*>(part),
                    nsplit, n4, static_cast<uint2*>(out));
}

cudaError_t launch_gemm_mlp(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmA2,
                            const CUtensorMap& tmB2, const CUtensorMap& tmW, const MlpGemmParams& p, int num_sms,
                            cudaStream_t stream) {
  if ((p.epi != 1 && p.epi != 2) || p.RP < 16 || p.RP > 128 || p.RP % 16 || p.nsplit < 1 || p.per < 1)
    return cudaErrorInvalidValue;
  auto kernel = p.epi == 1 ? gemm_mlp_kernel<1> : gemm_mlp_kernel<2>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kMlSmem));
  if (e != cudaSuccess) return e;
  const int units = ((p.g.M + 127) / 128) * p.nsplit;
  const int grid = units < num_sms ? units : num_sms;
  return launch_pdl(kernel, dim3(grid), dim3(kMlThreads), kMlSmem, stream, tmA, tmB, tmA2, tmB2, tmW, p);
}

}  // namespace ft
