// Block-scaled FP4 GEMM on the 5th-generation tensor cores, with the
// low-rank up-projection accumulated into the same TMEM accumulator.
//
// FourTune §3.1/§3.3: the 4-bit backbone product runs on 4-bit tensor cores and
// is fused with the stabilizer/LoRA up-projection, since the branch outputs are
// summed anyway.  §3.2: the backward dX product reads the weight blocks
// transposed with the same codes and scales -- here the B operand is the
// nibble-transposed copy of R's codes and its scales are R's own scales laid
// out for the transposed operand.
//
//   out[m, n] = sum_k deq(A)[m, k] deq(B)[n, k]  (+ sum_j A2[m, j] B2[n, j])  (+ bias[n])
//
// Persistent kernel: one CTA per SM walks the 128 x BN output tiles (BN = 256)
// in row-major tile order, so that the CTAs of one wave share the rows of A and
// all of B in L2.  One pipeline stage = one K-block of 256 FP4 elements: the A
// and B code boxes (128-byte swizzled rows) and the K-block's scale blocks of
// both operands, kept in global memory in the MMA-ready layout (kernels.h) and
// brought into the stage by bulk copies beside the code boxes.  The scales must
// sit in TMEM when the MMAs run: the MMA reads A's scales of lane quadrant w
// from column base + w of that quadrant, and B's scales from all four columns
// of every quadrant, so B's scales are needed four times over.  Moving them with
// tcgen05.cp 32x128b.warpx4 (which replicates into the four quadrants) costs
// ~70 cycles a copy, 12 copies per K-block, on the same queue as the MMAs --
// more than the 4 MMAs of the K-block take.  Instead four scale warps, one per
// lane quadrant, read each stage's scale words from shared memory once the
// stage has landed and write them into their quadrant with tcgen05.st, which
// runs beside the MMAs.  (Loading the words from global memory one stage ahead
// instead, in registers, left the MMAs waiting on scale loads: 41.5 / 43.4 us
// against 39.4 / 39.3 us at FLUX width.)
// Warp roles:
//   warp 0 lane 0  producer: TMA code boxes and scale bulk copies per K-block;
//                  then the bf16 low-rank blocks A2 [128 x 64] and B2 (K-major
//                  [BN x 64] or MN-major [64 x BN] in four boxes)
//   warp 1         TMEM owner; lane 0 issues
//                  tcgen05.mma kind::mxf4nvf4.block_scale.block16 (M=128,
//                  N=BN, K=64) once a stage's codes and scales are in, then
//                  kind::f16 for the low-rank blocks
//   warps 12..15   scale warps: warp 12+q fills quadrant q's scale columns of
//                  each stage from the stage's scale blocks once the stage has
//                  landed (its full barrier, which also means the MMAs that
//                  read the columns' previous contents have completed)
//   warps 4..11    epilogue, warp w on TMEM lanes 32 (w % 4).. and half of the
//                  columns.  bf16 output: the warp's accumulator slice goes to
//                  registers (+ bias, packed to bf16), the accumulator is
//                  handed back to the MMA warp at once, and the rows are
//                  written while the next tile's MMAs run.  fp32 output hands
//                  it back after its last TMEM read.  Rows go out through a 1 KB per-warp
//                  smem transpose as 16-row x 32-byte (whole-sector) stores.
#include "common.cuh"
#include "kernels.h"

namespace ft {

constexpr int kGmStages = 4;
constexpr int kGmThreads = 512;      // warps 0-3 roles, 4-11 epilogue, 12-15 scale warps

template <int BN>
struct GemmLayout {
  static constexpr int kNC = BN / 128;                       // 128-row scale chunks of the B tile
  static constexpr uint32_t kA = 128 * 128;                  // A codes / A2 bf16 tile
  static constexpr uint32_t kB = BN * 128;                   // B codes / B2 bf16 tile
  static constexpr uint32_t kSFA = 4 * 512;                 // A's scale blocks of a K-block
  static constexpr uint32_t kSFB = kNC * 4 * 512;           // B's: [128-row chunk][k-step][512 B]
  static constexpr uint32_t kStage = kA + kB + kSFA + kSFB;  // multiple of 1024
  static constexpr uint32_t kEpi = 8 * 1024;                 // one transpose buffer per epilogue warp
  static constexpr uint32_t kSmem = 1024 + kGmStages * kStage + kEpi + 256;
  // TMEM columns: accumulator, then per stage 16 (SFA) + 16*kNC (SFB)
  static constexpr uint32_t kSfColsPerStage = 16 + 16 * kNC;
  static constexpr uint32_t kTmemUsed = BN + kGmStages * kSfColsPerStage;
  static constexpr uint32_t kTmemCols = kTmemUsed <= 256 ? 256 : 512;
};

// Warp-cooperative store of a 32-row x 32-byte block: lane l holds row l's 32
// bytes in w.  The block passes through the warp's 1 KB smem buffer with its
// two 16-byte chunks swapped on every other group of four rows (conflict-free
// in both directions), so that each global store instruction covers 16 rows x
// 32 contiguous bytes (whole sectors).  Rows at or past rows_left are skipped.
__device__ __forceinline__ void store_rows32(uint8_t* buf, const uint32_t (&w)[8], int lane, uint8_t* gbase,
                                             long long ld_bytes, int rows_left) {
#pragma unroll
  for (int j = 0; j < 2; ++j)
    *reinterpret_cast<uint4*>(buf + lane * 32 + ((j ^ ((lane >> 2) & 1)) << 4)) =
        make_uint4(w[4 * j], w[4 * j + 1], w[4 * j + 2], w[4 * j + 3]);
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    const int rr = (lane >> 1) + 16 * j, cc = lane & 1;
    const uint4 v = *reinterpret_cast<const uint4*>(buf + rr * 32 + ((cc ^ ((rr >> 2) & 1)) << 4));
    if (rr < rows_left) *reinterpret_cast<uint4*>(gbase + rr * ld_bytes + cc * 16) = v;
  }
  __syncwarp();
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

// SCALED: the 1x16 layout's product scale 2^(eA + eB) in the epilogue (its own
// instantiation, so that the block layout's accumulator readout -- on the
// next tile's critical path -- carries no extra multiply)
template <int BN, bool SCALED>
__global__ void __launch_bounds__(kGmThreads, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                    const GemmParams p) {
  using Lay = GemmLayout<BN>;
  static_assert(Lay::kNC == 2, "scale warps store the B scales of two 128-row chunks (32 columns)");
  static_assert(Lay::kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(Lay::kTmemUsed <= 512, "TMEM budget");
  static_assert(Lay::kSmem <= 232448, "shared memory budget");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = smem + kGmStages * Lay::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + Lay::kEpi);
  uint64_t* empty = full + kGmStages;
  uint64_t* acc_full = empty + kGmStages;   // MMA -> epilogue: tile accumulated
  uint64_t* acc_empty = acc_full + 1;       // epilogue -> MMA: accumulator read out
  uint64_t* mma_done = acc_empty + 1;       // every MMA of the CTA completed (teardown)
  uint64_t* sf_full = mma_done + 1;         // scale warps -> MMA: a stage's scales are in TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_full + kGmStages);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  volatile int* abortp = abort_flag;
  static_assert((3 * kGmStages + 3) * 8 + 8 <= 256, "barriers, TMEM slot and flag fit the tail");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool bf16main = p.main_bf16 != 0;   // 16-bit main product: 64-wide bf16 K-blocks, no scales
  const int KB = bf16main ? (p.K + 63) / 64 : (p.K + 255) / 256;   // main-product K-blocks
  const int KS = (p.K + 63) / 64;         // 64-wide k-steps: scale blocks per 128-row chunk
  const int EB = (p.R2 + 63) / 64;        // bf16 low-rank blocks
  const int T = KB + EB;                  // pipeline stages per tile
  const int tiles_n = (p.N + BN - 1) / BN;
  const int tiles = tiles_n * ((p.M + 127) / 128);
  const int nchunk_b = (p.N + 127) / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGmStages; ++s) {
      mbar_init(&full[s], 1);      // producer (expect_tx)
      mbar_init(&empty[s], 1);     // MMA commit
      mbar_init(&sf_full[s], 4);   // one arrive per scale warp
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 8);   // one arrive per epilogue warp
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Lay::kTmemCols);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
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
      int g = 0;   // stages issued by this CTA so far (ring position)
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x) {
        const int m0 = (tile / tiles_n) * 128, n0 = (tile % tiles_n) * BN;
        for (int i = 0; i < T; ++i) {
          const int s = g % kGmStages;
          const uint32_t ph = (g / kGmStages) & 1;
          if (!mbar_wait(&empty[s], ph ^ 1, p.status, abortp)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * Lay::kStage;
          if (i < KB) {
            // a K-block is 128 bytes of each row: 256 FP4 codes or 64 bf16 values
            const int kx = bf16main ? i * 64 : i * 128;
            if (bf16main) {
              mbar_arrive_expect_tx(&full[s], Lay::kA + Lay::kB);
            } else {
              // the K-block's MMA-ready scale blocks ride in the stage (bulk copies)
              const int nks = min(4, KS - 4 * i);
              const uint32_t sfbytes = static_cast<uint32_t>(nks) * 512u;
              const int nb = (n0 / 128 + 1 < nchunk_b) ? 2 : 1;
              mbar_arrive_expect_tx(&full[s], Lay::kA + Lay::kB + sfbytes * static_cast<uint32_t>(1 + nb));
              bulk_load(st + Lay::kA + Lay::kB, p.sfa + (static_cast<size_t>(m0 / 128) * KS + 4 * i) * 512, sfbytes,
                        &full[s]);
              for (int c = 0; c < nb; ++c)
                bulk_load(st + Lay::kA + Lay::kB + Lay::kSFA + c * 2048,
                          p.sfb + (static_cast<size_t>(n0 / 128 + c) * KS + 4 * i) * 512, sfbytes, &full[s]);
            }
            tma_load_2d(st, &tmA, &full[s], kx, m0);
            tma_load_2d(st + Lay::kA, &tmB, &full[s], kx, n0);
          } else {
            const int e = i - KB;
            mbar_arrive_expect_tx(&full[s], Lay::kA + Lay::kB);
            tma_load_2d(st, &tmA2, &full[s], e * 64, m0);
            if (p.b2_mn_major) {
#pragma unroll
              for (int c = 0; c < BN / 64; ++c)
                tma_load_2d(st + Lay::kA + 8192 * c, &tmB2, &full[s], n0 + 64 * c, e * 64);
            } else {
              tma_load_2d(st + Lay::kA, &tmB2, &full[s], e * 64, n0);
            }
          }
          ++g;
        }
      }
      if (*abortp) {  // let copies already in flight land before the CTA exits
        for (int j = max(0, g - kGmStages); j < g; ++j)
          mbar_wait_drain(&full[j % kGmStages], (j / kGmStages) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc4 = idesc_fp4_block16(128, BN);
      const uint32_t idesc16 = idesc_bf16(128, BN, false, p.b2_mn_major != 0);
      const uint32_t idesc16k = idesc_bf16(128, BN, false, false);
      int g = 0, j = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < tiles && ok; tile += gridDim.x, ++j) {
        // the epilogue must have read the previous tile's accumulator out
        if (j > 0 && !mbar_wait(acc_empty, (j - 1) & 1, p.status, abortp)) break;
        tc_fence_after();
        for (int i = 0; i < T; ++i) {
          const int s = g % kGmStages;
          const uint32_t ph = (g / kGmStages) & 1;
          if (!mbar_wait(&full[s], ph, p.status, abortp) || !mbar_wait(&sf_full[s], ph, p.status, abortp)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * Lay::kStage);
          const uint32_t b_addr = a_addr + Lay::kA;
          if (i < KB && bf16main) {
#pragma unroll
            for (int t = 0; t < 4; ++t)
              mma_bf16(tmem, desc_kmajor_sw128(a_addr + 32 * t), desc_kmajor_sw128(b_addr + 32 * t), idesc16k,
                       (i | t) != 0 ? 1u : 0u);
          } else if (i < KB) {
            const int nks = min(4, KS - 4 * i);
            const uint32_t sf_col = BN + s * Lay::kSfColsPerStage;
            for (int t = 0; t < nks; ++t)
              mma_fp4_block16(tmem, desc_kmajor_sw128(a_addr + 32 * t), desc_kmajor_sw128(b_addr + 32 * t), idesc4,
                              tmem + sf_col + 4 * t, tmem + sf_col + 16 + t * Lay::kNC * 4,
                              (i | t) != 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const uint64_t bdesc =
                  p.b2_mn_major ? desc_mnmajor_sw128(b_addr + 2048 * t, 8192) : desc_kmajor_sw128(b_addr + 32 * t);
              mma_bf16(tmem, desc_kmajor_sw128(a_addr + 32 * t), bdesc, idesc16, 1u);
            }
          }
          tc_commit(&empty[s]);
          ++g;
        }
        if (ok) tc_commit(acc_full);
      }
      tc_commit(mma_done);
      mbar_wait_drain(mma_done, 0, kWaitLimitNs);  // every MMA done before TMEM can be freed
    }
  } else if (warp >= 12) {
    // Scale warp of TMEM lane quadrant q.  Stage columns (from sf_col): A's
    // k-step t at 4t..4t+3, of which the MMA reads 4t+q here (the diagonal
    // word of the 512-byte block: rows 32q+lane, byte 16*lane + 4q); B's
    // k-step t, chunk c at 16+8t+4c..+3, all four (the block's words
    // 16*lane..16*lane+15, i.e. rows 32j+lane of the chunk, j = 0..3).
    const int q = warp & 3;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const int bx = static_cast<int>(blockIdx.x), gx = static_cast<int>(gridDim.x);
    const int G = (bx < tiles ? (tiles - 1 - bx) / gx + 1 : 0) * T;
    constexpr int NB = 4 * 4 * Lay::kNC;
    // each stage's scale blocks, from the stage once its copies have landed
    // (full[s] of this use implies the MMAs of the slot's previous use are done)
    for (int gg = 0; gg < G; ++gg) {
      const int s = gg % kGmStages;
      const uint32_t ph = (gg / kGmStages) & 1;
      bool okw = true;
      if (lane == 0) okw = mbar_wait(&full[s], ph, p.status, abortp);
      if (__shfl_sync(0xFFFFFFFFu, okw ? 1 : 0, 0) == 0) break;
      const int i = gg % T;
      if (i < KB && !bf16main) {
        const int tile = bx + (gg / T) * gx;
        const int nks = min(4, KS - 4 * i);
        const int nc = (tile % tiles_n) * Lay::kNC;
        const uint8_t* sf = smem + s * Lay::kStage + Lay::kA + Lay::kB;
        uint32_t b[NB];
#pragma unroll
        for (int c = 0; c < Lay::kNC; ++c) {
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            uint4 x = make_uint4(0u, 0u, 0u, 0u);   // zero scales past N (their codes are zero)
            if (t < nks && nc + c < nchunk_b)
              x = *reinterpret_cast<const uint4*>(sf + Lay::kSFA + c * 2048 + t * 512 + 16 * lane);
            b[4 * (t * Lay::kNC + c)] = x.x;
            b[4 * (t * Lay::kNC + c) + 1] = x.y;
            b[4 * (t * Lay::kNC + c) + 2] = x.z;
            b[4 * (t * Lay::kNC + c) + 3] = x.w;
          }
        }
        tc_fence_after();
        const uint32_t sf_col = BN + s * Lay::kSfColsPerStage;
#pragma unroll
        for (int t = 0; t < 4; ++t)
          tmem_st_32x32b_x4_rep(trow + sf_col + 4 * t,
                                t < nks ? *reinterpret_cast<const uint32_t*>(sf + t * 512 + 16 * lane + 4 * q) : 0u);
        tmem_st_32x32b_x32(trow + sf_col + 16, b);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_full[s]);
    }
  } else if (warp >= 4) {
    // two warps per TMEM lane quadrant, each owning half of the tile's columns
    const int q = warp & 3;
    const int c_lo = ((warp - 4) >> 2) * (BN / 2);
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c_lo);
    uint8_t* buf = epi + (warp - 4) * 1024;
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(p.bias);
    const long long ldb = p.ldo * (p.out_bf16 ? 2 : 4);   // output row stride in bytes
    const bool fast = p.out_bf16 != 0;
    // 1x16 groups: the product's per-tensor scale 2^(eA + eB), as one factor
    // when it is a float32 number, else as two (then f1 is exact and the
    // product's own range is exceeded anyway)
    float f1 = 1.0f, f2 = 1.0f;
    if (SCALED) {
      const int es = group16_exponent(__uint_as_float(*p.amax_a)) + group16_exponent(__uint_as_float(*p.amax_b));
      if (es >= -126 && es <= 127) {
        f1 = pow2_f32(es);
      } else {
        f1 = pow2_f32(es / 2);
        f2 = pow2_f32(es - es / 2);
      }
    }
    int j = 0;
    for (int tile = blockIdx.x; tile < tiles; tile += gridDim.x, ++j) {
      if (!mbar_wait(acc_full, j & 1, p.status, abortp)) break;
      __syncwarp();
      tc_fence_after();
      const int m0 = (tile / tiles_n) * 128, n0 = (tile % tiles_n) * BN + c_lo;
      const int row0 = m0 + 32 * q;              // first row of this warp's 32
      const int rows_left = p.M - row0;
      uint8_t* out_rows = static_cast<uint8_t*>(p.out) + static_cast<long long>(row0) * ldb;
      if (fast) {
        // the warp's half row to registers (+ bias, bf16), accumulator handed
        // back, then the stores.  Four rounds of 32 columns (two 16-column TMEM
        // loads in flight per wait): the packed row and one round fit the
        // register budget without spilling.
        uint32_t pk[BN / 4];
#pragma unroll
        for (int rd = 0; rd < BN / 64; ++rd) {
          uint32_t v[2][16];
          tmem_ld_32x32b_x16(taddr + 32 * rd, v[0]);
          tmem_ld_32x32b_x16(taddr + 32 * rd + 16, v[1]);
          uint4 bw[4];                                     // 32 bias values (bf16)
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
              float x0 = __uint_as_float(v[k][2 * e]), x1 = __uint_as_float(v[k][2 * e + 1]);
              if (SCALED) {
                x0 *= f1;
                x1 *= f1;
              }
              pk[16 * rd + 8 * k + e] = pack_bf16x2(fmaf(x0, f2, bf16_bits_to_f32(bb & 0xFFFFu)),
                                                    fmaf(x1, f2, bf16_bits_to_f32(bb >> 16)));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
        if (rows_left > 0) {
#pragma unroll
          for (int c = 0; c < BN / 32; ++c) {
            const int nb = n0 + 16 * c;
            if (nb >= p.N) break;
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = pk[8 * c + e];
            store_rows32(buf, w, lane, out_rows + static_cast<long long>(nb) * 2, ldb, rows_left);
          }
        }
      } else {
        // fp32 rows, 8 columns (32 bytes) at a time
        for (int c = 0; c < BN / 32; ++c) {
          uint32_t v[16];
          tmem_ld_32x32b_x16(taddr + 16 * c, v);
          tmem_ld_wait();
          if (rows_left <= 0) continue;
#pragma unroll
          for (int hlf = 0; hlf < 2; ++hlf) {
            const int nb = n0 + 16 * c + 8 * hlf;
            if (nb >= p.N) continue;
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              w[e] = __float_as_uint(fmaf(SCALED ? __uint_as_float(v[8 * hlf + e]) * f1 : __uint_as_float(v[8 * hlf + e]),
                                          f2, bias ? __bfloat162float(bias[nb + e]) : 0.0f));
            store_rows32(buf, w, lane, out_rows + static_cast<long long>(nb) * 4, ldb, rows_left);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_empty);
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, Lay::kTmemCols);
  }
}

cudaError_t launch_gemm_fp4(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmA2,
                            const CUtensorMap& tmB2, const GemmParams& p, int num_sms, cudaStream_t stream) {
  constexpr int BN = kGemmBN;
  auto kernel = p.amax_a ? gemm_fp4_kernel<BN, true> : gemm_fp4_kernel<BN, false>;
  const uint32_t smem = GemmLayout<BN>::kSmem;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const int tiles = ((p.N + BN - 1) / BN) * ((p.M + 127) / 128);
  const int grid = tiles < num_sms ? tiles : num_sms;
  return launch_pdl(kernel, dim3(grid), dim3(kGmThreads), smem, stream, tmA, tmB, tmA2, tmB2, p);
}

}  // namespace ft
