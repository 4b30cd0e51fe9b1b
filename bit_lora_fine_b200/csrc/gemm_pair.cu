// Block-scaled FP4 GEMM on CTA pairs: the tensor cores of two SMs share each
// 256 x 256 output tile (tcgen05 cta_group::2), with the low-rank up-projection
// accumulated into the same TMEM accumulator.
//
// FourTune §3.1/§3.3: the 4-bit backbone product runs on 4-bit tensor cores and
// is fused with the stabilizer/LoRA up-projection; §3.2: the backward dX
// product reads the weight blocks transposed with the same codes and scales.
//
//   out[m, n] = sum_k deq(A)[m, k] deq(B)[n, k]  (+ sum_j A2[m, j] B2[n, j])  (+ bias[n])
//
// Why pairs.  The single-CTA 128 x 256 tile streams 48 KB of operands from L2
// per 256-wide K-block and SM, and that stream (not the MMA) paces it.  In a
// pair, CTA r loads rows 128 r.. of the A tile and rows 128 r.. of the B tile
// (its half of N): 32 KB per K-block and SM for the same MMA work.  Each CTA
// loads only its own tiles into its own shared memory (no multicast); the
// leader (rank 0) issues the MMAs, which read both CTAs' operands and write
// each CTA's 128 accumulator rows into that CTA's tensor memory.
//
// Protocol (barriers live at the same shared-memory offsets in both CTAs):
//   full[s]     leader's: its producer's arrive.expect_tx of both CTAs' bytes,
//               and both CTAs' TMA completions (each CTA's loads name the
//               leader's barrier)
//   empty[s]    each CTA's: the leader's MMA commit, multicast to both
//   sf_full[s]  leader's: one arrive per leader scale warp (4) and one
//               forwarded from the peer (below)
//   acc_full    each CTA's: the leader's commit after a tile's last MMA
//   acc_empty   leader's: one arrive per leader epilogue warp (8) and one
//               forwarded from the peer
// The peer's scale and epilogue warps arrive on barriers of their own CTA
// (sf_ready[s], acc_done), and one otherwise idle thread of the peer forwards
// each completed phase to the leader.  An arrive with cluster-scope release
// waits for every memory operation its thread has in flight -- for a scale
// warp, the next stage's scale loads -- so the warps that keep loads in flight
// only ever release at CTA scope.
// Each CTA's four scale warps write its own tensor memory: A's scales of its
// 128 rows and B's scales of all 256 columns of the tile (the layout of the
// single-CTA kernel).  Every wait is bounded (see common.cuh); both CTAs meet
// at a cluster barrier before the pair frees its tensor memory.
//
// Warp roles (both CTAs): warp 0 lane 0 producer; warp 1 TMEM allocation (and
// in the leader, lane 0 issues the MMAs); warps 4..11 epilogue, warp w on TMEM
// lanes 32 (w % 4).. and half of the columns; warps 12..15 scale warps.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace ft {

namespace {

constexpr int kPrStages = 5;
constexpr int kPrThreads = 512;
constexpr int kPrBN = 256;                   // output columns per pair tile
constexpr int kPrBM = 256;                   // output rows per pair tile (128 per CTA)
constexpr uint32_t kPrA = 128 * 128;         // this CTA's A codes / A2 bf16 tile
constexpr uint32_t kPrB = 128 * 128;         // this CTA's half of the B tile
constexpr uint32_t kPrStage = kPrA + kPrB;   // 32 KB
constexpr uint32_t kPrEpi = 8 * 1024;        // one transpose buffer per epilogue warp
constexpr uint32_t kPrSmem = 1024 + kPrStages * kPrStage + kPrEpi + 256;
constexpr uint32_t kPrSfCols = 16 + 32;      // per stage: A's 4 k-steps x 4, B's 4 k-steps x 2 chunks x 4
constexpr uint32_t kPrTmemCols = 512;
static_assert(kPrBN + kPrStages * kPrSfCols <= kPrTmemCols, "TMEM budget");
static_assert(kPrSmem <= 232448, "shared memory budget");

__device__ __forceinline__ void pr_store_rows32(uint8_t* buf, const uint32_t (&w)[8], int lane, uint8_t* gbase,
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

__device__ __forceinline__ uint32_t pr_pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

}  // namespace

__global__ void __launch_bounds__(kPrThreads, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                     const GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* epi = smem + kPrStages * kPrStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(epi + kPrEpi);
  uint64_t* empty = full + kPrStages;
  uint64_t* sf_full = empty + kPrStages;
  uint64_t* acc_full = sf_full + kPrStages;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* mma_done = acc_empty + 1;
  uint64_t* sf_ready = mma_done + 1;         // [kPrStages] peer only: its scale warps
  uint64_t* acc_done = sf_ready + kPrStages; // peer only: its epilogue warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_done + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  volatile int* abortp = abort_flag;
  static_assert((4 * kPrStages + 4) * 8 + 8 <= 256, "barriers, TMEM slot and flag fit the tail");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  const int KB = (p.K + 255) / 256;       // FP4 K-blocks
  const int KS = (p.K + 63) / 64;         // 64-wide k-steps: scale blocks per 128-row chunk
  const int EB = (p.R2 + 63) / 64;        // bf16 low-rank blocks
  const int T = KB + EB;                  // pipeline stages per tile
  const int tiles_n = (p.N + kPrBN - 1) / kPrBN;
  const int tiles = tiles_n * ((p.M + kPrBM - 1) / kPrBM);
  const int nchunk_a = (p.M + 127) / 128;
  const int nchunk_b = (p.N + 127) / 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPrStages; ++s) {
      mbar_init(&full[s], 1);      // leader's producer (expect_tx of both CTAs' bytes)
      mbar_init(&empty[s], 1);     // leader's MMA commit
      mbar_init(&sf_full[s], 5);   // the leader's 4 scale warps + the peer's forwarded arrive
      mbar_init(&sf_ready[s], 4);  // the peer's scale warps
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 9);       // the leader's 8 epilogue warps + the peer's forwarded arrive
    mbar_init(acc_done, 8);        // the peer's epilogue warps
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, kPrTmemCols);
    tmem_relinquish_pair();
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
  cluster_sync_all();              // barriers initialized and TMEM allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait_prior();

  if (warp == 0) {
    if (lane == 0) {
      const uint32_t full0 = cluster_addr(&full[0], 0);   // the leader's full[0]
      int g = 0;
      bool ok = true;
      for (int tile = pair; tile < tiles && ok; tile += npairs) {
        const int m0 = (tile / tiles_n) * kPrBM + 128 * static_cast<int>(rank);
        const int n0 = (tile % tiles_n) * kPrBN + 128 * static_cast<int>(rank);
        for (int i = 0; i < T; ++i) {
          const int s = g % kPrStages;
          const uint32_t ph = (g / kPrStages) & 1;
          if (!mbar_wait_cluster(&empty[s], ph ^ 1, p.status, abortp)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kPrStage;
          const uint32_t fb = full0 + 8u * s;
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2 * kPrStage);
          if (i < KB) {
            tma_load_2d_pair(st, &tmA, fb, i * 128, m0);
            tma_load_2d_pair(st + kPrA, &tmB, fb, i * 128, n0);
          } else {
            const int e = i - KB;
            tma_load_2d_pair(st, &tmA2, fb, e * 64, m0);
            if (p.b2_mn_major) {
              tma_load_2d_pair(st + kPrA, &tmB2, fb, n0, e * 64);
              tma_load_2d_pair(st + kPrA + 8192, &tmB2, fb, n0 + 64, e * 64);
            } else {
              tma_load_2d_pair(st + kPrA, &tmB2, fb, e * 64, n0);
            }
          }
          ++g;
        }
      }
      if (*abortp && rank == 0) {  // let copies already in flight land before the pair exits
        for (int j = max(0, g - kPrStages); j < g; ++j)
          mbar_wait_drain(&full[j % kPrStages], (j / kPrStages) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      const uint32_t idesc4 = idesc_fp4_block16(256, kPrBN);
      const uint32_t idesc16 = idesc_bf16(256, kPrBN, false, p.b2_mn_major != 0);
      int g = 0, j = 0;
      bool ok = true;
      for (int tile = pair; tile < tiles && ok; tile += npairs, ++j) {
        // both CTAs' epilogues must have read the previous tile's accumulator out
        if (j > 0 && !mbar_wait_cluster(acc_empty, (j - 1) & 1, p.status, abortp)) break;
        tc_fence_after();
        for (int i = 0; i < T; ++i) {
          const int s = g % kPrStages;
          const uint32_t ph = (g / kPrStages) & 1;
          // sf_full completes once per use of the slot (the scale warps arrive for
          // every stage), so it is waited on for every stage to keep its phase
          if (!mbar_wait_cluster(&full[s], ph, p.status, abortp) ||
              !mbar_wait_cluster(&sf_full[s], ph, p.status, abortp)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + s * kPrStage);
          const uint32_t b_addr = a_addr + kPrA;
          if (i < KB) {
            const int nks = min(4, KS - 4 * i);
            const uint32_t sf_col = kPrBN + s * kPrSfCols;
            for (int t = 0; t < nks; ++t)
              mma_fp4_block16_pair(tmem, desc_kmajor_sw128(a_addr + 32 * t), desc_kmajor_sw128(b_addr + 32 * t),
                                   idesc4, tmem + sf_col + 4 * t, tmem + sf_col + 16 + 8 * t, (i | t) != 0 ? 1u : 0u);
          } else {
#pragma unroll
            for (int t = 0; t < 4; ++t) {
              const uint64_t bdesc =
                  p.b2_mn_major ? desc_mnmajor_sw128(b_addr + 2048 * t, 8192) : desc_kmajor_sw128(b_addr + 32 * t);
              mma_bf16_pair(tmem, desc_kmajor_sw128(a_addr + 32 * t), bdesc, idesc16, 1u);
            }
          }
          tc_commit_pair(&empty[s], 0x3);
          ++g;
        }
        if (ok) tc_commit_pair(acc_full, 0x3);
      }
      tc_commit_pair(mma_done, 0x1);
      mbar_wait_drain(mma_done, 0, kWaitLimitNs);  // every MMA done before TMEM can be freed
    }
  } else if (warp >= 12) {
    // Scale warp of TMEM lane quadrant q (this CTA's tensor memory).  Stage
    // columns (from sf_col): A's k-step t at 4t..4t+3, of which the MMA reads
    // 4t+q here (the diagonal word of the 512-byte block: rows 32q+lane of this
    // CTA's chunk); B's k-step t, chunk c at 16+8t+4c..+3, all four.
    const int q = warp & 3;
    const uint32_t trow = tmem + (static_cast<uint32_t>(32 * q) << 16);
    const int G = (pair < tiles ? (tiles - 1 - pair) / npairs + 1 : 0) * T;
    auto fetch = [&](int gg, uint32_t (&a)[4], uint32_t (&b)[32]) {
      const int tile = pair + (gg / T) * npairs;
      const int i = gg % T;
      const int nks = i < KB ? min(4, KS - 4 * i) : 0;
      const int mc = (tile / tiles_n) * 2 + static_cast<int>(rank), nc = (tile % tiles_n) * 2;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        a[t] = 0u;
        if (t < nks && mc < nchunk_a)
          a[t] = __ldg(reinterpret_cast<const uint32_t*>(p.sfa + (static_cast<size_t>(mc) * KS + 4 * i + t) * 512 +
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
    auto put = [&](int gg, const uint32_t (&a)[4], const uint32_t (&b)[32]) -> bool {
      const int s = gg % kPrStages;
      const uint32_t ph = (gg / kPrStages) & 1;
      bool okw = true;
      if (lane == 0) okw = mbar_wait_cluster(&empty[s], ph ^ 1, p.status, abortp);  // MMAs that read the slot are done
      okw = __shfl_sync(0xFFFFFFFFu, okw ? 1 : 0, 0) != 0;
      if (!okw) return false;
      tc_fence_after();
      if (gg % T < KB) {
        const uint32_t sf_col = kPrBN + s * kPrSfCols;
        uint32_t a16[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) a16[e] = a[e >> 2];
        tmem_st_32x32b_x16(trow + sf_col, a16);
        tmem_st_32x32b_x32(trow + sf_col + 16, b);
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(rank == 0 ? &sf_full[s] : &sf_ready[s]);
      return true;
    };
    // two register sets: stage gg+1's loads are in flight while stage gg is stored
    uint32_t a0[4], b0[32], a1[4], b1[32];
    if (G > 0) fetch(0, a0, b0);
    for (int gg = 0; gg < G; gg += 2) {
      if (gg + 1 < G) fetch(gg + 1, a1, b1);
      if (!put(gg, a0, b0) || gg + 1 >= G) break;
      if (gg + 2 < G) fetch(gg + 2, a0, b0);
      if (!put(gg + 1, a1, b1)) break;
    }
  } else if (warp >= 4) {
    // two warps per TMEM lane quadrant, each owning half of the tile's columns
    const int q = warp & 3;
    const int c_lo = ((warp - 4) >> 2) * (kPrBN / 2);
    const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(c_lo);
    uint64_t* acc_free = rank == 0 ? acc_empty : acc_done;   // the peer's are forwarded
    uint8_t* buf = epi + (warp - 4) * 1024;
    const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(p.bias);
    const long long ldb = p.ldo * (p.out_bf16 ? 2 : 4);   // output row stride in bytes
    int j = 0;
    for (int tile = pair; tile < tiles; tile += npairs, ++j) {
      if (!mbar_wait_cluster(acc_full, j & 1, p.status, abortp)) break;
      __syncwarp();
      tc_fence_after();
      const int m0 = (tile / tiles_n) * kPrBM + 128 * static_cast<int>(rank);
      const int n0 = (tile % tiles_n) * kPrBN + c_lo;
      const int row0 = m0 + 32 * q;              // first row of this warp's 32
      const int rows_left = p.M - row0;
      uint8_t* out_rows = static_cast<uint8_t*>(p.out) + static_cast<long long>(row0) * ldb;
      if (p.out_bf16) {
        // the warp's half row to registers (+ bias, bf16), accumulator handed
        // back, then the stores
        uint32_t pk[kPrBN / 4];
#pragma unroll
        for (int rd = 0; rd < kPrBN / 64; ++rd) {
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
              pk[16 * rd + 8 * k + e] = pr_pack_bf16x2(__uint_as_float(v[k][2 * e]) + bf16_bits_to_f32(bb & 0xFFFFu),
                                                       __uint_as_float(v[k][2 * e + 1]) + bf16_bits_to_f32(bb >> 16));
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_free);
        if (rows_left > 0) {
#pragma unroll
          for (int c = 0; c < kPrBN / 32; ++c) {
            const int nb = n0 + 16 * c;
            if (nb >= p.N) break;
            uint32_t w[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) w[e] = pk[8 * c + e];
            pr_store_rows32(buf, w, lane, out_rows + static_cast<long long>(nb) * 2, ldb, rows_left);
          }
        }
      } else {
        // fp32 rows, 8 columns (32 bytes) at a time
        for (int c = 0; c < kPrBN / 32; ++c) {
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
              w[e] = __float_as_uint(__uint_as_float(v[8 * hlf + e]) + (bias ? __bfloat162float(bias[nb + e]) : 0.0f));
            pr_store_rows32(buf, w, lane, out_rows + static_cast<long long>(nb) * 4, ldb, rows_left);
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(acc_free);
      }
    }
  } else if (warp == 2 && lane == 0 && rank == 1) {
    // the peer's forwarder of its scale warps' phases to the leader's sf_full
    const int G = (pair < tiles ? (tiles - 1 - pair) / npairs + 1 : 0) * T;
    const uint32_t sf_full0 = cluster_addr(&sf_full[0], 0);
    for (int gg = 0; gg < G; ++gg) {
      const int s = gg % kPrStages;
      if (!mbar_wait(&sf_ready[s], (gg / kPrStages) & 1, p.status, abortp)) break;
      mbar_arrive_remote(sf_full0 + 8u * s);
    }
  } else if (warp == 3 && lane == 0 && rank == 1) {
    // ... and of its epilogue warps' phases to the leader's acc_empty
    const uint32_t acc_empty0 = cluster_addr(acc_empty, 0);
    int j = 0;
    for (int tile = pair; tile < tiles; tile += npairs, ++j) {
      if (!mbar_wait(acc_done, j & 1, p.status, abortp)) break;
      mbar_arrive_remote(acc_empty0);
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();              // the peer is done with this CTA's barriers and TMEM
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, kPrTmemCols);
  }
}

cudaError_t launch_gemm_pair(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmA2,
                             const CUtensorMap& tmB2, const GemmParams& p, int num_sms, cudaStream_t stream) {
  if (p.epi_gelu_bwd) return cudaErrorInvalidValue;
  cudaError_t e =
      cudaFuncSetAttribute(gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kPrSmem));
  if (e != cudaSuccess) return e;
  const int tiles = ((p.N + kPrBN - 1) / kPrBN) * ((p.M + kPrBM - 1) / kPrBM);
  const int pairs = std::min(tiles, std::max(1, num_sms / 2));
  return launch_pdl_pair(gemm_pair_kernel, dim3(2 * pairs), dim3(kPrThreads), kPrSmem, stream, tmA, tmB, tmA2, tmB2,
                         p);
}

}  // namespace ft
