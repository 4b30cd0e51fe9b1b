// Block-scaled FP4 GEMM on the 5th-generation tensor cores, with the
// low-rank up-projection accumulated into the same TMEM accumulator.
//
// FourTune §3.1/§3.3: the 4-bit backbone product runs on 4-bit tensor cores and
// is fused with the stabilizer/LoRA up-projection, since the branch outputs are
// summed anyway.  §3.2: the backward dX product reads the weight blocks
// transposed with the same codes and scales -- here the B operand is the
// nibble-transposed copy of R's codes and the scale of (row, k-group) is read
// transposed from R's own [N/16, K/16] scale array.
//
//   out[m, n] = sum_k deq(A)[m, k] deq(B)[n, k]  (+ sum_j A2[m, j] B2[n, j])  (+ bias[n])
//
// CTA tile 128 x BN (BN = 256), K-block = 256 FP4 elements (one 128-byte
// swizzle row per operand row).  Warp roles:
//   warp 0 lane 0  TMA: A codes [128 x 128 B] and B codes [BN x 128 B] per
//                  K-block; every kSfChunk K-blocks the compact 16x16 scale
//                  tiles of those K-blocks (two small boxes into a 2-slot ring,
//                  so that a K-block costs two TMA boxes, not four); for the
//                  bf16 extra blocks A2 [128 x 64] and B2 (K-major [BN x 64] or
//                  MN-major [64 x BN] in four boxes) into the same slots
//   warp 1         TMEM owner; lane 0 copies the stage's scale vectors smem->TMEM
//                  (tcgen05.cp 32x128b.warpx4) and issues
//                  tcgen05.mma kind::mxf4nvf4.block_scale.block16 (M=128, N=BN,
//                  K=64) x 4 per K-block, then kind::f16 for the extra blocks
//   warp 2         expands the compact scales into the per-row layout the MMA
//                  reads (one 16-byte pattern per 16 rows)
//   warps 4..7     epilogue: TMEM -> registers (+ bias) -> fp32/bf16 rows staged
//                  in the now idle pipeline smem (128-byte swizzled boxes of 32
//                  rows) -> TMA tensor stores, which clip rows/columns past M, N.
//                  MLP backward variant (FourTune §3.3 MLP): reads the saved
//                  hidden h and writes d_h = bf16(acc * GELU'(h)) and bf16(GELU(h))
#include "common.cuh"
#include "kernels.h"

namespace ft {

constexpr int kGmStages = 4;
constexpr int kGmThreads = 256;
constexpr int kSfChunk = kGemmSfGroups / 16;  // K-blocks per compact-scale load
constexpr int kSfSlots = 2;

template <int BN>
struct GemmLayout {
  static constexpr uint32_t kA = 128 * 128;                  // A codes / A2 bf16 tile
  static constexpr uint32_t kB = BN * 128;                   // B codes / B2 bf16 tile
  static constexpr int kNC = BN / 128;                       // 128-row scale chunks of B
  static constexpr uint32_t kSFA = 4 * 512;                  // 4 MMA K-steps x 512 B
  static constexpr uint32_t kSFB = 4 * kNC * 512;
  static constexpr uint32_t kStage = kA + kB + kSFA + kSFB;  // multiple of 1024
  // compact scales of kSfChunk K-blocks: A 8 row-blocks x 64 groups; B BN/16
  // row-blocks x 64 groups (or, read transposed, 64 groups x BN/16 row-blocks)
  static constexpr uint32_t kCA = 8 * 16 * kSfChunk;
  static constexpr uint32_t kCB = (BN / 16) * 16 * kSfChunk;
  static constexpr uint32_t kCSlot = kCA + kCB;
  static constexpr uint32_t kSmem = 1024 + kGmStages * kStage + kSfSlots * kCSlot + 256;
  // TMEM columns: accumulator, then per stage 16 (SFA) + 16*kNC (SFB)
  static constexpr uint32_t kSfColsPerStage = 16 + 16 * kNC;
  static constexpr uint32_t kTmemUsed = BN + kGmStages * kSfColsPerStage;
  static constexpr uint32_t kTmemCols = kTmemUsed <= 256 ? 256 : 512;
};

template <int BN>
__global__ void __launch_bounds__(kGmThreads, 1)
    gemm_fp4_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
                    const __grid_constant__ CUtensorMap tmSFA, const __grid_constant__ CUtensorMap tmSFB,
                    const __grid_constant__ CUtensorMap tmOut, const __grid_constant__ CUtensorMap tmOut2,
                    const GemmParams p) {
  using Lay = GemmLayout<BN>;
  static_assert(Lay::kStage % 1024 == 0, "stage must keep 1024-byte alignment");
  static_assert(Lay::kTmemUsed <= 512, "TMEM budget");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* compact = smem + kGmStages * Lay::kStage;
  uint64_t* full = reinterpret_cast<uint64_t*>(compact + kSfSlots * Lay::kCSlot);
  uint64_t* sf_ready = full + kGmStages;
  uint64_t* empty = sf_ready + kGmStages;
  uint64_t* acc_full = empty + kGmStages;
  uint64_t* sf_full = acc_full + 1;       // [kSfSlots] compact scales landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sf_full + kSfSlots);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  volatile int* abortp = abort_flag;
  static_assert((3 * kGmStages + 1 + kSfSlots) * 8 + 8 <= 256, "barriers, TMEM slot and flag fit the tail");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN;
  const int m0 = blockIdx.y * 128;
  const int KB = (p.K + 255) / 256;       // FP4 K-blocks
  const int EB = (p.R2 + 63) / 64;        // bf16 extra blocks
  const int T = KB + EB;
  const int KG = p.K / 16;                // number of 16-wide K groups
  const int Mb = (p.M + 15) / 16, Nb = (p.N + 15) / 16;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGmStages; ++s) {
      mbar_init(&full[s], 1);      // producer (expect_tx)
      mbar_init(&sf_ready[s], 1);  // scale stager
      mbar_init(&empty[s], 1);     // MMA commit
    }
    mbar_init(acc_full, 1);
    for (int c = 0; c < kSfSlots; ++c) mbar_init(&sf_full[c], 1);
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
    tma_prefetch(&tmOut);
    if (p.epi_gelu_bwd) tma_prefetch(&tmOut2);
    if (EB) {
      tma_prefetch(&tmA2);
      tma_prefetch(&tmB2);
    }
    if (p.sf_tma) {
      tma_prefetch(&tmSFA);
      tma_prefetch(&tmSFB);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0, chunks = 0;
      for (int i = 0; i < T; ++i) {
        const int s = i % kGmStages;
        const uint32_t ph = (i / kGmStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.status, abortp)) break;
        uint8_t* st = smem + s * Lay::kStage;
        if (i < KB) {
          if (p.sf_tma && i % kSfChunk == 0) {
            // The slot of chunk c was last read for K-block kSfChunk (c - 1) - 1,
            // before the MMA of K-block i - kGmStages, whose commit released
            // stage s: the slot is free.
            const int c = i / kSfChunk;
            uint8_t* cs = compact + (c % kSfSlots) * Lay::kCSlot;
            uint64_t* bar = &sf_full[c % kSfSlots];
            mbar_arrive_expect_tx(bar, Lay::kCSlot);
            tma_load_2d(cs, &tmSFA, bar, c * 16 * kSfChunk, m0 / 16);
            if (p.sfb_transposed)
              tma_load_2d(cs + Lay::kCA, &tmSFB, bar, n0 / 16, c * 16 * kSfChunk);
            else
              tma_load_2d(cs + Lay::kCA, &tmSFB, bar, c * 16 * kSfChunk, n0 / 16);
            chunks = c + 1;
          }
          mbar_arrive_expect_tx(&full[s], Lay::kA + Lay::kB);
          tma_load_2d(st, &tmA, &full[s], i * 128, m0);
          tma_load_2d(st + Lay::kA, &tmB, &full[s], i * 128, n0);
        } else {
          const int e = i - KB;
          mbar_arrive_expect_tx(&full[s], Lay::kA + Lay::kB);
          tma_load_2d(st, &tmA2, &full[s], e * 64, m0);
          if (p.b2_mn_major) {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c) tma_load_2d(st + Lay::kA + 8192 * c, &tmB2, &full[s], n0 + 64 * c, e * 64);
          } else {
            tma_load_2d(st + Lay::kA, &tmB2, &full[s], e * 64, n0);
          }
        }
        issued = i + 1;
      }
      if (*abortp) {
        for (int i = max(0, issued - kGmStages); i < issued; ++i)
          mbar_wait_drain(&full[i % kGmStages], (i / kGmStages) & 1, 100000000ull);
        for (int c = max(0, chunks - kSfSlots); c < chunks; ++c)
          mbar_wait_drain(&sf_full[c % kSfSlots], (c / kSfSlots) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc4 = idesc_fp4_block16(128, BN);
      const uint32_t idesc16 = idesc_bf16(128, BN, false, p.b2_mn_major != 0);
      for (int i = 0; i < T; ++i) {
        const int s = i % kGmStages;
        const uint32_t ph = (i / kGmStages) & 1;
        if (!mbar_wait(&full[s], ph, p.status, abortp)) break;
        if (!mbar_wait(&sf_ready[s], ph, p.status, abortp)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + s * Lay::kStage);
        const uint32_t b_addr = a_addr + Lay::kA;
        if (i < KB) {
          const uint32_t sfa_addr = b_addr + Lay::kB;
          const uint32_t sfb_addr = sfa_addr + Lay::kSFA;
          const uint32_t sf_col = BN + s * Lay::kSfColsPerStage;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            tmem_cp_32x128b_x4(tmem + sf_col + 4 * t, desc_sf_copy(sfa_addr + t * 512));
#pragma unroll
            for (int c = 0; c < Lay::kNC; ++c)
              tmem_cp_32x128b_x4(tmem + sf_col + 16 + (t * Lay::kNC + c) * 4,
                                 desc_sf_copy(sfb_addr + (t * Lay::kNC + c) * 512));
          }
#pragma unroll
          for (int t = 0; t < 4; ++t)
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
      }
      tc_commit(acc_full);
      mbar_wait_drain(acc_full, 0, kWaitLimitNs);
    }
  } else if (warp == 2) {
    // Scale stager.  For K-block kb and MMA K-step t the MMA reads, for operand
    // row q (0..127 within a 128-row chunk), the 4 scales of K-groups
    // 16 kb + 4 t + j from TMEM lane q%32, column q/32, byte j.  tcgen05.cp
    // 32x128b.warpx4 fills that from a 512-byte smem chunk in which row q%32
    // holds 16 bytes: [q/32 = 0..3][j = 0..3].  Rows 0..15 of a chunk cover
    // 16-row blocks 0,2,4,6 of the chunk and rows 16..31 blocks 1,3,5,7, so a
    // chunk is two distinct 16-byte patterns, each repeated 16 times.
    const int nA = 4 * 2, nB = 4 * Lay::kNC * 2;
    for (int i = 0; i < T; ++i) {
      const int s = i % kGmStages;
      const uint32_t ph = (i / kGmStages) & 1;
      if (!mbar_wait(&empty[s], ph ^ 1, p.status, abortp)) break;
      if (i < KB) {
        const int c = i / kSfChunk, kk = i % kSfChunk;   // chunk, K-block within it
        if (p.sf_tma && kk == 0 && !mbar_wait(&sf_full[c % kSfSlots], (c / kSfSlots) & 1, p.status, abortp))
          break;
        uint8_t* sfa = smem + s * Lay::kStage + Lay::kA + Lay::kB;
        uint8_t* sfb = sfa + Lay::kSFA;
        const uint8_t* cA = compact + (c % kSfSlots) * Lay::kCSlot;
        const uint8_t* cB = cA + Lay::kCA;
        if (lane < nA + nB) {
          const bool isA = lane < nA;
          const int idx = isA ? lane : lane - nA;
          const int hh = idx & 1;
          const int t = isA ? idx >> 1 : idx / (2 * Lay::kNC);
          const int c = isA ? 0 : (idx >> 1) % Lay::kNC;
          uint32_t word[4];
          if (p.sf_tma) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int rb = c * 8 + hh + 2 * w;   // row-block within the tile
              const int g = 16 * kk + 4 * t;     // first K-group of this MMA step within the chunk
              if (isA) {
                word[w] = *reinterpret_cast<const uint32_t*>(cA + rb * (16 * kSfChunk) + g);
              } else if (!p.sfb_transposed) {
                word[w] = *reinterpret_cast<const uint32_t*>(cB + rb * (16 * kSfChunk) + g);
              } else {
                uint32_t wv = 0;
#pragma unroll
                for (int j = 0; j < 4; ++j) wv |= static_cast<uint32_t>(cB[(g + j) * (BN / 16) + rb]) << (8 * j);
                word[w] = wv;
              }
            }
          } else {
            const uint8_t* src = isA ? p.sfa : p.sfb;
            const long long rs = isA ? p.sfa_rs : p.sfb_rs;
            const long long gs = isA ? p.sfa_gs : p.sfb_gs;
            const int rb0 = (isA ? m0 : n0 + 128 * c) / 16 + hh;
            const int nrb = isA ? Mb : Nb;
            const int g0 = i * 16 + t * 4;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const int rb = rb0 + 2 * w;
              uint32_t wv = 0;
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int g = g0 + j;
                const uint32_t b = (rb < nrb && g < KG) ? src[rb * rs + g * gs] : 0u;
                wv |= b << (8 * j);
              }
              word[w] = wv;
            }
          }
          const uint4 pat = make_uint4(word[0], word[1], word[2], word[3]);
          uint8_t* chunk = isA ? sfa + t * 512 : sfb + (t * Lay::kNC + c) * 512;
          uint4* dst = reinterpret_cast<uint4*>(chunk + hh * 16 * 16);
#pragma unroll
          for (int r = 0; r < 16; ++r) dst[r] = pat;
          fence_proxy_async_smem();
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sf_ready[s]);
    }
  } else if (warp >= 4) {
    if (mbar_wait(acc_full, 0, p.status, abortp)) {
      __syncwarp();
      // Every MMA has completed, so every TMA load has landed and been consumed:
      // the pipeline smem is free.  Warp q stages its 32 rows x BN columns as
      // boxes of 32 rows x 128 bytes (128-byte swizzle, 4 KB each) at q * (BN/ebox) * 4 KB.
      tc_fence_after();
      const int q = warp & 3;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16);
      const __nv_bfloat16* bias = static_cast<const __nv_bfloat16*>(p.bias);
      const int ebox = p.out_bf16 ? 64 : 32;               // elements per 128-byte box row
      uint8_t* region = smem + q * (BN / ebox) * 4096;
      // GELU-backward: second bf16 tile (GELU(h)) staged after the first four warps' regions
      uint8_t* region2 = smem + 4 * (BN / 64) * 4096 + q * (BN / 64) * 4096;
      const int row = m0 + 32 * q + lane;
      for (int c0 = 0; c0 < BN; c0 += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(taddr + c0, v);
        tmem_ld_wait();
        float f[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) f[e] = __uint_as_float(v[e]);
        const int nb = n0 + c0;
        if (bias) {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (nb + e < p.N) f[e] += __bfloat162float(bias[nb + e]);
        }
        float g[32];
        if (p.epi_gelu_bwd) {
          // d_h = d_a * GELU'(h) and GELU(h), h read for this row's 32 columns
          float hv[32];
#pragma unroll
          for (int e = 0; e < 32; ++e) hv[e] = 0.0f;
          if (row < p.M && nb < p.N) {
            const uint4* hp = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.h) +
                                                             static_cast<long long>(row) * p.N + nb);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const uint4 u = hp[k];
              const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                hv[8 * k + 2 * e] = bf16_bits_to_f32(wd[e] & 0xFFFFu);
                hv[8 * k + 2 * e + 1] = bf16_bits_to_f32(wd[e] >> 16);
              }
            }
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            float dg;
            gelu_tanh_and_grad(hv[e], &g[e], &dg);
            f[e] *= dg;
          }
        }
        uint8_t* rowp = region + (c0 / ebox) * 4096 + lane * 128;
        if (p.out_bf16) {
          const int j0 = (c0 % 64) / 8;                    // first 16-byte chunk of this 32-column slice
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint32_t w[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 b = __floats2bfloat162_rn(f[8 * k + 2 * e], f[8 * k + 2 * e + 1]);
              w[e] = *reinterpret_cast<const uint32_t*>(&b);
            }
            *reinterpret_cast<uint4*>(rowp + (((j0 + k) ^ (lane & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
          }
          if (p.epi_gelu_bwd) {
            uint8_t* rowg = region2 + (c0 / 64) * 4096 + lane * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 b = __floats2bfloat162_rn(g[8 * k + 2 * e], g[8 * k + 2 * e + 1]);
                w[e] = *reinterpret_cast<const uint32_t*>(&b);
              }
              *reinterpret_cast<uint4*>(rowg + (((j0 + k) ^ (lane & 7)) * 16)) = make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 8; ++k)
            *reinterpret_cast<uint4*>(rowp + ((k ^ (lane & 7)) * 16)) =
                make_uint4(__float_as_uint(f[4 * k]), __float_as_uint(f[4 * k + 1]), __float_as_uint(f[4 * k + 2]),
                           __float_as_uint(f[4 * k + 3]));
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0 && m0 + 32 * q < p.M) {
        for (int b = 0; b < BN / ebox; ++b) {
          const int x = n0 + b * ebox;
          if (x < p.N) tma_store_2d(&tmOut, region + b * 4096, x, m0 + 32 * q);
          if (x < p.N && p.epi_gelu_bwd) tma_store_2d(&tmOut2, region2 + b * 4096, x, m0 + 32 * q);
        }
        bulk_commit();
        bulk_wait_read_all();
      }
      __syncwarp();
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
                            const CUtensorMap& tmB2, const CUtensorMap& tmSFA, const CUtensorMap& tmSFB,
                            const CUtensorMap& tmOut, const CUtensorMap& tmOut2, const GemmParams& p,
                            cudaStream_t stream) {
  constexpr int BN = kGemmBN;
  using Lay = GemmLayout<BN>;
  cudaError_t e = cudaFuncSetAttribute(gemm_fp4_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(Lay::kSmem));
  if (e != cudaSuccess) return e;
  dim3 grid((p.N + BN - 1) / BN, (p.M + 127) / 128);
  gemm_fp4_kernel<BN><<<grid, kGmThreads, Lay::kSmem, stream>>>(tmA, tmB, tmA2, tmB2, tmSFA, tmSFB, tmOut,
                                                                  tmOut2, p);
  return cudaGetLastError();
}

}  // namespace ft
