// Adapter gradients: out[p, j] (+)= sum_m T[m, p] V[m, v0 + j].
//
// FourTune §3.2: parameter gradients exist only for the LoRA adapter (no weight
// gradient for the frozen residual or stabilizer).  With L = X [S_dn | A] and
// P = G [S_up ; B]^T saved in bf16:
//   dA = X^T P[:, r_s:]   (T = X,  V = P, out [K, r] row-major)
//   dB = L[:, r_s:]^T G   (T = G,  V = L, out [r, N] row-major, written as dB^T)
// For the MLP's FC2, dA = bf16(GELU(h))^T P[:, r_s:] takes T = h (saved by the
// forward): the epilogue warps, idle during the main loop, replace each staged
// h tile by bf16(GELU_tanh(h)) in place before its MMAs (t_gelu), so GELU(h) is
// never stored.
// Both problems run in one launch (the CTA index selects the problem).  Each is
// a reduction over the M tokens of a tall bf16 matrix against a thin one:
// HBM-bound (T is read once).  The tensor cores take both operands MN-major
// straight from the TMA tiles: T tile [128 m x 128 p] (two 128-byte swizzled
// boxes of 64 p), V tile [128 m x 64 j]; tcgen05.mma kind::f16 M=128 (p),
// N=64 (j), K=16 (m), 8 per tile.  CTAs split M; the last CTA of a p-tile sums
// the fp32 partials in split order (deterministic).
#include "common.cuh"
#include "kernels.h"

namespace ft {

constexpr int kTgStages = 4;
constexpr int kTgThreads = 384;        // warps 4..11 transform T when t_gelu; 4..7 also drain the accumulator
constexpr int kTgXWarps = 8;
constexpr uint32_t kTgTBox = 128 * 128;            // 128 m rows x 64 bf16
constexpr uint32_t kTgStage = 2 * kTgTBox + kTgTBox;  // T (two boxes) + V
constexpr uint32_t kTgSmem = 1024 + kTgStages * kTgStage + 256;
static_assert((3 * kTgStages + 1) * 8 + 8 + 16 <= 256, "barriers, TMEM slot and flags fit the tail");

__global__ void __launch_bounds__(kTgThreads, 1)
    tgrad_kernel(const __grid_constant__ CUtensorMap tmT0, const __grid_constant__ CUtensorMap tmV0,
                 const __grid_constant__ CUtensorMap tmT1, const __grid_constant__ CUtensorMap tmV1,
                 const TgradParams p0, const TgradParams p1) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTgStages * kTgStage);
  uint64_t* empty = full + kTgStages;
  uint64_t* acc_full = empty + kTgStages;
  uint64_t* ready = acc_full + 1;           // [kTgStages] t_gelu: the stage's T tile transformed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ready + kTgStages);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* s_last = abort_flag + 1;
  volatile int* s_ok = s_last + 1;  // [4]
  volatile int* abortp = abort_flag;

  // which problem and tile this CTA owns
  const int tiles0 = ((p0.P + 127) / 128) * p0.nsplit;
  const bool second = static_cast<int>(blockIdx.x) >= tiles0;
  const TgradParams& p = second ? p1 : p0;
  const CUtensorMap* tmT = second ? &tmT1 : &tmT0;
  const CUtensorMap* tmV = second ? &tmV1 : &tmV0;
  const int local = second ? static_cast<int>(blockIdx.x) - tiles0 : static_cast<int>(blockIdx.x);
  const int ptile = local / p.nsplit;
  const int split = local % p.nsplit;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pbase = ptile * 128;
  const int MT = (p.M + 127) / 128;
  const int mt0 = split * p.mt_per_split;
  const int mt1 = min(MT, mt0 + p.mt_per_split);
  const int nt = max(0, mt1 - mt0);
  const int Ppad = ((p.P + 127) / 128) * 128;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTgStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&ready[s], kTgXWarps);
    }
    mbar_init(acc_full, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(tmT);
    tma_prefetch(tmV);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_launch_dependents();
  pdl_wait_prior();

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nt; ++i) {
        const int s = i % kTgStages;
        const uint32_t ph = (i / kTgStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.status, abortp)) break;
        uint8_t* st = smem + s * kTgStage;
        const int my = (mt0 + i) * 128;
        mbar_arrive_expect_tx(&full[s], kTgStage);
        tma_load_2d(st, tmT, &full[s], pbase, my);
        tma_load_2d(st + kTgTBox, tmT, &full[s], pbase + 64, my);
        tma_load_2d(st + 2 * kTgTBox, tmV, &full[s], p.v0, my);
        issued = i + 1;
      }
      if (*abortp) {
        for (int i = max(0, issued - kTgStages); i < issued; ++i)
          mbar_wait_drain(&full[i % kTgStages], (i / kTgStages) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, 64, true, true);
      for (int i = 0; i < nt; ++i) {
        const int s = i % kTgStages;
        const uint32_t ph = (i / kTgStages) & 1;
        if (!mbar_wait(&full[s], ph, p.status, abortp)) break;
        if (p.t_gelu && !mbar_wait(&ready[s], ph, p.status, abortp)) break;
        tc_fence_after();
        const uint32_t ta = smem_u32(smem + s * kTgStage);
        const uint32_t va = ta + 2 * kTgTBox;
#pragma unroll
        for (int t = 0; t < 8; ++t)
          mma_bf16(tmem, desc_mnmajor_sw128(ta + 2048 * t, kTgTBox), desc_mnmajor_sw128(va + 2048 * t, kTgTBox),
                   idesc, (i | t) != 0 ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      tc_commit(acc_full);
      mbar_wait_drain(acc_full, 0, kWaitLimitNs);
    }
  } else if (warp >= 4) {
    bool ok = true;
    if (p.t_gelu) {
      // the T part of every stage (two 16 KB boxes of bf16 h) -> bf16(GELU(h)), in
      // place, by eight warps (enough in flight to hide the exponential's latency)
      const int t = static_cast<int>(threadIdx.x) - 128;   // 0..255
      for (int i = 0; i < nt && ok; ++i) {
        const int s = i % kTgStages;
        bool okw = true;
        if (lane == 0) okw = mbar_wait(&full[s], (i / kTgStages) & 1, p.status, abortp);
        ok = __shfl_sync(0xFFFFFFFFu, okw ? 1 : 0, 0) != 0;
        if (!ok) break;
        uint4* tile = reinterpret_cast<uint4*>(smem + s * kTgStage);
#pragma unroll 4
        for (int k = t; k < static_cast<int>(2 * kTgTBox / 16); k += 32 * kTgXWarps) {
          uint4 x = tile[k];
          uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(gelu_tanh(bf16_bits_to_f32(w[e] & 0xFFFFu)),
                                                           gelu_tanh(bf16_bits_to_f32(w[e] >> 16)));
            w[e] = *reinterpret_cast<const uint32_t*>(&b);
          }
          tile[k] = make_uint4(w[0], w[1], w[2], w[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ready[s]);
      }
    }
    if (warp < 8) {   // warps 8..11 only transform
      const bool mine = ok && (nt > 0) && mbar_wait(acc_full, 0, p.status, abortp);
      if (lane == 0) s_ok[warp - 4] = mine ? 1 : 0;
      named_bar_sync(1, 128);
      const bool go = s_ok[0] && s_ok[1] && s_ok[2] && s_ok[3];
      if (go) {
        __syncwarp();
        tc_fence_after();
        const int q = warp & 3;
        const int prow = pbase + 32 * q + lane;
        const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16);
        float acc[64];
        {
          uint32_t a[32], b[32];
          tmem_ld_32x32b_x32(taddr, a);
          tmem_ld_32x32b_x32(taddr + 32, b);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            acc[e] = __uint_as_float(a[e]);
            acc[32 + e] = __uint_as_float(b[e]);
          }
        }
        bool write = true;
        if (p.nsplit > 1) {
          // only the r columns that are output travel through the partials
          const int nq = (p.r + 3) / 4;
          float4* dst = reinterpret_cast<float4*>(p.part + (static_cast<long long>(split) * Ppad + prow) * 64);
#pragma unroll
          for (int e = 0; e < 16; ++e)
            if (e < nq) dst[e] = make_float4(acc[4 * e], acc[4 * e + 1], acc[4 * e + 2], acc[4 * e + 3]);
          // one thread's acq_rel counter increment publishes the CTA's partial
          // (ordered before it by the barrier) and, in the last CTA, orders its
          // partial reads (after the next barrier) after all other increments
          named_bar_sync(1, 128);
          if (threadIdx.x == 128) {
            const int prev = atomic_add_acq_rel_gpu(&p.counters[ptile], 1);
            *s_last = (prev == p.nsplit - 1);
          }
          named_bar_sync(1, 128);
          write = *s_last != 0;
          if (write) {
            // sum every split's partial row in split order (vector loads, registers
            // only), two splits' loads in flight at a time
#pragma unroll
            for (int e = 0; e < 64; ++e) acc[e] = 0.0f;
            for (int sp = 0; sp < p.nsplit; sp += 2) {
              const float4* src0 = reinterpret_cast<const float4*>(p.part + (static_cast<long long>(sp) * Ppad + prow) * 64);
              const float4* src1 = src0 + static_cast<long long>(Ppad) * 16;
              const bool two = sp + 1 < p.nsplit;
#pragma unroll
              for (int h = 0; h < 2; ++h) {   // 8 float4 of each split per round (registers)
                float4 x0[8], x1[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  if (8 * h + e < nq) {
                    x0[e] = __ldcg(src0 + 8 * h + e);
                    if (two) x1[e] = __ldcg(src1 + 8 * h + e);
                  }
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                  if (8 * h + e < nq) {
                    const int c = 4 * (8 * h + e);
                    acc[c] += x0[e].x;
                    acc[c + 1] += x0[e].y;
                    acc[c + 2] += x0[e].z;
                    acc[c + 3] += x0[e].w;
                    if (two) {
                      acc[c] += x1[e].x;
                      acc[c + 1] += x1[e].y;
                      acc[c + 2] += x1[e].z;
                      acc[c + 3] += x1[e].w;
                    }
                  }
                }
              }
            }
            if (threadIdx.x == 128) p.counters[ptile] = 0;
          }
        }
        if (write && prow < p.P) {
#pragma unroll
          for (int j = 0; j < 64; ++j) {
            if (j < p.r) {
              float* o = p.out + prow * p.out_sp + j * p.out_sj;
              *o = p.accumulate ? *o + acc[j] : acc[j];
            }
          }
        }
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

cudaError_t launch_tgrad2(const CUtensorMap& tmT0, const CUtensorMap& tmV0, const TgradParams& p0,
                          const CUtensorMap& tmT1, const CUtensorMap& tmV1, const TgradParams& p1,
                          cudaStream_t stream) {
  cudaError_t e =
      cudaFuncSetAttribute(tgrad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kTgSmem));
  if (e != cudaSuccess) return e;
  const int tiles0 = ((p0.P + 127) / 128) * p0.nsplit;
  const int tiles1 = ((p1.P + 127) / 128) * p1.nsplit;
  return launch_pdl(tgrad_kernel, dim3(tiles0 + tiles1), dim3(kTgThreads), kTgSmem, stream, tmT0, tmV0, tmT1, tmV1,
                    p0, p1);
}

}  // namespace ft
