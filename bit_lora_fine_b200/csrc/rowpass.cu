// Fused input pass: 16x16-block FP4 quantization of a bf16 row tile and its
// low-rank projection, reading the input from HBM once.
//
// FourTune §3.3 "LoRA Fusion": all three branches share the same input during
// quantization and down-projection, so one kernel quantizes X for the 4-bit
// branch and computes L = X [S_dn | A] for the stabilizer and LoRA branches.
// The backward uses the same kernel on the incoming gradient G with [S_up; B]
// (P = G [S_up; B]^T).
//
// CTA = 128 rows x a contiguous range of 64-column tiles (split-K when M alone
// gives too few CTAs; two CTAs fit on an SM for R <= 64).  Warp roles:
//   warp 0 lane 0  TMA producer: input tile [128 x 64] bf16 (128-byte rows,
//                  128-byte swizzle) and the projection tile, into a 4-stage ring
//   warp 1         TMEM owner; lane 0 issues tcgen05.mma kind::f16 (M=128,
//                  N=R rounded as below, K=16) x 4 per tile into TMEM
//   warps 4..11    each quantizes one 16-row block of the same smem tile, then
//                  the eight drain the accumulator (two warps per TMEM lane
//                  quadrant).  One split: L in bf16 straight from TMEM.  Several
//                  splits: the splits of a row tile form a thread-block cluster;
//                  each CTA parks its fp32 partial in its own (now idle) smem and
//                  every CTA sums one slice of rows over all ranks in rank order
//                  through distributed shared memory (deterministic, no global
//                  partials).  A global-memory variant (partials in scratch, the
//                  last CTA of the row tile sums them) serves the static-scratch
//                  entry point.
// The projection matrix is read either K-major (W^T [R, K], rows of 128 bytes,
// N = R) or MN-major (D [K, R] with R contiguous: TMA boxes of 64 k-rows x 64
// r, N = R rounded up to 64, the extra columns zero-filled by the TMA).
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace ft {

constexpr int kRpStages = 4;
constexpr int kRpThreads = 384;
constexpr int kRpQuantWarps = 8;
constexpr uint32_t kRpXBytes = 128 * 128;  // 128 rows x 64 bf16

__host__ __device__ constexpr int rp_mn_chunks(int R) { return (R + 63) / 64; }
__host__ __device__ constexpr int rp_n_mma(int R, int mn) { return mn ? 64 * rp_mn_chunks(R) : R; }
__host__ __device__ constexpr uint32_t rp_w_bytes(int R, int mn) {
  return mn ? 8192u * rp_mn_chunks(R) : static_cast<uint32_t>(R) * 128u;
}
__host__ __device__ constexpr uint32_t rp_stage_bytes(int R, int mn) {
  return kRpXBytes + ((rp_w_bytes(R, mn) + 1023u) & ~1023u);
}
__host__ __device__ constexpr uint32_t rp_smem_bytes(int R, int mn) {
  return 1024 + kRpStages * rp_stage_bytes(R, mn) + 256;
}

template <int RCOLS, bool GELU>
__global__ void __launch_bounds__(kRpThreads, 2)  // two CTAs per SM: registers <= 80
    rowpass_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                   const RowpassParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int R = p.R;
  const int mn = p.w_mn_major;
  const int nmma = rp_n_mma(R, mn);
  const uint32_t w_bytes = rp_w_bytes(R, mn);
  const uint32_t stage_bytes = rp_stage_bytes(R, mn);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kRpStages * stage_bytes);
  uint64_t* empty = full + kRpStages;
  uint64_t* acc_full = empty + kRpStages;
  uint64_t* ready = acc_full + 1;  // [kRpStages] GELU mode: transformed tile written back
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(ready + kRpStages);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  int* s_last = abort_flag + 1;
  volatile int* s_ok = s_last + 1;  // [kRpQuantWarps]
  volatile int* abortp = abort_flag;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128;
  const int split = blockIdx.y;
  const int KT = (p.K + 63) / 64;
  const int kt0 = split * p.kt_per_split;
  const int kt1 = min(KT, kt0 + p.kt_per_split);
  const int nt = max(0, kt1 - kt0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kRpQuantWarps);  // MMA commit + one arrive per quantizer warp
    }
    mbar_init(acc_full, 1);
    for (int s = 0; s < kRpStages; ++s) mbar_init(&ready[s], kRpQuantWarps);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, RCOLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch(&tmX);
    tma_prefetch(&tmW);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      for (int i = 0; i < nt; ++i) {
        const int s = i % kRpStages;
        const uint32_t ph = (i / kRpStages) & 1;
        if (!mbar_wait(&empty[s], ph ^ 1, p.status, abortp)) break;
        uint8_t* st = smem + s * stage_bytes;
        const int kc = (kt0 + i) * 64;
        mbar_arrive_expect_tx(&full[s], kRpXBytes + w_bytes);
        tma_load_2d(st, &tmX, &full[s], kc, m0);
        if (mn) {
          for (int c = 0; c < rp_mn_chunks(R); ++c)
            tma_load_2d(st + kRpXBytes + 8192 * c, &tmW, &full[s], 64 * c, kc);
        } else {
          tma_load_2d(st + kRpXBytes, &tmW, &full[s], kc, 0);
        }
        issued = i + 1;
      }
      if (*abortp) {  // let copies already in flight land before the CTA exits
        for (int i = max(0, issued - kRpStages); i < issued; ++i)
          mbar_wait_drain(&full[i % kRpStages], (i / kRpStages) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, nmma, false, mn != 0);
      for (int i = 0; i < nt; ++i) {
        const int s = i % kRpStages;
        const uint32_t ph = (i / kRpStages) & 1;
        if (!mbar_wait(&full[s], ph, p.status, abortp)) break;
        if (GELU && !mbar_wait(&ready[s], ph, p.status, abortp)) break;
        tc_fence_after();
        const uint32_t xa = smem_u32(smem + s * stage_bytes);
        const uint32_t wa = xa + kRpXBytes;
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const uint64_t bdesc = mn ? desc_mnmajor_sw128(wa + 2048 * t, 8192) : desc_kmajor_sw128(wa + 32 * t);
          mma_bf16(tmem, desc_kmajor_sw128(xa + 32 * t), bdesc, idesc, (i | t) != 0 ? 1u : 0u);
        }
        tc_commit(&empty[s]);
      }
      tc_commit(acc_full);
      mbar_wait_drain(acc_full, 0, kWaitLimitNs);  // every MMA done before TMEM can be freed
    }
  } else if (warp >= 4) {
    const int w8 = warp - 4;        // 16-row block of the tile this warp quantizes
    const int h = lane & 1;         // 32-column half of the 64-column tile
    const int r = w8 * 16 + (lane >> 1);
    const long long half_k = p.K / 2;
    const int kblocks = p.K / 16;
    const bool block_row_ok = m0 + w8 * 16 < p.M;
    bool ok = true;
    for (int i = 0; i < nt; ++i) {
      const int s = i % kRpStages;
      const uint32_t ph = (i / kRpStages) & 1;
      if (!mbar_wait(&full[s], ph, p.status, abortp)) {
        ok = false;
        break;
      }
      uint8_t* tile = smem + s * stage_bytes;
      float v[32];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int phys = (4 * h + q) ^ (r & 7);
        const uint4 u = *reinterpret_cast<const uint4*>(tile + r * 128 + phys * 16);
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[q * 8 + 2 * e] = bf16_bits_to_f32(wd[e] & 0xFFFFu);
          v[q * 8 + 2 * e + 1] = bf16_bits_to_f32(wd[e] >> 16);
        }
      }
      if (GELU) {
        // a = GELU(h) in fp32; bf16(a) goes back into the tile for the down-projection
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = gelu_tanh(v[e]);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t wd[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1]);
            wd[e] = *reinterpret_cast<const uint32_t*>(&b);
          }
          const int phys = (4 * h + q) ^ (r & 7);
          *reinterpret_cast<uint4*>(tile + r * 128 + phys * 16) = make_uint4(wd[0], wd[1], wd[2], wd[3]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&ready[s]);
          mbar_arrive(&empty[s]);
        }
      } else {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);  // the tile is in registers: release the stage early
      }
      float amax[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        float a = 0.0f;
#pragma unroll
        for (int e = 0; e < 16; ++e) a = fmaxf(a, fabsf(v[16 * j + e]));
#pragma unroll
        for (int off = 2; off < 32; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
        amax[j] = a;
      }
      const int cstart = (kt0 + i) * 64 + 32 * h;
      const bool inside = block_row_ok && cstart < p.K;
      if (inside || p.sf_mma) {
        // rows past M and columns past K were zero-filled by the TMA: their scale is 0
        uint32_t packed[4], sc[2];
        if (GELU)
          quantize_2blocks_div(v, amax, packed, sc);
        else
          quantize_2blocks(v, amax, packed, sc);
        if (inside) {
          *reinterpret_cast<uint4*>(p.codes + static_cast<long long>(m0 + r) * half_k + cstart / 2) =
              make_uint4(packed[0], packed[1], packed[2], packed[3]);
          if ((lane >> 1) == 0) {
            const long long srow = (m0 / 16 + w8) * static_cast<long long>(kblocks);
            p.scales[srow + cstart / 16] = static_cast<uint8_t>(sc[0]);
            p.scales[srow + cstart / 16 + 1] = static_cast<uint8_t>(sc[1]);
          }
          if (GELU && p.dbg_a) {
            float4* dst = reinterpret_cast<float4*>(p.dbg_a + static_cast<long long>(m0 + r) * p.K + cstart);
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
          }
        }
        if (p.sf_mma) {
          // MMA-ready copy: groups 2h, 2h+1 of k-step kt0+i for row r of chunk blockIdx.x
          const size_t o = (static_cast<size_t>(blockIdx.x) * KT + (kt0 + i)) * 512 + (r & 31) * 16 + (r >> 5) * 4 + 2 * h;
          *reinterpret_cast<uint16_t*>(p.sf_mma + o) = static_cast<uint16_t>(sc[0] | (sc[1] << 8));
        }
      }
    }

    // ---- epilogue: accumulator -> L (bf16) or fp32 partials.  All eight warps
    // agree on whether to run it, so the named barriers below are always
    // reached by all of them.
    const bool mine = ok && mbar_wait(acc_full, 0, p.status, abortp);
    if (lane == 0) s_ok[w8] = mine ? 1 : 0;
    named_bar_sync(1, 32 * kRpQuantWarps);
    bool go = true;
#pragma unroll
    for (int w = 0; w < kRpQuantWarps; ++w) go = go && s_ok[w];
    if (go) {
      __syncwarp();
      tc_fence_after();
      const int q = warp & 3;                       // TMEM lane quadrant of this warp
      const int row = m0 + 32 * q + lane;
      const uint32_t taddr = tmem + (static_cast<uint32_t>(32 * q) << 16);
      const bool row_ok = row < p.M;
      const int half = (warp - 4) >> 2;             // which 16-column chunks this warp drains
      float* parked = reinterpret_cast<float*>(smem) + (32 * q + lane) * (R + 4);
      for (int c0 = 16 * half; c0 < R; c0 += 32) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(taddr + c0, v);
        tmem_ld_wait();
        if (p.cluster_reduce) {                     // park the partial in this CTA's smem
          float4* dst = reinterpret_cast<float4*>(parked + c0);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                 __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
          continue;
        }
        if (!row_ok) continue;
        if (p.nsplit == 1) {
          uint32_t w[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const __nv_bfloat162 b = __floats2bfloat162_rn(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1]));
            w[e] = *reinterpret_cast<const uint32_t*>(&b);
          }
          uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.L) + static_cast<long long>(row) * R + c0);
          dst[0] = make_uint4(w[0], w[1], w[2], w[3]);
          dst[1] = make_uint4(w[4], w[5], w[6], w[7]);
        } else {
          float4* dst = reinterpret_cast<float4*>(p.part + (static_cast<long long>(split) * p.M + row) * R + c0);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_float4(__uint_as_float(v[4 * e]), __uint_as_float(v[4 * e + 1]),
                                 __uint_as_float(v[4 * e + 2]), __uint_as_float(v[4 * e + 3]));
        }
      }
      if (p.nsplit > 1 && !p.cluster_reduce) {
        // the last CTA of this row tile to finish sums every split's partial, in split order
        __threadfence();
        named_bar_sync(1, 32 * kRpQuantWarps);
        if (threadIdx.x == 128) {
          const int prev = atomicAdd(&p.counters[blockIdx.x], 1);
          *s_last = (prev == p.nsplit - 1);
        }
        named_bar_sync(1, 32 * kRpQuantWarps);
        if (*s_last) {
          __threadfence();
          if (row_ok) {
            for (int c0 = 8 * half; c0 < R; c0 += 16) {
              float acc[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) acc[e] = 0.0f;
              for (int sp = 0; sp < p.nsplit; ++sp) {
                const float4* src =
                    reinterpret_cast<const float4*>(p.part + (static_cast<long long>(sp) * p.M + row) * R + c0);
                const float4 a = __ldcg(src), b = __ldcg(src + 1);
                acc[0] += a.x; acc[1] += a.y; acc[2] += a.z; acc[3] += a.w;
                acc[4] += b.x; acc[5] += b.y; acc[6] += b.z; acc[7] += b.w;
              }
              uint32_t w[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const __nv_bfloat162 bb = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
                w[e] = *reinterpret_cast<const uint32_t*>(&bb);
              }
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.L) + static_cast<long long>(row) * R + c0) =
                  make_uint4(w[0], w[1], w[2], w[3]);
            }
          }
          if (threadIdx.x == 128) p.counters[blockIdx.x] = 0;
        }
      }
    }
  }

  if (p.cluster_reduce) {
    // every split of this row tile has parked its partial: rank c sums rows
    // [c * rows_per, (c + 1) * rows_per) over ranks 0..nsplit-1 in order
    __syncwarp();
    cluster_sync_all();
    if (warp >= 4) {
      const int ns = p.nsplit;
      const int rows_per = (128 + ns - 1) / ns;
      const int r_lo = static_cast<int>(cluster_ctarank()) * rows_per;
      const int r_hi = min(128, r_lo + rows_per);
      const int c4n = R / 4;
      const uint32_t base = smem_u32(smem);
      for (int idx = threadIdx.x - 128; idx < (r_hi - r_lo) * c4n; idx += 32 * kRpQuantWarps) {
        const int rl = r_lo + idx / c4n;
        const int c = 4 * (idx % c4n);
        const uint32_t off = base + static_cast<uint32_t>((rl * (R + 4) + c) * 4);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int j = 0; j < ns; ++j) {
          const float4 v = ld_cluster_f4(map_cluster(off, static_cast<uint32_t>(j)));
          acc.x += v.x;
          acc.y += v.y;
          acc.z += v.z;
          acc.w += v.w;
        }
        const int grow = m0 + rl;
        if (grow < p.M) {
          const __nv_bfloat162 b0 = __floats2bfloat162_rn(acc.x, acc.y);
          const __nv_bfloat162 b1 = __floats2bfloat162_rn(acc.z, acc.w);
          *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.L) + static_cast<long long>(grow) * R + c) =
              make_uint2(*reinterpret_cast<const uint32_t*>(&b0), *reinterpret_cast<const uint32_t*>(&b1));
        }
      }
    }
    __syncwarp();
    cluster_sync_all();  // no CTA leaves while another may still read its smem
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, RCOLS);
  }
}

template <int RCOLS, bool GELU>
static cudaError_t launch_rowpass_t(const CUtensorMap& tmX, const CUtensorMap& tmW, const RowpassParams& p,
                                    cudaStream_t stream) {
  const uint32_t smem = rp_smem_bytes(p.R, p.w_mn_major);
  cudaError_t e = cudaFuncSetAttribute(rowpass_kernel<RCOLS, GELU>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((p.M + 127) / 128, p.nsplit);
  cfg.blockDim = dim3(kRpThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = p.cluster_reduce ? p.nsplit : 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, rowpass_kernel<RCOLS, GELU>, tmX, tmW, p);
}

cudaError_t launch_rowpass(const CUtensorMap& tmX, const CUtensorMap& tmW, const RowpassParams& p,
                           cudaStream_t stream) {
  const int n = rp_n_mma(p.R, p.w_mn_major);
  if (p.gelu_input) {
    if (n <= 32) return launch_rowpass_t<32, true>(tmX, tmW, p, stream);
    if (n <= 64) return launch_rowpass_t<64, true>(tmX, tmW, p, stream);
    return launch_rowpass_t<128, true>(tmX, tmW, p, stream);
  }
  if (n <= 32) return launch_rowpass_t<32, false>(tmX, tmW, p, stream);
  if (n <= 64) return launch_rowpass_t<64, false>(tmX, tmW, p, stream);
  return launch_rowpass_t<128, false>(tmX, tmW, p, stream);
}

int rowpass_ctas_per_sm(int R, int w_mn_major) {
  return rp_smem_bytes(R, w_mn_major) * 2 <= 227u * 1024u ? 2 : 1;
}

// ---------------------------------------------------------------------------
// Allocation-free variant of the row pass.  Its split-K partial sums, split
// counters and status word live in this file-scope device array instead of a
// caller-provided workspace, for callers that cannot allocate device memory.
// Every GPU that loads the library holds the array until the process exits.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_rowpass_static_scratch[kRowpassStaticScratchBytes];

// Device address of the array for the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// cudaGetSymbolAddress once per device (with that device current) and cached.
cudaError_t rowpass_static_scratch(void** out) {
  static void* addr[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_rowpass_static_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace ft
