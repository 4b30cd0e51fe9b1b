// Fused input pass: 16x16-block FP4 quantization of a bf16 row tile and its
// low-rank projection, reading the input from HBM once.
//
// FourTune §3.3 "LoRA Fusion": all three branches share the same input during
// quantization and down-projection, so one kernel quantizes X for the 4-bit
// branch and computes L = X [S_dn | A] for the stabilizer and LoRA branches.
// The backward uses the same kernel on the incoming gradient G with [S_up; B]
// (P = G [S_up; B]^T).
//
// CTA = 128 rows x a contiguous range of 64-column tiles; when M alone gives
// too few CTAs for the SMs the K range is split (split-K).  Warp roles:
//   warp 0 lane 0  TMA producer: input tile [128 x 64] bf16 (128-byte rows,
//                  128-byte swizzle) and the projection tile, into a ring of
//                  p.stages slots
//   warp 1         TMEM owner; lane 0 issues tcgen05.mma kind::f16 (M=128,
//                  N=R rounded as below, K=16) x 4 per tile into TMEM
//   warps 4..19    sixteen quantizer warps: warp w takes the 16-row block w/2
//                  and the 32-column half w%2 of the smem tile, a lane one
//                  16x16 block row (block amax by warp shuffles), so that the
//                  ALU work of the quantizer is spread over enough warps to
//                  hide its latency.  The same sixteen warps then drain the
//                  accumulator (four per TMEM lane quadrant, 16 columns
//                  each).  One split: L in bf16 straight from TMEM.  Several
//                  splits: each CTA writes its fp32 partial to scratch, and
//                  the last CTA of the row tile (split counter) sums them in
//                  split order (deterministic), rounding once, with a batch of
//                  splits of two 4-column pieces in flight per thread.
// The projection matrix is read either K-major (W^T [R, K], rows of 128 bytes,
// N = R) or MN-major (D [K, R] with R contiguous: TMA boxes of 64 k-rows x 64
// r, N = R rounded up to 64, the extra columns zero-filled by the TMA).
#include <mutex>

#include "common.cuh"
#include "kernels.h"

namespace ft {

constexpr int kRpStages = 8;               // largest ring (p.stages <= this)
constexpr int kRpQuantWarps = 16;
constexpr int kRpThreads = 32 * (4 + kRpQuantWarps);
constexpr uint32_t kRpXBytes = 128 * 128;  // 128 rows x 64 bf16
constexpr int kRpSumBatch = 4;             // split partials loaded per batch by the last CTA
constexpr int kRpSumItems = 2;             // 4-column pieces per thread and pass of that sum
constexpr uint32_t kRpTail = 512;          // barriers, TMEM slot, flags

__host__ __device__ constexpr int rp_mn_chunks(int R) { return (R + 63) / 64; }
__host__ __device__ constexpr int rp_n_mma(int R, int mn) { return mn ? 64 * rp_mn_chunks(R) : R; }
__host__ __device__ constexpr uint32_t rp_w_bytes(int R, int mn) {
  return mn ? 8192u * rp_mn_chunks(R) : static_cast<uint32_t>(R) * 128u;
}
__host__ __device__ constexpr uint32_t rp_stage_bytes(int R, int mn) {
  return kRpXBytes + ((rp_w_bytes(R, mn) + 1023u) & ~1023u);
}
__host__ __device__ constexpr uint32_t rp_smem_bytes(int R, int mn, int stages) {
  return 1024 + stages * rp_stage_bytes(R, mn) + kRpTail;
}

template <int RCOLS>
__global__ void __launch_bounds__(kRpThreads, 1)
    rowpass_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                   const RowpassParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int R = p.R;
  const int mn = p.w_mn_major;
  const int nmma = rp_n_mma(R, mn);
  const uint32_t w_bytes = rp_w_bytes(R, mn);
  const uint32_t stage_bytes = rp_stage_bytes(R, mn);
  const int NS = p.stages;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + NS * stage_bytes);
  uint64_t* empty = full + NS;
  uint64_t* acc_full = empty + NS;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
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
  const uint64_t lim = p.wait_ns ? p.wait_ns : kWaitLimitNs;
  // test hook: in CTA (0, 0) the producer leaves this stage out, so the waits
  // for it expire and the bounded-wait abort path runs (never set otherwise)
  const int skip = (blockIdx.x == 0 && blockIdx.y == 0) ? p.fault_skip_stage : -1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + kRpQuantWarps);  // MMA commit + one arrive per quantizer warp
    }
    mbar_init(acc_full, 1);
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
  pdl_launch_dependents();
  pdl_wait_prior();

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      int s = 0;                 // ring slot and its phase parity (no division by the runtime depth)
      uint32_t ph = 0;
      for (int i = 0; i < nt; ++i, s = (s + 1 == NS) ? 0 : s + 1, ph ^= (s == 0) ? 1u : 0u) {
        if (!mbar_wait(&empty[s], ph ^ 1, p.status, abortp, lim)) break;
        issued = i + 1;
        if (i == skip) continue;
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
      }
      if (*abortp) {  // let copies already in flight land before the CTA exits
        for (int i = max(0, issued - NS); i < issued; ++i)  // once, on the abort path only
          if (i != skip) mbar_wait_drain(&full[i % NS], (i / NS) & 1, 100000000ull);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, nmma, false, mn != 0);
      int s = 0;
      uint32_t ph = 0;
      for (int i = 0; i < nt; ++i, s = (s + 1 == NS) ? 0 : s + 1, ph ^= (s == 0) ? 1u : 0u) {
        if (!mbar_wait(&full[s], ph, p.status, abortp, lim)) break;
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
    const int w16 = warp - 4;
    const int blk = w16 >> 1;                 // 16-row block of the tile
    const int colw = (w16 & 1) * 32 + (lane & 1) * 16;   // this lane's 16 columns within the tile
    const int r = blk * 16 + (lane >> 1);     // this lane's row within the tile
    const long long half_k = p.K / 2;
    const int kblocks = p.K / 16;
    const bool block_row_ok = m0 + blk * 16 < p.M;
    // 1x16 groups: this lane's 16 values are one group; the tensor's 2^-e
    const bool g16 = p.group16 != 0;
    const float g16_inv = g16 ? pow2_f32(-group16_exponent(__uint_as_float(*p.amax))) : 1.0f;
    bool ok = true;
    int s = 0;
    uint32_t ph = 0;
    for (int i = 0; i < nt; ++i, s = (s + 1 == NS) ? 0 : s + 1, ph ^= (s == 0) ? 1u : 0u) {
      if (!mbar_wait(&full[s], ph, p.status, abortp, lim)) {
        ok = false;
        break;
      }
      uint8_t* tile = smem + s * stage_bytes;
      float v[16];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int phys = (colw / 8 + q) ^ (r & 7);
        const uint4 u = *reinterpret_cast<const uint4*>(tile + r * 128 + phys * 16);
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          v[q * 8 + 2 * e] = bf16_bits_to_f32(wd[e] & 0xFFFFu);
          v[q * 8 + 2 * e + 1] = bf16_bits_to_f32(wd[e] >> 16);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);  // the tile is in registers: release the stage early
      float m[8];                               // this lane's 16 magnitudes, tree-reduced
#pragma unroll
      for (int e = 0; e < 8; ++e) m[e] = fmaxf(fabsf(v[e]), fabsf(v[e + 8]));
#pragma unroll
      for (int w = 4; w >= 1; w >>= 1)
#pragma unroll
        for (int e = 0; e < w; ++e) m[e] = fmaxf(m[e], m[e + w]);
      float amax = max16_same_parity(m[0], lane);   // over the block's 16 rows
      if (g16) {                                    // the lane's own group, scaled (exact: 2^-e)
        amax = m[0] * g16_inv;
#pragma unroll
        for (int e = 0; e < 16; ++e) v[e] *= g16_inv;
      }
      const int cstart = (kt0 + i) * 64 + colw;
      const bool inside = block_row_ok && cstart < p.K;
      if (!p.no_quant && (inside || p.sf_mma)) {
        // rows past M and columns past K were zero-filled by the TMA: their scale is 0
        uint32_t packed[2], sc;
        quantize_1block(v, amax, packed, &sc);
        if (inside) {
          *reinterpret_cast<uint2*>(p.codes + static_cast<long long>(m0 + r) * half_k + cstart / 2) =
              make_uint2(packed[0], packed[1]);
          if (g16)
            p.scales[static_cast<long long>(m0 + r) * kblocks + cstart / 16] = static_cast<uint8_t>(sc);
          else if ((lane >> 1) == 0)
            p.scales[(m0 / 16 + blk) * static_cast<long long>(kblocks) + cstart / 16] = static_cast<uint8_t>(sc);
        }
        if (p.sf_mma) {
          // MMA-ready copy: group colw/16 of k-step kt0+i for row r of chunk blockIdx.x
          const size_t o = (static_cast<size_t>(blockIdx.x) * KT + (kt0 + i)) * 512 + (r & 31) * 16 + (r >> 5) * 4 +
                           colw / 16;
          p.sf_mma[o] = static_cast<uint8_t>(sc);
        }
      }
    }

    // ---- epilogue (all sixteen quantizer warps): accumulator -> L (bf16) or
    // fp32 partials.  All agree on whether to run it, so the named barriers
    // below are always reached by all of them.
    {
      const bool mine = ok && mbar_wait(acc_full, 0, p.status, abortp, lim);
      if (lane == 0) s_ok[w16] = mine ? 1 : 0;
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
        for (int c0 = 16 * (w16 >> 2); c0 < R; c0 += 64) {   // this warp's 16-column chunks
          uint32_t v[16];
          tmem_ld_32x32b_x16(taddr + c0, v);
          tmem_ld_wait();
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
        if (p.nsplit > 1) {
          // the last CTA of this row tile to finish sums every split's partial, in
          // split order.  One thread's acq_rel counter increment publishes the
          // CTA's partial writes (ordered before it by the barrier) and, in the
          // last CTA, orders the partial reads (after the next barrier) after
          // every other CTA's increment.
          named_bar_sync(1, 32 * kRpQuantWarps);
          if (threadIdx.x == 128) {
            const int prev = atomic_add_acq_rel_gpu(&p.counters[blockIdx.x], 1);
            *s_last = (prev == p.nsplit - 1);
          }
          named_bar_sync(1, 32 * kRpQuantWarps);
          if (*s_last) {
            // pieces of 4 columns; a thread takes kRpSumItems of them per pass, with
            // a batch of splits of all of them in flight before the in-order sums
            constexpr int kT = 32 * kRpQuantWarps;
            const int c4n = R / 4;
            const int npiece = 128 * c4n;
            const int tid = static_cast<int>(threadIdx.x) - 128;
            for (int base = tid; base < npiece; base += kRpSumItems * kT) {
              float4 acc[kRpSumItems];
              long long off[kRpSumItems];
              bool live[kRpSumItems];
#pragma unroll
              for (int j = 0; j < kRpSumItems; ++j) {
                const int idx = base + j * kT;
                const int grow = m0 + idx / c4n;
                live[j] = idx < npiece && grow < p.M;
                off[j] = static_cast<long long>(grow) * R + 4 * (idx % c4n);
                acc[j] = make_float4(0.0f, 0.0f, 0.0f, 0.0f);
              }
              for (int sp0 = 0; sp0 < p.nsplit; sp0 += kRpSumBatch) {
                float4 a[kRpSumBatch][kRpSumItems];
#pragma unroll
                for (int b = 0; b < kRpSumBatch; ++b)
#pragma unroll
                  for (int j = 0; j < kRpSumItems; ++j)
                    if (live[j] && sp0 + b < p.nsplit)
                      a[b][j] = __ldcg(reinterpret_cast<const float4*>(
                          p.part + static_cast<long long>(sp0 + b) * p.M * R + off[j]));
#pragma unroll
                for (int b = 0; b < kRpSumBatch; ++b)
#pragma unroll
                  for (int j = 0; j < kRpSumItems; ++j)
                    if (live[j] && sp0 + b < p.nsplit) {
                      acc[j].x += a[b][j].x;
                      acc[j].y += a[b][j].y;
                      acc[j].z += a[b][j].z;
                      acc[j].w += a[b][j].w;
                    }
              }
#pragma unroll
              for (int j = 0; j < kRpSumItems; ++j) {
                if (!live[j]) continue;
                const __nv_bfloat162 lo = __floats2bfloat162_rn(acc[j].x, acc[j].y);
                const __nv_bfloat162 hi = __floats2bfloat162_rn(acc[j].z, acc[j].w);
                *reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(p.L) + off[j]) =
                    make_uint2(*reinterpret_cast<const uint32_t*>(&lo), *reinterpret_cast<const uint32_t*>(&hi));
              }
            }
            if (threadIdx.x == 128) p.counters[blockIdx.x] = 0;
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
    tmem_dealloc(tmem, RCOLS);
  }
}

template <int RCOLS>
static cudaError_t launch_rowpass_t(const CUtensorMap& tmX, const CUtensorMap& tmW, const RowpassParams& p,
                                    cudaStream_t stream) {
  const uint32_t smem = rp_smem_bytes(p.R, p.w_mn_major, p.stages);
  cudaError_t e = cudaFuncSetAttribute(rowpass_kernel<RCOLS>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(rowpass_kernel<RCOLS>, dim3((p.M + 127) / 128, p.nsplit), dim3(kRpThreads), smem, stream, tmX,
                    tmW, p);
}

cudaError_t launch_rowpass(const CUtensorMap& tmX, const CUtensorMap& tmW, const RowpassParams& p,
                           cudaStream_t stream) {
  if (p.stages < 2 || p.stages > kRpStages || rp_smem_bytes(p.R, p.w_mn_major, p.stages) > 232448u)
    return cudaErrorInvalidValue;
  const int n = rp_n_mma(p.R, p.w_mn_major);
  if (n <= 32) return launch_rowpass_t<32>(tmX, tmW, p, stream);
  if (n <= 64) return launch_rowpass_t<64>(tmX, tmW, p, stream);
  return launch_rowpass_t<128>(tmX, tmW, p, stream);
}

int rowpass_stages(int R, int w_mn_major) {
  const int fit = (232448 - 1024 - static_cast<int>(kRpTail)) / static_cast<int>(rp_stage_bytes(R, w_mn_major));
  return fit < kRpStages ? fit : kRpStages;
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
