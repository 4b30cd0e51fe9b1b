// The 1x16 group-wise NVFP4 layout: the granularity comparator of FourTune §4.3
// ("Impact of Quantization Granularity", Table 5), in NVFP4's full form of §2.3
// (a per-tensor scale above the per-group E4M3 scales).
//
//   per tensor: e = group16_exponent(max|T|) (2^e: the least power of two with
//               max|T| / (6 * 2^e) <= 448), T' = T * 2^-e (exact: a power of two)
//   per 1x16 group of T' (16 consecutive elements of a row): the block rules of
//               the 16x16 layout on one row -- a = max|t'|, sc = E4M3(fp32(a)/6),
//               code = E2M1(fp32(t') / dec(sc))
// The GEMM's product then carries 2^(eA + eB), applied in its epilogue; the
// low-rank factor that shares its accumulator is pre-scaled by 2^-(eA + eB).
// Unlike the 16x16 blocks, a transposed operand cannot reuse these groups: the
// backward's R^T is quantized on its own (groups along N).
//
// Kernels: the per-tensor maximum (one atomicMax of float bits per warp: the
// maximum does not depend on the order), the standalone group quantizer (the
// frozen weight in both orientations), and the power-of-two rescale of a bf16
// factor.  The activations' and gradients' groups are quantized by the row
// pass (rowpass.cu) in its group16 mode.
#include "common.cuh"
#include "kernels.h"

namespace ft {

namespace {

// max |x| over a bf16 tensor of n8 * 8 elements -> atomicMax into *word (the
// float bits of the maximum; non-negative floats order like their bits)
__global__ void __launch_bounds__(256) tensor_amax_kernel(const uint4* __restrict__ x, long long n8,
                                                          uint32_t* __restrict__ word) {
  pdl_launch_dependents();
  pdl_wait_prior();   // the word was cleared by the previous launch
  uint32_t m = 0u;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n8;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const uint4 u = __ldg(x + i);
    const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      m = max(m, w[k] & 0x7FFFu);
      m = max(m, (w[k] >> 16) & 0x7FFFu);
    }
  }
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  if ((threadIdx.x & 31) == 0 && m) atomicMax(word, m << 16);
}

// One thread per output group: Q [orows, ocols] is W [rows, cols]
// (transposed = 0) or W^T (transposed = 1); a group is 16 consecutive columns
// of Q.  Adjacent threads take adjacent groups of a row (transposed = 0: each
// reads 32 contiguous bytes) or adjacent rows of Q (transposed = 1: the 16
// loads of a group are 16 rows of W, each coalesced across the warp).
__global__ void __launch_bounds__(256) quantize_group16_kernel(const __nv_bfloat16* __restrict__ w, int rows,
                                                               int cols, int transposed,
                                                               const uint32_t* __restrict__ amax_word,
                                                               uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                               uint8_t* __restrict__ sf_mma) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const int orows = transposed ? cols : rows, ocols = transposed ? rows : cols;
  const int ngroups = ocols / 16;
  const long long idx = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<long long>(orows) * ngroups) return;
  int orow, g;
  if (transposed) {
    orow = static_cast<int>(idx % orows);
    g = static_cast<int>(idx / orows);
  } else {
    orow = static_cast<int>(idx / ngroups);
    g = static_cast<int>(idx % ngroups);
  }
  const float inv = pow2_f32(-group16_exponent(__uint_as_float(*amax_word)));
  float v[16];
  if (transposed) {
    const unsigned short* src = reinterpret_cast<const unsigned short*>(w) + static_cast<long long>(16 * g) * cols + orow;
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = bf16_bits_to_f32(src[static_cast<long long>(j) * cols]) * inv;
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(w + static_cast<long long>(orow) * cols + 16 * g);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const uint4 u = src[q];
      const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[8 * q + 2 * e] = bf16_bits_to_f32(wd[e] & 0xFFFFu) * inv;
        v[8 * q + 2 * e + 1] = bf16_bits_to_f32(wd[e] >> 16) * inv;
      }
    }
  }
  float a = 0.0f;
#pragma unroll
  for (int j = 0; j < 16; ++j) a = fmaxf(a, fabsf(v[j]));
  uint32_t packed[2], sc;
  quantize_block_row<16>(v, a, packed, &sc);   // bf16 values times 2^-e: the exact division-free path
  *reinterpret_cast<uint2*>(codes + static_cast<long long>(orow) * (ocols / 2) + 8 * g) = make_uint2(packed[0], packed[1]);
  scales[static_cast<long long>(orow) * ngroups + g] = static_cast<uint8_t>(sc);
  if (sf_mma) sf_mma[sf_mma_offset(orow, g, (ocols + 63) / 64)] = static_cast<uint8_t>(sc);
}

// dst = src * 2^-(eA + eB), eA and eB the per-tensor exponents of the two
// maxima (exact: a power-of-two scaling of a bf16 value)
__global__ void __launch_bounds__(256) scale_pow2_kernel(const __nv_bfloat16* __restrict__ src,
                                                         __nv_bfloat16* __restrict__ dst, long long n,
                                                         const uint32_t* __restrict__ amax_a,
                                                         const uint32_t* __restrict__ amax_b) {
  pdl_launch_dependents();
  pdl_wait_prior();
  const int k = -(group16_exponent(__uint_as_float(*amax_a)) + group16_exponent(__uint_as_float(*amax_b)));
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    dst[i] = __float2bfloat16_rn(ldexpf(__bfloat162float(src[i]), k));
}

}  // namespace

cudaError_t launch_tensor_amax(const void* x, long long n, uint32_t* word, int num_sms, cudaStream_t stream) {
  if (n % 8) return cudaErrorInvalidValue;
  const long long n8 = n / 8;
  const long long want = (n8 + 255) / 256;
  const int grid = static_cast<int>(want < 4LL * num_sms ? (want > 0 ? want : 1) : 4LL * num_sms);
  return launch_pdl(tensor_amax_kernel, dim3(grid), dim3(256), 0, stream, static_cast<const uint4*>(x), n8, word);
}

cudaError_t launch_quantize_group16(const void* w, int rows, int cols, int transposed, const uint32_t* amax_word,
                                    uint8_t* codes, uint8_t* scales, uint8_t* sf_mma, cudaStream_t stream) {
  const int ocols = transposed ? rows : cols;
  if (rows <= 0 || cols <= 0 || ocols % 16 || (!transposed && cols % 8)) return cudaErrorInvalidValue;
  const long long groups = static_cast<long long>(transposed ? cols : rows) * (ocols / 16);
  const long long blocks = (groups + 255) / 256;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  return launch_pdl(quantize_group16_kernel, dim3(static_cast<unsigned>(blocks)), dim3(256), 0, stream,
                    static_cast<const __nv_bfloat16*>(w), rows, cols, transposed, amax_word, codes, scales, sf_mma);
}

cudaError_t launch_scale_pow2(const void* src, void* dst, long long n, const uint32_t* amax_a, const uint32_t* amax_b,
                              int num_sms, cudaStream_t stream) {
  const long long want = (n + 255) / 256;
  const int grid = static_cast<int>(want < 2LL * num_sms ? (want > 0 ? want : 1) : 2LL * num_sms);
  return launch_pdl(scale_pow2_kernel, dim3(grid), dim3(256), 0, stream, static_cast<const __nv_bfloat16*>(src),
                    static_cast<__nv_bfloat16*>(dst), n, amax_a, amax_b);
}

}  // namespace ft
