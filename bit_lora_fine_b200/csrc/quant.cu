// Standalone 16x16-block FP4 quantizer and the nibble transpose of its codes.
//
// FourTune §3.2 / §4.3: each 16x16 block carries one scale, so the transposed
// operand of the backward GEMM is the same codes re-packed along the other
// dimension with the same scale bytes (no requantization).
//
// Per block: a = max|t|; s = a / 6 (fp32 division, round to nearest);
// sc = E4M3(s) (round to nearest even, saturate at 448); if sc decodes to 0
// every code is +0, else code = E2M1(t / dec(sc)) (fp32 division, round to
// nearest even, saturate at +-6, sign kept).  Codes: even column in the low
// nibble of byte [row, col/2]; scales: one byte per block, [rows/16, cols/16].
// Also: the workspace-header clear that every API call launches first.
#include <algorithm>

#include "common.cuh"
#include "kernels.h"

namespace ft {

// One warp quantizes a 16-row x 64-column strip (up to four blocks).
// Lane l owns row (l >> 1) of the strip and the 32-column half (l & 1).
template <typename T>
__device__ __forceinline__ void load32(const T* src, float* v);

template <>
__device__ __forceinline__ void load32<__nv_bfloat16>(const __nv_bfloat16* src, float* v) {
  const uint4* p = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 u = p[q];
    uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      v[q * 8 + 2 * e] = bf16_bits_to_f32(w[e] & 0xFFFFu);
      v[q * 8 + 2 * e + 1] = bf16_bits_to_f32(w[e] >> 16);
    }
  }
}

__global__ void __launch_bounds__(256) quantize_block16_kernel(const __nv_bfloat16* __restrict__ x, int rows,
                                                               int cols, long long ld, uint8_t* __restrict__ codes,
                                                               uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int strips_per_row = (cols + 63) / 64;
  const long long nstrips = static_cast<long long>(rows / 16) * strips_per_row;
  if (warp >= nstrips) return;
  const int rb = static_cast<int>(warp / strips_per_row);
  const int c0 = static_cast<int>(warp % strips_per_row) * 64;
  const int r = rb * 16 + (lane >> 1);
  const int h = lane & 1;
  const int cstart = c0 + 32 * h;
  const bool live = cstart < cols;           // cols % 16 == 0: a half may hold one or two blocks
  const int nblk = live ? min(2, (cols - cstart) / 16) : 0;

  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = 0.0f;
  if (nblk == 2) {
    load32(x + static_cast<long long>(r) * ld + cstart, v);
  } else if (nblk == 1) {
    const uint4* p = reinterpret_cast<const uint4*>(x + static_cast<long long>(r) * ld + cstart);
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      uint4 u = p[q];
      uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[q * 8 + 2 * e] = bf16_bits_to_f32(w[e] & 0xFFFFu);
        v[q * 8 + 2 * e + 1] = bf16_bits_to_f32(w[e] >> 16);
      }
    }
  }

  float amax[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[16 * j + i]));
    // reduce over the 16 lanes that share this half (lane bit 0 fixed)
#pragma unroll
    for (int off = 2; off < 32; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
    amax[j] = a;
  }

  if (nblk == 0) return;
  uint32_t packed[4], sc[2];
  quantize_2blocks(v, amax, packed, sc);
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    if (j >= nblk) break;
    const int cb = cstart + 16 * j;
    *reinterpret_cast<uint2*>(codes + static_cast<long long>(r) * (cols / 2) + cb / 2) =
        make_uint2(packed[2 * j], packed[2 * j + 1]);
    if ((lane >> 1) == 0) scales[static_cast<long long>(rb) * (cols / 16) + cb / 16] = static_cast<uint8_t>(sc[j]);
  }
}

// The same strip decomposition for float32 input of any precision: two blocks per
// lane through quantize_1block_f32 (the IEEE-quotient semantics without a division
// per element).
__global__ void __launch_bounds__(256) quantize_block16_f32_kernel(const float* __restrict__ x, int rows, int cols,
                                                                   long long ld, uint8_t* __restrict__ codes,
                                                                   uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const long long warp = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int strips_per_row = (cols + 63) / 64;
  const long long nstrips = static_cast<long long>(rows / 16) * strips_per_row;
  if (warp >= nstrips) return;
  const int rb = static_cast<int>(warp / strips_per_row);
  const int c0 = static_cast<int>(warp % strips_per_row) * 64;
  const int r = rb * 16 + (lane >> 1);
  const int cstart = c0 + 32 * (lane & 1);
  const int nblk = cstart < cols ? min(2, (cols - cstart) / 16) : 0;
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = 0.0f;
  const float4* src = reinterpret_cast<const float4*>(x + static_cast<long long>(r) * ld + cstart);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    if (q < 4 * nblk) {
      const float4 f = src[q];
      v[4 * q] = f.x;
      v[4 * q + 1] = f.y;
      v[4 * q + 2] = f.z;
      v[4 * q + 3] = f.w;
    }
  }
  float amax[2];
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) a = fmaxf(a, fabsf(v[16 * j + i]));
#pragma unroll
    for (int off = 2; off < 32; off <<= 1) a = fmaxf(a, __shfl_xor_sync(0xFFFFFFFFu, a, off));
    amax[j] = a;
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) {
    if (j >= nblk) break;
    uint32_t packed[2], sc;
    quantize_1block_f32(v + 16 * j, amax[j], packed, &sc);
    const int cb = cstart + 16 * j;
    *reinterpret_cast<uint2*>(codes + static_cast<long long>(r) * (cols / 2) + cb / 2) = make_uint2(packed[0], packed[1]);
    if ((lane >> 1) == 0) scales[static_cast<long long>(rb) * (cols / 16) + cb / 16] = static_cast<uint8_t>(sc);
  }
}

cudaError_t launch_quantize_block16_f32(const float* x, int rows, int cols, long long ld, uint8_t* codes,
                                        uint8_t* scales, cudaStream_t stream) {
  const long long nstrips = static_cast<long long>(rows / 16) * ((cols + 63) / 64);
  if (nstrips == 0) return cudaSuccess;
  const int block = 256;
  const long long grid = (nstrips * 32 + block - 1) / block;
  quantize_block16_f32_kernel<<<static_cast<unsigned>(grid), block, 0, stream>>>(x, rows, cols, ld, codes, scales);
  return cudaGetLastError();
}

// codes_t[c, r/2] = nibble (r & 1) <- code of element (r, c)
__global__ void transpose_codes_kernel(const uint8_t* __restrict__ codes, int rows, int cols,
                                       uint8_t* __restrict__ codes_t) {
  const long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long total = static_cast<long long>(cols) * (rows / 2);
  if (i >= total) return;
  const int c = static_cast<int>(i / (rows / 2));
  const int rp = static_cast<int>(i % (rows / 2));
  const uint8_t b0 = codes[static_cast<long long>(2 * rp) * (cols / 2) + c / 2];
  const uint8_t b1 = codes[static_cast<long long>(2 * rp + 1) * (cols / 2) + c / 2];
  const uint32_t n0 = (c & 1) ? (b0 >> 4) : (b0 & 0xF);
  const uint32_t n1 = (c & 1) ? (b1 >> 4) : (b1 & 0xF);
  codes_t[i] = static_cast<uint8_t>(n0 | (n1 << 4));
}

cudaError_t launch_quantize_block16(const void* x, int rows, int cols, long long ld, uint8_t* codes,
                                    uint8_t* scales, cudaStream_t stream) {
  const long long nstrips = static_cast<long long>(rows / 16) * ((cols + 63) / 64);
  if (nstrips == 0) return cudaSuccess;
  const long long threads = nstrips * 32;
  const int block = 256;
  const long long grid = (threads + block - 1) / block;
  quantize_block16_kernel<<<static_cast<unsigned>(grid), block, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(x), rows, cols, ld, codes, scales);
  return cudaGetLastError();
}

cudaError_t launch_transpose_codes(const uint8_t* codes, int rows, int cols, uint8_t* codes_t,
                                   cudaStream_t stream) {
  const long long total = static_cast<long long>(cols) * (rows / 2);
  if (total == 0) return cudaSuccess;
  const int block = 256;
  transpose_codes_kernel<<<static_cast<unsigned>((total + block - 1) / block), block, 0, stream>>>(codes, rows,
                                                                                                  cols, codes_t);
  return cudaGetLastError();
}

// Compact block16 scales -> MMA-ready layout (kernels.h), one thread per byte.
// Non-transposed: operand [rows, cols] = the quantized matrix, scale(rb, g) =
// scales[rb * (cols/16) + g].  Transposed: operand = the quantized matrix's
// transpose (FourTune §3.2: same scale bytes), scale(rb, g) = scales[g * (rows/16) + rb].
__global__ void sf_mma_kernel(const uint8_t* __restrict__ scales, int rows, int cols, int transposed,
                              uint8_t* __restrict__ out, long long n) {
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= n) return;
  const int ks = (cols + 63) / 64;
  const long long blk = i / 512;
  const int b = static_cast<int>(i % 512);
  const long long chunk = blk / ks;
  const int t = static_cast<int>(blk % ks);
  const long long r = chunk * 128 + ((b % 16) / 4) * 32 + b / 16;
  const int g = 4 * t + (b % 4);
  uint8_t v = 0;
  if (r < rows && g < cols / 16) {
    const long long rb = r / 16;
    v = transposed ? scales[static_cast<long long>(g) * (rows / 16) + rb] : scales[rb * (cols / 16) + g];
  }
  out[i] = v;
}

// Zero n16 16-byte words at p (a workspace header: status word, split
// counters), in stream order: launched with programmatic dependent launch, it
// releases the next kernel at once (whose prologue then overlaps) and waits for
// the previous grid before it writes.  A memset in its place would end the
// chain of dependent launches between the previous kernel and the next.
__global__ void clear_words_kernel(uint4* __restrict__ p, int n16) {
  pdl_launch_dependents();
  pdl_wait_prior();
  for (int i = threadIdx.x + blockIdx.x * blockDim.x; i < n16; i += blockDim.x * gridDim.x)
    p[i] = make_uint4(0u, 0u, 0u, 0u);
}

cudaError_t launch_clear_words(void* p, size_t bytes, cudaStream_t stream) {
  if (bytes == 0) return cudaSuccess;
  if ((bytes % 16) || (reinterpret_cast<uintptr_t>(p) % 16)) return cudaErrorInvalidValue;
  const long long n16 = static_cast<long long>(bytes / 16);
  const int blocks = static_cast<int>(std::min<long long>((n16 + 255) / 256, 64));
  return launch_pdl(clear_words_kernel, dim3(blocks), dim3(256), 0, stream, static_cast<uint4*>(p),
                    static_cast<int>(n16));
}

cudaError_t launch_sf_mma(const uint8_t* scales, int rows, int cols, int transposed, uint8_t* out,
                          cudaStream_t stream) {
  const long long n = static_cast<long long>(sf_mma_bytes(rows, cols));
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  sf_mma_kernel<<<static_cast<unsigned>((n + threads - 1) / threads), threads, 0, stream>>>(scales, rows, cols,
                                                                                          transposed, out, n);
  return cudaGetLastError();
}

// Dequantized values of a block16 matrix [rows, cols] as bf16: value =
// E2M1(code) * E4M3(scale of its 16x16 block), exact in bf16 (at most 2 + 4
// significant bits, magnitudes 2^-10 .. 2688).  transposed = 0 writes
// out[r, c] [rows, cols]; transposed = 1 writes the transpose out[c, r]
// [cols, rows] (FourTune §3.2: the transposed operand keeps its codes and
// scales).  One thread per pair of output elements (a byte of codes when not
// transposed).  The 16-bit precision variants (§4.3) use it to give their GEMMs
// the 4-bit weight as the tensor cores would see it.
__global__ void dequantize_block16_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                          int rows, int cols, int transposed, uint32_t* __restrict__ out,
                                          long long npairs) {
  const long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x;
  if (i >= npairs) return;
  float v[2];
  if (!transposed) {
    // output pair i = row r, columns 2j, 2j+1 = one code byte
    const long long r = i / (cols / 2);
    const int j = static_cast<int>(i % (cols / 2));
    const float d = e4m3_to_f32(scales[(r / 16) * (cols / 16) + (2 * j) / 16]);
    const uint32_t byte = codes[i];
#pragma unroll
    for (int e = 0; e < 2; ++e) v[e] = e2m1_to_f32((byte >> (4 * e)) & 0xFu) * d;
  } else {
    // output pair i = output row c (an input column), output columns 2j, 2j+1
    // (input rows 2j, 2j+1, one 16-row block)
    const long long c = i / (rows / 2);
    const int j = static_cast<int>(i % (rows / 2));
    const float d = e4m3_to_f32(scales[((2 * j) / 16) * (cols / 16) + c / 16]);
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const uint32_t byte = codes[static_cast<long long>(2 * j + e) * (cols / 2) + c / 2];
      v[e] = e2m1_to_f32((byte >> (4 * (c & 1))) & 0xFu) * d;
    }
  }
  const __nv_bfloat162 b = __floats2bfloat162_rn(v[0], v[1]);
  out[i] = *reinterpret_cast<const uint32_t*>(&b);
}

// Residual weight of the stabilizer split (FourTune §3.1): R[n, k] =
// bf16(W[n, k] - sum_j S_dn[k, j] S_up[j, n]), the rank-r_s product summed in
// fp32 and the difference rounded once.  A block of 256 threads covers 16 rows
// n x 64 columns k; it stages S_up[:, n0:n0+16] and S_dn[k0:k0+64, :] in shared
// memory (fp32) and each thread computes four outputs of one row.
constexpr int kResRows = 16, kResCols = 64, kResMaxRank = 128;
__global__ void __launch_bounds__(256) stabilizer_residual_kernel(const __nv_bfloat16* __restrict__ W, int N, int K,
                                                                  const __nv_bfloat16* __restrict__ S_dn,
                                                                  const __nv_bfloat16* __restrict__ S_up, int r_s,
                                                                  __nv_bfloat16* __restrict__ R) {
  __shared__ float sup[kResMaxRank][kResRows];
  __shared__ float sdn[kResCols][kResMaxRank + 1];
  const int n0 = blockIdx.y * kResRows, k0 = blockIdx.x * kResCols;
  for (int i = threadIdx.x; i < r_s * kResRows; i += blockDim.x) {
    const int j = i / kResRows, nn = i % kResRows;
    sup[j][nn] = n0 + nn < N ? __bfloat162float(S_up[static_cast<long long>(j) * N + n0 + nn]) : 0.0f;
  }
  for (int i = threadIdx.x; i < r_s * kResCols; i += blockDim.x) {
    const int kk = i / r_s, j = i % r_s;
    sdn[kk][j] = k0 + kk < K ? __bfloat162float(S_dn[static_cast<long long>(k0 + kk) * r_s + j]) : 0.0f;
  }
  __syncthreads();
  const int nn = threadIdx.x / 16, kq = (threadIdx.x % 16) * 4;
  const int n = n0 + nn;
  if (n >= N) return;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int k = k0 + kq + e;
    if (k >= K) break;
    float acc = 0.0f;
    for (int j = 0; j < r_s; ++j) acc = fmaf(sdn[kq + e][j], sup[j][nn], acc);
    const long long o = static_cast<long long>(n) * K + k;
    R[o] = __float2bfloat16_rn(__bfloat162float(W[o]) - acc);
  }
}

cudaError_t launch_stabilizer_residual(const void* W, int N, int K, const void* S_dn, const void* S_up, int r_s,
                                       void* R, cudaStream_t stream) {
  if (r_s < 1 || r_s > kResMaxRank) return cudaErrorInvalidValue;
  const dim3 grid((K + kResCols - 1) / kResCols, (N + kResRows - 1) / kResRows);
  stabilizer_residual_kernel<<<grid, 256, 0, stream>>>(
      static_cast<const __nv_bfloat16*>(W), N, K, static_cast<const __nv_bfloat16*>(S_dn),
      static_cast<const __nv_bfloat16*>(S_up), r_s, static_cast<__nv_bfloat16*>(R));
  return cudaGetLastError();
}

cudaError_t launch_dequantize_block16(const uint8_t* codes, const uint8_t* scales, int rows, int cols,
                                      int transposed, void* out, cudaStream_t stream) {
  const long long npairs = static_cast<long long>(rows) * cols / 2;
  if (npairs == 0) return cudaSuccess;
  const int threads = 256;
  dequantize_block16_kernel<<<static_cast<unsigned>((npairs + threads - 1) / threads), threads, 0, stream>>>(
      codes, scales, rows, cols, transposed, static_cast<uint32_t*>(out), npairs);
  return cudaGetLastError();
}

}  // namespace ft
