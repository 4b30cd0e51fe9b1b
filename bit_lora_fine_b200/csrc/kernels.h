// Internal host-side interface between the C-ABI layer (api.cu) and the kernel
// files.  Not installed; the public interface is include/fourtune/fourtune.h.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ft {

// Quantize the rows of a bf16 input and project it onto R low-rank directions:
// codes/scales = block16(X), L = bf16(X W) where W is either D [K, R] (R
// contiguous, read MN-major) or W^T [R, K] (K contiguous, read K-major).
struct RowpassParams {
  int M, K, R;
  int w_mn_major;                        // 1: D [K, R]; 0: W^T [R, K]
  int kt_per_split, nsplit;              // 64-column tiles per CTA along K, number of K splits
  int stages;                            // TMA ring depth, 2..rowpass_stages()
  int no_quant;                          // only L: no codes or scales (the 16-bit precision variants)
  // 1x16 groups (group16.cu): each row's 16 columns get their own scale, the
  // values scaled by 2^-e of the tensor maximum in *amax (float bits); scales
  // [M, K/16].  0: 16x16 blocks, scales [M/16, K/16].
  int group16;
  const uint32_t* amax;
  uint8_t* codes;                        // [M, K/2]
  uint8_t* scales;                       // [M/16, K/16]
  uint8_t* sf_mma;                       // the same scales in the MMA-ready layout (null = not written)
  void* L;                               // bf16 [M, R]
  float* part;                           // fp32 [nsplit, M, R] when nsplit > 1
  int* counters;                         // [ceil(M/128)], zero on entry, left zero (nsplit > 1)
  int* status;
  unsigned long long wait_ns;            // limit of every bounded wait (0: the default, 2 s)
  int fault_skip_stage;                  // test hook: CTA (0, 0) never loads this stage (-1: none)
};

// MMA-ready scale layout of a block16 operand with `rows` rows (along M or N)
// and `cols` columns along K: for each 128-row chunk c and each 64-column
// k-step t, one 512-byte block at byte ((c * KS) + t) * 512, KS = ceil(cols/64).
// Inside a block, the scale of row r (r % 128 = 32 q + l) and of the step's
// 16-column group j (0..3) sits at byte 16 l + 4 q + j -- the order in which
// tcgen05.cp 32x128b.warpx4 moves 512 bytes into the TMEM columns that the
// block-scaled MMA reads.  Rows past `rows` and groups past cols/16 hold 0.
__host__ __device__ constexpr size_t sf_mma_bytes(long long rows, long long cols) {
  return static_cast<size_t>((rows + 127) / 128) * static_cast<size_t>((cols + 63) / 64) * 512u;
}
__host__ __device__ constexpr long long sf_mma_offset(long long r, long long g, long long ks) {
  return ((r / 128) * ks + g / 4) * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (g % 4);
}

// out = deq(A) deq(B)^T (+ A2 * B2^T) (+ bias); A [M, K], B [N, K] packed E2M1,
// their scales in the MMA-ready layout (sfa: rows = M, sfb: rows = N, cols = K).
// A2 [M, R2] bf16; B2 is [N, R2] (K-major) or U [R2, N] (b2_mn_major).
struct GemmParams {
  int M, N, K, R2;
  int b2_mn_major;
  const uint8_t* sfa;
  const uint8_t* sfb;
  const void* bias;                      // bf16 [N] or null
  void* out;
  long long ldo;
  int out_bf16;
  int* status;
  // 16-bit main product (the precision variants): A [M, K] and B [N, K] are
  // bf16 (K contiguous) instead of block16 codes; sfa, sfb unused
  int main_bf16;
  // 1x16 groups: the accumulator is scaled by 2^(eA + eB), the per-tensor
  // exponents of the maxima in *amax_a, *amax_b (float bits), before the bias
  // (null: no scaling).  The low-rank factor B2 must come pre-scaled by the
  // inverse (launch_scale_pow2).
  const uint32_t* amax_a;
  const uint32_t* amax_b;
};

// The MLP's 4-bit GEMMs with their fused epilogues (FourTune §3.3 "MLP
// Fusion").  The main product is GemmParams' (A [M, K] and B [N, K] block16
// codes with MMA-ready scales, + A2 B2^T low-rank blocks); per output tile the
// epilogue forms a bf16 tensor T [M, N] and
//   epi == 1 (FC1 forward):  h = bf16(acc + bias) -> out_h;  a = GELU(h) fp32
//            (-> dbg if set);  Q(a) -> q_*;  T = bf16(a)
//   epi == 2 (FC2 dX):       d_h = bf16(acc * GELU'(h)) -> out_h;  Q(d_h) -> q_*;
//            T = d_h
// and projects it: part [nsplit, M, RP] = T Wp over each unit's N tiles (fp32,
// accumulated in TMEM), Wp [N, RP] read from D2 [N, RP] (wp_mn_major = 1) or
// from U1 [RP, N] (0); launch_proj_reduce then forms bf16(sum of the partials
// in split order).
struct MlpGemmParams {
  GemmParams g;                          // main product (M, N, K, R2, scales, bias, status)
  int epi;                               // 1 or 2 (above)
  const void* h;                         // epi 2: bf16 [M, N]
  void* out_h;                           // bf16 [M, N]: h (epi 1) or d_h (epi 2)
  float* dbg;                            // epi 1: fp32 a [M, N] or null
  uint8_t* q_codes;                      // [M, N/2]
  uint8_t* q_scales;                     // [M/16, N/16]
  uint8_t* q_sf;                         // MMA-ready scales of Q(T) (rows M, cols N)
  int RP;                                // projection rank (16..128, multiple of 16)
  int wp_mn_major;
  int nsplit, per;                       // units: N tiles [sp*per, +per) of one 128-row tile
  float* part;                           // fp32 [nsplit, M, RP]
};
cudaError_t launch_gemm_mlp(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmA2,
                            const CUtensorMap& tmB2, const CUtensorMap& tmW, const MlpGemmParams& p, int num_sms,
                            cudaStream_t stream);
// out [M, RP] bf16 = sum over s = 0 .. nsplit - 1 (in that order) of part [s, M, RP] (fp32)
cudaError_t launch_proj_reduce(const float* part, int nsplit, int M, int RP, void* out, int num_sms,
                               cudaStream_t stream);

// out[p, j] (+)= sum_m T[m, p] * V[m, v0 + j]   for p < P, j < r (r <= 64)
struct TgradParams {
  int M, P, r, v0;
  int t_gelu;                            // T is h: use bf16(GELU_tanh(T)) (the MLP's FC2 dA)
  int mt_per_split, nsplit;              // 128-row tiles per CTA along M, number of M splits
  float* out;
  long long out_sp, out_sj;
  int accumulate;
  float* part;                           // fp32 [nsplit, ceil(P/128)*128, 64] when nsplit > 1
  int* counters;                         // [ceil(P/128)], zero on entry, left zero
  int* status;
};

cudaError_t launch_quantize_block16(const void* x, int rows, int cols, long long ld, uint8_t* codes,
                                    uint8_t* scales, cudaStream_t stream);
cudaError_t launch_quantize_block16_f32(const float* x, int rows, int cols, long long ld, uint8_t* codes,
                                        uint8_t* scales, cudaStream_t stream);
// R = bf16(W - (S_dn S_up)^T) [N, K] (the stabilizer split's residual), see quant.cu
cudaError_t launch_stabilizer_residual(const void* W, int N, int K, const void* S_dn, const void* S_up, int r_s,
                                       void* R, cudaStream_t stream);
// bf16 values of a block16 matrix (or of its transpose), see quant.cu
cudaError_t launch_dequantize_block16(const uint8_t* codes, const uint8_t* scales, int rows, int cols,
                                      int transposed, void* out, cudaStream_t stream);
cudaError_t launch_transpose_codes(const uint8_t* codes, int rows, int cols, uint8_t* codes_t,
                                   cudaStream_t stream);
cudaError_t launch_rowpass(const CUtensorMap& tmX, const CUtensorMap& tmW, const RowpassParams& p,
                           cudaStream_t stream);
// Deepest TMA ring of the row pass that one CTA's shared memory holds (one CTA per SM).
int rowpass_stages(int R, int w_mn_major);
// persistent: min(tiles, num_sms) CTAs
cudaError_t launch_gemm_fp4(const CUtensorMap& tmA, const CUtensorMap& tmB, const CUtensorMap& tmA2,
                            const CUtensorMap& tmB2, const GemmParams& p, int num_sms, cudaStream_t stream);
// zero `bytes` (a multiple of 16, 16-aligned) at p after the previous kernel, in a
// dependent launch (see quant.cu)
cudaError_t launch_clear_words(void* p, size_t bytes, cudaStream_t stream);
// 1x16 groups (group16.cu): max|x| of a bf16 tensor (n a multiple of 8) into
// *word (atomicMax of float bits: the word must start at 0); the group
// quantizer of W [rows, cols] (transposed: of W^T) with codes [orows, ocols/2],
// scales [orows, ocols/16] and the MMA-ready copy (null: not written; rows and
// groups past the matrix are left as they are); dst = src * 2^-(eA + eB)
cudaError_t launch_tensor_amax(const void* x, long long n, uint32_t* word, int num_sms, cudaStream_t stream);
cudaError_t launch_quantize_group16(const void* w, int rows, int cols, int transposed, const uint32_t* amax_word,
                                    uint8_t* codes, uint8_t* scales, uint8_t* sf_mma, cudaStream_t stream);
cudaError_t launch_scale_pow2(const void* src, void* dst, long long n, const uint32_t* amax_a, const uint32_t* amax_b,
                              int num_sms, cudaStream_t stream);
// compact block16 scales -> MMA-ready layout of the operand [rows, cols]; with
// `transposed`, the operand is the transpose of the quantized matrix, whose
// compact scales are [cols/16, rows/16]
cudaError_t launch_sf_mma(const uint8_t* scales, int rows, int cols, int transposed, uint8_t* out,
                          cudaStream_t stream);
cudaError_t launch_tgrad2(const CUtensorMap& tmT0, const CUtensorMap& tmV0, const TgradParams& p0,
                          const CUtensorMap& tmT1, const CUtensorMap& tmV1, const TgradParams& p1,
                          cudaStream_t stream);

// Size of the row pass's file-scope scratch array (allocation-free entry point)
// and the lookup of its device address on the current device.
constexpr size_t kRowpassStaticScratchBytes = size_t(16) << 20;
cudaError_t rowpass_static_scratch(void** out);

// tile sizes the host needs for tensor-map boxes and workspace sizing
constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;

}  // namespace ft
