/*
 * fourtune.h -- C ABI of the B200 (sm_100a) FourTune layer library.
 *
 * The layer is the triple-branch hybrid-precision linear of "FourTune: Towards
 * Fully 4-Bit Efficient Post-Training for Diffusion Models" (§3.1): a frozen
 * 4-bit residual weight R, a frozen bf16 low-rank stabilizer (S_dn, S_up) and a
 * trainable bf16 LoRA adapter (A, B), all fed the same input:
 *
 *     y = deq(Q(X) Q(R)^T) + (X S_dn) S_up + (X A) B  (+ bias)
 *
 * with weights, activations and gradients quantized to 4 bits (W4A4G4, §3).
 * Q is 16x16-block quantization (§3.2, §4.3 "Impact of Quantization
 * Granularity"): FP4 E2M1 codes, one FP8 E4M3 scale per 16x16 block,
 * round-to-nearest-even.  Because a block's scale belongs to the block, the
 * backward product Q(G) Q(R) reads R's blocks transposed with the same codes and
 * scales, no requantization (§3.2).
 *
 * Conventions (every entry point):
 *   - Return value: FT_OK (0) or a negative FT_ERR_* code; nothing is launched
 *     when an argument check fails.
 *   - All tensor pointers are DEVICE pointers owned by the caller; the library
 *     never allocates device memory.  Scratch space is the caller's `ws` buffer
 *     of at least *_workspace_size(...) bytes, 256-byte aligned; it must not be
 *     shared by calls that may run concurrently.
 *   - Calls are asynchronous on `stream` (a cudaStream_t passed as void*; NULL is
 *     the legacy default stream).  A kernel whose internal wait times out
 *     records it in the workspace; fourtune_device_status() reports it
 *     (FT_ERR_TIMEOUT; FT_ERR_UNSUPPORTED if the MLP's fused GEMM found its
 *     dynamic shared memory not 1024-byte aligned and did nothing).
 *   - bf16 tensors are arrays of IEEE bfloat16 bit patterns (ft_bf16), row-major,
 *     16-byte aligned.  Dimensions must be multiples of 16; K and N must also be
 *     multiples of 32 (4-bit rows are copied in 16-byte units).
 *   - Block16 tensor of a [rows, cols] matrix: codes uint8 [rows, cols/2]
 *     (column 2i in the low nibble of byte i, 2i+1 in the high nibble) and
 *     scales uint8 [rows/16, cols/16] (E4M3 bit patterns).
 *   - Requires an sm_100 device (B200); FT_ERR_UNSUPPORTED otherwise.
 */
#ifndef FOURTUNE_FOURTUNE_H_
#define FOURTUNE_FOURTUNE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FT_API __attribute__((visibility("default")))
#else
#define FT_API
#endif

typedef uint16_t ft_bf16;

enum {
  FT_OK = 0,
  FT_ERR_INVALID_ARG = -1, /* null pointer, bad enum, rank out of range */
  FT_ERR_SHAPE = -2,       /* a dimension is not a multiple of 16 (or 32 where stated) */
  FT_ERR_ALIGN = -3,       /* a pointer is not 16-byte aligned (256 for the workspace) */
  FT_ERR_WORKSPACE = -4,   /* ws_bytes smaller than the *_workspace_size() value */
  FT_ERR_CUDA = -5,        /* a CUDA runtime call or kernel launch failed */
  FT_ERR_TIMEOUT = -6,     /* a kernel's bounded wait expired (device status) */
  FT_ERR_UNSUPPORTED = -7  /* not an sm_100 device, or a size the library does not handle */
};

enum { FT_DTYPE_F32 = 0, FT_DTYPE_BF16 = 1 };

/* One triple-branch linear layer, y[M, N] from x[M, K]  (§3.1, §3.2).
 *   R_codes   [N, K/2]  block16 codes of the frozen residual weight R [N, K]
 *   R_scales  [N/16, K/16]
 *   R_codes_t [K, N/2]  the same codes nibble-transposed (codes of R^T); the
 *                       scales of R^T are R_scales read transposed.  Required by
 *                       the backward (fourtune_quantize_block16 writes it).
 *   R_sf      R_scales rearranged for the tensor cores: fourtune_mma_scales of
 *             R_scales with rows = N, cols = K, transposed = 0
 *   R_sf_t    the same for R^T: rows = K, cols = N, transposed = 1.  Required
 *             by the backward.  Both are frozen like R and prepared once.
 *   D [K, r_s + r] = [S_dn | A]   down-projections, bf16 row-major: the frozen
 *                       stabilizer's S_dn in columns 0..r_s-1, the LoRA A after it
 *   U [r_s + r, N] = [S_up ; B]   up-projections, bf16 row-major: S_up rows first,
 *                       then the LoRA B
 *   bias [N] frozen bf16 or NULL
 * The stabilizer and the adapter share the input (§3.3), so their factors are
 * stored concatenated along the rank and applied as one product each way; A
 * and B are views into D and U (A has row stride r_s + r).
 * Ranks: r_s >= 0, 16 <= r <= 64, r_s + r <= 128, each a multiple of 16. */
typedef struct {
  int64_t K, N, r_s, r;
  const uint8_t* R_codes;
  const uint8_t* R_scales;
  const uint8_t* R_codes_t;
  const ft_bf16* D;
  const ft_bf16* U;
  const ft_bf16* bias;
  const uint8_t* R_sf;
  const uint8_t* R_sf_t;
} ft_linear_t;

/* Block16 quantization of a bf16 matrix x [rows, cols] with row stride `ld`
 * elements (§2.3 Round(W/s), §3.2, §4.3): per 16x16 block, s = amax/6 in fp32,
 * scale = E4M3(s) (nearest-even, saturating at 448, subnormals kept), codes =
 * E2M1(x / scale) (nearest-even, saturating at +-6, sign kept; all +0 when the
 * scale is 0).  Writes codes [rows, cols/2], scales [rows/16, cols/16] and, if
 * codes_t is not NULL, the transposed codes [cols, rows/2].  Used offline for
 * the frozen residual weight.  rows, cols multiples of 16; ld multiple of 8. */
FT_API int fourtune_quantize_block16(const ft_bf16* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes,
                              uint8_t* scales, uint8_t* codes_t, void* stream);

/* The same block16 quantization of a float32 matrix x [rows, cols] (row stride
 * `ld` elements, a multiple of 4): element codes follow the IEEE float32 quotient
 * x / dec(scale), exactly as for bf16 input, for inputs of any precision (the
 * MLP's fp32 GELU output is quantized this way, §3.3).  x 16-byte aligned,
 * codes 8-byte aligned. */
FT_API int fourtune_quantize_block16_f32(const float* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes,
                                         uint8_t* scales, void* stream);

/* Nibble transpose of block16 codes: codes [rows, cols/2] -> codes_t [cols, rows/2]
 * (§3.2: the transposed operand keeps its codes and scales). */
FT_API int fourtune_transpose_codes(const uint8_t* codes, int64_t rows, int64_t cols, uint8_t* codes_t, void* stream);

/* The block16 scales of an operand rearranged in the order the block-scaled
 * tensor-core MMA consumes them (§3.1: the 4-bit products run on 4-bit tensor
 * cores).  The operand is a [rows, cols] matrix with cols along the reduction
 * dimension; its scales are `scales` [rows/16, cols/16], or, with transposed =
 * 1, the operand is the transpose of the quantized matrix and `scales` is that
 * matrix's [cols/16, rows/16] array (§3.2: the transposed operand keeps its
 * scales).  Output: fourtune_mma_scales_size(rows, cols) bytes, 16-byte
 * aligned: for each 128-row chunk c and 64-column step t a 512-byte block at
 * ((c * ceil(cols/64)) + t) * 512 holding the scale of row r = 128 c + 32 q + l
 * and column group 4 t + j at byte 16 l + 4 q + j (0 past the matrix).
 * rows, cols multiples of 16. */
FT_API size_t fourtune_mma_scales_size(int64_t rows, int64_t cols);
FT_API int fourtune_mma_scales(const uint8_t* scales, int64_t rows, int64_t cols, int transposed, uint8_t* out,
                               void* stream);

/* Stabilizer split (§3.1: a frozen full-precision low-rank component is
 * isolated from the backbone weight and only the rest is quantized).  Given the
 * weight W [N, K] (y = X W^T) and rank-r_s factors S_dn [K, r_s], S_up [r_s, N]
 * of W^T (bf16; the paper cites SVDQuant, read as the truncated SVD of W^T
 * with the singular values split evenly between the factors -- a
 * factorization the caller computes), writes the residual
 *   R [N, K] = bf16(W - (S_dn S_up)^T)
 * (the rank-r_s product summed in fp32, the difference rounded once), which
 * fourtune_quantize_block16 then quantizes.  1 <= r_s <= 128; bf16 arrays
 * row-major and contiguous.  Run once per frozen weight. */
FT_API int fourtune_stabilizer_residual(const ft_bf16* W, int64_t N, int64_t K, const ft_bf16* S_dn,
                                        const ft_bf16* S_up, int64_t r_s, ft_bf16* R, void* stream);

/* The 4-bit product alone, a building block (the unfused form of the layer is
 * the paper's fusion ablation, §4.3 Fig. 9):
 *   out [M, N] = deq(A) deq(B)^T (+ bias)
 * A [M, K] and B [N, K] block16 codes ([rows, K/2] bytes), their scales in the
 * MMA-ready layout (A_sf = fourtune_mma_scales(A's scales, M, K, 0), B_sf the
 * same for B; for R^T, R_sf_t).  out fp32 or bf16 row-major (stride N).  ws:
 * at least 256 bytes, 256-byte aligned (its status word; fourtune_device_status
 * reads it).  M multiple of 16, N and K of 32. */
FT_API int fourtune_gemm_block16(const uint8_t* A_codes, const uint8_t* A_sf, const uint8_t* B_codes,
                                 const uint8_t* B_sf, int64_t M, int64_t N, int64_t K, const ft_bf16* bias, void* out,
                                 int out_dtype, void* ws, size_t ws_bytes, void* stream);

/* Workspace bytes for fourtune_linear_fwd / fourtune_linear_bwd with M tokens. */
FT_API size_t fourtune_linear_fwd_workspace_size(const ft_linear_t* layer, int64_t M);
FT_API size_t fourtune_linear_bwd_workspace_size(const ft_linear_t* layer, int64_t M);

/* Forward (§3.1, §3.3 LoRA fusion).  X [M, K] bf16.  Writes
 *   Y [M, N] (y_dtype FT_DTYPE_F32 or FT_DTYPE_BF16, row stride N)
 *   L_saved [M, r_s + r] bf16 = bf16(X D), kept for the backward.
 * One pass reads X once, quantizes it and computes L; the 4-bit GEMM then adds
 * L [S_up ; B] and the bias in its accumulator. */
FT_API int fourtune_linear_fwd(const ft_linear_t* layer, const ft_bf16* X, int64_t M, void* Y, int y_dtype,
                        ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream);

/* Backward (§3.2).  dY [M, N] bf16 (the incoming gradient G), X and L_saved from
 * the forward.  Writes
 *   dX [M, K] = deq(Q(G)) deq(Q(R)) + P D^T   (dx_dtype F32 or BF16)
 *   dA [K, r] fp32 = X^T P[:, r_s:]     dB [r, N] fp32 = L[:, r_s:]^T G
 * with P = bf16(G U^T).  accumulate = 1 adds into dA and dB, 0
 * overwrites.  R, S and bias receive no gradient.
 * Streams: after the G pass, dA and dB run on a library-owned stream (one per
 * device, created on first use) beside the dX GEMM, which gets the other SMs;
 * that stream waits for `stream` first and `stream` waits for it before the
 * call returns, so all work of the call is ordered on `stream` as seen by the
 * caller.  Calls from several host threads are safe; their dA/dB share the
 * library stream (so they run one after another there). */
FT_API int fourtune_linear_bwd(const ft_linear_t* layer, const ft_bf16* dY, const ft_bf16* X, const ft_bf16* L_saved,
                        int64_t M, void* dX, int dx_dtype, float* dA, float* dB, int accumulate, void* ws,
                        size_t ws_bytes, void* stream);

/* The same calls, recording caller-created CUDA events (cudaEvent_t as void*) on
 * `stream` around each kernel they launch: events[2k] before and events[2k+1]
 * after kernel k (NULL entries and k >= n_events/2 are skipped).  Kernels, in
 * order -- forward: 0 fused X pass (quantize + X D), 1 FP4 GEMM with
 * up-projection; backward: 0 fused G pass (quantize + G U^T), 1 dA and dB (run
 * while G is still in L2), 2 FP4 dX GEMM.  With events every kernel runs on
 * `stream` on all SMs, one after another (no library stream).  Used for live
 * per-kernel timing. */
FT_API int fourtune_linear_fwd_timed(const ft_linear_t* layer, const ft_bf16* X, int64_t M, void* Y, int y_dtype,
                                     ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream,
                                     void* const* events, int n_events);
FT_API int fourtune_linear_bwd_timed(const ft_linear_t* layer, const ft_bf16* dY, const ft_bf16* X,
                                     const ft_bf16* L_saved, int64_t M, void* dX, int dx_dtype, float* dA,
                                     float* dB, int accumulate, void* ws, size_t ws_bytes, void* stream,
                                     void* const* events, int n_events);

/* Precision variants (§4.3, Table 4: W4A16G4, W4A4G16, W4A16G16 beside the
 * paper's W4A4G4).  The weight stays the 4-bit R; a 16-bit activation or
 * gradient enters its product unquantized, so that product runs on the bf16
 * tensor cores against R's dequantized values:
 *   fourtune_dequantize_block16: out = deq(codes, scales) as bf16, exact (an
 *     E2M1 value times an E4M3 scale has at most 6 significant bits):
 *     [rows, cols], or with transposed = 1 its transpose [cols, rows].  For the
 *     layer: W16 = deq(Q(R)) [N, K] (transposed = 0 of R_codes/R_scales),
 *     W16_t = deq(Q(R))^T [K, N] (transposed = 1).  Frozen: prepared once.
 *     out 4-byte aligned.
 *   fourtune_linear_fwd_a16: y = X W16^T + L [S_up ; B] (+ bias),
 *     L = bf16(X [S_dn | A]) -- fourtune_linear_fwd with a 16-bit activation.
 *   fourtune_linear_bwd_g16: dX = G W16_t^T + P [S_dn | A]^T (G = dY in bf16),
 *     dA, dB as in fourtune_linear_bwd -- the backward with a 16-bit gradient.
 * W4A16G4 = _fwd_a16 + fourtune_linear_bwd; W4A4G16 = fourtune_linear_fwd +
 * _bwd_g16; W4A16G16 = _fwd_a16 + _bwd_g16.  Given a bf16 weight in place of
 * W16 (and W16_t = its transpose) and r_s = 0, the same two calls are the
 * standard bf16 LoRA layer the paper compares against (§4.2).  These calls read
 * only K, N, r_s, r, D, U and bias of the layer (the codes fields may be NULL);
 * their workspaces are sized by the two *_workspace_size calls below. */
FT_API size_t fourtune_linear_fwd_a16_workspace_size(const ft_linear_t* layer, int64_t M);
FT_API size_t fourtune_linear_bwd_g16_workspace_size(const ft_linear_t* layer, int64_t M);
FT_API int fourtune_dequantize_block16(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                       int transposed, ft_bf16* out, void* stream);
FT_API int fourtune_linear_fwd_a16(const ft_linear_t* layer, const ft_bf16* W16, const ft_bf16* X, int64_t M,
                                   void* Y, int y_dtype, ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream);
FT_API int fourtune_linear_bwd_g16(const ft_linear_t* layer, const ft_bf16* W16_t, const ft_bf16* dY,
                                   const ft_bf16* X, const ft_bf16* L_saved, int64_t M, void* dX, int dx_dtype,
                                   float* dA, float* dB, int accumulate, void* ws, size_t ws_bytes, void* stream);

/* The 1x16 group-wise layer (the quantization-granularity comparator of §4.3,
 * Table 5, in NVFP4's full form of §2.3): the same triple-branch layer with
 * X, G and the frozen weight quantized in 1x16 groups -- 16 consecutive
 * elements of a row along each GEMM's reduction dimension share one E4M3
 * scale -- below a per-tensor scale 2^e, e the least integer with
 * max|T| <= 6 * 448 * 2^e (at least -126; 0 for an all-zero tensor).  A group
 * of T' = T * 2^-e follows the block rules on one row: s = max|t'| / 6 in
 * fp32, scale = E4M3(s), codes = E2M1(t' / scale).  The forward GEMM reads
 * Q16(R) [N, K] (groups along K); the backward's dX reads Q16(R^T) [K, N]
 * (groups along N) -- a transposed operand cannot reuse 1x16 groups, which is
 * the cost the 16x16 blocks avoid (§3.2).  The product of two tensors carries
 * 2^(eA + eB), applied to the accumulator before the bias; the low-rank factor
 * sharing that accumulator (U forward, D for dX) is pre-scaled by the inverse
 * into the workspace, an exact power-of-two step.
 *
 * fourtune_quantize_1x16: W [rows, cols] bf16 -> Q16(W) (transposed = 0,
 *   output [rows, cols]) or Q16(W^T) (transposed = 1, output [cols, rows]):
 *   codes [orows, ocols/2], scales [orows, ocols/16] and, when sf_mma is not
 *   NULL, the MMA-ready copy (fourtune_mma_scales_size(orows, ocols) bytes,
 *   fully written).  amax_word: 16 bytes of device memory, 16-byte aligned,
 *   cleared by the call; its first word receives the float32 bits of max|W|,
 *   the per-tensor scale's source, which the layer reads.  rows % 32 == 0 and
 *   cols % 32 == 0; W, codes 16-byte aligned.  Offline for the frozen weight;
 *   also the standalone parity probe of the group quantizer.
 * ft_linear_1x16_t: Q16(R) and Q16(R^T) (codes and MMA-ready scales, both
 *   from one fourtune_quantize_1x16 call each on the bf16 R), R_amax the word
 *   those calls wrote, and the low-rank factors and bias as in ft_linear_t.
 * fourtune_linear_fwd_1x16 / _bwd_1x16: fourtune_linear_fwd / _bwd with the
 *   1x16 layout (one more pass each: the maximum of X or G).  The _timed
 *   kernels, in order -- forward: 0 max|X|, 1 X pass, 2 U rescale, 3 FP4 GEMM;
 *   backward: 0 max|G|, 1 G pass, 2 D rescale, 3 dA and dB, 4 FP4 dX GEMM.
 *   fourtune_linear_1x16_ws_offsets gives the workspace offsets of Q16(X)
 *   (backward = 0) or Q16(G) (backward = 1): codes [M, C/2], scales [M, C/16],
 *   the tensor's maximum word and (backward) P [M, r_s + r] bf16. */
typedef struct {
  int64_t K, N, r_s, r;
  const uint8_t* R_codes;     /* Q16(R)   [N, K/2] */
  const uint8_t* R_sf;        /* its MMA-ready scales (rows N, cols K) */
  const uint8_t* Rt_codes;    /* Q16(R^T) [K, N/2] */
  const uint8_t* Rt_sf;       /* its MMA-ready scales (rows K, cols N) */
  const uint32_t* R_amax;     /* device word: float32 bits of max|R| */
  const ft_bf16* D;
  const ft_bf16* U;
  const ft_bf16* bias;
} ft_linear_1x16_t;
FT_API int fourtune_quantize_1x16(const ft_bf16* W, int64_t rows, int64_t cols, int transposed, uint32_t* amax_word,
                                  uint8_t* codes, uint8_t* scales, uint8_t* sf_mma, void* stream);
FT_API size_t fourtune_linear_fwd_1x16_workspace_size(const ft_linear_1x16_t* layer, int64_t M);
FT_API size_t fourtune_linear_bwd_1x16_workspace_size(const ft_linear_1x16_t* layer, int64_t M);
FT_API int fourtune_linear_fwd_1x16(const ft_linear_1x16_t* layer, const ft_bf16* X, int64_t M, void* Y, int y_dtype,
                                    ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream);
FT_API int fourtune_linear_bwd_1x16(const ft_linear_1x16_t* layer, const ft_bf16* dY, const ft_bf16* X,
                                    const ft_bf16* L_saved, int64_t M, void* dX, int dx_dtype, float* dA, float* dB,
                                    int accumulate, void* ws, size_t ws_bytes, void* stream);
FT_API int fourtune_linear_fwd_1x16_timed(const ft_linear_1x16_t* layer, const ft_bf16* X, int64_t M, void* Y,
                                          int y_dtype, ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream,
                                          void* const* events, int n_events);
FT_API int fourtune_linear_bwd_1x16_timed(const ft_linear_1x16_t* layer, const ft_bf16* dY, const ft_bf16* X,
                                          const ft_bf16* L_saved, int64_t M, void* dX, int dx_dtype, float* dA,
                                          float* dB, int accumulate, void* ws, size_t ws_bytes, void* stream,
                                          void* const* events, int n_events);
FT_API int fourtune_linear_1x16_ws_offsets(const ft_linear_1x16_t* layer, int64_t M, int backward, size_t* codes_off,
                                           size_t* scales_off, size_t* amax_off, size_t* P_off);

/* The MLP pair (§3.3 "MLP Fusion"): y = FC2(GELU_tanh(FC1(X))), both layers
 * triple-branch, fc1 [K1 -> H], fc2 [H -> N2] (fc1->N == fc2->K).
 * Forward: the X pass, then FC1's 4-bit GEMM (+ L1 U1 + b1) whose epilogue
 * forms h = bf16(FC1(X)) (saved), a = GELU_tanh(h) in fp32 and FC2's input
 * bf16(a), shared by FC2's three branches: Q(bf16(a)) (FC2's 4-bit input) and
 * the fp32 partials of bf16(a) D2 per run of N tiles (a small reduction sums
 * them in split order into L2 = bf16(bf16(a) D2), FC2's low-rank input) --
 * the hidden activation is never stored -- then FC2's 4-bit GEMM
 * (+ L2 U2 + b2).  Writes Y [M, N2], h_saved [M, H], L1_saved
 * [M, r_s1 + r1], L2_saved [M, r_s2 + r2]; dbg_a, when not NULL, receives the
 * fp32 a [M, H] (for inspection). */
FT_API size_t fourtune_mlp_fwd_workspace_size(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M);
FT_API int fourtune_mlp_fwd(const ft_linear_t* fc1, const ft_linear_t* fc2, const ft_bf16* X, int64_t M, void* Y,
                            int y_dtype, ft_bf16* h_saved, ft_bf16* L1_saved, ft_bf16* L2_saved, float* dbg_a,
                            void* ws, size_t ws_bytes, void* stream);

/* MLP backward.  FC2's G pass, then FC2's dX GEMM whose epilogue forms
 * d_h = bf16(d_a GELU'(h)) -- FC1's incoming gradient, taken by all three of
 * its branches -- with Q(d_h) (FC1's 4-bit gradient) and the partials of
 * d_h U1^T (summed by the reduction into P1 = bf16(d_h U1^T)).
 * FC2's dA2 = bf16(GELU(h))^T P2[:, r_s2:] recomputes GELU(h) from h (nothing
 * of the activation is stored).  Writes dX [M, K1] and the four adapter
 * gradients (fp32; accumulate = 1 adds).  FC1's dA1/dB1 run beside FC1's dX
 * GEMM on the library stream, as in fourtune_linear_bwd. */
FT_API size_t fourtune_mlp_bwd_workspace_size(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M);
FT_API int fourtune_mlp_bwd(const ft_linear_t* fc1, const ft_linear_t* fc2, const ft_bf16* dY, const ft_bf16* X,
                            const ft_bf16* h_saved, const ft_bf16* L1_saved, const ft_bf16* L2_saved, int64_t M,
                            void* dX, int dx_dtype, float* dA1, float* dB1, float* dA2, float* dB2, int accumulate,
                            void* ws, size_t ws_bytes, void* stream);

/* The MLP calls with per-kernel CUDA events, as fourtune_linear_*_timed.  Kernels,
 * in order -- forward: 0 X pass, 1 FC1 GEMM with the GELU / Q(a) / L2 epilogue,
 * 2 L2 reduction, 3 FC2 GEMM; backward: 0 G pass (FC2), 1 FC2 dX GEMM with the
 * GELU' / Q(d_h) / P1 epilogue, 2 P1 reduction, 3 FC2 dA/dB, 4 FC1 dA/dB, 5 FC1
 * dX GEMM. */
FT_API int fourtune_mlp_fwd_timed(const ft_linear_t* fc1, const ft_linear_t* fc2, const ft_bf16* X, int64_t M,
                                  void* Y, int y_dtype, ft_bf16* h_saved, ft_bf16* L1_saved, ft_bf16* L2_saved,
                                  float* dbg_a, void* ws, size_t ws_bytes, void* stream, void* const* events,
                                  int n_events);
FT_API int fourtune_mlp_bwd_timed(const ft_linear_t* fc1, const ft_linear_t* fc2, const ft_bf16* dY,
                                  const ft_bf16* X, const ft_bf16* h_saved, const ft_bf16* L1_saved,
                                  const ft_bf16* L2_saved, int64_t M, void* dX, int dx_dtype, float* dA1, float* dB1,
                                  float* dA2, float* dB2, int accumulate, void* ws, size_t ws_bytes, void* stream,
                                  void* const* events, int n_events);

/* Workspace byte offsets of the MLP's intermediate tensors (inspection, tests):
 * forward: Q(a) codes [M, H/2] and scales [M/16, H/16]; backward: d_h (bf16
 * [M, H]) and Q(d_h) codes and scales; a_off is set to SIZE_MAX (bf16(GELU(h))
 * is not stored). */
FT_API int fourtune_mlp_fwd_ws_offsets(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M, size_t* qa_codes,
                                       size_t* qa_scales);
FT_API int fourtune_mlp_bwd_ws_offsets(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M, size_t* dh_off,
                                       size_t* a_off, size_t* qdh_codes, size_t* qdh_scales);

/* Byte offsets, inside the workspace of the last fwd / bwd call with these sizes,
 * of the block16 activation (fwd: Q(X)) or gradient (bwd: Q(G)) codes and scales,
 * and (bwd) of P [M, r_s + r] bf16.  For inspection and tests; unused -> NULL. */
FT_API int fourtune_linear_fwd_ws_offsets(const ft_linear_t* layer, int64_t M, size_t* codes_off, size_t* scales_off);
FT_API int fourtune_linear_bwd_ws_offsets(const ft_linear_t* layer, int64_t M, size_t* codes_off, size_t* scales_off,
                                   size_t* P_off);

/* Fused row pass without a workspace.  The FourTune paper has no counterpart to
 * this entry point; it exists for callers that cannot allocate device memory
 * to hand the library a workspace -- plugin or embedding hosts that own all
 * device memory and offer no scratch allocator, and runtimes that forbid any
 * allocation once they have started.  It computes what the forward's first
 * kernel computes, for any bf16 input X [M, K] and down-projection rows
 * W [R, K] (bf16, K contiguous; for the layer, W = D^T = [S_dn | A]^T):
 *   codes [M, K/2], scales [M/16, K/16] = block16(X)   and   L [M, R] = bf16(X W^T).
 * The caller still owns X, W and the outputs.  Scratch (split-K partial sums,
 * split counters, status word) lives in one device array inside the library,
 * FT_STATIC_SCRATCH_BYTES (16 MiB) on every GPU that loads the library, kept
 * until the process exits; no cudaMalloc, cudaFree or other allocation is made.
 * The first call on a device looks up the array's device address on that
 * device and keeps it for the life of the process, so make that first call
 * before any stream capture begins; a cudaDeviceReset (or anything else that
 * tears down the device's primary context) invalidates the kept address, and
 * the entry point must not be called on that device afterwards.  Every call
 * shares the array: calls that overlap on the GPU (other streams, other host
 * threads) race and corrupt each other's results; serialize them.  The split
 * rule is the workspace path's, so the outputs are bit-identical to the
 * forward's.  Returns FT_ERR_WORKSPACE when the problem needs more scratch than
 * the array holds (only for M in the millions of tokens), FT_ERR_UNSUPPORTED
 * for R outside 16..128 (multiples of 16), else as the other calls.  An
 * expired wait is recorded in the array: fourtune_quant_down_static_status
 * reports it. */
#define FT_STATIC_SCRATCH_BYTES (16u << 20)
FT_API int fourtune_quant_down_static(const ft_bf16* X, int64_t M, int64_t K, const ft_bf16* W, int64_t R,
                                      uint8_t* codes, uint8_t* scales, ft_bf16* L, void* stream);

/* Status of the last fourtune_quant_down_static call on the current device
 * (no counterpart in the paper): synchronizes `stream` and returns
 * FT_ERR_TIMEOUT if one of its kernel waits expired (the outputs are then
 * incomplete), FT_ERR_CUDA on a CUDA error, else FT_OK.  Allocates nothing. */
FT_API int fourtune_quant_down_static_status(void* stream);

/* Test hook for the failure path (no counterpart in the paper).  Runs the fused
 * row pass of fourtune_quant_down_static with its bookkeeping in the caller's
 * `ws` (256-byte aligned; at least 256 + 4 ceil(M/128) + 64 M R bytes is always
 * enough) and with every kernel wait limited to `wait_ns` (1e6 .. 1e9 ns), and
 * makes the first CTA's producer leave its first stage unloaded: the waits for
 * that stage expire, the CTA records FT_ERR_TIMEOUT in ws, stops waiting,
 * drains the copies it started and frees its tensor memory.  The outputs of
 * that CTA's rows are then incomplete; fourtune_device_status(ws) returns
 * FT_ERR_TIMEOUT.  Nothing faults or traps: the GPU stays usable. */
FT_API int fourtune_test_wait_timeout(const ft_bf16* X, int64_t M, int64_t K, const ft_bf16* W, int64_t R,
                                      uint8_t* codes, uint8_t* scales, ft_bf16* L, void* ws, size_t ws_bytes,
                                      int64_t wait_ns, void* stream);

/* Synchronizes `stream` and returns FT_ERR_TIMEOUT if a kernel of the last call
 * that used `ws` recorded an expired wait, FT_ERR_CUDA on a CUDA error, else FT_OK. */
FT_API int fourtune_device_status(const void* ws, void* stream);

/* Static description of an FT_* code. */
FT_API const char* fourtune_error_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* FOURTUNE_FOURTUNE_H_ */
