// C ABI entry points: argument checks, workspace carving, tensor-map
// construction and the launch sequence of each call.  No device allocation and
// no host synchronization happen here (except fourtune_device_status).
#include <algorithm>
#include <cstring>
#include <mutex>

#include "fourtune/fourtune.h"
#include "kernels.h"

namespace {

using ft::GemmParams;
using ft::RowpassParams;
using ft::TgradParams;

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 2-D row-major map: `inner` elements per row (contiguous), `outer` rows of
// `row_bytes` bytes; box = box_inner x box_outer.  Out-of-range elements read 0.
bool make_map(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}
// bf16 [rows, cols], boxes of 64 columns (128 bytes, 128-byte swizzle) x box_rows
bool map_bf16(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, cols, rows, cols * 2, 64, box_rows,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}
// block16 codes of a [rows, cols] matrix: [rows, cols/2] bytes, boxes of 128 bytes x box_rows
bool map_codes(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, cols / 2, rows, cols / 2, 128, box_rows,
                  CU_TENSOR_MAP_SWIZZLE_128B);
}
// GEMM output [rows, cols] fp32 or bf16: boxes of 128 bytes x 32 rows, 128-byte swizzle
bool map_out(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, bool bf16) {
  return bf16 ? make_map(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, cols, rows, cols * 2, 64, 32,
                         CU_TENSOR_MAP_SWIZZLE_128B)
              : make_map(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, base, cols, rows, cols * 4, 32, 32,
                         CU_TENSOR_MAP_SWIZZLE_128B);
}
// compact scales [rows, cols] bytes, unswizzled boxes of 16 bytes x box_rows
bool map_scales(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint32_t box_rows) {
  return make_map(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, cols, rows, cols, 16, box_rows,
                  CU_TENSOR_MAP_SWIZZLE_NONE);
}

struct DevInfo {
  int ok = 0;  // 1 = sm_100, -1 = other
  int num_sms = 0;
};

int device_info(DevInfo* out) {
  static DevInfo cache[64];
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return FT_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev].ok == 0) {
    int major = 0, minor = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return FT_ERR_CUDA;
    cache[dev].ok = (major == 10 && minor == 0) ? 1 : -1;
    cache[dev].num_sms = sms;
  }
  *out = cache[dev];
  return out->ok == 1 ? FT_OK : FT_ERR_UNSUPPORTED;
}
int num_sms_or_default() {
  DevInfo di;
  device_info(&di);
  return di.num_sms > 0 ? di.num_sms : 148;
}

inline bool al16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline int cdiv(int64_t a, int64_t b) { return static_cast<int>((a + b - 1) / b); }

int check_layer(const ft_linear_t* L, bool need_t) {
  if (!L || !L->R_codes || !L->R_scales || !L->D || !L->U) return FT_ERR_INVALID_ARG;
  if (need_t && !L->R_codes_t) return FT_ERR_INVALID_ARG;
  if (L->K <= 0 || L->N <= 0 || L->K % 32 || L->N % 32) return FT_ERR_SHAPE;
  if (L->r_s < 0 || L->r < 16 || L->r_s % 16 || L->r % 16 || L->r > 64 || L->r_s + L->r > 128)
    return FT_ERR_UNSUPPORTED;
  if (L->K > (1 << 30) || L->N > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(L->R_codes) || !al16(L->D) || !al16(L->U) || (L->R_codes_t && !al16(L->R_codes_t)) ||
      (L->bias && !al16(L->bias)))
    return FT_ERR_ALIGN;
  return FT_OK;
}

// ---------------------------------------------------------------- split choice
struct RowSplit {
  int nsplit, kt_per_split;
};
// enough CTAs for every SM (two per SM when they fit), never more splits than tiles
RowSplit row_split(int64_t M, int64_t K, int64_t R, int mn, int num_sms, int max_split) {
  const int MT = cdiv(M, 128), KT = cdiv(K, 64);
  const int target = num_sms * ft::rowpass_ctas_per_sm(static_cast<int>(R), mn);
  const int ns = MT >= target ? 1 : std::max(1, std::min({KT, target / MT, max_split}));
  const int per = cdiv(KT, ns);
  return {cdiv(KT, per), per};
}
struct MSplit {
  int nsplit, mt_per_split;
};
MSplit m_split(int64_t M, int64_t P, int ctas) {
  const int MT = cdiv(M, 128), PT = cdiv(P, 128);
  const int ns = PT >= ctas ? 1 : std::max(1, std::min(MT, ctas / PT));
  const int per = cdiv(MT, ns);
  return {cdiv(MT, per), per};
}

// ---------------------------------------------------------------- workspace
// Every layout starts with a header (status word + split counters) that each
// call clears before its first kernel.
struct FwdWs {
  size_t header, counters, codes, scales, part, total;
  RowSplit rs;
};
FwdWs fwd_layout(const ft_linear_t* L, int64_t M, int num_sms) {
  FwdWs w{};
  const int64_t R = L->r_s + L->r;
  w.rs = row_split(M, L->K, R, 1, num_sms, ft::kRowpassMaxClusterSplit);
  w.counters = 16;
  w.header = up256(16 + 4 * static_cast<size_t>(cdiv(M, 128)));
  size_t o = w.header;
  w.codes = o;
  o = up256(o + static_cast<size_t>(M * L->K / 2));
  w.scales = o;
  o = up256(o + static_cast<size_t>((M / 16) * (L->K / 16)));
  w.part = o;  // unused: split partials are reduced inside the cluster
  w.total = o;
  return w;
}

struct BwdWs {
  size_t header, cnt_rp, cnt_dA, cnt_dB, codes, scales, P, part_rp, part_dA, part_dB, total;
  RowSplit rs;
  MSplit sA, sB;
};
BwdWs bwd_layout(const ft_linear_t* L, int64_t M, int num_sms) {
  BwdWs w{};
  const int64_t R = L->r_s + L->r;
  w.rs = row_split(M, L->N, R, 0, num_sms, ft::kRowpassMaxClusterSplit);
  w.sA = m_split(M, L->K, std::max(1, num_sms / 2));
  w.sB = m_split(M, L->N, std::max(1, num_sms / 2));
  const int MT = cdiv(M, 128), KTl = cdiv(L->K, 128), NTl = cdiv(L->N, 128);
  w.cnt_rp = 16;
  w.cnt_dA = w.cnt_rp + 4 * static_cast<size_t>(MT);
  w.cnt_dB = w.cnt_dA + 4 * static_cast<size_t>(KTl);
  w.header = up256(w.cnt_dB + 4 * static_cast<size_t>(NTl));
  size_t o = w.header;
  w.codes = o;
  o = up256(o + static_cast<size_t>(M * L->N / 2));
  w.scales = o;
  o = up256(o + static_cast<size_t>((M / 16) * (L->N / 16)));
  w.P = o;
  o = up256(o + static_cast<size_t>(M * R * 2));
  w.part_rp = o;  // unused: split partials are reduced inside the cluster
  w.part_dA = o;
  if (w.sA.nsplit > 1) o = up256(o + static_cast<size_t>(w.sA.nsplit) * KTl * 128 * 64 * 4);
  w.part_dB = o;
  if (w.sB.nsplit > 1) o = up256(o + static_cast<size_t>(w.sB.nsplit) * NTl * 128 * 64 * 4);
  w.total = o;
  return w;
}

int cuda_err(cudaError_t e) { return e == cudaSuccess ? FT_OK : FT_ERR_CUDA; }

// Optional per-kernel timing: events[2k] / events[2k+1] are recorded on the
// launching stream right before / after kernel k of the call (when provided).
struct Events {
  void* const* ev;
  int n;
  cudaError_t mark(int k, int side, cudaStream_t s) const {
    const int i = 2 * k + side;
    if (!ev || i >= n || !ev[i]) return cudaSuccess;
    return cudaEventRecord(static_cast<cudaEvent_t>(ev[i]), s);
  }
};
#define FT_LAUNCH(k, expr)                                      \
  do {                                                          \
    if (evs.mark((k), 0, s) != cudaSuccess) return FT_ERR_CUDA; \
    if ((expr) != cudaSuccess) return FT_ERR_CUDA;              \
    if (evs.mark((k), 1, s) != cudaSuccess) return FT_ERR_CUDA; \
  } while (0)

// scales can come by TMA when every compact scale row is a whole number of 16-byte units
bool scales_by_tma(int64_t K, int64_t N, const void* a, const void* b) {
  return K % 256 == 0 && N % 256 == 0 && al16(a) && al16(b);
}

}  // namespace

extern "C" {

const char* fourtune_error_string(int code) {
  switch (code) {
    case FT_OK: return "ok";
    case FT_ERR_INVALID_ARG: return "invalid argument";
    case FT_ERR_SHAPE: return "unsupported shape (dimensions must be multiples of 16, K and N of 32)";
    case FT_ERR_ALIGN: return "misaligned pointer";
    case FT_ERR_WORKSPACE: return "workspace too small (or problem larger than the static scratch)";
    case FT_ERR_CUDA: return "CUDA error";
    case FT_ERR_TIMEOUT: return "a kernel wait timed out";
    case FT_ERR_UNSUPPORTED: return "unsupported device or size";
    default: return "unknown error";
  }
}

int fourtune_quantize_block16(const ft_bf16* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes,
                              uint8_t* scales, uint8_t* codes_t, void* stream) {
  if (!x || !codes || !scales) return FT_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16 || ld < cols || ld % 8) return FT_ERR_SHAPE;
  if (rows > (1 << 30) || cols > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(x)) return FT_ERR_ALIGN;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaError_t e =
      ft::launch_quantize_block16(x, static_cast<int>(rows), static_cast<int>(cols), ld, codes, scales, s);
  if (e == cudaSuccess && codes_t)
    e = ft::launch_transpose_codes(codes, static_cast<int>(rows), static_cast<int>(cols), codes_t, s);
  return cuda_err(e);
}

int fourtune_transpose_codes(const uint8_t* codes, int64_t rows, int64_t cols, uint8_t* codes_t, void* stream) {
  if (!codes || !codes_t) return FT_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16) return FT_ERR_SHAPE;
  if (rows > (1 << 30) || cols > (1 << 30)) return FT_ERR_UNSUPPORTED;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  return cuda_err(ft::launch_transpose_codes(codes, static_cast<int>(rows), static_cast<int>(cols), codes_t,
                                             static_cast<cudaStream_t>(stream)));
}

size_t fourtune_linear_fwd_workspace_size(const ft_linear_t* layer, int64_t M) {
  if (check_layer(layer, false) || M <= 0 || M % 16) return 0;
  return fwd_layout(layer, M, num_sms_or_default()).total;
}

size_t fourtune_linear_bwd_workspace_size(const ft_linear_t* layer, int64_t M) {
  if (check_layer(layer, true) || M <= 0 || M % 16) return 0;
  return bwd_layout(layer, M, num_sms_or_default()).total;
}

int fourtune_linear_fwd_ws_offsets(const ft_linear_t* layer, int64_t M, size_t* codes_off, size_t* scales_off) {
  int st = check_layer(layer, false);
  if (st) return st;
  FwdWs w = fwd_layout(layer, M, num_sms_or_default());
  if (codes_off) *codes_off = w.codes;
  if (scales_off) *scales_off = w.scales;
  return FT_OK;
}

int fourtune_linear_bwd_ws_offsets(const ft_linear_t* layer, int64_t M, size_t* codes_off, size_t* scales_off,
                                   size_t* P_off) {
  int st = check_layer(layer, true);
  if (st) return st;
  BwdWs w = bwd_layout(layer, M, num_sms_or_default());
  if (codes_off) *codes_off = w.codes;
  if (scales_off) *scales_off = w.scales;
  if (P_off) *P_off = w.P;
  return FT_OK;
}

int fourtune_linear_fwd(const ft_linear_t* layer, const ft_bf16* X, int64_t M, void* Y, int y_dtype,
                        ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream) {
  return fourtune_linear_fwd_timed(layer, X, M, Y, y_dtype, L_saved, ws, ws_bytes, stream, nullptr, 0);
}

int fourtune_linear_fwd_timed(const ft_linear_t* layer, const ft_bf16* X, int64_t M, void* Y, int y_dtype,
                              ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream, void* const* events,
                              int n_events) {
  const Events evs{events, n_events};
  int st = check_layer(layer, false);
  if (st) return st;
  if (!X || !Y || !L_saved || !ws) return FT_ERR_INVALID_ARG;
  if (y_dtype != FT_DTYPE_F32 && y_dtype != FT_DTYPE_BF16) return FT_ERR_INVALID_ARG;
  if (M <= 0 || M % 16) return FT_ERR_SHAPE;
  if (M > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(X) || !al16(Y) || !al16(L_saved) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return FT_ERR_ALIGN;
  DevInfo di;
  if ((st = device_info(&di))) return st;
  const FwdWs w = fwd_layout(layer, M, di.num_sms);
  if (ws_bytes < w.total) return FT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int64_t K = layer->K, N = layer->N, R = layer->r_s + layer->r;
  int* status = reinterpret_cast<int*>(base);
  if (cudaMemsetAsync(base, 0, w.header, s) != cudaSuccess) return FT_ERR_CUDA;

  // X pass: Q(X) and L = bf16(X D), D = [S_dn | A] read MN-major
  CUtensorMap tmX, tmW;
  if (!map_bf16(&tmX, X, K, M, 128) || !map_bf16(&tmW, layer->D, R, K, 64)) return FT_ERR_CUDA;
  RowpassParams rp{};
  rp.M = static_cast<int>(M);
  rp.K = static_cast<int>(K);
  rp.R = static_cast<int>(R);
  rp.w_mn_major = 1;
  rp.kt_per_split = w.rs.kt_per_split;
  rp.nsplit = w.rs.nsplit;
  rp.cluster_reduce = w.rs.nsplit > 1;
  rp.codes = base + w.codes;
  rp.scales = base + w.scales;
  rp.L = L_saved;
  rp.part = reinterpret_cast<float*>(base + w.part);
  rp.counters = reinterpret_cast<int*>(base + w.counters);
  rp.status = status;
  FT_LAUNCH(0, ft::launch_rowpass(tmX, tmW, rp, s));

  // 4-bit GEMM + L U + bias, U = [S_up ; B] read MN-major
  CUtensorMap tmA, tmB, tmA2, tmB2, tmSA, tmSB;
  const bool sf_tma = scales_by_tma(K, N, base + w.scales, layer->R_scales);
  if (!map_codes(&tmA, base + w.codes, K, M, 128) || !map_codes(&tmB, layer->R_codes, K, N, ft::kGemmBN) ||
      !map_bf16(&tmA2, L_saved, R, M, 128) || !map_bf16(&tmB2, layer->U, N, R, 64))
    return FT_ERR_CUDA;
  if (sf_tma) {
    if (!map_scales(&tmSA, base + w.scales, K / 16, M / 16, 8) ||
        !map_scales(&tmSB, layer->R_scales, K / 16, N / 16, ft::kGemmBN / 16))
      return FT_ERR_CUDA;
  } else {
    tmSA = tmA;  // unused
    tmSB = tmA;
  }
  GemmParams gp{};
  gp.M = static_cast<int>(M);
  gp.N = static_cast<int>(N);
  gp.K = static_cast<int>(K);
  gp.R2 = static_cast<int>(R);
  gp.b2_mn_major = 1;
  gp.sf_tma = sf_tma ? 1 : 0;
  gp.sfb_transposed = 0;
  gp.sfa = base + w.scales;
  gp.sfa_rs = K / 16;
  gp.sfa_gs = 1;
  gp.sfb = layer->R_scales;
  gp.sfb_rs = K / 16;
  gp.sfb_gs = 1;
  gp.bias = layer->bias;
  gp.out = Y;
  gp.ldo = N;
  gp.out_bf16 = y_dtype == FT_DTYPE_BF16;
  gp.status = status;
  CUtensorMap tmO;
  if (!map_out(&tmO, Y, N, M, gp.out_bf16 != 0)) return FT_ERR_CUDA;
  FT_LAUNCH(1, ft::launch_gemm_fp4(tmA, tmB, tmA2, tmB2, tmSA, tmSB, tmO, gp, s));
  return FT_OK;
}

int fourtune_linear_bwd(const ft_linear_t* layer, const ft_bf16* dY, const ft_bf16* X, const ft_bf16* L_saved,
                        int64_t M, void* dX, int dx_dtype, float* dA, float* dB, int accumulate, void* ws,
                        size_t ws_bytes, void* stream) {
  return fourtune_linear_bwd_timed(layer, dY, X, L_saved, M, dX, dx_dtype, dA, dB, accumulate, ws, ws_bytes, stream,
                                   nullptr, 0);
}

int fourtune_linear_bwd_timed(const ft_linear_t* layer, const ft_bf16* dY, const ft_bf16* X,
                              const ft_bf16* L_saved, int64_t M, void* dX, int dx_dtype, float* dA, float* dB,
                              int accumulate, void* ws, size_t ws_bytes, void* stream, void* const* events,
                              int n_events) {
  const Events evs{events, n_events};
  int st = check_layer(layer, true);
  if (st) return st;
  if (!dY || !X || !L_saved || !dX || !dA || !dB || !ws) return FT_ERR_INVALID_ARG;
  if (dx_dtype != FT_DTYPE_F32 && dx_dtype != FT_DTYPE_BF16) return FT_ERR_INVALID_ARG;
  if (M <= 0 || M % 16) return FT_ERR_SHAPE;
  if (M > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(dY) || !al16(X) || !al16(L_saved) || !al16(dX) || !al16(dA) || !al16(dB) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return FT_ERR_ALIGN;
  DevInfo di;
  if ((st = device_info(&di))) return st;
  const BwdWs w = bwd_layout(layer, M, di.num_sms);
  if (ws_bytes < w.total) return FT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  const int64_t K = layer->K, N = layer->N, R = layer->r_s + layer->r;
  int* status = reinterpret_cast<int*>(base);
  if (cudaMemsetAsync(base, 0, w.header, s) != cudaSuccess) return FT_ERR_CUDA;

  // G pass: Q(G) and P = bf16(G U^T), U = [S_up ; B] [R, N] read K-major
  CUtensorMap tmG, tmU;
  if (!map_bf16(&tmG, dY, N, M, 128) || !map_bf16(&tmU, layer->U, N, R, static_cast<uint32_t>(R)))
    return FT_ERR_CUDA;
  RowpassParams rp{};
  rp.M = static_cast<int>(M);
  rp.K = static_cast<int>(N);
  rp.R = static_cast<int>(R);
  rp.w_mn_major = 0;
  rp.kt_per_split = w.rs.kt_per_split;
  rp.nsplit = w.rs.nsplit;
  rp.cluster_reduce = w.rs.nsplit > 1;
  rp.codes = base + w.codes;
  rp.scales = base + w.scales;
  rp.L = base + w.P;
  rp.part = reinterpret_cast<float*>(base + w.part_rp);
  rp.counters = reinterpret_cast<int*>(base + w.cnt_rp);
  rp.status = status;
  FT_LAUNCH(0, ft::launch_rowpass(tmG, tmU, rp, s));

  // dX = deq(Q(G)) deq(Q(R)) + P D^T : B operand = R^T codes, R's scales read transposed,
  // D = [S_dn | A] [K, R] read K-major
  CUtensorMap tmA, tmB, tmA2, tmB2, tmSA, tmSB;
  const bool sf_tma = scales_by_tma(K, N, base + w.scales, layer->R_scales);
  if (!map_codes(&tmA, base + w.codes, N, M, 128) || !map_codes(&tmB, layer->R_codes_t, N, K, ft::kGemmBN) ||
      !map_bf16(&tmA2, base + w.P, R, M, 128) || !map_bf16(&tmB2, layer->D, R, K, ft::kGemmBN))
    return FT_ERR_CUDA;
  if (sf_tma) {
    if (!map_scales(&tmSA, base + w.scales, N / 16, M / 16, 8) ||
        !map_scales(&tmSB, layer->R_scales, K / 16, N / 16, 16))
      return FT_ERR_CUDA;
  } else {
    tmSA = tmA;  // unused
    tmSB = tmA;
  }
  GemmParams gp{};
  gp.M = static_cast<int>(M);
  gp.N = static_cast<int>(K);
  gp.K = static_cast<int>(N);
  gp.R2 = static_cast<int>(R);
  gp.b2_mn_major = 0;
  gp.sf_tma = sf_tma ? 1 : 0;
  gp.sfb_transposed = 1;
  gp.sfa = base + w.scales;
  gp.sfa_rs = N / 16;
  gp.sfa_gs = 1;
  gp.sfb = layer->R_scales;  // scale of (row k of R^T, group g over N) = R_scales[g, k/16]
  gp.sfb_rs = 1;
  gp.sfb_gs = K / 16;
  gp.bias = nullptr;
  gp.out = dX;
  gp.ldo = K;
  gp.out_bf16 = dx_dtype == FT_DTYPE_BF16;
  gp.status = status;
  CUtensorMap tmO;
  if (!map_out(&tmO, dX, K, M, gp.out_bf16 != 0)) return FT_ERR_CUDA;
  FT_LAUNCH(1, ft::launch_gemm_fp4(tmA, tmB, tmA2, tmB2, tmSA, tmSB, tmO, gp, s));

  // dA = X^T P[:, r_s:] and dB = L[:, r_s:]^T G (computed as dB^T, stored transposed), one launch
  CUtensorMap tmTa, tmVa, tmTb, tmVb;
  if (!map_bf16(&tmTa, X, K, M, 128) || !map_bf16(&tmVa, base + w.P, R, M, 128) ||
      !map_bf16(&tmTb, dY, N, M, 128) || !map_bf16(&tmVb, L_saved, R, M, 128))
    return FT_ERR_CUDA;
  TgradParams ta{}, tb{};
  ta.M = tb.M = static_cast<int>(M);
  ta.r = tb.r = static_cast<int>(layer->r);
  ta.v0 = tb.v0 = static_cast<int>(layer->r_s);
  ta.accumulate = tb.accumulate = accumulate ? 1 : 0;
  ta.status = tb.status = status;
  ta.P = static_cast<int>(K);
  ta.mt_per_split = w.sA.mt_per_split;
  ta.nsplit = w.sA.nsplit;
  ta.out = dA;
  ta.out_sp = layer->r;
  ta.out_sj = 1;
  ta.part = reinterpret_cast<float*>(base + w.part_dA);
  ta.counters = reinterpret_cast<int*>(base + w.cnt_dA);
  tb.P = static_cast<int>(N);
  tb.mt_per_split = w.sB.mt_per_split;
  tb.nsplit = w.sB.nsplit;
  tb.out = dB;
  tb.out_sp = 1;
  tb.out_sj = N;
  tb.part = reinterpret_cast<float*>(base + w.part_dB);
  tb.counters = reinterpret_cast<int*>(base + w.cnt_dB);
  FT_LAUNCH(2, ft::launch_tgrad2(tmTa, tmVa, ta, tmTb, tmVb, tb, s));
  return FT_OK;
}

int fourtune_quant_down_static(const ft_bf16* X, int64_t M, int64_t K, const ft_bf16* W, int64_t R,
                               uint8_t* codes, uint8_t* scales, ft_bf16* L, void* stream) {
  if (!X || !W || !codes || !scales || !L) return FT_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || M % 16 || K % 32) return FT_ERR_SHAPE;
  if (R < 16 || R % 16 || R > 128 || M > (1 << 30) || K > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(X) || !al16(W) || !al16(codes) || !al16(L)) return FT_ERR_ALIGN;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  // W^T [R, K] read K-major (the backward pass's layout) with its own split choice
  const RowSplit rs = row_split(M, K, R, 0, di.num_sms, 1 << 20);
  const size_t header = up256(16 + 4 * static_cast<size_t>(cdiv(M, 128)));
  const size_t need = header + (rs.nsplit > 1 ? static_cast<size_t>(rs.nsplit) * M * R * 4 : 0);
  if (need > ft::kRowpassStaticScratchBytes) return FT_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (ft::rowpass_static_scratch(&scratch) != cudaSuccess) return FT_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(scratch);
  // status word and split counters must start at zero; the array keeps what the last call left
  if (cudaMemsetAsync(base, 0, header, s) != cudaSuccess) return FT_ERR_CUDA;
  CUtensorMap tmX, tmW;
  if (!map_bf16(&tmX, X, K, M, 128) || !map_bf16(&tmW, W, K, R, static_cast<uint32_t>(R))) return FT_ERR_CUDA;
  RowpassParams rp{};
  rp.M = static_cast<int>(M);
  rp.K = static_cast<int>(K);
  rp.R = static_cast<int>(R);
  rp.w_mn_major = 0;
  rp.kt_per_split = rs.kt_per_split;
  rp.nsplit = rs.nsplit;
  rp.cluster_reduce = 0;  // partials in the static scratch, summed by the last CTA
  rp.codes = codes;
  rp.scales = scales;
  rp.L = L;
  rp.part = reinterpret_cast<float*>(base + header);
  rp.counters = reinterpret_cast<int*>(base + 16);
  rp.status = reinterpret_cast<int*>(base);
  return cuda_err(ft::launch_rowpass(tmX, tmW, rp, s));
}

int fourtune_device_status(const void* ws, void* stream) {
  if (!ws) return FT_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int h = 0;
  if (cudaMemcpyAsync(&h, ws, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FT_ERR_CUDA;
  return h == 0 ? FT_OK : FT_ERR_TIMEOUT;
}

}  // extern "C"
