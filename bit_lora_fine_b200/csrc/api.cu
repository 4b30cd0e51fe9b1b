// C ABI entry points: argument checks, workspace carving, tensor-map
// construction and the launch sequence of each call.  No device allocation and
// no host synchronization happen here (except fourtune_device_status).
#include <algorithm>
#include <cstring>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "fourtune/fourtune.h"
#include "kernels.h"

// One NVTX range around each entry point (visible in timeline profilers; costs
// nothing when no tool is attached).
struct FtRange {
  explicit FtRange(const char* name) { nvtxRangePushA(name); }
  ~FtRange() { nvtxRangePop(); }
};
#define FT_RANGE(name) const FtRange ft_range_(name)

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
int cuda_err(cudaError_t e) { return e == cudaSuccess ? FT_OK : FT_ERR_CUDA; }

int check_layer(const ft_linear_t* L, bool need_t) {
  if (!L || !L->R_codes || !L->R_scales || !L->R_sf || !L->D || !L->U) return FT_ERR_INVALID_ARG;
  if (need_t && (!L->R_codes_t || !L->R_sf_t)) return FT_ERR_INVALID_ARG;
  if (L->K <= 0 || L->N <= 0 || L->K % 32 || L->N % 32) return FT_ERR_SHAPE;
  if (L->r_s < 0 || L->r < 16 || L->r_s % 16 || L->r % 16 || L->r > 64 || L->r_s + L->r > 128)
    return FT_ERR_UNSUPPORTED;
  if (L->K > (1 << 30) || L->N > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(L->R_codes) || !al16(L->R_sf) || !al16(L->D) || !al16(L->U) || (L->R_codes_t && !al16(L->R_codes_t)) ||
      (L->R_sf_t && !al16(L->R_sf_t)) || (L->bias && !al16(L->bias)))
    return FT_ERR_ALIGN;
  return FT_OK;
}
int check_mlp(const ft_linear_t* fc1, const ft_linear_t* fc2, bool need_t) {
  int st = check_layer(fc1, need_t);
  if (st) return st;
  if ((st = check_layer(fc2, need_t))) return st;
  return fc1->N == fc2->K ? FT_OK : FT_ERR_SHAPE;
}
inline int64_t rank_all(const ft_linear_t* L) { return L->r_s + L->r; }

// ---------------------------------------------------------------- split choice
struct RowSplit {
  int nsplit, kt_per_split, stages;
};
// One CTA per SM with the deepest ring: enough CTAs for every SM (split-K when
// the 128-row tiles alone are too few), never more splits than K tiles.
constexpr int kRowMaxSplit = 16;
RowSplit row_split(int64_t M, int64_t K, int64_t R, int mn, int num_sms, int max_split) {
  const int MT = cdiv(M, 128), KT = cdiv(K, 64);
  const int ns = MT >= num_sms ? 1 : std::max(1, std::min({KT, num_sms / MT, max_split}));
  const int per = cdiv(KT, ns);
  return {cdiv(KT, per), per, ft::rowpass_stages(static_cast<int>(R), mn)};
}
// fp32 split partials of one row pass (0 without a split)
size_t rp_part_bytes(int64_t M, int64_t K, int64_t R, int mn, int num_sms) {
  const RowSplit rs = row_split(M, K, R, mn, num_sms, kRowMaxSplit);
  return rs.nsplit > 1 ? static_cast<size_t>(rs.nsplit) * static_cast<size_t>(M) * static_cast<size_t>(R) * 4 : 0;
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

// ---------------------------------------------------------------- workspace carving
struct Carver {
  size_t o = 0;
  size_t take(size_t bytes) {
    const size_t at = o;
    o = up256(o + bytes);
    return at;
  }
};
// block16 activations of a [M, C] matrix: codes, compact scales and the same
// scales in the MMA-ready layout the GEMM loads
struct Q16 {
  size_t codes, scales, sf;
  void carve(Carver& c, int64_t M, int64_t C) {
    codes = c.take(static_cast<size_t>(M * C / 2));
    scales = c.take(static_cast<size_t>((M / 16) * (C / 16)));
    sf = c.take(ft::sf_mma_bytes(M, C));
  }
};
// dA/dB launch of one layer: splits (serial run on all SMs; side run beside the
// dX GEMM on side_sms SMs), counters (in the header) and partials
struct GradPair {
  MSplit sA, sB;   // serial
  MSplit cA, cB;   // beside the dX GEMM
  int side_sms;
  size_t cntA, cntB;
  size_t partA, partB;
};
size_t grad_counter_words(const ft_linear_t* L) { return cdiv(L->K, 128) + cdiv(L->N, 128); }
// SMs given to dA/dB when they run beside the dX GEMM, which then gets the
// rest: split in proportion to the two kernels' work at the per-SM rates
// measured on this part when they share the GPU (FP4 GEMM ~14 TFLOP/s, dA/dB
// ~44 GB/s of X and G per SM -- both are paced per SM by TMA latency, not by
// the GPU-wide L2 or HBM bandwidth).  The GEMM's time goes in whole waves of
// output tiles, so it keeps the fewest SMs that give it the same number of
// waves and dA/dB take the rest; even, 8 .. half of the SMs.  0 (run them one
// after the other) on parts with fewer than 16 SMs.
int grad_side_sms(const ft_linear_t* L, int64_t M, int num_sms) {
  if (num_sms < 16) return 0;
  const double t_gemm = 2.0 * static_cast<double>(M) * L->N * L->K / 14.0e12;
  const double t_grad = 2.0 * static_cast<double>(M) * static_cast<double>(L->K + L->N) / 44.0e9;
  int n = static_cast<int>(std::lround(num_sms * t_grad / (t_grad + t_gemm)));
  n = std::max(8, std::min(num_sms / 2, n));
  const int64_t tiles = static_cast<int64_t>(cdiv(L->K, ft::kGemmBN)) * cdiv(M, ft::kGemmBM);   // dX output tiles
  const int64_t waves = (tiles + (num_sms - n) - 1) / (num_sms - n);
  const int64_t keep = (tiles + waves - 1) / waves;   // fewest SMs with that many waves (<= num_sms - n)
  n = std::max(n, num_sms - static_cast<int>(keep));
  n = std::min(num_sms / 2, n);
  return n & ~1;
}
// Serial: dA reads X from HBM; dB reads G, which the G pass has just streamed
// through L2, so dA gets two thirds of the SMs.  Side: each planned for the
// side SMs (one split per 128-row output tile when that fills them).
void plan_grads(GradPair& g, const ft_linear_t* L, int64_t M, int num_sms) {
  g.sA = m_split(M, L->K, std::max(1, 2 * num_sms / 3));
  g.sB = m_split(M, L->N, std::max(1, num_sms / 3));
  g.side_sms = grad_side_sms(L, M, num_sms);
  g.cA = m_split(M, L->K, std::max(1, g.side_sms));
  g.cB = m_split(M, L->N, std::max(1, g.side_sms));
}
size_t split_part_bytes(const MSplit& m, int64_t P) {
  return m.nsplit > 1 ? static_cast<size_t>(m.nsplit) * cdiv(P, 128) * 128 * 64 * 4 : 0;
}
// partials of dA (then dB), large enough for both plans
size_t grad_part_a(const GradPair& g, const ft_linear_t* L) {
  return std::max(split_part_bytes(g.sA, L->K), split_part_bytes(g.cA, L->K));
}
size_t grad_partial_bytes(const GradPair& g, const ft_linear_t* L) {
  return grad_part_a(g, L) + std::max(split_part_bytes(g.sB, L->N), split_part_bytes(g.cB, L->N));
}

// Each layout starts with a header of `header` bytes (status word, split
// counters) that every call clears first.
// Linear forward: header (status, row-pass split counters) | Q(X) | row-pass partials
struct FwdWs {
  size_t header, rp_cnt, rp_part, total;
  Q16 qx;
};
FwdWs fwd_layout(const ft_linear_t* L, int64_t M, int num_sms) {
  FwdWs w{};
  Carver c;
  w.rp_cnt = 16;
  c.take(w.header = up256(16 + 4 * static_cast<size_t>(cdiv(M, 128))));
  w.qx.carve(c, M, L->K);
  w.rp_part = c.take(rp_part_bytes(M, L->K, rank_all(L), 1, num_sms));
  w.total = c.o;
  return w;
}

// Linear backward: header (status, dA/dB and row-pass counters) | Q(G) | P |
// dA/dB partials | row-pass partials
struct BwdWs {
  size_t header, P, rp_cnt, rp_part, total;
  Q16 qg;
  GradPair g;
};
BwdWs bwd_layout(const ft_linear_t* L, int64_t M, int num_sms) {
  BwdWs w{};
  plan_grads(w.g, L, M, num_sms);
  Carver c;
  w.g.cntA = 16;
  w.g.cntB = w.g.cntA + 4 * static_cast<size_t>(cdiv(L->K, 128));
  w.rp_cnt = 16 + 4 * grad_counter_words(L);
  c.take(w.header = up256(w.rp_cnt + 4 * static_cast<size_t>(cdiv(M, 128))));
  w.qg.carve(c, M, L->N);
  w.P = c.take(static_cast<size_t>(M * rank_all(L) * 2));
  w.g.partA = c.take(grad_partial_bytes(w.g, L));
  w.g.partB = w.g.partA + grad_part_a(w.g, L);
  w.rp_part = c.take(rp_part_bytes(M, L->N, rank_all(L), 0, num_sms));
  w.total = c.o;
  return w;
}

// Units of the MLP's fused GEMMs (gemm_mlp.cu): a 128-row tile's N tiles split
// into nsplit runs of `per` (each unit writes one fp32 partial of the
// projection, summed by launch_proj_reduce).
struct MlpUnits {
  int nsplit, per;
};
MlpUnits plan_units(int64_t M, int64_t N, int num_sms) {
  // units of `per` consecutive N tiles of one 128-row tile: the makespan (tiles
  // on the busiest CTA) first, then as few splits (fp32 partials) as possible
  const int MT = cdiv(M, 128), NT = cdiv(N, 256);
  auto span_of = [&](int ns, int* nsr_out) {
    const int per = cdiv(NT, ns);
    const int nsr = cdiv(NT, per);
    if (nsr_out) *nsr_out = nsr;
    return static_cast<int64_t>(cdiv(static_cast<int64_t>(MT) * nsr, num_sms)) * per;
  };
  int64_t best = span_of(NT, nullptr);
  for (int ns = 1; ns < NT; ++ns) best = std::min(best, span_of(ns, nullptr));
  for (int ns = 1; ns <= NT; ++ns) {
    int nsr = 0;
    if (span_of(ns, &nsr) <= best) return {nsr, cdiv(NT, ns)};
  }
  return {NT, 1};
}
size_t proj_part_bytes(int64_t M, int64_t N, int64_t RP, int num_sms) {
  return static_cast<size_t>(plan_units(M, N, num_sms).nsplit) * static_cast<size_t>(M) * static_cast<size_t>(RP) * 4;
}

// MLP forward: header (status, row-pass counters) | Q(X) |
// Q(a) | row-pass partials | FC1 projection partials (L2)
struct MlpFwdWs {
  size_t header, rp_cnt, rp_part, pj_part, total;
  Q16 qx, qa;
};
MlpFwdWs mlp_fwd_layout(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M, int num_sms) {
  MlpFwdWs w{};
  Carver c;
  w.rp_cnt = 16;
  c.take(w.header = up256(w.rp_cnt + 4 * static_cast<size_t>(cdiv(M, 128))));
  w.qx.carve(c, M, fc1->K);
  w.qa.carve(c, M, fc1->N);
  w.rp_part = c.take(rp_part_bytes(M, fc1->K, rank_all(fc1), 1, num_sms));
  w.pj_part = c.take(proj_part_bytes(M, fc1->N, rank_all(fc2), num_sms));
  w.total = c.o;
  return w;
}

// MLP backward: header (status, counters of both layers' dA/dB, row-pass
// counters) | Q(G) | P2 | d_h | Q(d_h) | P1 | dA/dB
// partials (shared by the two dA/dB launches) | row-pass partials | FC2-dX
// projection partials (P1)
struct MlpBwdWs {
  size_t header, P2, dh, P1, rp_cnt, rp_part, pj_part, total;
  Q16 qg, qdh;
  GradPair g2, g1;
};
MlpBwdWs mlp_bwd_layout(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M, int num_sms) {
  MlpBwdWs w{};
  plan_grads(w.g2, fc2, M, num_sms);
  plan_grads(w.g1, fc1, M, num_sms);
  const int64_t H = fc1->N;
  Carver c;
  w.g2.cntA = 16;
  w.g2.cntB = w.g2.cntA + 4 * static_cast<size_t>(cdiv(fc2->K, 128));
  w.g1.cntA = w.g2.cntB + 4 * static_cast<size_t>(cdiv(fc2->N, 128));
  w.g1.cntB = w.g1.cntA + 4 * static_cast<size_t>(cdiv(fc1->K, 128));
  w.rp_cnt = 16 + 4 * (grad_counter_words(fc2) + grad_counter_words(fc1));
  c.take(w.header = up256(w.rp_cnt + 4 * static_cast<size_t>(cdiv(M, 128))));
  w.qg.carve(c, M, fc2->N);
  w.P2 = c.take(static_cast<size_t>(M * rank_all(fc2) * 2));
  w.dh = c.take(static_cast<size_t>(M * H * 2));
  w.qdh.carve(c, M, H);
  w.P1 = c.take(static_cast<size_t>(M * rank_all(fc1) * 2));
  const size_t part = c.take(std::max(grad_partial_bytes(w.g2, fc2), grad_partial_bytes(w.g1, fc1)));
  w.g2.partA = w.g1.partA = part;
  w.g2.partB = part + grad_part_a(w.g2, fc2);
  w.g1.partB = part + grad_part_a(w.g1, fc1);
  w.rp_part = c.take(rp_part_bytes(M, fc2->N, rank_all(fc2), 0, num_sms));
  w.pj_part = c.take(proj_part_bytes(M, H, rank_all(fc1), num_sms));
  w.total = c.o;
  return w;
}

// ---------------------------------------------------------------- timing hooks
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

// ---------------------------------------------------------------- side stream
// The backward runs dA/dB beside the dX GEMM (independent; both paced per SM,
// so splitting the SMs between them beats running them one after the other).
// One library-owned non-blocking stream per device carries dA/dB: it waits for
// the caller's stream at the fork and the caller's stream waits for it at the
// join, so the call keeps single-stream semantics for the caller.  The enqueue
// of fork .. join is serialised by a lock so that concurrent callers cannot
// interleave their event records.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_side_mu;
int side_stream(SideStream** out) {
  static SideStream ss[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FT_ERR_CUDA;
  if (dev < 0 || dev >= 64) return FT_ERR_UNSUPPORTED;
  SideStream& x = ss[dev];
  if (!x.s) {
    if (cudaStreamCreateWithFlags(&x.s, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&x.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&x.join, cudaEventDisableTiming) != cudaSuccess)
      return FT_ERR_CUDA;
  }
  *out = &x;
  return FT_OK;
}

// ---------------------------------------------------------------- launch helpers
// Fused row pass over X [M, K] bf16: Q(X) -> (codes, scales), L = bf16(X W)
// with W = D [K, R] (w_mn) or W^T [R, K].
int run_rowpass(const void* X, int64_t M, int64_t K, const void* W, int64_t R, bool w_mn, uint8_t* codes, uint8_t* scales, uint8_t* sf_mma, void* L, float* part, int* counters,
                int* status, int num_sms, cudaStream_t s, bool no_quant = false, const uint32_t* amax16 = nullptr) {
  CUtensorMap tmX, tmW;
  if (!map_bf16(&tmX, X, K, M, 128)) return FT_ERR_CUDA;
  if (w_mn ? !map_bf16(&tmW, W, R, K, 64) : !map_bf16(&tmW, W, K, R, static_cast<uint32_t>(R))) return FT_ERR_CUDA;
  const RowSplit rs = row_split(M, K, R, w_mn ? 1 : 0, num_sms, kRowMaxSplit);
  RowpassParams rp{};
  rp.M = static_cast<int>(M);
  rp.K = static_cast<int>(K);
  rp.R = static_cast<int>(R);
  rp.w_mn_major = w_mn ? 1 : 0;
  rp.kt_per_split = rs.kt_per_split;
  rp.nsplit = rs.nsplit;
  rp.stages = rs.stages;
  rp.codes = codes;
  rp.scales = scales;
  rp.sf_mma = sf_mma;
  rp.L = L;
  rp.part = part;
  rp.counters = counters;
  rp.status = status;
  rp.fault_skip_stage = -1;
  rp.no_quant = no_quant ? 1 : 0;
  rp.group16 = amax16 ? 1 : 0;   // 1x16 groups below the per-tensor scale of *amax16
  rp.amax = amax16;
  return cuda_err(ft::launch_rowpass(tmX, tmW, rp, s));
}

// FP4 GEMM.  Forward form: A = Q(act) [M, K], B = layer's R [N, K] with R_sf,
// B2 = U [R2, N] (MN-major).  Transposed form (dX): B = R^T from R_codes_t with
// R_sf_t, B2 = D [N_out, R2] (K-major).  Scales of both operands in the
// MMA-ready layout.
struct GemmArgs {
  int64_t M, N, K, R2;
  const uint8_t* a_codes;
  const uint8_t* a_sf;          // MMA-ready scales of A (rows M, cols K)
  const uint8_t* b_codes;       // R_codes [N, K/2] or R_codes_t [N, K/2] (transposed form)
  const uint8_t* b_sf;          // R_sf or R_sf_t (rows N, cols K)
  bool transposed;
  const void* A2;               // bf16 [M, R2]
  const void* B2;               // U [R2, N] (forward) or D [N, R2] (transposed)
  const void* bias;
  void* out;
  bool out_bf16;
  bool main_bf16;               // 16-bit main product: a_codes = A [M, K], b_codes = B [N, K] bf16
  const uint32_t* amax_a;       // 1x16 groups: the operands' maxima (the product's 2^(eA + eB)), else null
  const uint32_t* amax_b;
};
int run_gemm(const GemmArgs& a, int* status, int num_sms, cudaStream_t s) {
  const uint32_t b_rows = static_cast<uint32_t>(ft::kGemmBN);
  CUtensorMap tmA, tmB, tmA2, tmB2;
  const bool maps_ok = a.main_bf16
                           ? map_bf16(&tmA, a.a_codes, a.K, a.M, 128) && map_bf16(&tmB, a.b_codes, a.K, a.N, b_rows)
                           : map_codes(&tmA, a.a_codes, a.K, a.M, 128) && map_codes(&tmB, a.b_codes, a.K, a.N, b_rows);
  if (!maps_ok) return FT_ERR_CUDA;
  if (a.R2 == 0) {          // no low-rank blocks: the kernel never reads these maps
    tmA2 = tmA;
    tmB2 = tmB;
  } else {
    if (!map_bf16(&tmA2, a.A2, a.R2, a.M, 128)) return FT_ERR_CUDA;
    if (a.transposed ? !map_bf16(&tmB2, a.B2, a.R2, a.N, b_rows) : !map_bf16(&tmB2, a.B2, a.N, a.R2, 64))
      return FT_ERR_CUDA;
  }
  GemmParams gp{};
  gp.M = static_cast<int>(a.M);
  gp.N = static_cast<int>(a.N);
  gp.K = static_cast<int>(a.K);
  gp.R2 = static_cast<int>(a.R2);
  gp.b2_mn_major = a.transposed ? 0 : 1;
  gp.sfa = a.a_sf;
  gp.sfb = a.b_sf;
  gp.bias = a.bias;
  gp.out = a.out;
  gp.ldo = a.N;
  gp.out_bf16 = a.out_bf16 ? 1 : 0;
  gp.status = status;
  gp.main_bf16 = a.main_bf16 ? 1 : 0;
  gp.amax_a = a.amax_a;
  gp.amax_b = a.amax_b;
  return cuda_err(ft::launch_gemm_fp4(tmA, tmB, tmA2, tmB2, gp, num_sms, s));
}

// dA = T_A^T V_A[:, r_s:] ([K, r]) and dB = (L[:, r_s:]^T G) ([r, N]) of one layer, one launch
int run_grads(const ft_linear_t* L, int64_t M, const void* X, const void* P, const void* G, const void* Lsaved,
              float* dA, float* dB, bool accumulate, const GradPair& g, bool side, uint8_t* base, int* status,
              cudaStream_t s, bool x_gelu = false) {
  const MSplit& sa = side ? g.cA : g.sA;
  const MSplit& sb = side ? g.cB : g.sB;
  const int64_t R = rank_all(L);
  CUtensorMap tmTa, tmVa, tmTb, tmVb;
  if (!map_bf16(&tmTa, X, L->K, M, 128) || !map_bf16(&tmVa, P, R, M, 128) || !map_bf16(&tmTb, G, L->N, M, 128) ||
      !map_bf16(&tmVb, Lsaved, R, M, 128))
    return FT_ERR_CUDA;
  TgradParams ta{}, tb{};
  ta.M = tb.M = static_cast<int>(M);
  ta.r = tb.r = static_cast<int>(L->r);
  ta.v0 = tb.v0 = static_cast<int>(L->r_s);
  ta.accumulate = tb.accumulate = accumulate ? 1 : 0;
  ta.status = tb.status = status;
  ta.P = static_cast<int>(L->K);
  ta.t_gelu = x_gelu ? 1 : 0;
  ta.mt_per_split = sa.mt_per_split;
  ta.nsplit = sa.nsplit;
  ta.out = dA;
  ta.out_sp = L->r;
  ta.out_sj = 1;
  ta.part = reinterpret_cast<float*>(base + g.partA);
  ta.counters = reinterpret_cast<int*>(base + g.cntA);
  tb.P = static_cast<int>(L->N);
  tb.mt_per_split = sb.mt_per_split;
  tb.nsplit = sb.nsplit;
  tb.out = dB;
  tb.out_sp = 1;
  tb.out_sj = L->N;
  tb.part = reinterpret_cast<float*>(base + g.partB);
  tb.counters = reinterpret_cast<int*>(base + g.cntB);
  return cuda_err(ft::launch_tgrad2(tmTa, tmVa, ta, tmTb, tmVb, tb, s));
}

// One of the MLP's fused GEMMs (gemm_mlp.cu): the main product as run_gemm, the
// epilogue of `epi`, and the projection T Wp -> proj_out (Wp = D2 [N, RP]
// MN-major for epi 1, U1 [RP, N] K-major for epi 2).
struct MlpGemmArgs {
  GemmArgs g;
  int epi;
  const void* h;
  void* out_h;
  float* dbg;
  uint8_t *q_codes, *q_scales, *q_sf;
  const void* Wp;
  int64_t RP;
  void* proj_out;
  float* part;
};
int run_gemm_mlp(const MlpGemmArgs& m, int* status, int num_sms, cudaStream_t s) {
  const GemmArgs& a = m.g;
  CUtensorMap tmA, tmB, tmA2, tmB2, tmW;
  if (!map_codes(&tmA, a.a_codes, a.K, a.M, 128) || !map_codes(&tmB, a.b_codes, a.K, a.N, ft::kGemmBN) ||
      !map_bf16(&tmA2, a.A2, a.R2, a.M, 128))
    return FT_ERR_CUDA;
  if (a.transposed ? !map_bf16(&tmB2, a.B2, a.R2, a.N, ft::kGemmBN) : !map_bf16(&tmB2, a.B2, a.N, a.R2, 64))
    return FT_ERR_CUDA;
  const bool wmn = m.epi == 1;
  if (wmn ? !map_bf16(&tmW, m.Wp, m.RP, a.N, 64) : !map_bf16(&tmW, m.Wp, a.N, m.RP, static_cast<uint32_t>(m.RP)))
    return FT_ERR_CUDA;
  const MlpUnits un = plan_units(a.M, a.N, num_sms);
  ft::MlpGemmParams mp{};
  mp.g.M = static_cast<int>(a.M);
  mp.g.N = static_cast<int>(a.N);
  mp.g.K = static_cast<int>(a.K);
  mp.g.R2 = static_cast<int>(a.R2);
  mp.g.b2_mn_major = a.transposed ? 0 : 1;
  mp.g.sfa = a.a_sf;
  mp.g.sfb = a.b_sf;
  mp.g.bias = a.bias;
  mp.g.out_bf16 = 1;
  mp.g.status = status;
  mp.epi = m.epi;
  mp.h = m.h;
  mp.out_h = m.out_h;
  mp.dbg = m.dbg;
  mp.q_codes = m.q_codes;
  mp.q_scales = m.q_scales;
  mp.q_sf = m.q_sf;
  mp.RP = static_cast<int>(m.RP);
  mp.wp_mn_major = wmn ? 1 : 0;
  mp.nsplit = un.nsplit;
  mp.per = un.per;
  mp.part = m.part;
  return cuda_err(ft::launch_gemm_mlp(tmA, tmB, tmA2, tmB2, tmW, mp, num_sms, s));
}
// the split-order sum of the fused GEMM's fp32 projection partials -> bf16 proj_out
int run_proj_reduce(const MlpGemmArgs& m, int num_sms, cudaStream_t s) {
  const MlpUnits un = plan_units(m.g.M, m.g.N, num_sms);
  return cuda_err(ft::launch_proj_reduce(m.part, un.nsplit, static_cast<int>(m.g.M), static_cast<int>(m.RP),
                                         m.proj_out, num_sms, s));
}

#define FT_TRY(k, expr)                                          \
  do {                                                           \
    if (evs.mark((k), 0, s) != cudaSuccess) return FT_ERR_CUDA;  \
    const int rc_ = (expr);                                      \
    if (rc_ != FT_OK) return rc_;                                \
    if (evs.mark((k), 1, s) != cudaSuccess) return FT_ERR_CUDA;  \
  } while (0)

// The dX GEMM on the caller's stream, on all but gp.side_sms SMs, and dA/dB
// beside it on the side stream (fork before, join after: see SideStream).  The
// GEMM is launched first so that its persistent CTAs take their SMs as the
// previous kernel leaves them; dA/dB fill the rest.
int gemm_and_grads_side(const GemmArgs& g, const ft_linear_t* L, int64_t M, const void* X, const void* P,
                        const void* G, const void* Lsaved, float* dA, float* dB, bool accumulate, const GradPair& gp,
                        uint8_t* base, int* status, int num_sms, cudaStream_t s) {
  std::lock_guard<std::mutex> lock(g_side_mu);
  SideStream* ss = nullptr;
  int st = side_stream(&ss);
  if (st) return st;
  if (cudaEventRecord(ss->fork, s) != cudaSuccess) return FT_ERR_CUDA;
  if ((st = run_gemm(g, status, num_sms - gp.side_sms, s))) return st;
  if (cudaStreamWaitEvent(ss->s, ss->fork, 0) != cudaSuccess) return FT_ERR_CUDA;
  if ((st = run_grads(L, M, X, P, G, Lsaved, dA, dB, accumulate, gp, true, base, status, ss->s))) return st;
  if (cudaEventRecord(ss->join, ss->s) != cudaSuccess || cudaStreamWaitEvent(s, ss->join, 0) != cudaSuccess)
    return FT_ERR_CUDA;
  return FT_OK;
}

size_t kmajor_rowpass_scratch(int64_t M, int64_t K, int64_t R, int num_sms, size_t* header) {
  const RowSplit rs = row_split(M, K, R, 0, num_sms, kRowMaxSplit);
  *header = up256(16 + 4 * static_cast<size_t>(cdiv(M, 128)));
  return *header + (rs.nsplit > 1 ? static_cast<size_t>(rs.nsplit) * M * R * 4 : 0);
}
int check_quant_down(const ft_bf16* X, int64_t M, int64_t K, const ft_bf16* W, int64_t R, uint8_t* codes,
                     uint8_t* scales, ft_bf16* L) {
  if (!X || !W || !codes || !scales || !L) return FT_ERR_INVALID_ARG;
  if (M <= 0 || K <= 0 || M % 16 || K % 32) return FT_ERR_SHAPE;
  if (R < 16 || R % 16 || R > 128 || M > (1 << 30) || K > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(X) || !al16(W) || !al16(codes) || !al16(L)) return FT_ERR_ALIGN;
  return FT_OK;
}
int launch_kmajor_rowpass(const ft_bf16* X, int64_t M, int64_t K, const ft_bf16* W, int64_t R, uint8_t* codes,
                          uint8_t* scales, ft_bf16* L, uint8_t* base, size_t header, int num_sms, int fault_skip_stage,
                          unsigned long long wait_ns, cudaStream_t s) {
  const RowSplit rs = row_split(M, K, R, 0, num_sms, kRowMaxSplit);
  // status word and split counters must start at zero
  if (ft::launch_clear_words(base, header, s) != cudaSuccess) return FT_ERR_CUDA;
  CUtensorMap tmX, tmW;
  if (!map_bf16(&tmX, X, K, M, 128) || !map_bf16(&tmW, W, K, R, static_cast<uint32_t>(R))) return FT_ERR_CUDA;
  RowpassParams rp{};
  rp.M = static_cast<int>(M);
  rp.K = static_cast<int>(K);
  rp.R = static_cast<int>(R);
  rp.w_mn_major = 0;
  rp.kt_per_split = rs.kt_per_split;
  rp.nsplit = rs.nsplit;
  rp.stages = rs.stages;
  rp.codes = codes;
  rp.scales = scales;
  rp.L = L;
  rp.part = reinterpret_cast<float*>(base + header);
  rp.counters = reinterpret_cast<int*>(base + 16);
  rp.status = reinterpret_cast<int*>(base);
  rp.wait_ns = wait_ns;
  rp.fault_skip_stage = fault_skip_stage;
  return cuda_err(ft::launch_rowpass(tmX, tmW, rp, s));
}
int read_status_word(const void* dev_word, cudaStream_t s) {
  int h = 0;
  if (cudaMemcpyAsync(&h, dev_word, sizeof(int), cudaMemcpyDeviceToHost, s) != cudaSuccess) return FT_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return FT_ERR_CUDA;
  return h == 0 ? FT_OK : h == 2 ? FT_ERR_UNSUPPORTED : FT_ERR_TIMEOUT;
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
  FT_RANGE("fourtune_quantize_block16");
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

int fourtune_quantize_block16_f32(const float* x, int64_t rows, int64_t cols, int64_t ld, uint8_t* codes,
                                  uint8_t* scales, void* stream) {
  FT_RANGE("fourtune_quantize_block16_f32");
  if (!x || !codes || !scales) return FT_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16 || ld < cols || ld % 4) return FT_ERR_SHAPE;
  if (rows > (1 << 30) || cols > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(x) || (reinterpret_cast<uintptr_t>(codes) & 7u)) return FT_ERR_ALIGN;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  return cuda_err(ft::launch_quantize_block16_f32(x, static_cast<int>(rows), static_cast<int>(cols), ld, codes, scales,
                                                  static_cast<cudaStream_t>(stream)));
}

int fourtune_transpose_codes(const uint8_t* codes, int64_t rows, int64_t cols, uint8_t* codes_t, void* stream) {
  FT_RANGE("fourtune_transpose_codes");
  if (!codes || !codes_t) return FT_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16) return FT_ERR_SHAPE;
  if (rows > (1 << 30) || cols > (1 << 30)) return FT_ERR_UNSUPPORTED;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  return cuda_err(ft::launch_transpose_codes(codes, static_cast<int>(rows), static_cast<int>(cols), codes_t,
                                             static_cast<cudaStream_t>(stream)));
}

size_t fourtune_mma_scales_size(int64_t rows, int64_t cols) {
  FT_RANGE("fourtune_mma_scales_size");
  if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16 || rows > (1 << 30) || cols > (1 << 30)) return 0;
  return ft::sf_mma_bytes(rows, cols);
}

int fourtune_mma_scales(const uint8_t* scales, int64_t rows, int64_t cols, int transposed, uint8_t* out,
                        void* stream) {
  FT_RANGE("fourtune_mma_scales");
  if (!scales || !out || (transposed != 0 && transposed != 1)) return FT_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16) return FT_ERR_SHAPE;
  if (rows > (1 << 30) || cols > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(out)) return FT_ERR_ALIGN;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  return cuda_err(ft::launch_sf_mma(scales, static_cast<int>(rows), static_cast<int>(cols), transposed, out,
                                    static_cast<cudaStream_t>(stream)));
}

// ---------------------------------------------------------------- linear
size_t fourtune_linear_fwd_workspace_size(const ft_linear_t* layer, int64_t M) {
  FT_RANGE("fourtune_linear_fwd_workspace_size");
  if (check_layer(layer, false) || M <= 0 || M % 16) return 0;
  return fwd_layout(layer, M, num_sms_or_default()).total;
}

size_t fourtune_linear_bwd_workspace_size(const ft_linear_t* layer, int64_t M) {
  FT_RANGE("fourtune_linear_bwd_workspace_size");
  if (check_layer(layer, true) || M <= 0 || M % 16) return 0;
  return bwd_layout(layer, M, num_sms_or_default()).total;
}

int fourtune_linear_fwd_ws_offsets(const ft_linear_t* layer, int64_t M, size_t* codes_off, size_t* scales_off) {
  FT_RANGE("fourtune_linear_fwd_ws_offsets");
  int st = check_layer(layer, false);
  if (st) return st;
  const FwdWs w = fwd_layout(layer, M, num_sms_or_default());
  if (codes_off) *codes_off = w.qx.codes;
  if (scales_off) *scales_off = w.qx.scales;
  return FT_OK;
}

int fourtune_linear_bwd_ws_offsets(const ft_linear_t* layer, int64_t M, size_t* codes_off, size_t* scales_off,
                                   size_t* P_off) {
  FT_RANGE("fourtune_linear_bwd_ws_offsets");
  int st = check_layer(layer, true);
  if (st) return st;
  const BwdWs w = bwd_layout(layer, M, num_sms_or_default());
  if (codes_off) *codes_off = w.qg.codes;
  if (scales_off) *scales_off = w.qg.scales;
  if (P_off) *P_off = w.P;
  return FT_OK;
}

int fourtune_linear_fwd(const ft_linear_t* layer, const ft_bf16* X, int64_t M, void* Y, int y_dtype,
                        ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream) {
  FT_RANGE("fourtune_linear_fwd");
  return fourtune_linear_fwd_timed(layer, X, M, Y, y_dtype, L_saved, ws, ws_bytes, stream, nullptr, 0);
}

int fourtune_linear_fwd_timed(const ft_linear_t* layer, const ft_bf16* X, int64_t M, void* Y, int y_dtype,
                              ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream, void* const* events,
                              int n_events) {
  FT_RANGE("fourtune_linear_fwd_timed");
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
  int* status = reinterpret_cast<int*>(base);
  if (ft::launch_clear_words(base, w.header, s) != cudaSuccess) return FT_ERR_CUDA;
  const int64_t K = layer->K, N = layer->N, R = rank_all(layer);
  uint8_t* qc = base + w.qx.codes;
  uint8_t* qs = base + w.qx.scales;
  uint8_t* qf = base + w.qx.sf;
  // X pass: Q(X) and L = bf16(X D)
  FT_TRY(0, run_rowpass(X, M, K, layer->D, R, true, qc, qs, qf, L_saved,
                        reinterpret_cast<float*>(base + w.rp_part), reinterpret_cast<int*>(base + w.rp_cnt), status,
                        di.num_sms, s));
  // 4-bit GEMM + L U + bias
  GemmArgs g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.R2 = R;
  g.a_codes = qc;
  g.a_sf = qf;
  g.b_codes = layer->R_codes;
  g.b_sf = layer->R_sf;
  g.transposed = false;
  g.A2 = L_saved;
  g.B2 = layer->U;
  g.bias = layer->bias;
  g.out = Y;
  g.out_bf16 = y_dtype == FT_DTYPE_BF16;
  FT_TRY(1, run_gemm(g, status, di.num_sms, s));
  return FT_OK;
}

int fourtune_linear_bwd(const ft_linear_t* layer, const ft_bf16* dY, const ft_bf16* X, const ft_bf16* L_saved,
                        int64_t M, void* dX, int dx_dtype, float* dA, float* dB, int accumulate, void* ws,
                        size_t ws_bytes, void* stream) {
  FT_RANGE("fourtune_linear_bwd");
  return fourtune_linear_bwd_timed(layer, dY, X, L_saved, M, dX, dx_dtype, dA, dB, accumulate, ws, ws_bytes, stream,
                                   nullptr, 0);
}

int fourtune_linear_bwd_timed(const ft_linear_t* layer, const ft_bf16* dY, const ft_bf16* X,
                              const ft_bf16* L_saved, int64_t M, void* dX, int dx_dtype, float* dA, float* dB,
                              int accumulate, void* ws, size_t ws_bytes, void* stream, void* const* events,
                              int n_events) {
  FT_RANGE("fourtune_linear_bwd_timed");
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
  int* status = reinterpret_cast<int*>(base);
  if (ft::launch_clear_words(base, w.header, s) != cudaSuccess) return FT_ERR_CUDA;
  const int64_t K = layer->K, N = layer->N, R = rank_all(layer);
  uint8_t* gc = base + w.qg.codes;
  uint8_t* gs = base + w.qg.scales;
  uint8_t* gf = base + w.qg.sf;
  void* P = base + w.P;
  // G pass: Q(G) and P = bf16(G U^T), U [R, N] read K-major
  FT_TRY(0, run_rowpass(dY, M, N, layer->U, R, false, gc, gs, gf, P,
                        reinterpret_cast<float*>(base + w.rp_part), reinterpret_cast<int*>(base + w.rp_cnt), status,
                        di.num_sms, s));
  // dX = deq(Q(G)) deq(Q(R)) + P D^T, and dA = X^T P[:, r_s:], dB = L[:, r_s:]^T G
  GemmArgs g{};
  g.M = M;
  g.N = K;
  g.K = N;
  g.R2 = R;
  g.a_codes = gc;
  g.a_sf = gf;
  g.b_codes = layer->R_codes_t;
  g.b_sf = layer->R_sf_t;
  g.transposed = true;
  g.A2 = P;
  g.B2 = layer->D;
  g.out = dX;
  g.out_bf16 = dx_dtype == FT_DTYPE_BF16;
  if (evs.ev || w.g.side_sms == 0) {
    // timed (or a small part): one after the other (dA/dB first, while G is
    // still in L2), so that every kernel has its own event pair
    FT_TRY(1, run_grads(layer, M, X, P, dY, L_saved, dA, dB, accumulate != 0, w.g, false, base, status, s));
    FT_TRY(2, run_gemm(g, status, di.num_sms, s));
  } else {
    st = gemm_and_grads_side(g, layer, M, X, P, dY, L_saved, dA, dB, accumulate != 0, w.g, base, status,
                             di.num_sms, s);
    if (st) return st;
  }
  return FT_OK;
}

// ---------------------------------------------------------------- 1x16 groups
namespace {
int check_layer_1x16(const ft_linear_1x16_t* L) {
  if (!L || !L->R_codes || !L->R_sf || !L->Rt_codes || !L->Rt_sf || !L->R_amax || !L->D || !L->U)
    return FT_ERR_INVALID_ARG;
  if (L->K <= 0 || L->N <= 0 || L->K % 32 || L->N % 32) return FT_ERR_SHAPE;
  if (L->r_s < 0 || L->r < 16 || L->r_s % 16 || L->r % 16 || L->r > 64 || L->r_s + L->r > 128)
    return FT_ERR_UNSUPPORTED;
  if (L->K > (1 << 30) || L->N > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(L->R_codes) || !al16(L->R_sf) || !al16(L->Rt_codes) || !al16(L->Rt_sf) || !al16(L->D) ||
      !al16(L->U) || (L->bias && !al16(L->bias)) || (reinterpret_cast<uintptr_t>(L->R_amax) & 3u))
    return FT_ERR_ALIGN;
  return FT_OK;
}
// the shapes and low-rank factors, for the helpers shared with the block layout
ft_linear_t view_1x16(const ft_linear_1x16_t* L) {
  ft_linear_t v{};
  v.K = L->K;
  v.N = L->N;
  v.r_s = L->r_s;
  v.r = L->r;
  v.D = L->D;
  v.U = L->U;
  v.bias = L->bias;
  return v;
}
// 1x16 activations of a [M, C] matrix: codes, compact scales [M, C/16], MMA-ready scales
struct Q1x16 {
  size_t codes, scales, sf;
  void carve(Carver& c, int64_t M, int64_t C) {
    codes = c.take(static_cast<size_t>(M * C / 2));
    scales = c.take(static_cast<size_t>(M * (C / 16)));
    sf = c.take(ft::sf_mma_bytes(M, C));
  }
};
// header: status (byte 0), the tensor's maximum word (byte 8), split counters from 16
constexpr size_t kAmaxWord = 8;
// forward: header | Q16(X) | row-pass partials | U rescaled
struct Fwd1x16Ws {
  size_t header, rp_cnt, rp_part, Us, total;
  Q1x16 qx;
};
Fwd1x16Ws fwd_1x16_layout(const ft_linear_t* L, int64_t M, int num_sms) {
  Fwd1x16Ws w{};
  Carver c;
  w.rp_cnt = 16;
  c.take(w.header = up256(16 + 4 * static_cast<size_t>(cdiv(M, 128))));
  w.qx.carve(c, M, L->K);
  w.rp_part = c.take(rp_part_bytes(M, L->K, rank_all(L), 1, num_sms));
  w.Us = c.take(static_cast<size_t>(rank_all(L) * L->N * 2));
  w.total = c.o;
  return w;
}
// backward: header (status, maximum, dA/dB and row-pass counters) | Q16(G) | P |
// dA/dB partials | row-pass partials | D rescaled
struct Bwd1x16Ws {
  size_t header, P, rp_cnt, rp_part, Ds, total;
  Q1x16 qg;
  GradPair g;
};
Bwd1x16Ws bwd_1x16_layout(const ft_linear_t* L, int64_t M, int num_sms) {
  Bwd1x16Ws w{};
  plan_grads(w.g, L, M, num_sms);
  Carver c;
  w.g.cntA = 16;
  w.g.cntB = w.g.cntA + 4 * static_cast<size_t>(cdiv(L->K, 128));
  w.rp_cnt = 16 + 4 * grad_counter_words(L);
  c.take(w.header = up256(w.rp_cnt + 4 * static_cast<size_t>(cdiv(M, 128))));
  w.qg.carve(c, M, L->N);
  w.P = c.take(static_cast<size_t>(M * rank_all(L) * 2));
  w.g.partA = c.take(grad_partial_bytes(w.g, L));
  w.g.partB = w.g.partA + grad_part_a(w.g, L);
  w.rp_part = c.take(rp_part_bytes(M, L->N, rank_all(L), 0, num_sms));
  w.Ds = c.take(static_cast<size_t>(L->K * rank_all(L) * 2));
  w.total = c.o;
  return w;
}
}  // namespace

int fourtune_quantize_1x16(const ft_bf16* W, int64_t rows, int64_t cols, int transposed, uint32_t* amax_word,
                           uint8_t* codes, uint8_t* scales, uint8_t* sf_mma, void* stream) {
  FT_RANGE("fourtune_quantize_1x16");
  if (!W || !amax_word || !codes || !scales || (transposed != 0 && transposed != 1)) return FT_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows % 32 || cols % 32) return FT_ERR_SHAPE;
  if (rows > (1 << 30) || cols > (1 << 30) || rows * cols > (1LL << 40)) return FT_ERR_UNSUPPORTED;
  if (!al16(W) || !al16(codes) || !al16(amax_word) || (sf_mma && !al16(sf_mma))) return FT_ERR_ALIGN;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t orows = transposed ? cols : rows, ocols = transposed ? rows : cols;
  // the maximum word (16 bytes cleared) and the MMA-ready padding start at zero
  if (ft::launch_clear_words(amax_word, 16, s) != cudaSuccess) return FT_ERR_CUDA;
  if (sf_mma && ft::launch_clear_words(sf_mma, ft::sf_mma_bytes(orows, ocols), s) != cudaSuccess) return FT_ERR_CUDA;
  if (ft::launch_tensor_amax(W, rows * cols, amax_word, di.num_sms, s) != cudaSuccess) return FT_ERR_CUDA;
  return cuda_err(ft::launch_quantize_group16(W, static_cast<int>(rows), static_cast<int>(cols), transposed, amax_word,
                                             codes, scales, sf_mma, s));
}

size_t fourtune_linear_fwd_1x16_workspace_size(const ft_linear_1x16_t* layer, int64_t M) {
  FT_RANGE("fourtune_linear_fwd_1x16_workspace_size");
  if (check_layer_1x16(layer) || M <= 0 || M % 16) return 0;
  const ft_linear_t v = view_1x16(layer);
  return fwd_1x16_layout(&v, M, num_sms_or_default()).total;
}

size_t fourtune_linear_bwd_1x16_workspace_size(const ft_linear_1x16_t* layer, int64_t M) {
  FT_RANGE("fourtune_linear_bwd_1x16_workspace_size");
  if (check_layer_1x16(layer) || M <= 0 || M % 16) return 0;
  const ft_linear_t v = view_1x16(layer);
  return bwd_1x16_layout(&v, M, num_sms_or_default()).total;
}

int fourtune_linear_1x16_ws_offsets(const ft_linear_1x16_t* layer, int64_t M, int backward, size_t* codes_off,
                                    size_t* scales_off, size_t* amax_off, size_t* P_off) {
  FT_RANGE("fourtune_linear_1x16_ws_offsets");
  int st = check_layer_1x16(layer);
  if (st) return st;
  if (M <= 0 || M % 16) return FT_ERR_SHAPE;
  const ft_linear_t v = view_1x16(layer);
  if (backward) {
    const Bwd1x16Ws w = bwd_1x16_layout(&v, M, num_sms_or_default());
    if (codes_off) *codes_off = w.qg.codes;
    if (scales_off) *scales_off = w.qg.scales;
    if (P_off) *P_off = w.P;
  } else {
    const Fwd1x16Ws w = fwd_1x16_layout(&v, M, num_sms_or_default());
    if (codes_off) *codes_off = w.qx.codes;
    if (scales_off) *scales_off = w.qx.scales;
    if (P_off) *P_off = 0;
  }
  if (amax_off) *amax_off = kAmaxWord;
  return FT_OK;
}

int fourtune_linear_fwd_1x16(const ft_linear_1x16_t* layer, const ft_bf16* X, int64_t M, void* Y, int y_dtype,
                             ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream) {
  FT_RANGE("fourtune_linear_fwd_1x16");
  return fourtune_linear_fwd_1x16_timed(layer, X, M, Y, y_dtype, L_saved, ws, ws_bytes, stream, nullptr, 0);
}

int fourtune_linear_fwd_1x16_timed(const ft_linear_1x16_t* layer, const ft_bf16* X, int64_t M, void* Y, int y_dtype,
                                   ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream, void* const* events,
                                   int n_events) {
  FT_RANGE("fourtune_linear_fwd_1x16_timed");
  const Events evs{events, n_events};
  int st = check_layer_1x16(layer);
  if (st) return st;
  if (!X || !Y || !L_saved || !ws) return FT_ERR_INVALID_ARG;
  if (y_dtype != FT_DTYPE_F32 && y_dtype != FT_DTYPE_BF16) return FT_ERR_INVALID_ARG;
  if (M <= 0 || M % 16) return FT_ERR_SHAPE;
  if (M > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(X) || !al16(Y) || !al16(L_saved) || (reinterpret_cast<uintptr_t>(ws) & 255u)) return FT_ERR_ALIGN;
  DevInfo di;
  if ((st = device_info(&di))) return st;
  const ft_linear_t v = view_1x16(layer);
  const Fwd1x16Ws w = fwd_1x16_layout(&v, M, di.num_sms);
  if (ws_bytes < w.total) return FT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(base);
  uint32_t* amax = reinterpret_cast<uint32_t*>(base + kAmaxWord);
  if (ft::launch_clear_words(base, w.header, s) != cudaSuccess) return FT_ERR_CUDA;
  const int64_t K = layer->K, N = layer->N, R = rank_all(&v);
  uint8_t* qc = base + w.qx.codes;
  uint8_t* qf = base + w.qx.sf;
  void* Us = base + w.Us;
  FT_TRY(0, cuda_err(ft::launch_tensor_amax(X, M * K, amax, di.num_sms, s)));
  // X pass: Q16(X) (below 2^e of max|X|) and L = bf16(X D)
  FT_TRY(1, run_rowpass(X, M, K, layer->D, R, true, qc, base + w.qx.scales, qf, L_saved,
                        reinterpret_cast<float*>(base + w.rp_part), reinterpret_cast<int*>(base + w.rp_cnt), status,
                        di.num_sms, s, false, amax));
  // U rescaled by 2^-(eX + eR): it shares the accumulator the epilogue scales by 2^(eX + eR)
  FT_TRY(2, cuda_err(ft::launch_scale_pow2(layer->U, Us, R * N, amax, layer->R_amax, di.num_sms, s)));
  GemmArgs g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.R2 = R;
  g.a_codes = qc;
  g.a_sf = qf;
  g.b_codes = layer->R_codes;
  g.b_sf = layer->R_sf;
  g.transposed = false;
  g.A2 = L_saved;
  g.B2 = Us;
  g.bias = layer->bias;
  g.out = Y;
  g.out_bf16 = y_dtype == FT_DTYPE_BF16;
  g.amax_a = amax;
  g.amax_b = layer->R_amax;
  FT_TRY(3, run_gemm(g, status, di.num_sms, s));
  return FT_OK;
}

int fourtune_linear_bwd_1x16(const ft_linear_1x16_t* layer, const ft_bf16* dY, const ft_bf16* X,
                             const ft_bf16* L_saved, int64_t M, void* dX, int dx_dtype, float* dA, float* dB,
                             int accumulate, void* ws, size_t ws_bytes, void* stream) {
  FT_RANGE("fourtune_linear_bwd_1x16");
  return fourtune_linear_bwd_1x16_timed(layer, dY, X, L_saved, M, dX, dx_dtype, dA, dB, accumulate, ws, ws_bytes,
                                        stream, nullptr, 0);
}

int fourtune_linear_bwd_1x16_timed(const ft_linear_1x16_t* layer, const ft_bf16* dY, const ft_bf16* X,
                                   const ft_bf16* L_saved, int64_t M, void* dX, int dx_dtype, float* dA, float* dB,
                                   int accumulate, void* ws, size_t ws_bytes, void* stream, void* const* events,
                                   int n_events) {
  FT_RANGE("fourtune_linear_bwd_1x16_timed");
  const Events evs{events, n_events};
  int st = check_layer_1x16(layer);
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
  const ft_linear_t v = view_1x16(layer);
  const Bwd1x16Ws w = bwd_1x16_layout(&v, M, di.num_sms);
  if (ws_bytes < w.total) return FT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(base);
  uint32_t* amax = reinterpret_cast<uint32_t*>(base + kAmaxWord);
  if (ft::launch_clear_words(base, w.header, s) != cudaSuccess) return FT_ERR_CUDA;
  const int64_t K = layer->K, N = layer->N, R = rank_all(&v);
  uint8_t* gc = base + w.qg.codes;
  uint8_t* gf = base + w.qg.sf;
  void* P = base + w.P;
  void* Ds = base + w.Ds;
  FT_TRY(0, cuda_err(ft::launch_tensor_amax(dY, M * N, amax, di.num_sms, s)));
  // G pass: Q16(G) and P = bf16(G U^T), U [R, N] read K-major
  FT_TRY(1, run_rowpass(dY, M, N, layer->U, R, false, gc, base + w.qg.scales, gf, P,
                        reinterpret_cast<float*>(base + w.rp_part), reinterpret_cast<int*>(base + w.rp_cnt), status,
                        di.num_sms, s, false, amax));
  FT_TRY(2, cuda_err(ft::launch_scale_pow2(layer->D, Ds, K * R, amax, layer->R_amax, di.num_sms, s)));
  // dX = deq(Q16(G)) deq(Q16(R^T))^T + P D^T: B is Q16(R^T) [K, N], B2 = D rescaled
  GemmArgs g{};
  g.M = M;
  g.N = K;
  g.K = N;
  g.R2 = R;
  g.a_codes = gc;
  g.a_sf = gf;
  g.b_codes = layer->Rt_codes;
  g.b_sf = layer->Rt_sf;
  g.transposed = true;
  g.A2 = P;
  g.B2 = Ds;
  g.out = dX;
  g.out_bf16 = dx_dtype == FT_DTYPE_BF16;
  g.amax_a = amax;
  g.amax_b = layer->R_amax;
  if (evs.ev || w.g.side_sms == 0) {
    FT_TRY(3, run_grads(&v, M, X, P, dY, L_saved, dA, dB, accumulate != 0, w.g, false, base, status, s));
    FT_TRY(4, run_gemm(g, status, di.num_sms, s));
  } else {
    st = gemm_and_grads_side(g, &v, M, X, P, dY, L_saved, dA, dB, accumulate != 0, w.g, base, status, di.num_sms,
                             s);
    if (st) return st;
  }
  return FT_OK;
}

// ---------------------------------------------------------------- 16-bit precision variants
namespace {
// the layer fields the 16-bit variants use (the low-rank factors; no 4-bit weight)
int check_layer16(const ft_linear_t* L) {
  if (!L || !L->D || !L->U) return FT_ERR_INVALID_ARG;
  if (L->K <= 0 || L->N <= 0 || L->K % 32 || L->N % 32) return FT_ERR_SHAPE;
  if (L->r_s < 0 || L->r < 16 || L->r_s % 16 || L->r % 16 || L->r > 64 || L->r_s + L->r > 128)
    return FT_ERR_UNSUPPORTED;
  if (L->K > (1 << 30) || L->N > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(L->D) || !al16(L->U) || (L->bias && !al16(L->bias))) return FT_ERR_ALIGN;
  return FT_OK;
}
}  // namespace

int fourtune_stabilizer_residual(const ft_bf16* W, int64_t N, int64_t K, const ft_bf16* S_dn, const ft_bf16* S_up,
                                 int64_t r_s, ft_bf16* R, void* stream) {
  FT_RANGE("fourtune_stabilizer_residual");
  if (!W || !S_dn || !S_up || !R) return FT_ERR_INVALID_ARG;
  if (N <= 0 || K <= 0) return FT_ERR_SHAPE;
  if (r_s < 1 || r_s > 128 || N > (1 << 30) || K > (1 << 30)) return FT_ERR_UNSUPPORTED;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  return cuda_err(ft::launch_stabilizer_residual(W, static_cast<int>(N), static_cast<int>(K), S_dn, S_up,
                                                 static_cast<int>(r_s), R, static_cast<cudaStream_t>(stream)));
}

int fourtune_gemm_block16(const uint8_t* A_codes, const uint8_t* A_sf, const uint8_t* B_codes, const uint8_t* B_sf,
                          int64_t M, int64_t N, int64_t K, const ft_bf16* bias, void* out, int out_dtype, void* ws,
                          size_t ws_bytes, void* stream) {
  FT_RANGE("fourtune_gemm_block16");
  if (!A_codes || !A_sf || !B_codes || !B_sf || !out || !ws) return FT_ERR_INVALID_ARG;
  if (out_dtype != FT_DTYPE_F32 && out_dtype != FT_DTYPE_BF16) return FT_ERR_INVALID_ARG;
  if (M <= 0 || N <= 0 || K <= 0 || M % 16 || N % 32 || K % 32) return FT_ERR_SHAPE;
  if (M > (1 << 30) || N > (1 << 30) || K > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(A_codes) || !al16(A_sf) || !al16(B_codes) || !al16(B_sf) || !al16(out) || (bias && !al16(bias)) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return FT_ERR_ALIGN;
  if (ws_bytes < 256) return FT_ERR_WORKSPACE;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (ft::launch_clear_words(ws, 256, s) != cudaSuccess) return FT_ERR_CUDA;
  GemmArgs g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.R2 = 0;
  g.a_codes = A_codes;
  g.a_sf = A_sf;
  g.b_codes = B_codes;
  g.b_sf = B_sf;
  g.bias = bias;
  g.out = out;
  g.out_bf16 = out_dtype == FT_DTYPE_BF16;
  return run_gemm(g, static_cast<int*>(ws), di.num_sms, s);
}

size_t fourtune_linear_fwd_a16_workspace_size(const ft_linear_t* layer, int64_t M) {
  FT_RANGE("fourtune_linear_fwd_a16_workspace_size");
  if (check_layer16(layer) || M <= 0 || M % 16) return 0;
  return fwd_layout(layer, M, num_sms_or_default()).total;
}

size_t fourtune_linear_bwd_g16_workspace_size(const ft_linear_t* layer, int64_t M) {
  FT_RANGE("fourtune_linear_bwd_g16_workspace_size");
  if (check_layer16(layer) || M <= 0 || M % 16) return 0;
  return bwd_layout(layer, M, num_sms_or_default()).total;
}

int fourtune_dequantize_block16(const uint8_t* codes, const uint8_t* scales, int64_t rows, int64_t cols,
                                int transposed, ft_bf16* out, void* stream) {
  FT_RANGE("fourtune_dequantize_block16");
  if (!codes || !scales || !out || (transposed != 0 && transposed != 1)) return FT_ERR_INVALID_ARG;
  if (rows <= 0 || cols <= 0 || rows % 16 || cols % 16) return FT_ERR_SHAPE;
  if (rows > (1 << 30) || cols > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (reinterpret_cast<uintptr_t>(out) & 3u) return FT_ERR_ALIGN;
  DevInfo di;
  int st = device_info(&di);
  if (st) return st;
  return cuda_err(ft::launch_dequantize_block16(codes, scales, static_cast<int>(rows), static_cast<int>(cols),
                                                transposed, out, static_cast<cudaStream_t>(stream)));
}

int fourtune_linear_fwd_a16(const ft_linear_t* layer, const ft_bf16* W16, const ft_bf16* X, int64_t M, void* Y,
                            int y_dtype, ft_bf16* L_saved, void* ws, size_t ws_bytes, void* stream) {
  FT_RANGE("fourtune_linear_fwd_a16");
  int st = check_layer16(layer);
  if (st) return st;
  if (!W16 || !X || !Y || !L_saved || !ws) return FT_ERR_INVALID_ARG;
  if (y_dtype != FT_DTYPE_F32 && y_dtype != FT_DTYPE_BF16) return FT_ERR_INVALID_ARG;
  if (M <= 0 || M % 16) return FT_ERR_SHAPE;
  if (M > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(W16) || !al16(X) || !al16(Y) || !al16(L_saved) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return FT_ERR_ALIGN;
  DevInfo di;
  if ((st = device_info(&di))) return st;
  const FwdWs w = fwd_layout(layer, M, di.num_sms);
  if (ws_bytes < w.total) return FT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(base);
  if (ft::launch_clear_words(base, w.header, s) != cudaSuccess) return FT_ERR_CUDA;
  const int64_t K = layer->K, N = layer->N, R = rank_all(layer);
  // L = bf16(X D) only (the activation is not quantized)
  st = run_rowpass(X, M, K, layer->D, R, true, nullptr, nullptr, nullptr, L_saved,
                   reinterpret_cast<float*>(base + w.rp_part), reinterpret_cast<int*>(base + w.rp_cnt), status,
                   di.num_sms, s, true);
  if (st) return st;
  GemmArgs g{};
  g.M = M;
  g.N = N;
  g.K = K;
  g.R2 = R;
  g.a_codes = reinterpret_cast<const uint8_t*>(X);
  g.b_codes = reinterpret_cast<const uint8_t*>(W16);
  g.main_bf16 = true;
  g.transposed = false;
  g.A2 = L_saved;
  g.B2 = layer->U;
  g.bias = layer->bias;
  g.out = Y;
  g.out_bf16 = y_dtype == FT_DTYPE_BF16;
  return run_gemm(g, status, di.num_sms, s);
}

int fourtune_linear_bwd_g16(const ft_linear_t* layer, const ft_bf16* W16_t, const ft_bf16* dY, const ft_bf16* X,
                            const ft_bf16* L_saved, int64_t M, void* dX, int dx_dtype, float* dA, float* dB,
                            int accumulate, void* ws, size_t ws_bytes, void* stream) {
  FT_RANGE("fourtune_linear_bwd_g16");
  int st = check_layer16(layer);
  if (st) return st;
  if (!W16_t || !dY || !X || !L_saved || !dX || !dA || !dB || !ws) return FT_ERR_INVALID_ARG;
  if (dx_dtype != FT_DTYPE_F32 && dx_dtype != FT_DTYPE_BF16) return FT_ERR_INVALID_ARG;
  if (M <= 0 || M % 16) return FT_ERR_SHAPE;
  if (M > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(W16_t) || !al16(dY) || !al16(X) || !al16(L_saved) || !al16(dX) || !al16(dA) || !al16(dB) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return FT_ERR_ALIGN;
  DevInfo di;
  if ((st = device_info(&di))) return st;
  const BwdWs w = bwd_layout(layer, M, di.num_sms);
  if (ws_bytes < w.total) return FT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(base);
  if (ft::launch_clear_words(base, w.header, s) != cudaSuccess) return FT_ERR_CUDA;
  const int64_t K = layer->K, N = layer->N, R = rank_all(layer);
  void* P = base + w.P;
  // P = bf16(G U^T) only (the gradient is not quantized)
  st = run_rowpass(dY, M, N, layer->U, R, false, nullptr, nullptr, nullptr, P,
                   reinterpret_cast<float*>(base + w.rp_part), reinterpret_cast<int*>(base + w.rp_cnt), status,
                   di.num_sms, s, true);
  if (st) return st;
  GemmArgs g{};
  g.M = M;
  g.N = K;
  g.K = N;
  g.R2 = R;
  g.a_codes = reinterpret_cast<const uint8_t*>(dY);
  g.b_codes = reinterpret_cast<const uint8_t*>(W16_t);
  g.main_bf16 = true;
  g.transposed = true;
  g.A2 = P;
  g.B2 = layer->D;
  g.out = dX;
  g.out_bf16 = dx_dtype == FT_DTYPE_BF16;
  if (w.g.side_sms == 0) {
    if ((st = run_grads(layer, M, X, P, dY, L_saved, dA, dB, accumulate != 0, w.g, false, base, status, s)))
      return st;
    return run_gemm(g, status, di.num_sms, s);
  }
  return gemm_and_grads_side(g, layer, M, X, P, dY, L_saved, dA, dB, accumulate != 0, w.g, base, status, di.num_sms,
                             s);
}

// ---------------------------------------------------------------- MLP
size_t fourtune_mlp_fwd_workspace_size(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M) {
  FT_RANGE("fourtune_mlp_fwd_workspace_size");
  if (check_mlp(fc1, fc2, false) || M <= 0 || M % 16) return 0;
  return mlp_fwd_layout(fc1, fc2, M, num_sms_or_default()).total;
}

size_t fourtune_mlp_bwd_workspace_size(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M) {
  FT_RANGE("fourtune_mlp_bwd_workspace_size");
  if (check_mlp(fc1, fc2, true) || M <= 0 || M % 16) return 0;
  return mlp_bwd_layout(fc1, fc2, M, num_sms_or_default()).total;
}

int fourtune_mlp_fwd_ws_offsets(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M, size_t* qa_codes,
                                size_t* qa_scales) {
  FT_RANGE("fourtune_mlp_fwd_ws_offsets");
  int st = check_mlp(fc1, fc2, false);
  if (st) return st;
  const MlpFwdWs w = mlp_fwd_layout(fc1, fc2, M, num_sms_or_default());
  if (qa_codes) *qa_codes = w.qa.codes;
  if (qa_scales) *qa_scales = w.qa.scales;
  return FT_OK;
}

int fourtune_mlp_bwd_ws_offsets(const ft_linear_t* fc1, const ft_linear_t* fc2, int64_t M, size_t* dh_off,
                                size_t* a_off, size_t* qdh_codes, size_t* qdh_scales) {
  FT_RANGE("fourtune_mlp_bwd_ws_offsets");
  int st = check_mlp(fc1, fc2, true);
  if (st) return st;
  const MlpBwdWs w = mlp_bwd_layout(fc1, fc2, M, num_sms_or_default());
  if (dh_off) *dh_off = w.dh;
  if (a_off) *a_off = SIZE_MAX;   // bf16(GELU(h)) is not stored (recomputed from h where needed)
  if (qdh_codes) *qdh_codes = w.qdh.codes;
  if (qdh_scales) *qdh_scales = w.qdh.scales;
  return FT_OK;
}

int fourtune_mlp_fwd(const ft_linear_t* fc1, const ft_linear_t* fc2, const ft_bf16* X, int64_t M, void* Y,
                     int y_dtype, ft_bf16* h_saved, ft_bf16* L1_saved, ft_bf16* L2_saved, float* dbg_a, void* ws,
                     size_t ws_bytes, void* stream) {
  FT_RANGE("fourtune_mlp_fwd");
  return fourtune_mlp_fwd_timed(fc1, fc2, X, M, Y, y_dtype, h_saved, L1_saved, L2_saved, dbg_a, ws, ws_bytes, stream,
                                nullptr, 0);
}

int fourtune_mlp_fwd_timed(const ft_linear_t* fc1, const ft_linear_t* fc2, const ft_bf16* X, int64_t M, void* Y,
                           int y_dtype, ft_bf16* h_saved, ft_bf16* L1_saved, ft_bf16* L2_saved, float* dbg_a,
                           void* ws, size_t ws_bytes, void* stream, void* const* events, int n_events) {
  FT_RANGE("fourtune_mlp_fwd_timed");
  const Events evs{events, n_events};
  int st = check_mlp(fc1, fc2, false);
  if (st) return st;
  if (!X || !Y || !h_saved || !L1_saved || !L2_saved || !ws) return FT_ERR_INVALID_ARG;
  if (y_dtype != FT_DTYPE_F32 && y_dtype != FT_DTYPE_BF16) return FT_ERR_INVALID_ARG;
  if (M <= 0 || M % 16) return FT_ERR_SHAPE;
  if (M > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(X) || !al16(Y) || !al16(h_saved) || !al16(L1_saved) || !al16(L2_saved) || (dbg_a && !al16(dbg_a)) ||
      (reinterpret_cast<uintptr_t>(ws) & 255u))
    return FT_ERR_ALIGN;
  DevInfo di;
  if ((st = device_info(&di))) return st;
  const MlpFwdWs w = mlp_fwd_layout(fc1, fc2, M, di.num_sms);
  if (ws_bytes < w.total) return FT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(base);
  if (ft::launch_clear_words(base, w.header, s) != cudaSuccess) return FT_ERR_CUDA;
  const int64_t K1 = fc1->K, H = fc1->N, N2 = fc2->N, R1 = rank_all(fc1), R2 = rank_all(fc2);
  // FC1: X pass (Q(X), L1)
  FT_TRY(0, run_rowpass(X, M, K1, fc1->D, R1, true, base + w.qx.codes, base + w.qx.scales,
                        base + w.qx.sf, L1_saved, reinterpret_cast<float*>(base + w.rp_part),
                        reinterpret_cast<int*>(base + w.rp_cnt), status, di.num_sms, s));
  // FC1's 4-bit GEMM + L1 U1 + b1 with the fused epilogue: h (saved), a =
  // GELU(h), Q(a) for FC2's 4-bit branch, L2 = bf16(bf16(a) D2) for its low-rank ones
  MlpGemmArgs m{};
  m.g.M = M;
  m.g.N = H;
  m.g.K = K1;
  m.g.R2 = R1;
  m.g.a_codes = base + w.qx.codes;
  m.g.a_sf = base + w.qx.sf;
  m.g.b_codes = fc1->R_codes;
  m.g.b_sf = fc1->R_sf;
  m.g.A2 = L1_saved;
  m.g.B2 = fc1->U;
  m.g.bias = fc1->bias;
  m.epi = 1;
  m.out_h = h_saved;
  m.dbg = dbg_a;
  m.q_codes = base + w.qa.codes;
  m.q_scales = base + w.qa.scales;
  m.q_sf = base + w.qa.sf;
  m.Wp = fc2->D;
  m.RP = R2;
  m.proj_out = L2_saved;
  m.part = reinterpret_cast<float*>(base + w.pj_part);
  FT_TRY(1, run_gemm_mlp(m, status, di.num_sms, s));
  FT_TRY(2, run_proj_reduce(m, di.num_sms, s));
  // FC2: 4-bit GEMM + L2 U2 + b2 -> Y
  GemmArgs g2{};
  g2.M = M;
  g2.N = N2;
  g2.K = H;
  g2.R2 = R2;
  g2.a_codes = base + w.qa.codes;
  g2.a_sf = base + w.qa.sf;
  g2.b_codes = fc2->R_codes;
  g2.b_sf = fc2->R_sf;
  g2.A2 = L2_saved;
  g2.B2 = fc2->U;
  g2.bias = fc2->bias;
  g2.out = Y;
  g2.out_bf16 = y_dtype == FT_DTYPE_BF16;
  FT_TRY(3, run_gemm(g2, status, di.num_sms, s));
  return FT_OK;
}

int fourtune_mlp_bwd(const ft_linear_t* fc1, const ft_linear_t* fc2, const ft_bf16* dY, const ft_bf16* X,
                     const ft_bf16* h_saved, const ft_bf16* L1_saved, const ft_bf16* L2_saved, int64_t M, void* dX,
                     int dx_dtype, float* dA1, float* dB1, float* dA2, float* dB2, int accumulate, void* ws,
                     size_t ws_bytes, void* stream) {
  FT_RANGE("fourtune_mlp_bwd");
  return fourtune_mlp_bwd_timed(fc1, fc2, dY, X, h_saved, L1_saved, L2_saved, M, dX, dx_dtype, dA1, dB1, dA2, dB2,
                                accumulate, ws, ws_bytes, stream, nullptr, 0);
}

int fourtune_mlp_bwd_timed(const ft_linear_t* fc1, const ft_linear_t* fc2, const ft_bf16* dY, const ft_bf16* X,
                           const ft_bf16* h_saved, const ft_bf16* L1_saved, const ft_bf16* L2_saved, int64_t M,
                           void* dX, int dx_dtype, float* dA1, float* dB1, float* dA2, float* dB2, int accumulate,
                           void* ws, size_t ws_bytes, void* stream, void* const* events, int n_events) {
  FT_RANGE("fourtune_mlp_bwd_timed");
  const Events evs{events, n_events};
  int st = check_mlp(fc1, fc2, true);
  if (st) return st;
  if (!dY || !X || !h_saved || !L1_saved || !L2_saved || !dX || !dA1 || !dB1 || !dA2 || !dB2 || !ws)
    return FT_ERR_INVALID_ARG;
  if (dx_dtype != FT_DTYPE_F32 && dx_dtype != FT_DTYPE_BF16) return FT_ERR_INVALID_ARG;
  if (M <= 0 || M % 16) return FT_ERR_SHAPE;
  if (M > (1 << 30)) return FT_ERR_UNSUPPORTED;
  if (!al16(dY) || !al16(X) || !al16(h_saved) || !al16(L1_saved) || !al16(L2_saved) || !al16(dX) || !al16(dA1) ||
      !al16(dB1) || !al16(dA2) || !al16(dB2) || (reinterpret_cast<uintptr_t>(ws) & 255u))
    return FT_ERR_ALIGN;
  DevInfo di;
  if ((st = device_info(&di))) return st;
  const MlpBwdWs w = mlp_bwd_layout(fc1, fc2, M, di.num_sms);
  if (ws_bytes < w.total) return FT_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  int* status = reinterpret_cast<int*>(base);
  if (ft::launch_clear_words(base, w.header, s) != cudaSuccess) return FT_ERR_CUDA;
  const int64_t K1 = fc1->K, H = fc1->N, N2 = fc2->N, R1 = rank_all(fc1), R2 = rank_all(fc2);
  void* P2 = base + w.P2;
  void* dh = base + w.dh;
  void* P1 = base + w.P1;
  // FC2 backward: G pass (Q(G), P2)
  FT_TRY(0, run_rowpass(dY, M, N2, fc2->U, R2, false, base + w.qg.codes, base + w.qg.scales,
                        base + w.qg.sf, P2, reinterpret_cast<float*>(base + w.rp_part),
                        reinterpret_cast<int*>(base + w.rp_cnt), status, di.num_sms, s));
  // FC2's dX GEMM with the fused epilogue: d_h = bf16(d_a GELU'(h)) (FC1's
  // incoming gradient), Q(d_h) for FC1's 4-bit branch, P1 = bf16(d_h U1^T)
  MlpGemmArgs m{};
  m.g.M = M;
  m.g.N = H;
  m.g.K = N2;
  m.g.R2 = R2;
  m.g.a_codes = base + w.qg.codes;
  m.g.a_sf = base + w.qg.sf;
  m.g.b_codes = fc2->R_codes_t;
  m.g.b_sf = fc2->R_sf_t;
  m.g.transposed = true;
  m.g.A2 = P2;
  m.g.B2 = fc2->D;
  m.epi = 2;
  m.h = h_saved;
  m.out_h = dh;
  m.q_codes = base + w.qdh.codes;
  m.q_scales = base + w.qdh.scales;
  m.q_sf = base + w.qdh.sf;
  m.Wp = fc1->U;
  m.RP = R1;
  m.proj_out = P1;
  m.part = reinterpret_cast<float*>(base + w.pj_part);
  FT_TRY(1, run_gemm_mlp(m, status, di.num_sms, s));
  FT_TRY(2, run_proj_reduce(m, di.num_sms, s));
  // FC2 adapter gradients: dA2 on bf16(GELU(h)) (recomputed from h), dB2 on G
  FT_TRY(3, run_grads(fc2, M, h_saved, P2, dY, L2_saved, dA2, dB2, accumulate != 0, w.g2, false, base, status, s,
                      true));
  // FC1 dX GEMM and adapter gradients (on d_h)
  GemmArgs g1{};
  g1.M = M;
  g1.N = K1;
  g1.K = H;
  g1.R2 = R1;
  g1.a_codes = base + w.qdh.codes;
  g1.a_sf = base + w.qdh.sf;
  g1.b_codes = fc1->R_codes_t;
  g1.b_sf = fc1->R_sf_t;
  g1.transposed = true;
  g1.A2 = P1;
  g1.B2 = fc1->D;
  g1.out = dX;
  g1.out_bf16 = dx_dtype == FT_DTYPE_BF16;
  if (evs.ev || w.g1.side_sms == 0) {
    FT_TRY(4, run_grads(fc1, M, X, P1, dh, L1_saved, dA1, dB1, accumulate != 0, w.g1, false, base, status, s));
    FT_TRY(5, run_gemm(g1, status, di.num_sms, s));
  } else {
    st = gemm_and_grads_side(g1, fc1, M, X, P1, dh, L1_saved, dA1, dB1, accumulate != 0, w.g1, base, status,
                             di.num_sms, s);
    if (st) return st;
  }
  return FT_OK;
}

// ---------------------------------------------------------------- static-scratch row pass
// Row pass over X [M, K] with W^T [R, K] read K-major, its split bookkeeping at
// `base` (status word, split counters, then partials); `fault_skip_stage` and
// `wait_ns` are the test hook of fourtune_test_wait_timeout (-1 and 0 otherwise).

int fourtune_quant_down_static(const ft_bf16* X, int64_t M, int64_t K, const ft_bf16* W, int64_t R,
                               uint8_t* codes, uint8_t* scales, ft_bf16* L, void* stream) {
  FT_RANGE("fourtune_quant_down_static");
  int st = check_quant_down(X, M, K, W, R, codes, scales, L);
  if (st) return st;
  DevInfo di;
  if ((st = device_info(&di))) return st;
  // split partials in the library's static array
  size_t header = 0;
  if (kmajor_rowpass_scratch(M, K, R, di.num_sms, &header) > ft::kRowpassStaticScratchBytes) return FT_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (ft::rowpass_static_scratch(&scratch) != cudaSuccess) return FT_ERR_CUDA;
  return launch_kmajor_rowpass(X, M, K, W, R, codes, scales, L, static_cast<uint8_t*>(scratch), header, di.num_sms, -1,
                               0, static_cast<cudaStream_t>(stream));
}

int fourtune_quant_down_static_status(void* stream) {
  FT_RANGE("fourtune_quant_down_static_status");
  void* scratch = nullptr;
  if (ft::rowpass_static_scratch(&scratch) != cudaSuccess) return FT_ERR_CUDA;
  return read_status_word(scratch, static_cast<cudaStream_t>(stream));
}

int fourtune_test_wait_timeout(const ft_bf16* X, int64_t M, int64_t K, const ft_bf16* W, int64_t R, uint8_t* codes,
                               uint8_t* scales, ft_bf16* L, void* ws, size_t ws_bytes, int64_t wait_ns,
                               void* stream) {
  FT_RANGE("fourtune_test_wait_timeout");
  int st = check_quant_down(X, M, K, W, R, codes, scales, L);
  if (st) return st;
  if (!ws) return FT_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(ws) & 255u) return FT_ERR_ALIGN;
  if (wait_ns < 1000000 || wait_ns > 1000000000) return FT_ERR_INVALID_ARG;
  DevInfo di;
  if ((st = device_info(&di))) return st;
  size_t header = 0;
  if (kmajor_rowpass_scratch(M, K, R, di.num_sms, &header) > ws_bytes) return FT_ERR_WORKSPACE;
  return launch_kmajor_rowpass(X, M, K, W, R, codes, scales, L, static_cast<uint8_t*>(ws), header, di.num_sms, 0,
                               static_cast<unsigned long long>(wait_ns), static_cast<cudaStream_t>(stream));
}

int fourtune_device_status(const void* ws, void* stream) {
  FT_RANGE("fourtune_device_status");
  if (!ws) return FT_ERR_INVALID_ARG;
  return read_status_word(ws, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
