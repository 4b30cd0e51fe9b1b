// Device-side building blocks for the sm_100a kernels: mbarriers with bounded
// waits, TMA tile loads, tcgen05 (TMEM alloc, MMA, smem->TMEM copy, TMEM
// loads) and the shared-memory matrix descriptors they consume.
//
// Every wait on an mbarrier is bounded in time: on expiry the waiting thread
// records FT_DEV_TIMEOUT in the call's status word and raises a CTA-local abort
// flag so that the other roles stop waiting too; nothing traps.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ft {

// status word values written by kernels (0 = ok)
constexpr int kDevTimeout = 1;
constexpr int kDevUnsupported = 2;   // a launch found its shared memory misaligned
// a wait that has not completed after this many nanoseconds gives up
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase of `bar` with the given parity.  Returns false if
// the CTA was aborted or the wait expired after `limit_ns` (then status/abort
// are set).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int* status,
                                          volatile int* abort_flag, uint64_t limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  uint32_t n = 0;
  while (!mbar_try_wait(bar, parity)) {
    if ((++n & 63u) == 0) {
      if (*abort_flag) return false;
      if (global_ns() - t0 > limit_ns) {
        *abort_flag = 1;
        if (status) atomicCAS(status, 0, kDevTimeout);
        return false;
      }
    }
  }
  return true;
}

// Bounded wait used on the way out (draining copies or MMAs already in flight):
// ignores the abort flag, gives up silently after `limit_ns`.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  const uint64_t t0 = global_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_ns() - t0 > limit_ns) return false;
  }
  return true;
}

// ------------------------------------------------------------------ dependent launch
// Programmatic dependent launch (kernels launched with launch_pdl): the next
// kernel on the stream may be scheduled once every CTA of this grid has issued
// launch_dependents (its CTAs then run their prologue on SMs this grid has
// left); wait_prior blocks until the previous grid has completed and its
// memory operations are visible.  Every kernel here calls both right after
// its prologue (barriers, TMEM, tensor-map prefetch) and before touching
// global memory, so no read or write can race the neighbouring kernels.
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void pdl_wait_prior() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ proxies
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
// bar.sync is the aligned barrier: reconverge the warp first
__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  __syncwarp();
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier over `nthreads` threads that also returns, to every thread, the
// OR of their predicates (bar.red.or): warps that must leave a loop together
// (because one of them saw an expired wait or an abort) decide it in the same
// operation that synchronizes them, so none is left waiting at a later barrier.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t out;
  __syncwarp();
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(out)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
      : "memory");
  return out != 0;
}

// ------------------------------------------------------------------ TMA
// Split-K counter: returns the old value.  acq_rel at gpu scope: the release
// half publishes every write ordered before this thread's atomic (the CTA's
// partial, through the CTA barrier that precedes it); the acquire half orders
// the reads that follow (through the next CTA barrier, the last CTA's loads of
// the other CTAs' partials) after every earlier increment's release.  One
// atomic in place of fence, atomic, fence.
__device__ __forceinline__ int atomic_add_acq_rel_gpu(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
// pull the 128-byte line holding p into L2 (no registers, no completion)
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<uint64_t>(p)));
}
__device__ __forceinline__ void tma_prefetch(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
// 2-D tiled load of one box into shared memory, completing on `bar`.
// The innermost coordinate x is in elements and must keep x*elemsize a
// multiple of 16 bytes (all callers use multiples of 64 elements / 128 bytes).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// Plain (untiled) bulk copy of `bytes` contiguous bytes global -> shared,
// completing on `bar`; both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// 2-D tiled store of one box from shared memory (bulk-group completion).
// Elements of the box outside the tensor are not written.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// wait until every committed bulk store has finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// arrive on `bar` once every tcgen05 operation issued so far by this thread completes
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 inputs, fp32 accumulate
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= (A * sfA) * (B * sfB)^T, packed E2M1 operands, one UE4M3 scale per
// 16 elements along K (K = 64 per instruction), fp32 accumulate.
__device__ __forceinline__ void mma_fp4_block16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}" ::"r"(
          d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
      : "memory");
}

// copy 32 rows x 128 bits from smem into TMEM, replicated into all four
// 32-lane sub-partitions (the layout the block-scaled MMA reads scales from)
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// 32 lanes x 32 columns of 32-bit TMEM words -> 32 registers per thread
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
        "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]),
        "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]),
        "=r"(v[30]), "=r"(v[31])
      : "r"(taddr));
}
// 32 lanes x 16 columns -> 16 registers per thread
__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
        "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 16 / 32 registers per thread -> 32 lanes x 16 / 32 columns of TMEM (the
// warp's own lane quadrant); complete once tmem_st_wait returns
__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]), "r"(v[8]),
      "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]), "r"(v[16]),
      "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]),
      "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
// one word per thread -> the same word in 4 consecutive columns of the warp's lane quadrant
__device__ __forceinline__ void tmem_st_32x32b_x4_rep(uint32_t taddr, uint32_t w) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x4.b32 [%0], {%1,%1,%1,%1};" ::"r"(taddr), "r"(w) : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ------------------------------------------------------------------ descriptors
// Shared-memory matrix descriptor (sm_100 format): start address, leading and
// stride byte offsets (>>4), version 1, layout type in bits 61..63.
constexpr uint32_t kLayoutNone = 0;
constexpr uint32_t kLayoutSw128 = 2;

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;
  d |= static_cast<uint64_t>(layout) << 61;
  return d;
}
// K-major operand stored as 128-byte rows with the 128-byte swizzle (what a TMA
// box of 128-byte rows with CU_TENSOR_MAP_SWIZZLE_128B writes): 8-row groups
// are 1024 bytes apart.  Advancing along K inside the swizzle atom is a plain
// start-address offset.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  return smem_desc(saddr, 16, 1024, kLayoutSw128);
}
// MN-major operand in 128-byte-swizzled rows: each 128-byte row holds 64
// consecutive MN elements for one K index; `mn_chunk_bytes` is the distance
// between consecutive 64-element MN chunks, 8-K groups are 1024 bytes apart.
__device__ __forceinline__ uint64_t desc_mnmajor_sw128(uint32_t saddr, uint32_t mn_chunk_bytes) {
  return smem_desc(saddr, mn_chunk_bytes, 1024, kLayoutSw128);
}
// Source of tcgen05.cp 32x128b: 32 rows of 16 bytes, contiguous
__device__ __forceinline__ uint64_t desc_sf_copy(uint32_t saddr) { return smem_desc(saddr, 0, 128, kLayoutNone); }

// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4)                                   // D format: f32
         | (1u << 7)                                 // A format: bf16
         | (1u << 10)                                // B format: bf16
         | (static_cast<uint32_t>(a_mn_major) << 15)  // A major
         | (static_cast<uint32_t>(b_mn_major) << 16)  // B major
         | (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}
// Instruction descriptor, kind::mxf4nvf4 block-scaled: E2M1 A/B, UE4M3 scales,
// K = 64 per instruction, scale-factor ids 0 (column-aligned scale addresses).
__host__ __device__ constexpr uint32_t idesc_fp4_block16(int M, int N) {
  return (1u << 7)      // A format: E2M1
         | (1u << 10)   // B format: E2M1
         | (static_cast<uint32_t>(N >> 3) << 17) |
         (0u << 23)     // scale format: UE4M3
         | (static_cast<uint32_t>(M >> 4) << 24);
}

// ------------------------------------------------------------------ conversions
// E4M3 encode of a non-negative float (round to nearest even, saturate at 448)
__device__ __forceinline__ uint32_t f32_to_e4m3(float s) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(s));
  return r & 0xFFu;
}
__device__ __forceinline__ float e4m3_to_f32(uint32_t code) {
  uint32_t h2;
  uint16_t c = static_cast<uint16_t>(code & 0xFFu);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}
// one E2M1 code (low 4 bits) -> its value, by the hardware conversion
__device__ __forceinline__ float e2m1_to_f32(uint32_t code) {
  uint32_t h2;
  const uint16_t c = static_cast<uint16_t>(code & 0xFu);
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u16 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}" : "=r"(h2) : "h"(c));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}
// eight floats -> 32 bits of E2M1 codes, element i in bits 4i..4i+3: the
// hardware conversion rounds to nearest even, saturates at +-6 and keeps the
// sign of zero (the parity tests check every E2M1 tie, both signs, against the
// oracle's table search)
__device__ __forceinline__ uint32_t f32x8_to_e2m1(const float* v) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return r;
}

// Block16 quantization of consecutive bf16 values of one row, given the block
// maximum: scale = E4M3(amax / 6) (IEEE division), code = E2M1(v / dec(scale))
// rounded to nearest even, all +0 when the scale decodes to 0.
//
// The per-element division is replaced by an exact equivalent.  v is bf16 (at
// most 8 significant bits) and d = dec(scale) an E4M3 value (at most 4), so v/d
// is either exactly one of the E2M1 rounding ties (0.25, 0.75, 1.25, 1.75, 2.5,
// 3.5, 5, either sign) or at least 1/255 (relative) away from every one of them
// (the difference of two such products is a multiple of the smaller power of
// two).  q = v * (1/d), with the reciprocal correctly rounded, is within 2^-22
// (relative) of v/d; rounding q to 19 mantissa bits therefore lands exactly on
// the tie when v/d is one and otherwise moves q by less than 2^-19, never across
// a tie.  The nearest-even conversion of that q is the code of v/d, i.e. of the
// IEEE quotient fp32(v / d) (which can only equal a tie when v/d does).
__device__ __forceinline__ float snap19(float q) {
  return __uint_as_float((__float_as_uint(q) + 0x8u) & ~0xFu);
}
// N (a multiple of 8) values of one block row and the block maximum -> N/8 words
// of codes (element i in bits 4(i%8).. of word i/8) and the scale byte.
// fp32(a / 6) for a bf16 value a (the block maximum of bf16 inputs), correctly
// rounded without a division, by the correction step for division by a constant
// known in advance of Brisebarre, Muller and Raina ("Accelerating correctly
// rounded floating-point division when the divisor is known in advance", IEEE
// Trans. Computers 53(8), 2004): q0 = RN(a * RN(1/6)) is at most one ulp off; the
// residual a - 6 q0 is exact in one fused multiply-add, and q0 + RN(residual) *
// RN(1/6) lands on the correctly rounded quotient for every finite bf16 a
// (checked exhaustively against IEEE division on the GPU by the scale tests of
// every bf16 block maximum).
__device__ __forceinline__ float div6_bf16(float a) {
  constexpr float kSixth = 1.0f / 6.0f;
  const float q0 = a * kSixth;
  const float r = fmaf(-q0, 6.0f, a);
  return fmaf(r, kSixth, q0);
}
template <int N>
__device__ __forceinline__ void quantize_block_row(const float* v, float amax, uint32_t* packed, uint32_t* sc) {
  *sc = f32_to_e4m3(div6_bf16(amax));
  const float d = e4m3_to_f32(*sc);
  if (d == 0.0f) {
#pragma unroll
    for (int w = 0; w < N / 8; ++w) packed[w] = 0u;
    return;
  }
  const float rd = __frcp_rn(d);
  float q[N];
#pragma unroll
  for (int e = 0; e < N; ++e) q[e] = snap19(v[e] * rd);
#pragma unroll
  for (int w = 0; w < N / 8; ++w) packed[w] = f32x8_to_e2m1(q + 8 * w);
}
__device__ __forceinline__ void quantize_1block(const float* v, float amax, uint32_t* packed, uint32_t* sc) {
  quantize_block_row<16>(v, amax, packed, sc);
}
__device__ __forceinline__ void quantize_2blocks(const float* v, const float* amax, uint32_t* packed,
                                                 uint32_t* sc) {
#pragma unroll
  for (int j = 0; j < 2; ++j) quantize_1block(v + 16 * j, amax[j], packed + 2 * j, sc + j);
}

// Block16 quantization of 16 float32 values (one block) of any precision (the
// GELU output), with the semantics of the IEEE quotient fp32(v / d) but no
// division per element.  q = v * RN(1/d) lies within 2^-22.4 (relative) of the
// quotient, so the code of the quotient is the code of q unless an E2M1 rounding
// threshold lies within [q (1 - 2^-21), q (1 + 2^-21)]: the codes of those two
// ends (the conversion is monotonic in |x|) detect it, and only then is the
// quotient computed by IEEE division.  Same outputs as quantize_1block.
template <int N>
__device__ __forceinline__ void quantize_block_row_f32(const float* v, float amax, uint32_t* packed, uint32_t* sc) {
  *sc = f32_to_e4m3(__fdiv_rn(amax, 6.0f));
  const float d = e4m3_to_f32(*sc);
  if (d == 0.0f) {
#pragma unroll
    for (int w = 0; w < N / 8; ++w) packed[w] = 0u;
    return;
  }
  const float rd = __frcp_rn(d);
  constexpr float kDown = 1.0f - 0x1p-21f, kUp = 1.0f + 0x1p-21f;
  float lo[N], hi[N];
#pragma unroll
  for (int e = 0; e < N; ++e) {
    const float q = v[e] * rd;
    lo[e] = q * kDown;
    hi[e] = q * kUp;
  }
  bool near = false;
#pragma unroll
  for (int w = 0; w < N / 8; ++w) {
    packed[w] = f32x8_to_e2m1(lo + 8 * w);
    near = near || packed[w] != f32x8_to_e2m1(hi + 8 * w);
  }
  if (near) {
    float q[N];
#pragma unroll
    for (int e = 0; e < N; ++e) q[e] = __fdiv_rn(v[e], d);
#pragma unroll
    for (int w = 0; w < N / 8; ++w) packed[w] = f32x8_to_e2m1(q + 8 * w);
  }
}
__device__ __forceinline__ void quantize_1block_f32(const float* v, float amax, uint32_t* packed, uint32_t* sc) {
  quantize_block_row_f32<16>(v, amax, packed, sc);
}

// GELU, tanh form: 0.5 h (1 + tanh(sqrt(2/pi) (h + 0.044715 h^3))), evaluated
// through 0.5 (1 + tanh(u)) = 1 / (1 + e^{-2u}) =: s (no cancellation for very
// negative h), so GELU(h) = h s.  Its derivative, with 1 - tanh(u)^2 = 4 s (1 - s)
// and 1 - s = s e^{-2u}: GELU'(h) = s + 2 h s (1 - s) sqrt(2/pi) (1 + 3 * 0.044715 h^2).
// e^{-2u} = 2^(-2 log2(e) u) on the hardware base-2 exponential and s on the
// hardware reciprocal (PTX ex2.approx / rcp.approx: relative errors near
// 2^-22; with the rounding of the exponent's product, e^{-2u} is within ~6e-6
// for |u| <= 44).  Their limits need no special cases: for u < -44.3 e^{-2u}
// is +inf and s = 1/inf = +0, so GELU = h * 0 = -0 (true value below 3e-39 |h|);
// for u > 44 e^{-2u} = 0, s = 1 and GELU = h (exact in fp32).  The derivative
// takes GELU' = 0 for u < -40 and 1 for u > 40 (true values within 1e-32 of
// those), as selects, so that s (1 - s) = s * s e^{-2u} is never inf * 0.
constexpr float kGeluC = 0.7978845608028654f;   // sqrt(2/pi)
constexpr float kGeluK = 0.044715f;
constexpr float kGeluM2Log2e = -2.8853900817779268f;   // -2 log2(e)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// u = sqrt(2/pi) (h + 0.044715 h^3)
__device__ __forceinline__ float gelu_u(float h) { return h * fmaf(kGeluC * kGeluK, h * h, kGeluC); }
__device__ __forceinline__ float gelu_tanh(float h) {
  const float e = ex2_approx(kGeluM2Log2e * gelu_u(h));
  return h * rcp_approx(1.0f + e);
}
__device__ __forceinline__ void gelu_tanh_and_grad(float h, float* g, float* dg) {
  const float u = gelu_u(h);
  const float e = ex2_approx(kGeluM2Log2e * u);
  const float s = rcp_approx(1.0f + e);
  *g = h * s;
  const float d = fmaf(2.0f * h * s * (e * s), kGeluC * fmaf(3.0f * kGeluK, h * h, 1.0f), s);
  *dg = u > 40.0f ? 1.0f : (u < -40.0f ? 0.0f : d);
}

__device__ __forceinline__ float bf16_bits_to_f32(uint32_t b) { return __uint_as_float(b << 16); }

// ------------------------------------------------------------------ 1x16 groups
// Per-tensor scale of the 1x16 group-wise layout (the granularity comparator of
// FourTune §4.3, Table 5): 2^e with e the least integer such that
// amax <= 2688 * 2^e (2688 = 6 * 448: the E2M1 times the E4M3 maximum), at
// least -126; 0 for amax = 0.  amax is a non-negative finite float.  With
// amax = m 2^E (1 <= m < 2) and 2688 = 1.3125 * 2^11: e = E - 11, plus one when
// m > 1.3125 (m's fraction bits above 0x280000).
__device__ __forceinline__ int group16_exponent(float amax) {
  if (!(amax > 0.0f)) return 0;
  uint32_t b = __float_as_uint(amax);
  int E = static_cast<int>(b >> 23) - 127;
  if ((b >> 23) == 0) {                      // subnormal: normalize (exact)
    b = __float_as_uint(amax * 16777216.0f);
    E = static_cast<int>(b >> 23) - 127 - 24;
  }
  const int e = E - 11 + ((b & 0x7FFFFFu) > 0x280000u ? 1 : 0);
  return e < -126 ? -126 : e;
}
// 2^k for -126 <= k <= 127
__device__ __forceinline__ float pow2_f32(int k) { return __uint_as_float(static_cast<uint32_t>(k + 127) << 23); }

// Maximum of a non-negative float over the 16 lanes of the warp whose lane bit 0
// equals this lane's (two half-warp groups, reduced at once).  Non-negative
// IEEE floats order like their bit patterns, so one integer max reduction does it.
__device__ __forceinline__ float max16_same_parity(float a, int lane) {
  const unsigned mask = (lane & 1) ? 0xAAAAAAAAu : 0x55555555u;
  return __uint_as_float(__reduce_max_sync(mask, __float_as_uint(a)));
}

// Launch with programmatic stream serialization (see pdl_wait_prior).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

}  // namespace ft
