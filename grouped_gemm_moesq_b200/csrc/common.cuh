// Shared device helpers of the moesq CUDA library (sm_100a only).
//
//  * NVFP4 codecs: E2M1 values (paper App. A, Fig. 3 grid) and UE4M3 block
//    scales (paper Sec. 3.4, Eq. 5), converted with the hardware's
//    round-to-nearest-even saturating conversions.
//  * The NVFP4 block quantiser of Eq. 3 / Eq. 5 in binary32 with one
//    rounding per operation (explicit _rn intrinsics, no contraction).
//  * PTX wrappers for mbarriers, TMA / bulk copies and tcgen05.
//  * The device error word and bounded waits (every wait gives up after a
//    time limit, records the error and lets the kernel return).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace moesq {

// ------------------------------------------------------------- error word
enum DevErrKind : int { kErrTimeout = 4, kErrFault = 5 };
enum DevErrWhere : int {
  kWhereGemmProducer = 1, kWhereGemmMma = 2, kWhereGemmEpilogue = 3, kWhereGemmCounts = 4,
  kWhereRoute = 5, kWhereQuant = 6, kWhereDebug = 7, kWhereSwiglu = 8, kWhereCombine = 9, kWhereConvert = 10
};

__device__ int g_error_word;   // 0 = no error; (where << 8) | kind

__device__ __forceinline__ void record_error(int where, int kind) {
  atomicCAS(&g_error_word, 0, (where << 8) | kind);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ------------------------------------------------------------------ codecs
// Clears the sign bit of every E2M1 nibble whose magnitude is zero, so that
// a result of -0 is written as +0.
__device__ __forceinline__ uint32_t e2m1_canon_zero(uint32_t v) {
  uint32_t nz = ((v & 0x77777777u) + 0x77777777u) & 0x88888888u;  // bit 3 set iff magnitude != 0
  return (v & 0x77777777u) | (v & nz);
}

// Eight floats -> four bytes of E2M1 codes, element 2i in the low nibble of
// byte i; round to nearest even, saturating at +-6.
__device__ __forceinline__ uint32_t e2m1x8(const float (&x)[8]) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(x[0]), "f"(x[1]), "f"(x[2]), "f"(x[3]), "f"(x[4]), "f"(x[5]), "f"(x[6]), "f"(x[7]));
  return e2m1_canon_zero(r);
}

// Two floats -> one byte of E2M1 codes (lo in the low nibble).
__device__ __forceinline__ uint32_t e2m1x2(float lo, float hi) {
  uint32_t r;
  asm("{\n\t.reg .b8 b0;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "mov.b32 %0, {b0, b0, b0, b0};\n\t}"
      : "=r"(r) : "f"(lo), "f"(hi));
  return e2m1_canon_zero(r & 0xFFu);
}

// Non-negative float -> UE4M3 code, RNE with saturation to 448.
__device__ __forceinline__ uint32_t ue4m3_encode(float x) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(x));
  return r & 0x7Fu;
}

// UE4M3 code -> value (exact): e = 0: m * 2^-9, else (8 + m) * 2^(e - 10).
__device__ __forceinline__ float ue4m3_value(uint32_t c) {
  uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return __uint2float_rn(m) * 0.001953125f;
  return __uint_as_float(((e + 120u) << 23) | (m << 20));
}

// Eq. 5: gamma = 448 / (amax / 6); 1 for an all-zero tensor.
__device__ __forceinline__ float nvfp4_global_scale(float amax) {
  if (!(amax > 0.0f)) return 1.0f;
  return __fdiv_rn(448.0f, __fdiv_rn(amax, 6.0f));
}

// Eq. 5 block scale code: RNE_E4M3(gamma * amax_b / 6).
__device__ __forceinline__ uint32_t block_scale_code(float gamma, float amax_b) {
  return ue4m3_encode(__fdiv_rn(__fmul_rn(gamma, amax_b), 6.0f));
}

// Eq. 3 / Eq. 5: s_b = UE4M3(code) / gamma; value / s_b rounded onto E2M1.
__device__ __forceinline__ float block_step(uint32_t code, float gamma) {
  return __fdiv_rn(ue4m3_value(code), gamma);
}
// Eight values of one block -> four bytes of codes: each code is the E2M1
// rounding of the correctly rounded quotient q = fl(v / s_b), given
// r = fl(1 / s_b) (rfin: r is finite).
//
// The code of q only depends on where q lies relative to the E2M1 decision
// points (0.25, 0.75, ..., 5) and on exact ties there, and E2M1 rounding is
// monotone in the magnitude.  y = fl(v * r) is within (2^-23 + 2^-48)|x| of
// x = v / s_b, and q within 2^-24 |x| of x, so q lies strictly inside
// [y (1 - 2^-20), y (1 + 2^-20)] (both ends rounded).  When the two ends
// round to the same codes, every value between them does, q included, and
// those codes are returned.  Otherwise (a value within about 2^-20 of a
// decision point), or when r is not finite, the quotients are formed exactly.
__device__ __forceinline__ uint32_t quant8_r(const float* v, float s_b, float r, bool rfin) {
  if (rfin) {
    float lo[8], hi[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float y = __fmul_rn(v[i], r);
      lo[i] = __fmul_rn(y, 0x1.ffffep-1f);     // 1 - 2^-20
      hi[i] = __fmul_rn(y, 0x1.00001p+0f);     // 1 + 2^-20
    }
    const uint32_t cl = e2m1x8(lo), ch = e2m1x8(hi);
    if (cl == ch) return cl;
  }
  float q[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) q[i] = __fdiv_rn(v[i], s_b);
  return e2m1x8(q);
}

// SwiGLU of one feature: SiLU(g) * u with SiLU(g) = g / (1 + e^-g) in
// binary32 with the hardware exponential and divide (a few ulp; for
// g < -88 the denominator overflows and the quotient is 0).  Every kernel
// that forms h uses this one function, so fused and unfused paths agree
// bit for bit.
__device__ __forceinline__ float silu_mul(float g, float u) {
  return __fmul_rn(__fdividef(g, __fadd_rn(1.0f, __expf(-g))), u);
}

// Eight values of one block -> four bytes of codes (x / s_b onto E2M1).
__device__ __forceinline__ uint32_t quant8(const float (&v)[8], float s_b, bool zero_block) {
  if (zero_block) return 0u;
  const float r = __frcp_rn(s_b);
  return quant8_r(v, s_b, r, isfinite(r));
}

// One whole 32-element scale block -> 16 bytes of codes (element 2i in the
// low nibble of byte i).
__device__ __forceinline__ uint4 quant32(const float (&v)[32], float s_b, bool zero_block) {
  if (zero_block) return make_uint4(0u, 0u, 0u, 0u);
  const float r = __frcp_rn(s_b);
  const bool rfin = isfinite(r);
  uint4 o;
  o.x = quant8_r(v, s_b, r, rfin);
  o.y = quant8_r(v + 8, s_b, r, rfin);
  o.z = quant8_r(v + 16, s_b, r, rfin);
  o.w = quant8_r(v + 24, s_b, r, rfin);
  return o;
}

// Quantises the 32-element block v with global scale gamma: stores the 16
// code bytes at dst and returns the block's scale code.
__device__ __forceinline__ uint32_t quantize_block32(const float (&v)[32], float gamma, uint8_t* dst) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(v[i]));
  const uint32_t code = block_scale_code(gamma, a);
  *reinterpret_cast<uint4*>(dst) = quant32(v, block_step(code, gamma), code == 0);
  return code;
}

__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ uint32_t f32_to_bf16_bits(float f) {
  return (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(f));
}

// Offset of the scale of (row, scale index sidx) in the MMA scale layout
// [rows/128][K/128][32][4][4] (K given as the number of 128-wide blocks kb).
__device__ __forceinline__ size_t mma_scale_offset(int64_t row, int sidx, int kb) {
  int64_t rb = row >> 7;
  int r = (int)(row & 127);
  return ((size_t)(rb * kb + (sidx >> 2)) << 9) + (size_t)((r & 31) * 16 + (r >> 5) * 4 + (sidx & 3));
}

// ------------------------------------------------------------------ smem / mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" :: "r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" :: "r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}

// Bounded wait: true once the phase of `parity` has completed; false after
// `timeout_ns` or once *abort is set by another role of the CTA.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                          volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((spin & 15u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
  }
}

// Named barrier `id` over `nthreads` threads (whole warps), returning
// whether any participating thread passed v = true.
__device__ __forceinline__ bool bar_red_or(int id, int nthreads, bool v) {
  uint32_t r;
  asm volatile("{\n\t.reg .pred p, q;\n\t"
               "setp.ne.u32 q, %1, 0;\n\t"
               "bar.red.or.pred p, %2, %3, q;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(r) : "r"((uint32_t)v), "r"(id), "r"(nthreads) : "memory");
  return r != 0;
}

__device__ __forceinline__ void bar_sync_named(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" :: "r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------------------ TMA / bulk copies
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* tmap, uint32_t bar, int x, int y,
                                            uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;"
      :: "r"(dst), "l"(tmap), "r"(bar), "r"(x), "r"(y), "l"(policy) : "memory");
}

__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;"
      :: "r"(dst), "l"(src), "r"(bytes), "r"(bar), "l"(policy) : "memory");
}

// Programmatic dependent launch: the kernels of a layer step let the next
// grid launch as soon as all of their CTAs are running (launch_dependents),
// and wait for the previous grid to finish, its memory visible, before
// touching global memory (wait; returns at once without a predecessor).
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}

__device__ __forceinline__ void prefetch_tmap(const void* tmap) {
  asm volatile("prefetch.tensormap [%0];" :: "l"(tmap) : "memory");
}

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               :: "r"(dst_smem), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(bar) : "memory");
}
// smem (128 rows x 16 B) -> TMEM lanes 0..127, 4 columns
__device__ __forceinline__ void tc_cp_128x128b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x128b [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}
// smem (128 rows x 32 B) -> TMEM lanes 0..127, 8 columns
__device__ __forceinline__ void tc_cp_128x256b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.128x256b [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}
// smem (32 rows x 16 B) -> TMEM lanes 0..31 of each of the 4 sub-partitions, 4 columns
__device__ __forceinline__ void tc_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}

// Sparse block-scaled FP4 MMA (M = 128, K = 128 dense / 64 stored per row of
// A, one UE4M3 scale per 32 dense K of each operand): D (+)= A * B^T.
__device__ __forceinline__ void tc_mma_sp_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                               uint32_t e_tmem, uint32_t idesc, uint32_t sfa_tmem,
                                               uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.sp.cta_group::1.kind::mxf4nvf4.block_scale.block16"
               " [%0], %1, %2, [%7], %3, [%5], [%6], p;\n\t}"
               :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate),
                  "r"(sfa_tmem), "r"(sfb_tmem), "r"(e_tmem) : "memory");
}

// Dense block-scaled FP4 MMA (M = 128, K = 64, one UE4M3 scale per 16 K of
// each operand): D (+)= A * B^T.
__device__ __forceinline__ void tc_mma_nvf4(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t sfa_tmem, uint32_t sfb_tmem, uint32_t accumulate) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16"
               " [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
               :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem),
                  "r"(sfb_tmem) : "memory");
}

__device__ __forceinline__ void tmem_ld_32x32b_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x16.b32"
               " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
                 "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
                 "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
               : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05 "matrix descriptor"): start
// address, leading / stride byte offsets (16-byte units), version 1 at bit
// 46, layout type at bits 61-63 (0 none, 2 128B swizzle, 4 64B swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes,
                                              uint32_t layout) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)(layout & 7u) << 61;
  return d;
}

// Instruction descriptor of the sparse block-scaled E2M1 x E2M1 MMA with
// UE4M3 scales, K-major A and B, M = 128 and N rows of B.
__device__ __forceinline__ uint32_t idesc_sp_nvf4(uint32_t n) {
  return (1u << 2)              // sparse
       | (1u << 7)              // A format E2M1
       | (1u << 10)             // B format E2M1
       | ((n >> 3) << 17)       // N / 8
       | (0u << 23)             // scale format UE4M3
       | ((128u >> 4) << 24);   // M / 16
}

}  // namespace moesq
