// Tensor-core throughput benchmark for the block-scaled FP4 MMA the grouped
// GEMM is built on (tcgen05.mma kind::mxf4nvf4, UE4M3 scales per 16 K).
//
// Every CTA stages one operand image in shared memory and its scale and
// metadata columns in tensor memory once, then one thread issues `iters`
// groups of two MMAs back to back into one TMEM accumulator (M = 128,
// N = n; dense: K = 64 per MMA, sparse .sp: K = 128 dense-equivalent per
// MMA) and waits for their completion through tcgen05.commit.  With COPIES,
// each group is preceded by the shared-to-tensor-memory copies the grouped
// GEMM issues per 256-wide K step (metadata, two weight-scale and
// ceil(n / 128) x 2 token-scale blocks), so the rate includes their share
// of the tensor pipe.  The operand
// contents do not change the instruction's timing, so the images are zero.
// The measured rate (MMAs x 2 M N K / time) is this GPU's ceiling for the
// shapes the GEMM issues, with no memory traffic behind it.
#pragma once
#include "common.cuh"

namespace moesq {

constexpr int kPeakThreads = 128;
// shared memory: A image 128 x 64 B (64-byte swizzle) at 0, B image
// 256 x 128 B (128-byte swizzle) at 8 KB, 2 KB of zero bytes for the
// metadata / scale copies at 40 KB, the mbarrier and TMEM address after
constexpr int kPeakOffB = 8192;
constexpr int kPeakOffZ = kPeakOffB + 256 * 128;
constexpr int kPeakOffBar = kPeakOffZ + 2048;
constexpr int kPeakSmemBytes = kPeakOffBar + 64 + 1024;

template <bool SPARSE, bool COPIES>
__global__ void __launch_bounds__(kPeakThreads, 1)
mma_peak_kernel(int n, int iters, uint32_t tmem_cols, uint64_t timeout_ns, unsigned long long* cycles_out) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  uint32_t* tptr = reinterpret_cast<uint32_t*>(smem + kPeakOffBar + 8);
  const uint32_t bar = sbase + kPeakOffBar;
  for (int i = threadIdx.x; i < kPeakOffBar / 16; i += blockDim.x)
    reinterpret_cast<uint4*>(smem)[i] = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async();                       // generic-proxy zeros visible to the tensor core
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  if (threadIdx.x < 32) {
    tmem_alloc(smem_u32(tptr), tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tptr;
  if (threadIdx.x == 0) {
    // metadata (4 columns) and scales (A: 8, B: up to 16 columns) after the accumulator
    const uint32_t tbuf = tmem + (uint32_t)n;
    const uint32_t z = sbase + kPeakOffZ;
    tc_cp_128x128b(tbuf, smem_desc(z, 16, 128, 0));
    for (int c = 0; c < 7; ++c) tc_cp_32x128b_x4(tbuf + 4 + 4 * c, smem_desc(z, 16, 128, 0));
    const uint32_t idesc = SPARSE ? idesc_sp_nvf4((uint32_t)n) : (idesc_sp_nvf4((uint32_t)n) & ~(1u << 2));
    const uint64_t t0 = clock64();
    for (int it = 0; it < iters; ++it) {
      if (COPIES) {
        tc_cp_128x128b(tbuf, smem_desc(z, 16, 128, 0));
        tc_cp_32x128b_x4(tbuf + 4, smem_desc(z, 16, 128, 0));
        tc_cp_32x128b_x4(tbuf + 8, smem_desc(z + 512, 16, 128, 0));
        for (int c = 0; c < (n + 127) / 128; ++c) {
          tc_cp_32x128b_x4(tbuf + 12 + 8 * c, smem_desc(z + 1024, 16, 128, 0));
          tc_cp_32x128b_x4(tbuf + 16 + 8 * c, smem_desc(z + 1536, 16, 128, 0));
        }
      }
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        const uint64_t adesc = smem_desc(sbase + kb * 32, 16, 512, 4);
        const uint64_t bdesc = smem_desc(sbase + kPeakOffB + kb * (SPARSE ? 64 : 32), 16, 1024, 2);
        const uint32_t acc = (it | kb) != 0 ? 1u : 0u;
        if (SPARSE) {
          tc_mma_sp_nvf4(tmem, adesc, bdesc, tbuf + 2 * kb, idesc, tbuf + 4 + 4 * kb, tbuf + 12, acc);
        } else {
          tc_mma_nvf4(tmem, adesc, bdesc, idesc, tbuf + 4 + 4 * kb, tbuf + 12, acc);
        }
      }
    }
    tc_commit(bar);
    int zero = 0;
    if (!mbar_wait(bar, 0, timeout_ns, &zero)) record_error(kWhereDebug, kErrTimeout);
    const uint64_t t1 = clock64();
    if (cycles_out) atomicMax(cycles_out, (unsigned long long)(t1 - t0));
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

}  // namespace moesq
