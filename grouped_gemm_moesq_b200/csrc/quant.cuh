// Activation-side kernels: NVFP4 quantisation of activations (plain and
// fused with the dispatch scatter), SwiGLU + requantisation, the
// router-weighted combine and the amax reductions behind the static global
// scales.  The quantising kernels give each lane one whole 32-element scale
// block (64-byte loads, one scale per lane, 16-byte code stores), so the
// block's scale and step are computed once.
#pragma once
#include "common.cuh"

namespace moesq {

__device__ __forceinline__ void load8_bf16(const uint16_t* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
  v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}

__device__ __forceinline__ void load32_bf16(const uint16_t* p, float (&v)[32]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + j);
    v[8 * j + 0] = bf16lo(u.x); v[8 * j + 1] = bf16hi(u.x); v[8 * j + 2] = bf16lo(u.y); v[8 * j + 3] = bf16hi(u.y);
    v[8 * j + 4] = bf16lo(u.z); v[8 * j + 5] = bf16hi(u.z); v[8 * j + 6] = bf16lo(u.w); v[8 * j + 7] = bf16hi(u.w);
  }
}

// One warp task = (token t, 1024-element chunk c of x[t], slot group g):
// lane l loads the scale block [1024 c + 32 l, +32) and takes its amax once,
// then quantises it for the token's slots j = g, g + S, ... (S =
// slot_groups) with the slot's expert gamma into the slot's row (the fused
// dispatch + quantisation): the block scale code depends on the slot only
// through gamma.  S = 1 shares one load among all k slots; with few tokens
// the host splits the slots over S = k warps so that enough warps run.
// Indices stay 32-bit (T * k * S, rows, K and the task count are below
// 2^31).  Plain form (slot_to_row == nullptr): one slot, gamma[0], row = t.
__global__ void __launch_bounds__(256) quantize_act_kernel(const uint16_t* __restrict__ x, int T, int K, int k,
                                                           const int32_t* __restrict__ topk_ids,
                                                           const int32_t* __restrict__ slot_to_row, int E,
                                                           const float* __restrict__ gamma, int rows_cap,
                                                           uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
                                                           int slot_groups) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int nslots = slot_to_row ? k : 1;
  const int chunks = (K + 1023) >> 10;
  const int ntasks = T * chunks * slot_groups;
  const int wstride = gridDim.x * (blockDim.x >> 5);
  const int KB = K / 128;
  for (int task = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < ntasks; task += wstride) {
    const int grp = task % slot_groups;
    const int tc = task / slot_groups;
    const int t = tc / chunks;
    const int k0 = (tc - t * chunks) * 1024 + lane * 32;
    // lane j < nslots holds slot j's row and gamma (row -1: invalid slot)
    int my_row = -1;
    float my_g = 0.0f;
    if (lane < nslots) {
      if (slot_to_row) {
        const int slot = t * k + lane;
        const int e = topk_ids[slot], row = slot_to_row[slot];
        if (e >= 0 && e < E && row >= 0 && row < rows_cap) {
          my_row = row;
          my_g = gamma[e];
        } else if (k0 == lane * 32 && lane % slot_groups == grp) {   // once per slot (first chunk)
          record_error(kWhereQuant, kErrFault);
        }
      } else {
        my_row = t;
        my_g = gamma[0];
      }
    }
    const bool act = k0 < K;
    float v[32];
    float a = 0.0f;
    if (act) {
      load32_bf16(x + (size_t)t * K + k0, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(v[i]));
    }
    for (int j = grp; j < nslots; j += slot_groups) {
      const int row = __shfl_sync(0xffffffffu, my_row, j);
      const float g = __shfl_sync(0xffffffffu, my_g, j);
      if (row < 0 || !act) continue;
      const uint32_t code = block_scale_code(g, a);
      *reinterpret_cast<uint4*>(codes + (size_t)row * (K / 2) + k0 / 2) = quant32(v, block_step(code, g), code == 0);
      scales[mma_scale_offset(row, k0 / 32, KB)] = (uint8_t)code;
    }
  }
}

// SwiGLU + requantisation: one warp per routed slot; per 1024-element chunk
// of h, lane l the scale block [1024 c + 32 l, +32); the slot's expert and
// row come from the routing arrays.  With amax_bits set (calibration) the
// per-expert amax of h is accumulated instead.  gu_layout gives the column
// order of y_gu: 0 = [gate 0..I) | up 0..I)], 1 = per 128 columns 64 gate
// features then the same 64 up features (the kernel row order of weights
// packed with MOESQ_LAYOUT_SWIGLU).
__global__ void __launch_bounds__(256) swiglu_quant_kernel(const uint16_t* __restrict__ y_gu, int I, int R, int E,
                                                           const int32_t* __restrict__ topk_ids,
                                                           const int32_t* __restrict__ slot_to_row, int rows_cap,
                                                           const float* __restrict__ gamma_h,
                                                           uint8_t* __restrict__ h_codes, uint8_t* __restrict__ h_scales,
                                                           unsigned int* __restrict__ amax_bits, int gu_layout) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int wstride = gridDim.x * (blockDim.x >> 5);
  for (int slot = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); slot < R; slot += wstride) {
    const int e = topk_ids[slot];
    const int row = slot_to_row[slot];
    if (e < 0 || e >= E || row < 0 || row >= rows_cap) {
      if (lane == 0) record_error(kWhereSwiglu, kErrFault);
      continue;
    }
    const uint16_t* yr = y_gu + (size_t)row * (2 * I);
    const float g_h = amax_bits ? 0.0f : gamma_h[e];
    float amax = 0.0f;
    for (int c0 = 0; c0 < I; c0 += 1024) {
      const int i0 = c0 + lane * 32;
      if (i0 >= I) continue;
      float h[32], u[32];
      const int gcol = gu_layout ? ((i0 >> 6) << 7) + (i0 & 63) : i0;
      load32_bf16(yr + gcol, h);                        // gate
      load32_bf16(yr + (gu_layout ? gcol + 64 : I + i0), u);   // up
#pragma unroll
      for (int i = 0; i < 32; ++i) h[i] = silu_mul(h[i], u[i]);
      if (amax_bits) {           // calibration: per-expert amax of h
#pragma unroll
        for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(h[i]));
        continue;
      }
      const uint32_t code = quantize_block32(h, g_h, h_codes + (size_t)row * (I / 2) + i0 / 2);
      h_scales[mma_scale_offset(row, i0 / 32, I / 128)] = (uint8_t)code;
    }
    if (amax_bits) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      if (lane == 0) atomicMax(amax_bits + e, __float_as_uint(amax));
    }
  }
}

// Router-weighted combine: one CTA per (token, chunk of up to kCombineCols
// columns).  One thread bulk-copies the chunk of each of the token's k rows
// into shared memory, all completing on one mbarrier (the copies keep many
// bytes in flight per SM without holding registers); then thread i sums
// columns [8 i, 8 i + 8) over the k rows in slot order (fp32, j = 0 .. k-1,
// w_j * y_j) and writes them as bf16.  A slot whose row is outside
// [0, rows_cap) contributes nothing and sets the error word.
constexpr int kCombineCols = 2048;
constexpr int kCombineThreads = kCombineCols / 8;

__global__ void __launch_bounds__(kCombineThreads) combine_kernel(const uint16_t* __restrict__ y, int H, int T, int k,
                                                                  const float* __restrict__ topk_w,
                                                                  const int32_t* __restrict__ slot_to_row,
                                                                  int rows_cap, uint16_t* __restrict__ out,
                                                                  uint64_t timeout_ns) {
  extern __shared__ __align__(128) uint8_t comb_smem[];           // [k][kCombineCols] bf16
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_row[32];
  __shared__ float s_w[32];
  __shared__ int s_abort;
  pdl_trigger();
  pdl_wait();
  const int nch = (H + kCombineCols - 1) / kCombineCols;
  const int t = (int)blockIdx.x / nch;
  const int h0 = ((int)blockIdx.x - t * nch) * kCombineCols;
  const int cols = min(kCombineCols, H - h0);
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x < k) {
    int row = slot_to_row[(size_t)t * k + threadIdx.x];
    if (row < 0 || row >= rows_cap) {
      record_error(kWhereCombine, kErrFault);
      row = -1;
    }
    s_row[threadIdx.x] = row;
    s_w[threadIdx.x] = topk_w[(size_t)t * k + threadIdx.x];
  }
  if (threadIdx.x == 0) {
    s_abort = 0;
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t bytes = 0;
    for (int j = 0; j < k; ++j) bytes += s_row[j] >= 0 ? (uint32_t)cols * 2u : 0u;
    mbar_arrive_expect_tx(b, bytes);
    const uint64_t pol = policy_evict_first();
    for (int j = 0; j < k; ++j)
      if (s_row[j] >= 0)
        bulk_load(smem_u32(comb_smem + (size_t)j * kCombineCols * 2), y + (size_t)s_row[j] * H + h0,
                  (uint32_t)cols * 2u, b, pol);
  }
  const bool ok = mbar_wait(b, 0, timeout_ns, &s_abort);
  if (!ok && threadIdx.x == 0) record_error(kWhereCombine, kErrTimeout);
  const int c = threadIdx.x * 8;
  if (ok && c < cols) {
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
      if (s_row[j] < 0) continue;
      const float wj = s_w[j];
      const uint4 raw = *reinterpret_cast<const uint4*>(comb_smem + ((size_t)j * kCombineCols + c) * 2);
      const uint32_t wd[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float v = (i & 1) ? bf16hi(wd[i >> 1]) : bf16lo(wd[i >> 1]);
        acc[i] = __fadd_rn(acc[i], __fmul_rn(wj, v));
      }
    }
    uint4 o;
    o.x = f32_to_bf16_bits(acc[0]) | (f32_to_bf16_bits(acc[1]) << 16);
    o.y = f32_to_bf16_bits(acc[2]) | (f32_to_bf16_bits(acc[3]) << 16);
    o.z = f32_to_bf16_bits(acc[4]) | (f32_to_bf16_bits(acc[5]) << 16);
    o.w = f32_to_bf16_bits(acc[6]) | (f32_to_bf16_bits(acc[7]) << 16);
    *reinterpret_cast<uint4*>(out + (size_t)t * H + h0 + c) = o;
  }
  if (!ok) {                     // let copies still in flight land before the CTA's memory is reused
    int zero = 0;
    mbar_wait(b, 0, timeout_ns, &zero);
  }
}

// amax of n bf16 values -> atomicMax into *amax_bits (float bits).
__global__ void __launch_bounds__(256) amax_bf16_kernel(const uint16_t* __restrict__ x, int64_t n,
                                                        unsigned int* __restrict__ amax_bits) {
  float a = 0.0f;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += stride)
    a = fmaxf(a, fabsf(__uint_as_float((uint32_t)x[i] << 16)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax_bits, __float_as_uint(a));
}

// Per-expert amax of the tokens routed to each expert (calibration).
__global__ void __launch_bounds__(256) routed_amax_kernel(const uint16_t* __restrict__ x, int T, int K, int k,
                                                          const int32_t* __restrict__ topk_ids, int E,
                                                          unsigned int* __restrict__ amax_bits) {
  const int lane = threadIdx.x & 31;
  const int64_t nslots = (int64_t)T * k;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t slot = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); slot < nslots; slot += wstride) {
    const int e = topk_ids[slot];
    if (e < 0 || e >= E) continue;
    const uint16_t* xr = x + (slot / k) * K;
    float a = 0.0f;
    for (int i = lane; i < K; i += 32) a = fmaxf(a, fabsf(__uint_as_float((uint32_t)xr[i] << 16)));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if (lane == 0) atomicMax(amax_bits + e, __float_as_uint(a));
  }
}

// amax (float bits, in place) -> Eq. 5 gamma.  fill_missing: experts with
// amax 0 take the largest amax over all n entries first.  One CTA.
__global__ void __launch_bounds__(1024) amax_to_gamma_kernel(float* __restrict__ v, int n, int fill_missing) {
  __shared__ float s_max;
  if (threadIdx.x == 0) s_max = 0.0f;
  __syncthreads();
  float a = 0.0f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) a = fmaxf(a, v[i]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
  if ((threadIdx.x & 31) == 0) atomicMax(reinterpret_cast<unsigned int*>(&s_max), __float_as_uint(a));
  __syncthreads();
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    float x = v[i];
    if (fill_missing && !(x > 0.0f)) x = s_max;
    v[i] = nvfp4_global_scale(x);
  }
}

// Watchdog self-test: wait on a barrier that nothing signals.
__global__ void debug_wait_kernel(uint64_t timeout_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(smem_u32(&bar), 1);
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!mbar_wait(smem_u32(&bar), 0, timeout_ns, &abort_flag)) record_error(kWhereDebug, kErrTimeout);
  }
  __syncthreads();
}

}  // namespace moesq
