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

// One warp task = (slot, 1024-element chunk of the slot's token): lane l
// quantises the scale block [1024 c + 32 l, +32) of x[t] with the slot's
// expert gamma into the slot's row (the fused dispatch + quantisation).
// Consecutive tasks walk the chunks, then the k slots of a token, so the
// token's row is re-read from L2.  Plain form (slot_to_row == nullptr): one
// slot per token, gamma[0], row = t.
__global__ void __launch_bounds__(256) quantize_act_kernel(const uint16_t* __restrict__ x, int T, int K, int k,
                                                           const int32_t* __restrict__ topk_ids,
                                                           const int32_t* __restrict__ slot_to_row, int E,
                                                           const float* __restrict__ gamma, int rows_cap,
                                                           uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int chunks = (K + 1023) / 1024;
  const int nslots = slot_to_row ? k : 1;
  const int64_t ntasks = (int64_t)T * nslots * chunks;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < ntasks; task += wstride) {
    const int64_t slot = task / chunks;
    const int c = (int)(task - slot * chunks);
    const int64_t t = slot / nslots;
    int64_t row = t;
    float g;
    if (slot_to_row) {
      const int e = topk_ids[slot];
      row = slot_to_row[slot];
      if (e < 0 || e >= E || row < 0 || row >= rows_cap) {
        if (lane == 0) record_error(kWhereQuant, kErrFault);
        continue;
      }
      g = gamma[e];
    } else {
      g = gamma[0];
    }
    const int k0 = c * 1024 + lane * 32;
    if (k0 >= K) continue;
    float v[32];
    load32_bf16(x + t * K + k0, v);
    const uint32_t code = quantize_block32(v, g, codes + row * (K / 2) + k0 / 2);
    scales[mma_scale_offset(row, k0 / 32, K / 128)] = (uint8_t)code;
  }
}

// SwiGLU + requantisation: one warp task = (slot, 1024 outputs), lane l the
// scale block [1024 c + 32 l, +32) of h; the slot's expert and row come from
// the routing arrays.  With amax_bits set (calibration) the per-expert amax
// of h is accumulated instead.
__global__ void __launch_bounds__(256) swiglu_quant_kernel(const uint16_t* __restrict__ y_gu, int I, int R, int E,
                                                           const int32_t* __restrict__ topk_ids,
                                                           const int32_t* __restrict__ slot_to_row, int rows_cap,
                                                           const float* __restrict__ gamma_h,
                                                           uint8_t* __restrict__ h_codes, uint8_t* __restrict__ h_scales,
                                                           unsigned int* __restrict__ amax_bits) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int chunks = (I + 1023) / 1024;
  const int64_t ntasks = (int64_t)R * chunks;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < ntasks; task += wstride) {
    const int64_t slot = task / chunks;
    const int c = (int)(task - slot * chunks);
    const int e = topk_ids[slot];
    const int64_t row = slot_to_row[slot];
    if (e < 0 || e >= E || row < 0 || row >= rows_cap) {
      if (lane == 0) record_error(kWhereSwiglu, kErrFault);
      continue;
    }
    const int i0 = c * 1024 + lane * 32;
    const bool active = i0 < I;
    float h[32];
    if (active) {
      float u[32];
      load32_bf16(y_gu + row * (2 * I) + i0, h);          // gate
      load32_bf16(y_gu + row * (2 * I) + I + i0, u);      // up
      // SiLU(g) = g / (1 + e^-g) in binary32 with the hardware exponential
      // and divide (a few ulp; for g < -88 the denominator overflows and
      // the quotient is 0)
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float sg = __fdividef(h[i], __fadd_rn(1.0f, __expf(-h[i])));
        h[i] = __fmul_rn(sg, u[i]);
      }
    }
    if (amax_bits) {             // calibration: per-expert amax of h
      float a = 0.0f;
      if (active) {
#pragma unroll
        for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(h[i]));
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      if (lane == 0) atomicMax(amax_bits + e, __float_as_uint(a));
      continue;
    }
    if (!active) continue;
    const uint32_t code = quantize_block32(h, gamma_h[e], h_codes + row * (I / 2) + i0 / 2);
    h_scales[mma_scale_offset(row, i0 / 32, I / 128)] = (uint8_t)code;
  }
}

// Router-weighted combine: one warp task = (token, 256 columns).  Lane j < k
// fetches slot j's row and weight; the rows of up to 8 slots are then loaded
// together and summed in slot order (fp32, j = 0 .. k-1).
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y, int H, int T, int k,
                                                      const float* __restrict__ topk_w,
                                                      const int32_t* __restrict__ slot_to_row, int rows_cap,
                                                      uint16_t* __restrict__ out) {
  pdl_trigger();
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int chunks = (H + 255) / 256;
  const int64_t ntasks = (int64_t)T * chunks;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < ntasks; task += wstride) {
    const int64_t t = task / chunks;
    const int h0 = (int)(task % chunks) * 256 + lane * 8;
    const bool active = h0 < H;
    int my_row = -1;
    float my_w = 0.0f;
    if (lane < k) {
      my_row = slot_to_row[t * k + lane];
      my_w = topk_w[t * k + lane];
    }
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j0 = 0; j0 < k; j0 += 8) {
      uint4 raw[8];
      int rows[8];
      float ws[8];
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        rows[jj] = __shfl_sync(0xffffffffu, my_row, (j0 + jj) & 31);
        ws[jj] = __shfl_sync(0xffffffffu, my_w, (j0 + jj) & 31);
        raw[jj] = make_uint4(0u, 0u, 0u, 0u);
        if (active && j0 + jj < k && rows[jj] >= 0 && rows[jj] < rows_cap)
          raw[jj] = __ldg(reinterpret_cast<const uint4*>(y + (int64_t)rows[jj] * H + h0));
      }
#pragma unroll
      for (int jj = 0; jj < 8; ++jj) {
        if (j0 + jj >= k) break;
        if (rows[jj] < 0 || rows[jj] >= rows_cap) {
          if (lane == 0) record_error(kWhereCombine, kErrFault);
          continue;
        }
        const uint32_t wd[4] = {raw[jj].x, raw[jj].y, raw[jj].z, raw[jj].w};
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float v = (i & 1) ? bf16hi(wd[i >> 1]) : bf16lo(wd[i >> 1]);
          acc[i] = __fadd_rn(acc[i], __fmul_rn(ws[jj], v));
        }
      }
    }
    if (!active) continue;
    uint4 o;
    o.x = f32_to_bf16_bits(acc[0]) | (f32_to_bf16_bits(acc[1]) << 16);
    o.y = f32_to_bf16_bits(acc[2]) | (f32_to_bf16_bits(acc[3]) << 16);
    o.z = f32_to_bf16_bits(acc[4]) | (f32_to_bf16_bits(acc[5]) << 16);
    o.w = f32_to_bf16_bits(acc[6]) | (f32_to_bf16_bits(acc[7]) << 16);
    *reinterpret_cast<uint4*>(out + t * H + h0) = o;
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
