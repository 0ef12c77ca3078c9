// Activation-side kernels: NVFP4 quantisation of activations (plain and
// fused with the dispatch scatter), SwiGLU + requantisation, the
// router-weighted combine and the amax reductions behind the static global
// scales.  All are HBM / L2 bound: one warp streams 256 contiguous elements
// (16-byte loads per lane, 4 lanes per 32-element scale block).
#pragma once
#include "common.cuh"

namespace moesq {

// Quantises 8 values held by this lane; the 4 lanes of a 32-element block
// share amax through shuffles.  Returns the 4 code bytes; *code_out gets the
// block's scale code.
__device__ __forceinline__ uint32_t quantize_lane8(const float (&v)[8], float gamma, uint32_t* code_out) {
  float a = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
  a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
  const uint32_t code = block_scale_code(gamma, a);
  *code_out = code;
  return quant8(v, block_step(code, gamma), code == 0);
}

__device__ __forceinline__ void load8_bf16(const uint16_t* p, float (&v)[8]) {
  const uint4 u = __ldg(reinterpret_cast<const uint4*>(p));
  v[0] = bf16lo(u.x); v[1] = bf16hi(u.x); v[2] = bf16lo(u.y); v[3] = bf16hi(u.y);
  v[4] = bf16lo(u.z); v[5] = bf16hi(u.z); v[6] = bf16lo(u.w); v[7] = bf16hi(u.w);
}

// One warp task = (token t, 256-element chunk).  The chunk of x[t] is read
// once and the block amax computed once; it is then quantised for each of
// the token's k slots with that slot's expert gamma and written to the
// slot's row (the fused dispatch + quantisation).  Plain form
// (slot_to_row == nullptr): k = 1, gamma[0], row = t.
__global__ void __launch_bounds__(256) quantize_act_kernel(const uint16_t* __restrict__ x, int T, int K, int k,
                                                           const int32_t* __restrict__ topk_ids,
                                                           const int32_t* __restrict__ slot_to_row, int E,
                                                           const float* __restrict__ gamma, int rows_cap,
                                                           uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int chunks = K / 256;
  const int64_t ntasks = (int64_t)T * chunks;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < ntasks; task += wstride) {
    const int64_t t = task / chunks;
    const int c = (int)(task - t * chunks);
    const int k0 = c * 256 + lane * 8;
    // lane j < k holds slot j's row and gamma
    int64_t my_row = t;
    float my_gamma = 0.0f;
    bool my_ok = true;
    if (slot_to_row) {
      if (lane < k) {
        const int e = topk_ids[t * k + lane];
        my_row = slot_to_row[t * k + lane];
        my_ok = e >= 0 && e < E && my_row >= 0 && my_row < rows_cap;
        my_gamma = my_ok ? gamma[e] : 0.0f;
      }
    } else if (lane == 0) {
      my_gamma = gamma[0];
    }
    float v[8];
    load8_bf16(x + t * K + k0, v);
    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    const int nslots = slot_to_row ? k : 1;
    for (int j = 0; j < nslots; ++j) {
      const int64_t row = __shfl_sync(0xffffffffu, my_row, j);
      const float g = __shfl_sync(0xffffffffu, my_gamma, j);
      const bool ok = __shfl_sync(0xffffffffu, my_ok ? 1 : 0, j) != 0;
      if (!ok) {
        if (lane == 0) record_error(kWhereQuant, kErrFault);
        continue;
      }
      const uint32_t code = block_scale_code(g, a);
      const uint32_t q = quant8(v, block_step(code, g), code == 0);
      *reinterpret_cast<uint32_t*>(codes + row * (K / 2) + k0 / 2) = q;
      if ((lane & 3) == 0) scales[mma_scale_offset(row, k0 / 32, K / 128)] = (uint8_t)code;
    }
  }
}

// SwiGLU + requantisation: one warp task = (slot, 256 outputs); the slot's
// expert and row come from the routing arrays.
__global__ void __launch_bounds__(256) swiglu_quant_kernel(const uint16_t* __restrict__ y_gu, int I, int R, int E,
                                                           const int32_t* __restrict__ topk_ids,
                                                           const int32_t* __restrict__ slot_to_row, int rows_cap,
                                                           const float* __restrict__ gamma_h,
                                                           uint8_t* __restrict__ h_codes, uint8_t* __restrict__ h_scales,
                                                           unsigned int* __restrict__ amax_bits) {
  const int lane = threadIdx.x & 31;
  const int chunks = I / 256;
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
    const int i0 = c * 256 + lane * 8;
    float g[8], u[8], h[8];
    load8_bf16(y_gu + row * (2 * I) + i0, g);
    load8_bf16(y_gu + row * (2 * I) + I + i0, u);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float sg = __fdiv_rn(g[i], __fadd_rn(1.0f, expf(-g[i])));
      h[i] = __fmul_rn(sg, u[i]);
    }
    if (amax_bits) {             // calibration: per-expert amax of h
      float a = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(h[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
      if (lane == 0) atomicMax(amax_bits + e, __float_as_uint(a));
      continue;
    }
    uint32_t code;
    const uint32_t q = quantize_lane8(h, gamma_h[e], &code);
    *reinterpret_cast<uint32_t*>(h_codes + row * (I / 2) + i0 / 2) = q;
    if ((lane & 3) == 0) h_scales[mma_scale_offset(row, i0 / 32, I / 128)] = (uint8_t)code;
  }
}

// Router-weighted combine: one warp task = (token, 256 columns).
__global__ void __launch_bounds__(256) combine_kernel(const uint16_t* __restrict__ y, int H, int T, int k,
                                                      const float* __restrict__ topk_w,
                                                      const int32_t* __restrict__ slot_to_row, int rows_cap,
                                                      uint16_t* __restrict__ out) {
  const int lane = threadIdx.x & 31;
  const int chunks = (H + 255) / 256;
  const int64_t ntasks = (int64_t)T * chunks;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < ntasks; task += wstride) {
    const int64_t t = task / chunks;
    const int h0 = (int)(task % chunks) * 256 + lane * 8;
    if (h0 >= H) continue;
    float acc[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    for (int j = 0; j < k; ++j) {
      const int64_t row = slot_to_row[t * k + j];
      if (row < 0 || row >= rows_cap) { record_error(kWhereCombine, kErrFault); continue; }
      const float w = topk_w[t * k + j];
      float v[8];
      load8_bf16(y + row * H + h0, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] = __fadd_rn(acc[i], __fmul_rn(w, v[i]));
    }
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
