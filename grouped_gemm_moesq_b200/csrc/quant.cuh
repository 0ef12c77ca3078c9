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

// One warp task = (slot, 256-element chunk).  Dispatch form: slot (t, j)
// writes token t quantised with gamma[topk_ids[slot]] to row slot_to_row[slot].
// Plain form (slot_to_row == nullptr): slot t writes token t to row t with gamma[0].
__global__ void __launch_bounds__(256) quantize_act_kernel(const uint16_t* __restrict__ x, int T, int K, int k,
                                                           const int32_t* __restrict__ topk_ids,
                                                           const int32_t* __restrict__ slot_to_row, int E,
                                                           const float* __restrict__ gamma, int rows_cap,
                                                           uint8_t* __restrict__ codes, uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const int chunks = K / 256;
  const int64_t nslots = slot_to_row ? (int64_t)T * k : (int64_t)T;
  const int64_t ntasks = nslots * chunks;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < ntasks; task += wstride) {
    const int64_t slot = task / chunks;
    const int c = (int)(task % chunks);
    int64_t t, row;
    int e = 0;
    if (slot_to_row) {
      t = slot / k;
      row = slot_to_row[slot];
      e = topk_ids[slot];
      if (e < 0 || e >= E || row < 0 || row >= rows_cap) {
        if (lane == 0) record_error(kWhereQuant, kErrFault);
        continue;
      }
    } else {
      t = slot;
      row = slot;
    }
    const int k0 = c * 256 + lane * 8;
    float v[8];
    load8_bf16(x + t * K + k0, v);
    uint32_t code;
    const uint32_t q = quantize_lane8(v, gamma[e], &code);
    *reinterpret_cast<uint32_t*>(codes + row * (K / 2) + k0 / 2) = q;
    if ((lane & 3) == 0) scales[mma_scale_offset(row, k0 / 32, K / 128)] = (uint8_t)code;
  }
}

// Expert of compact position s: largest e with offsets[e] <= s.
__device__ __forceinline__ int expert_of(const int32_t* __restrict__ offsets, int E, int s) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (offsets[mid] <= s) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// SwiGLU + requantisation: one warp task = (compact row s, 256 outputs).
__global__ void __launch_bounds__(256) swiglu_quant_kernel(const uint16_t* __restrict__ y_gu, int I, int R, int E,
                                                           const int32_t* __restrict__ offsets,
                                                           const int32_t* __restrict__ row_offsets,
                                                           const float* __restrict__ gamma_h,
                                                           uint8_t* __restrict__ h_codes, uint8_t* __restrict__ h_scales,
                                                           unsigned int* __restrict__ amax_bits) {
  const int lane = threadIdx.x & 31;
  const int chunks = I / 256;
  const int64_t ntasks = (int64_t)R * chunks;
  const int64_t wstride = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t task = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); task < ntasks; task += wstride) {
    const int s = (int)(task / chunks);
    const int c = (int)(task % chunks);
    const int e = expert_of(offsets, E, s);
    const int64_t row = row_offsets[e] + (s - offsets[e]);
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
