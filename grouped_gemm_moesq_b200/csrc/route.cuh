// Routing and dispatch planning: top-k selection with softmax gate weights,
// per-expert counts, compact and expert-aligned offsets and the stable
// (expert, token, slot) permutation.  Integer outputs are exact and
// independent of thread scheduling: ranks come from per-block token bitmaps
// (atomicOr is order-free) and popcounts, never from atomic counters.
// Kernels: route_topk_kernel (one warp per token), then either
// route_finish_kernel (one CTA, T <= kRouteSmallMaxT) or route_count_kernel,
// route_scan_kernel and route_scatter_kernel (blocks of kRouteTPB tokens).
#pragma once
#include "common.cuh"

namespace moesq {

constexpr int kRouteTPB = 128;          // tokens per routing block
constexpr int kRouteWords = kRouteTPB / 32;
constexpr int kRouteSmallMaxT = 512;     // tokens whose counts / scan / scatter one CTA does
constexpr int kRouteMaxE = 512;
constexpr int kRouteMaxPerLane = kRouteMaxE / 32;

// Order-preserving map of a finite float to uint32 (-0 maps like +0; NaN
// maps to 0 and is never chosen while a number is left).
__device__ __forceinline__ uint32_t ordered_bits(float v) {
  if (v != v) return 0u;
  const uint32_t u = __float_as_uint(v == 0.0f ? 0.0f : v);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float from_ordered_bits(uint32_t o) {
  return __uint_as_float((o & 0x80000000u) ? (o & 0x7fffffffu) : ~o);
}

// Top-k of one token by one warp: PL logits per lane (lane + 32 i), softmax
// over all E, k picks by descending logit with ties to the lower id.  Each
// pick is two warp reductions (max of the ordered value, then min of the ids
// holding it).  Lane (id % 32) of each pick writes ids / weights and, when
// bitmap != nullptr, sets the token's bit (token index tl in its block; the
// bitmap holds `words` 32-bit words per expert).
template <int PL>
__device__ __forceinline__ void topk_one_token(const float* __restrict__ lr, int E, int k, int lane,
                                               int32_t* __restrict__ ids_out, float* __restrict__ w_out,
                                               uint32_t* bitmap, int words, int tl) {
  uint32_t o[PL];                        // ordered bits; the logit is recovered exactly from them
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < PL; ++i) {
    const int e = lane + 32 * i;
    const float x = (e < E) ? __ldg(lr + e) : -INFINITY;
    o[i] = (e < E) ? ordered_bits(x) : 0u;
    mx = fmaxf(mx, x);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float z = 0.0f;
#pragma unroll
  for (int i = 0; i < PL; ++i)
    if (lane + 32 * i < E) z += expf(from_ordered_bits(o[i]) - mx);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
  for (int j = 0; j < k; ++j) {
    uint32_t bo = 0;
    int be = 0x7fffffff;
#pragma unroll
    for (int i = 0; i < PL; ++i)
      if (o[i] > bo) { bo = o[i]; be = lane + 32 * i; }   // ids ascend with i: > keeps the lowest
    const uint32_t best = __reduce_max_sync(0xffffffffu, bo);
    const int win = __reduce_min_sync(0xffffffffu, (bo == best && be < E) ? be : 0x7fffffff);
    if (win >= E) {                      // only NaN logits leave no candidate
      // picks j .. k-1 get the sentinel id -1 (weight 0): the counting and
      // scatter kernels skip it, and the quantiser, SwiGLU and combine
      // report the slot through the error word
      if (lane == 0) {
        record_error(kWhereRoute, kErrFault);
        for (int jj = j; jj < k; ++jj) { ids_out[jj] = -1; w_out[jj] = 0.0f; }
      }
      return;
    }
    if ((win & 31) == lane) {
#pragma unroll
      for (int i = 0; i < PL; ++i)
        if (i == (win >> 5)) o[i] = 0u;  // taken
      ids_out[j] = win;
      w_out[j] = __fdiv_rn(expf(from_ordered_bits(best) - mx), z);
      if (bitmap) atomicOr(&bitmap[win * words + (tl >> 5)], 1u << (tl & 31));
    }
  }
}

// K1: one warp per token over the whole grid: ids and gate weights.
template <int PL>
__global__ void __launch_bounds__(256) route_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                         int32_t* __restrict__ topk_ids, float* __restrict__ topk_w) {
  pdl_trigger();
  pdl_wait();
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t >= T) return;
  topk_one_token<PL>(logits + (size_t)t * E, E, k, threadIdx.x & 31, topk_ids + (size_t)t * k,
                     topk_w + (size_t)t * k, nullptr, 0, 0);
}

// K1b: per 128-token block, per-expert counts from the block's token bitmaps.
__global__ void __launch_bounds__(256) route_count_kernel(int T, int E, int k, const int32_t* __restrict__ topk_ids,
                                                          int32_t* __restrict__ block_counts) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint32_t bitmap[];                 // [E][kRouteWords]
  for (int i = threadIdx.x; i < E * kRouteWords; i += blockDim.x) bitmap[i] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kRouteTPB;
  const int nslots = min(kRouteTPB, T - t0) * k;
  for (int i = threadIdx.x; i < nslots; i += blockDim.x) {
    const int tl = i / k;
    const int e = topk_ids[(size_t)t0 * k + i];
    if (e >= 0 && e < E) atomicOr(&bitmap[e * kRouteWords + (tl >> 5)], 1u << (tl & 31));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
#pragma unroll
    for (int w = 0; w < kRouteWords; ++w) c += __popc(bitmap[e * kRouteWords + w]);
    block_counts[(size_t)blockIdx.x * E + e] = c;
  }
}

// K2 (one CTA): per-expert totals, per-block exclusive bases (in place in
// block_counts), compact offsets and 128-aligned row offsets.
__global__ void __launch_bounds__(1024) route_scan_kernel(int32_t* __restrict__ block_counts, int nblk, int E,
                                                          int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                          int32_t* __restrict__ row_offsets) {
  pdl_trigger();
  pdl_wait();
  __shared__ int32_t s_cnt[kRouteMaxE];
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int run = 0;
    int b = 0;
    for (; b + 8 <= nblk; b += 8) {
      int c[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) c[u] = block_counts[(size_t)(b + u) * E + e];
#pragma unroll
      for (int u = 0; u < 8; ++u) { block_counts[(size_t)(b + u) * E + e] = run; run += c[u]; }
    }
    for (; b < nblk; ++b) {
      const int c = block_counts[(size_t)b * E + e];
      block_counts[(size_t)b * E + e] = run;
      run += c;
    }
    s_cnt[e] = run;
    counts[e] = run;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = (E + 31) / 32;
    const int e0 = lane * per;
    int sc = 0, sr = 0;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) { sc += s_cnt[e]; sr += (s_cnt[e] + 127) & ~127; }
    }
    int ic = sc, ir = sr;                      // inclusive warp scan of the lane sums
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int tc = __shfl_up_sync(0xffffffffu, ic, o);
      const int tr = __shfl_up_sync(0xffffffffu, ir, o);
      if (lane >= o) { ic += tc; ir += tr; }
    }
    int oc = ic - sc, orr = ir - sr;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) {
        offsets[e] = oc;
        row_offsets[e] = orr;
        oc += s_cnt[e];
        orr += (s_cnt[e] + 127) & ~127;
      }
    }
    if (lane == 31) { offsets[E] = ic; row_offsets[E] = ir; }
  }
}

// K3: stable scatter.  Rank of slot (t, j) within expert e = number of
// tokens before t (in this block) routed to e, from the block bitmap.
__global__ void __launch_bounds__(256) route_scatter_kernel(int T, int E, int k, const int32_t* __restrict__ topk_ids,
                                                            const int32_t* __restrict__ block_base,
                                                            const int32_t* __restrict__ offsets,
                                                            const int32_t* __restrict__ row_offsets,
                                                            int32_t* __restrict__ sorted_to_slot,
                                                            int32_t* __restrict__ slot_to_row) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint32_t bitmap[];                 // [E][kRouteWords]
  for (int i = threadIdx.x; i < E * kRouteWords; i += blockDim.x) bitmap[i] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kRouteTPB;
  const int nslots = min(kRouteTPB, T - t0) * k;
  for (int i = threadIdx.x; i < nslots; i += blockDim.x) {
    const int tl = i / k;
    const int e = topk_ids[(size_t)t0 * k + i];
    if (e >= 0 && e < E) atomicOr(&bitmap[e * kRouteWords + (tl >> 5)], 1u << (tl & 31));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nslots; i += blockDim.x) {
    const int tl = i / k;
    const int slot = t0 * k + i;
    const int e = topk_ids[slot];
    if (e < 0 || e >= E) {               // not counted: the slot has no row
      slot_to_row[slot] = -1;
      continue;
    }
    int rank = 0;
#pragma unroll
    for (int w = 0; w < kRouteWords; ++w) {
      const uint32_t word = bitmap[e * kRouteWords + w];
      if (w < (tl >> 5)) rank += __popc(word);
      else if (w == (tl >> 5)) rank += __popc(word & ((1u << (tl & 31)) - 1u));
    }
    const int local = block_base[(size_t)blockIdx.x * E + e] + rank;
    sorted_to_slot[offsets[e] + local] = slot;
    slot_to_row[slot] = row_offsets[e] + local;
  }
}

// Single-CTA finish of the routing for few tokens: from the top-k ids of
// route_topk_kernel, the expert bitmaps (words = ceil(T / 32) words per
// expert), counts, offsets and the stable scatter in one launch, with the
// same arithmetic as the multi-kernel path.
__global__ void __launch_bounds__(1024) route_finish_kernel(int T, int E, int k, const int32_t* __restrict__ topk_ids,
                                                            int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                                                            int32_t* __restrict__ row_offsets,
                                                            int32_t* __restrict__ sorted_to_slot,
                                                            int32_t* __restrict__ slot_to_row, int words) {
  pdl_trigger();
  pdl_wait();
  extern __shared__ uint32_t bitmap[];                 // [E][words]
  __shared__ int32_t s_cnt[kRouteMaxE];
  __shared__ int32_t s_off[kRouteMaxE];
  __shared__ int32_t s_roff[kRouteMaxE];
  for (int i = threadIdx.x; i < E * words; i += blockDim.x) bitmap[i] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < T * k; i += blockDim.x) {
    const int e = topk_ids[i], tl = i / k;
    if (e >= 0 && e < E) atomicOr(&bitmap[e * words + (tl >> 5)], 1u << (tl & 31));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    int c = 0;
    for (int w = 0; w < words; ++w) c += __popc(bitmap[e * words + w]);
    s_cnt[e] = c;
    counts[e] = c;
  }
  __syncthreads();
  if (warp == 0) {
    const int per = (E + 31) / 32, e0 = lane * per;
    int sc = 0, sr = 0;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) { sc += s_cnt[e]; sr += (s_cnt[e] + 127) & ~127; }
    }
    int ic = sc, ir = sr;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int tc = __shfl_up_sync(0xffffffffu, ic, off);
      const int tr = __shfl_up_sync(0xffffffffu, ir, off);
      if (lane >= off) { ic += tc; ir += tr; }
    }
    int oc = ic - sc, orr = ir - sr;
    for (int i = 0; i < per; ++i) {
      const int e = e0 + i;
      if (e < E) {
        s_off[e] = oc;
        s_roff[e] = orr;
        offsets[e] = oc;
        row_offsets[e] = orr;
        oc += s_cnt[e];
        orr += (s_cnt[e] + 127) & ~127;
      }
    }
    if (lane == 31) { offsets[E] = ic; row_offsets[E] = ir; }
  }
  __syncthreads();
  const int nslots = T * k;
  for (int i = threadIdx.x; i < nslots; i += blockDim.x) {
    const int tl = i / k;
    const int e = topk_ids[i];
    if (e < 0 || e >= E) {               // not counted: the slot has no row
      slot_to_row[i] = -1;
      continue;
    }
    int rank = 0;
    for (int w = 0; w < (tl >> 5); ++w) rank += __popc(bitmap[e * words + w]);
    rank += __popc(bitmap[e * words + (tl >> 5)] & ((1u << (tl & 31)) - 1u));
    sorted_to_slot[s_off[e] + rank] = i;
    slot_to_row[i] = s_roff[e] + rank;
  }
}

}  // namespace moesq
