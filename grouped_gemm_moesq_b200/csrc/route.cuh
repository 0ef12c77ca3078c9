// Routing and dispatch planning: top-k selection with softmax gate weights,
// per-expert counts, compact and expert-aligned offsets and the stable
// (expert, token, slot) permutation.  Integer outputs are exact and
// independent of thread scheduling: ranks come from per-block token bitmaps
// (atomicOr is order-free) and popcounts, never from atomic counters.
#pragma once
#include "common.cuh"

namespace moesq {

constexpr int kRouteTPB = 128;          // tokens per routing block
constexpr int kRouteWords = kRouteTPB / 32;
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

// K1: one warp per token (32 warps, 4 tokens each, per 128-token block):
// top-k by descending logit with ties to the lower id, softmax gate weights
// over all E logits, and the block's per-expert token bitmaps -> per-block
// counts [nblk][E].  Each pick is two warp reductions (max of the ordered
// value, then min of the ids holding it).
__global__ void __launch_bounds__(1024) route_topk_kernel(const float* __restrict__ logits, int T, int E, int k,
                                                          int32_t* __restrict__ topk_ids, float* __restrict__ topk_w,
                                                          int32_t* __restrict__ block_counts) {
  extern __shared__ uint32_t bitmap[];                 // [E][kRouteWords]
  for (int i = threadIdx.x; i < E * kRouteWords; i += blockDim.x) bitmap[i] = 0;
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nwarps = blockDim.x >> 5;
  const int per_lane = (E + 31) >> 5;
  for (int tl = warp; tl < kRouteTPB; tl += nwarps) {
    const int t = blockIdx.x * kRouteTPB + tl;
    if (t >= T) break;
    const float* lr = logits + (size_t)t * E;
    uint32_t o[kRouteMaxPerLane];          // ordered bits; the logit is recovered exactly from them
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < kRouteMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      const float x = (i < per_lane && e < E) ? __ldg(lr + e) : -INFINITY;
      o[i] = (i < per_lane && e < E) ? ordered_bits(x) : 0u;
      mx = fmaxf(mx, x);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float z = 0.0f;
#pragma unroll
    for (int i = 0; i < kRouteMaxPerLane; ++i) {
      const int e = lane + 32 * i;
      if (i < per_lane && e < E) z += expf(from_ordered_bits(o[i]) - mx);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
    uint32_t taken = 0;
    for (int j = 0; j < k; ++j) {
      uint32_t bo = 0;
      int be = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < kRouteMaxPerLane; ++i) {
        const int e = lane + 32 * i;
        if (i < per_lane && e < E && !(taken >> i & 1u) && o[i] > bo) {   // ids ascend with i: > keeps the lowest
          bo = o[i];
          be = e;
        }
      }
      const uint32_t best = __reduce_max_sync(0xffffffffu, bo);
      const int win = __reduce_min_sync(0xffffffffu, (bo == best && be < E) ? be : 0x7fffffff);
      if (win >= E) {                      // only NaN logits leave no candidate
        if (lane == 0) record_error(kWhereRoute, kErrFault);
        break;
      }
      if ((win & 31) == lane) {
        taken |= 1u << (win >> 5);
        topk_ids[(size_t)t * k + j] = win;
        topk_w[(size_t)t * k + j] = __fdiv_rn(expf(from_ordered_bits(bo) - mx), z);
        atomicOr(&bitmap[win * kRouteWords + (tl >> 5)], 1u << (tl & 31));
      }
    }
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
  extern __shared__ uint32_t bitmap[];                 // [E][kRouteWords]
  for (int i = threadIdx.x; i < E * kRouteWords; i += blockDim.x) bitmap[i] = 0;
  __syncthreads();
  const int t0 = blockIdx.x * kRouteTPB;
  const int nslots = min(kRouteTPB, T - t0) * k;
  for (int i = threadIdx.x; i < nslots; i += blockDim.x) {
    const int tl = i / k;
    const int e = topk_ids[(size_t)t0 * k + i];
    atomicOr(&bitmap[e * kRouteWords + (tl >> 5)], 1u << (tl & 31));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < nslots; i += blockDim.x) {
    const int tl = i / k;
    const int slot = t0 * k + i;
    const int e = topk_ids[slot];
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

}  // namespace moesq
