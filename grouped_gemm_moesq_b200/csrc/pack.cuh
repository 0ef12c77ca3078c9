// Weight packing: bf16 expert weights -> paired-4:8 sparse NVFP4.
//
// Support: per group of 8 K elements keep the two pairs of largest
// w0^2 + w1^2 (binary32), an exact tie keeping the lower pair index
// (paper App. A Eq. 6 pattern set; model card "exactly 2 pairs are kept").
// Scales: paper Sec. 3.4 Eq. 5 on the masked weights; values: Eq. 3.
// Outputs the storage form of the model card (values / mask / scales /
// gamma) and the kernel form read by the grouped GEMM (ktiles).  Also the
// converters between dense NVFP4 codes and that storage form (the model
// card's canonical rule for chunks with fewer than two nonzero bytes).
#pragma once
#include "common.cuh"

namespace moesq {

// Kept-pair bitmask (bit p = pair p) of one group of 8 values.
__device__ __forceinline__ uint32_t select_pairs(const float (&w)[8]) {
  float s[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) s[p] = __fadd_rn(__fmul_rn(w[2 * p], w[2 * p]), __fmul_rn(w[2 * p + 1], w[2 * p + 1]));
  uint32_t bits = 0;
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    int beaten = 0;
#pragma unroll
    for (int q = 0; q < 4; ++q)
      if (q != p && (s[q] > s[p] || (s[q] == s[p] && q < p))) ++beaten;
    if (beaten < 2) bits |= 1u << p;
  }
  return bits;
}

__device__ __forceinline__ void load_group(const uint16_t* src, float (&w)[8]) {
  uint4 v = *reinterpret_cast<const uint4*>(src);
  w[0] = bf16lo(v.x); w[1] = bf16hi(v.x); w[2] = bf16lo(v.y); w[3] = bf16hi(v.y);
  w[4] = bf16lo(v.z); w[5] = bf16hi(v.z); w[6] = bf16lo(v.w); w[7] = bf16hi(v.w);
}

// Pass 1: largest kept |w| per expert, accumulated as float bits (>= 0) with
// atomicMax into amax_bits[e].  One thread per group of 8.
__global__ void pack_amax_kernel(const uint16_t* __restrict__ w, int64_t n_groups,
                                 int64_t groups_per_expert, unsigned int* __restrict__ amax_bits) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g - (threadIdx.x & 31) < n_groups;
       g += stride) {
    float a = 0.0f;
    int64_t e = -1;
    if (g < n_groups) {
      float v[8];
      load_group(w + g * 8, v);
      uint32_t bits = select_pairs(v);
#pragma unroll
      for (int p = 0; p < 4; ++p)
        if (bits >> p & 1u) a = fmaxf(a, fmaxf(fabsf(v[2 * p]), fabsf(v[2 * p + 1])));
      e = g / groups_per_expert;
    }
    // groups_per_expert is a multiple of 32: a warp never spans two experts
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0 && e >= 0) atomicMax(amax_bits + e, __float_as_uint(a));
  }
}

// amax bits -> gamma (Eq. 5), in place.
__global__ void pack_gamma_kernel(float* __restrict__ gamma, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) gamma[i] = nvfp4_global_scale(gamma[i]);   // gamma[i] holds amax here
}

// Kernel-form tile of 128 weight rows x 256 dense K (see include/moesq.h).
constexpr int kKTileBytes = 11264;
constexpr int kKTileMeta = 8192;
constexpr int kKTileScales = 10240;

struct PackOut {
  uint8_t* values;    // [E][M][K/4]
  uint8_t* mask;      // [E][M][K/16]
  uint8_t* scales;    // [E][M][K/32]
  const float* gamma; // [E]
  uint8_t* ktiles;    // [E][M/128][K/256][kKTileBytes]
  int layout;         // kernel row order: 0 = as stored, 1 = gate/up interleaved by 64 rows
};

// Kernel-form row of storage row m of an M-row gate_up linear under layout
// 1: block b of 128 kernel rows holds gate rows [64 b, 64 b + 64) and then
// up rows M/2 + [64 b, 64 b + 64), so that one 128-row weight tile of the
// GEMM produces both halves of 64 SwiGLU features.
__device__ __forceinline__ int kernel_row(int m, int M, int layout) {
  if (!layout) return m;
  const int I = M >> 1;
  const int up = m >= I ? 1 : 0;
  const int f = m - up * I;
  return ((f >> 6) << 7) + up * 64 + (f & 63);
}

// Writes one 32-element block of an expert linear's packed form: the 8 code
// bytes (the two kept pairs of each of its 4 groups, in K order), the 4 pair
// bitmasks and the scale code, in the storage form and in the kernel-form
// tile (swizzled values, metadata nibbles i0 | i1 << 2 of the two kept pair
// indices, scales in the MMA layout).
__device__ __forceinline__ void store_block(const PackOut& out, int e, int m, int b, int M, int K, uint2 vbytes,
                                            const uint32_t (&bits4)[4], uint32_t code) {
  const int nb_row = K / 32, KT = K / 256, MB = M / 128;
  const int64_t row = (int64_t)e * M + m;
  *reinterpret_cast<uint2*>(out.values + row * (K / 4) + (int64_t)b * 8) = vbytes;
  const uint16_t mk = (uint16_t)(bits4[0] | (bits4[1] << 4) | (bits4[2] << 8) | (bits4[3] << 12));
  *reinterpret_cast<uint16_t*>(out.mask + row * (K / 16) + (int64_t)b * 2) = mk;
  out.scales[row * nb_row + b] = (uint8_t)code;
  uint32_t meta = 0;
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    const uint32_t bits = bits4[g];
    const uint32_t i0 = __ffs(bits) - 1;
    const uint32_t i1 = 31 - __clz(bits);
    meta |= (i0 | (i1 << 2)) << (4 * g);
  }
  const int mk_row = kernel_row(m, M, out.layout);
  const int mb = mk_row >> 7, r = mk_row & 127;
  const int kt = b >> 3, bt = b & 7;            // 32-block within the 256-wide K tile
  uint8_t* tile = out.ktiles + (((int64_t)e * MB + mb) * KT + kt) * kKTileBytes;
  const int chunk = (bt >> 1) ^ ((r >> 1) & 3);  // 16-byte chunk after the swizzle
  *reinterpret_cast<uint2*>(tile + r * 64 + chunk * 16 + (bt & 1) * 8) = vbytes;
  *reinterpret_cast<uint16_t*>(tile + kKTileMeta + r * 16 + bt * 2) = (uint16_t)meta;
  tile[kKTileScales + (bt >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (bt & 3)] = (uint8_t)code;
}

// Pass 2: one thread per 32-element block (4 groups, 16 kept values).
__global__ void pack_blocks_kernel(const uint16_t* __restrict__ w, int e_begin, int64_t n_blocks, int M,
                                   int K, PackOut out) {
  const int nb_row = K / 32;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_blocks; t += stride) {
    const int b = (int)(t % nb_row);
    const int64_t row_local = t / nb_row;          // e_local * M + m
    const int e = e_begin + (int)(row_local / M);
    const int m = (int)(row_local % M);
    const uint16_t* src = w + row_local * K + (int64_t)b * 32;

    float kept[16];                                 // kept values of the block, K order
    uint32_t bits4[4];
    float amax = 0.0f;
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      float v[8];
      load_group(src + 8 * g, v);
      uint32_t bits = select_pairs(v);
      bits4[g] = bits;
      int slot = 0;
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        if (bits >> p & 1u) {
          // slot is 0 or 1; written without dynamic register indexing
          float x0 = v[2 * p], x1 = v[2 * p + 1];
          if (slot == 0) { kept[4 * g + 0] = x0; kept[4 * g + 1] = x1; }
          else           { kept[4 * g + 2] = x0; kept[4 * g + 3] = x1; }
          amax = fmaxf(amax, fmaxf(fabsf(x0), fabsf(x1)));
          ++slot;
        }
      }
    }
    const float gamma = out.gamma[e];
    const uint32_t code = block_scale_code(gamma, amax);
    const float s_b = block_step(code, gamma);
    float h0[8], h1[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) { h0[i] = kept[i]; h1[i] = kept[8 + i]; }
    uint2 vbytes;
    vbytes.x = quant8(h0, s_b, code == 0);
    vbytes.y = quant8(h1, s_b, code == 0);

    store_block(out, e, m, b, M, K, vbytes, bits4, code);
  }
}

// Dense NVFP4 codes of a tensor in the paired pattern -> pair-bitmask storage
// and kernel form (model card, pair-bitmask v1): per 4-byte chunk the nonzero
// bytes are kept; a chunk with fewer than 2 nonzero bytes keeps its
// lowest-index zero bytes as well.  A chunk with more than 2 nonzero bytes is
// not in the pattern: the device error word is set and its lowest two
// nonzero bytes are kept.  One thread per 32-element block.
__global__ void import_dense_kernel(const uint8_t* __restrict__ codes, const uint8_t* __restrict__ scales,
                                    const float* __restrict__ gamma_in, int e_begin, int64_t n_blocks, int M, int K,
                                    PackOut out, float* __restrict__ gamma_out) {
  const int nb_row = K / 32;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_blocks; t += stride) {
    const int b = (int)(t % nb_row);
    const int64_t row_local = t / nb_row;
    const int e_local = (int)(row_local / M);
    const int m = (int)(row_local % M);
    const uint4 raw = *reinterpret_cast<const uint4*>(codes + row_local * (K / 2) + (int64_t)b * 16);
    const uint32_t words[4] = {raw.x, raw.y, raw.z, raw.w};
    uint32_t bits4[4], kept2[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t w = words[g];
      uint32_t nz = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) nz |= ((w >> (8 * i)) & 0xFFu) != 0u ? (1u << i) : 0u;
      if (__popc(nz) > 2) {                    // not in the pattern: keep the lowest two
        record_error(kWhereConvert, kErrFault);
        const uint32_t lo = nz & (0u - nz);
        const uint32_t rest = nz & ~lo;
        nz = lo | (rest & (0u - rest));
      }
      // fewer than two nonzero bytes: add the lowest-index zero bytes
      if (__popc(nz) < 2) nz |= ~nz & (nz + 1u);
      if (__popc(nz) < 2) nz |= ~nz & (nz + 1u);
      bits4[g] = nz;
      const uint32_t i0 = __ffs(nz) - 1, i1 = 31 - __clz(nz);
      kept2[g] = ((w >> (8 * i0)) & 0xFFu) | (((w >> (8 * i1)) & 0xFFu) << 8);
    }
    const uint2 vbytes = make_uint2(kept2[0] | (kept2[1] << 16), kept2[2] | (kept2[3] << 16));
    const uint32_t code = scales[row_local * nb_row + b];
    store_block(out, e_begin + e_local, m, b, M, K, vbytes, bits4, code);
    if (m == 0 && b == 0) gamma_out[e_begin + e_local] = gamma_in[e_local];
  }
}

// Pair-bitmask storage form -> dense NVFP4 codes [E][M][K/2] (the kept bytes
// at their chunk positions, zeros elsewhere).  One thread per 32-element block.
__global__ void export_dense_kernel(const uint8_t* __restrict__ values, const uint8_t* __restrict__ mask,
                                    int64_t n_blocks, int K, uint8_t* __restrict__ codes) {
  const int nb_row = K / 32;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_blocks; t += stride) {
    const int b = (int)(t % nb_row);
    const int64_t row = t / nb_row;
    const uint2 v = *reinterpret_cast<const uint2*>(values + row * (K / 4) + (int64_t)b * 8);
    const uint32_t mk = *reinterpret_cast<const uint16_t*>(mask + row * (K / 16) + (int64_t)b * 2);
    const uint32_t kept2[4] = {v.x & 0xFFFFu, v.x >> 16, v.y & 0xFFFFu, v.y >> 16};
    uint32_t words[4];
#pragma unroll
    for (int g = 0; g < 4; ++g) {
      const uint32_t nz = (mk >> (4 * g)) & 0xFu;
      if (__popc(nz) != 2) record_error(kWhereConvert, kErrFault);
      const uint32_t i0 = nz ? __ffs(nz) - 1 : 0, i1 = nz ? 31 - __clz(nz) : 1;
      words[g] = ((kept2[g] & 0xFFu) << (8 * i0)) | ((kept2[g] >> 8) << (8 * i1));
    }
    *reinterpret_cast<uint4*>(codes + row * (K / 2) + (int64_t)b * 16) = make_uint4(words[0], words[1], words[2],
                                                                                   words[3]);
  }
}

}  // namespace moesq
