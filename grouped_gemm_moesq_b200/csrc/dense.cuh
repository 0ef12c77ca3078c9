// Dense NVFP4 control: the baseline the paper measures its sparse kernel
// against (App. D.2, "Dense (transposed)": the same kernel orientation,
// differing only in sparsity).  Every weight is kept and quantised with one
// UE4M3 scale per 16 K elements (the NVFP4 group) under Eq. 5's per-tensor
// gamma (over the whole, unpruned expert linear); values by Eq. 3.
//
// Storage form: codes [E][M][K/2] (element 2i in the low nibble of byte i),
// scales [E][M][K/16] (UE4M3, row-major), gamma [E].  Kernel form: per
// (expert, 128-row block, 256-wide K step) an 18 KB tile: bytes 0-16383 the
// 128 rows of codes (128 B each) in the 128-byte swizzle the MMA's
// shared-memory descriptor expects (16-byte chunk c of row r at chunk
// c ^ (r & 7)), bytes 16384-18431 the scales of the four 64-wide K chunks in
// the MMA scale layout (chunk j, row 32 a + b, 16-wide group s at
// j * 512 + b * 16 + a * 4 + s).
#pragma once
#include "common.cuh"
#include "pack.cuh"

namespace moesq {

constexpr int kDTileBytes = 18432;
constexpr int kDTileScales = 16384;

struct DensePackOut {
  uint8_t* codes;     // [E][M][K/2]
  uint8_t* scales;    // [E][M][K/16]
  const float* gamma; // [E]
  uint8_t* dtiles;    // [E][M/128][K/256][kDTileBytes]
};

// Pass 1: largest |w| per expert (float bits, atomicMax).  One thread per
// group of 8; groups_per_expert is a multiple of 32.
__global__ void dense_amax_kernel(const uint16_t* __restrict__ w, int64_t n_groups, int64_t groups_per_expert,
                                  unsigned int* __restrict__ amax_bits) {
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g - (threadIdx.x & 31) < n_groups;
       g += stride) {
    float a = 0.0f;
    int64_t e = -1;
    if (g < n_groups) {
      float v[8];
      load_group(w + g * 8, v);
#pragma unroll
      for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
      e = g / groups_per_expert;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0 && e >= 0) atomicMax(amax_bits + e, __float_as_uint(a));
  }
}

// Pass 2: one thread per 16-element group: scale code, 8 code bytes, in the
// storage form and the kernel-form tile.
__global__ void dense_pack_kernel(const uint16_t* __restrict__ w, int e_begin, int64_t n_groups, int M, int K,
                                  DensePackOut out) {
  const int ng_row = K / 16, KT = K / 256, MB = M / 128;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n_groups; t += stride) {
    const int g = (int)(t % ng_row);
    const int64_t row_local = t / ng_row;          // e_local * M + m
    const int e = e_begin + (int)(row_local / M);
    const int m = (int)(row_local % M);
    float v0[8], v1[8];
    load_group(w + row_local * K + (int64_t)g * 16, v0);
    load_group(w + row_local * K + (int64_t)g * 16 + 8, v1);
    float amax = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fmaxf(fabsf(v0[i]), fabsf(v1[i])));
    const float gamma = out.gamma[e];
    const uint32_t code = block_scale_code(gamma, amax);
    const float s_b = block_step(code, gamma);
    const uint2 bytes = make_uint2(quant8(v0, s_b, code == 0), quant8(v1, s_b, code == 0));
    const int64_t row = (int64_t)e * M + m;
    *reinterpret_cast<uint2*>(out.codes + row * (K / 2) + (int64_t)g * 8) = bytes;
    out.scales[row * ng_row + g] = (uint8_t)code;
    const int mb = m >> 7, r = m & 127;
    const int kt = g >> 4, gt = g & 15;            // 16-group within the 256-wide K step
    uint8_t* tile = out.dtiles + (((int64_t)e * MB + mb) * KT + kt) * kDTileBytes;
    const int chunk = (gt >> 1) ^ (r & 7);         // 16-byte chunk after the swizzle
    *reinterpret_cast<uint2*>(tile + r * 128 + chunk * 16 + (gt & 1) * 8) = bytes;
    tile[kDTileScales + (gt >> 2) * 512 + (r & 31) * 16 + (r >> 5) * 4 + (gt & 3)] = (uint8_t)code;
  }
}

// Activation scales, one UE4M3 code per 32 K in the MMA scale layout
// [R/128][K/128][512], -> one per 16 K (each code twice) in the layout the
// dense MMA reads, [R/128][K/64][512] (chunk j of 64 K, row 32 a + b,
// 16-group s at b * 16 + a * 4 + s).  Value-exact: a 32-block's scale
// applies to both of its 16-element halves.  One thread per output word.
__global__ void expand_scales16_kernel(const uint8_t* __restrict__ s32, int64_t n_words, int K,
                                       uint8_t* __restrict__ s16) {
  const int KB64 = K / 64, KB128 = K / 128;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_words; i += stride) {
    // word i = output bytes 4i .. 4i+3 = one row's four 16-groups of a 64-chunk
    const int64_t blk = i >> 7;                    // 128 words (512 B) per (row block, 64-chunk)
    const int w = (int)(i & 127);                  // = b * 4 + a
    const int64_t rb = blk / KB64;
    const int j = (int)(blk - rb * KB64);
    const uint32_t src_word =
        *reinterpret_cast<const uint32_t*>(s32 + ((rb * KB128 + (j >> 1)) << 9) + (int64_t)w * 4);
    // the 64-chunk j covers 32-blocks 2j and 2j + 1: bytes (2j) & 3 and (2j + 1) & 3 of the source word
    const uint32_t lo = (src_word >> (8 * ((2 * j) & 3))) & 0xFFu;
    const uint32_t hi = (src_word >> (8 * ((2 * j + 1) & 3))) & 0xFFu;
    *reinterpret_cast<uint32_t*>(s16 + i * 4) = lo | (lo << 8) | (hi << 16) | (hi << 24);
  }
}

}  // namespace moesq
