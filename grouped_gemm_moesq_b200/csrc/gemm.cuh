// Grouped sparse NVFP4 GEMM on the sm_100a sparse tensor cores.
//
// For every expert e and valid row r of e:
//   y[r][m] = bf16( alpha_e * sum_k deq(a[r][k]) deq(W_e[m][k]) ),
//   alpha_e = 1 / (gamma_w[e] gamma_a[e]),
// in the paper's swap-AB form Y_e^T = W_e X_e^T (Sec. 3.4): the paired-4:8
// weight is the sparse operand A (M = 128 rows per tile), the token rows of
// the expert are operand B (N <= TN per tile), both block scales are applied
// inside the MMA and alpha_e in the epilogue (App. D.1).
//
// Design (two CTAs per SM, persistent, warp-specialised):
//   warp 0  producer: per 256-wide K step one bulk copy brings the weight
//           tile of the kernel form (11 KB, contiguous: 128 x 64 B of
//           pre-swizzled compressed values, 2 KB of metadata, 1 KB of scales);
//           TMA brings the token codes (TN x 128 B, 128-byte swizzle) and a bulk
//           copy their scales (1 KB) into an S-stage shared-memory ring.
//   warp 1  MMA issuer (one thread): per K step tcgen05.cp moves the
//           metadata and both scale blocks into one of 4 rotating TMEM
//           buffers, then two tcgen05.mma.sp.kind::mxf4nvf4.block_scale
//           (K = 128 dense each) accumulate in TMEM; tcgen05.commit frees the
//           stage.  A thread's copies and MMAs execute in issue order, so
//           they need no barrier between them; handing the copies to another
//           warp costs a commit/wait round trip per K step and measured
//           slower.  The second CTA of the SM is a second independent issue
//           stream, which keeps the tensor pipe busy.  With 64-row token tiles
//           the accumulator is double-buffered in TMEM so the epilogue of tile
//           i overlaps the main loop of tile i+1; with 128-row tiles the other
//           CTA covers the epilogue.
//   warps 2-5 epilogue: tcgen05.ld of the fp32 accumulator, times alpha_e,
//           rounded to bf16 and stored for the valid rows only; or, for a
//           gate_up stack in the SwiGLU kernel row order (SWIGLU), h =
//           SiLU(gate) * up requantised to NVFP4 (App. D.1 "fused SwiGLU
//           with requantization"), so that the bf16 gate_up output never
//           reaches memory.
// Work units are (expert, 128-row weight block, TN-row token block); the
// per-expert token counts stay on the device and every CTA derives the unit
// list from them (no host synchronisation).  Units are taken round-robin;
// consecutive units share the token block, so concurrently running CTAs
// reuse it from L2 while each streams its own weight block from HBM.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "dense.cuh"
#include "pack.cuh"

namespace moesq {

constexpr int kGemmMaxE = 512;
constexpr int kGemmThreads = 192;   // producer, MMA, 4 epilogue warps

// DENSE: the dense NVFP4 control (dense.cuh): per K step an 18 KB weight
// tile (128 x 128 B of codes, 128-byte swizzle, and per-16 scales), token
// scales one per 16 K (2 KB), four dense MMAs of K = 64 and eight scale
// copies; otherwise the same kernel.
// SWIGLU: the gate_up GEMM with SwiGLU and the NVFP4 requantisation of h
// in the epilogue (weights in the gate/up-interleaved kernel row order):
// y_gu never leaves the SM; the epilogue writes h codes and scales.
template <int TN, bool DENSE = false, bool SWIGLU = false>
struct GemmCfg {
  // Two CTAs share an SM: each issues its tcgen05 copies and MMAs from one
  // thread, and two such independent issue streams keep the tensor pipe
  // busier than one.
  static constexpr int kCtasPerSm = 2;
  static constexpr int kNAcc = (TN == 128) ? 1 : 2;     // accumulator buffers (TN columns each)
  static constexpr int kStages = DENSE ? ((TN == 128) ? 2 : 3) : ((TN == 128) ? 3 : (SWIGLU ? 4 : 5));
  static constexpr int kWBytes = DENSE ? kDTileBytes : kKTileBytes;   // weight tile of one K step
  static constexpr int kBBytes = TN * 128;       // token codes, 256 K
  static constexpr int kSfBytes = DENSE ? 2048 : 1024;   // token scales: 4 (or 2) x (32 x 16 B)
  static constexpr int kOffW = 0;
  static constexpr int kOffB = kOffW + kStages * kWBytes;
  static constexpr int kOffSfb = kOffB + kStages * kBBytes;
  // SwiGLU transpose buffer: 64 token rows of 128 bf16 (64 gate, then 64 up
  // features) padded to 272 bytes, so that 16-byte reads of 8 consecutive
  // rows hit 8 different bank groups
  static constexpr int kXRow = 272;
  static constexpr int kXBytes = SWIGLU ? 64 * kXRow : 0;
  static constexpr int kOffX = kOffSfb + kStages * kSfBytes;
  static constexpr int kOffBar = kOffX + kXBytes;
  static constexpr int kTBufs = 4;                       // rotating TMEM buffers of metadata + scales
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffTab = kOffMisc + 16;
  static constexpr int kSmemBytes = kOffTab + (3 * kGemmMaxE + 1) * 4 + 1024;
  static constexpr uint32_t kTmemCols = 256;            // half of an SM's tensor memory
  // TMEM buffer b (of kTBufs) at column kColBuf + kBufCols b: sparse:
  // metadata 4 columns, weight scales 8, token scales 8; dense: weight
  // scales 16, token scales 16
  static constexpr uint32_t kColBuf = kNAcc * TN;
  static constexpr uint32_t kBufCols = DENSE ? 32 : 20;
  static_assert(TN == 64 || TN == 128, "token tile");
  static_assert(kWBytes % 1024 == 0 && kBBytes % 1024 == 0, "1 KB aligned stages");
  static_assert(kCtasPerSm * (kSmemBytes + 1024) <= 228 * 1024, "shared memory of the CTAs of one SM");
  static_assert(kColBuf + kTBufs * kBufCols <= kTmemCols, "tensor memory");
};

struct GemmParams {
  const uint8_t* ktiles;
  const uint8_t* a_scales;
  const float* gamma_w;
  const float* gamma_a;
  const int32_t* counts;
  const int32_t* row_offsets;
  uint16_t* y;
  uint8_t* h_codes;      // SWIGLU: [rows_cap][M/4]
  uint8_t* h_scales;     // SWIGLU: MMA scale layout, M/2 columns
  const float* gamma_h;  // SWIGLU: [E]
  int E, M, K, rows_cap;
  uint64_t timeout_ns;
};

struct Tile {
  int e, mb, row0, nvalid, nmma, q;
};

// Unit t -> (expert, weight block, token block).  ntp = per-expert prefix of
// token blocks, rstart = aligned row start, cnt = rows of the expert.
template <int TN>
__device__ __forceinline__ Tile decode_tile(int t, int MB, int E, const int* ntp, const int* rstart, const int* cnt) {
  Tile tl;
  const int g = t / MB;
  tl.mb = t - g * MB;
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ntp[mid] <= g) lo = mid; else hi = mid - 1;
  }
  tl.e = lo;
  const int nb = g - ntp[lo];
  tl.row0 = rstart[lo] + nb * TN;
  tl.nvalid = min(TN, cnt[lo] - nb * TN);
  tl.nmma = (tl.nvalid + 15) & ~15;
  // 32-row group of the tile inside its 128-row scale block: 0 or 2 (TN is 64
  // or 128 and expert rows start 128-aligned), so the B-scale TMEM address
  // moves by an even number of columns only
  tl.q = (tl.row0 & 127) >> 5;
  return tl;
}

template <int TN, bool DENSE, bool SWIGLU = false>
__global__ void __launch_bounds__(kGemmThreads, GemmCfg<TN, DENSE, SWIGLU>::kCtasPerSm)
grouped_sparse_gemm_kernel(const __grid_constant__ CUtensorMap tm_b, const GemmParams p) {
  using C = GemmCfg<TN, DENSE, SWIGLU>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int MB = p.M / 128, KT = p.K / 256, KB = p.K / 128, E = p.E;
  const int KSF = DENSE ? p.K / 64 : KB;   // 512-byte token-scale blocks per 128 token rows

  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* ntp = reinterpret_cast<int*>(smem + C::kOffTab);   // [E+1]
  int* rstart = ntp + kGemmMaxE + 1;                       // [E]
  int* cnt = rstart + kGemmMaxE;                           // [E]
  auto bar = [&](int i) { return sbase + C::kOffBar + 8u * (uint32_t)i; };
  auto full_bar = [&](int s) { return bar(s); };
  auto empty_bar = [&](int s) { return bar(C::kStages + s); };
  auto accf_bar = [&](int b) { return bar(2 * C::kStages + b); };
  auto acce_bar = [&](int b) { return bar(2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = bar(2 * C::kStages + 4);

  // ---------------------------------------------------------------- set-up
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(accf_bar(b), 1); mbar_init(acce_bar(b), 4); }
    mbar_init(drain_bar, 1);
    fence_barrier_init();
    misc[1] = 0;
    prefetch_tmap(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(misc), C::kTmemCols);
    tmem_relinquish();
  }
  // the routing counts come from the previous kernels of the step
  pdl_trigger();
  pdl_wait();
  // expert table; validate the routing counts against the aligned row space
  int local_bad = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = p.counts[e], r0 = p.row_offsets[e], r1 = p.row_offsets[e + 1];
    // each expert's span starts on a 128-row boundary and holds its rows
    // (padded to 128); spans may leave gaps, e.g. a fixed capacity per expert
    const bool ok = c >= 0 && r0 >= 0 && (r0 & 127) == 0 && r1 - r0 >= ((c + 127) & ~127) && r1 <= p.rows_cap;
    local_bad |= ok ? 0 : 1;
    cnt[e] = ok ? c : 0;
    rstart[e] = r0;
    ntp[e + 1] = ok ? (c + TN - 1) / TN : 0;
  }
  tc_fence_before();
  const int bad = __syncthreads_or(local_bad);
  tc_fence_after();
  if (warp == 0) {                      // exclusive prefix of token blocks, in place
    const int per = (E + 31) / 32, e0 = lane * per;   // per <= 16 (E <= 512)
    int vals[16];
    int sum = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      vals[i] = (i < per && e0 + i < E) ? ntp[e0 + i + 1] : 0;
      sum += vals[i];
    }
    int inc = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += v;
    }
    __syncwarp();                       // every lane has read before any lane writes
    int run = inc - sum;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < per && e0 + i < E) { ntp[e0 + i] = run; run += vals[i]; }
    }
    if (lane == 31) ntp[E] = inc;
    if (lane == 0 && bad && blockIdx.x == 0) record_error(kWhereGemmCounts, kErrFault);
  }
  __syncthreads();
  const uint32_t tmem = misc[0];
  const int total = bad ? 0 : ntp[E] * MB;

  // ---------------------------------------------------------------- roles
  if (warp == 0) {
    if (lane == 0) {
      // weight tiles an expert reuses (more than one token block) stay in
      // L2; tiles read once are streamed with evict_first so they do not
      // push out the token tiles
      const uint64_t pol_keep = policy_evict_last();
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;     // per-stage bits for the drain on abort
      bool ok = true;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x) {
        const Tile tl = decode_tile<TN>(t, MB, E, ntp, rstart, cnt);
        const int nbox = (tl.nmma + 31) >> 5;
        const uint32_t bytes = C::kWBytes + C::kSfBytes + nbox * 4096;
        const uint8_t* wt = p.ktiles + ((int64_t)tl.e * MB + tl.mb) * KT * C::kWBytes;
        const uint64_t pol_w = (ntp[tl.e + 1] - ntp[tl.e] > 1) ? pol_keep : pol_stream;
        const uint8_t* xsc = p.a_scales + (int64_t)(tl.row0 >> 7) * KSF * 512;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait(empty_bar(stage), phase ^ 1u, p.timeout_ns, abort_flag)) {
            record_error(kWhereGemmProducer, kErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          const uint32_t fb = full_bar(stage);
          mbar_arrive_expect_tx(fb, bytes);
          bulk_load(sbase + C::kOffW + stage * C::kWBytes, wt + (int64_t)kt * C::kWBytes, C::kWBytes, fb, pol_w);
          bulk_load(sbase + C::kOffSfb + stage * C::kSfBytes, xsc + kt * C::kSfBytes, C::kSfBytes, fb, pol_x);
          for (int i = 0; i < nbox; ++i)
            tma_load_2d(sbase + C::kOffB + stage * C::kBBytes + i * 4096, &tm_b, fb, kt * 128, tl.row0 + 32 * i,
                        pol_x);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {                        // let the copies in flight land before the CTA exits
        int zero = 0;
        for (int s = 0; s < C::kStages; ++s)
          if (issued >> s & 1u) mbar_wait(full_bar(s), (issued_parity >> s) & 1u, p.timeout_ns, &zero);
      }
    }
  } else if (warp == 1) {
    // MMA issuer: per K step waits for the stage, moves its metadata and
    // both scale blocks into the next of kTBufs rotating TMEM buffers
    // (tcgen05.cp) and issues the two sparse MMAs that read them.  The
    // copies and MMAs of one thread run in issue order, so no barrier
    // separates them; the buffer rotation keeps a copy away from the
    // buffers the MMAs in flight still read.
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t g = 0;                   // K steps of this CTA so far (TMEM buffer = g % kTBufs)
      bool ok = true, any = false;
      int it = 0;
      for (int t = blockIdx.x; t < total && ok; t += gridDim.x, ++it) {
        const Tile tl = decode_tile<TN>(t, MB, E, ntp, rstart, cnt);
        const int buf = it % C::kNAcc;
        const uint32_t aph = (uint32_t)(it / C::kNAcc) & 1u;
        if (!mbar_wait(acce_bar(buf), aph ^ 1u, p.timeout_ns, abort_flag)) {
          record_error(kWhereGemmMma, kErrTimeout);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * TN);
        const uint32_t idesc = DENSE ? (idesc_sp_nvf4((uint32_t)tl.nmma) & ~(1u << 2)) : idesc_sp_nvf4((uint32_t)tl.nmma);
        for (int kt = 0; kt < KT; ++kt, ++g) {
          const int tb = (int)(g % C::kTBufs);
          if (!mbar_wait(full_bar(stage), phase, p.timeout_ns, abort_flag)) {
            record_error(kWhereGemmMma, kErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = sbase + C::kOffW + stage * C::kWBytes;
          const uint32_t sb = sbase + C::kOffB + stage * C::kBBytes;
          const uint32_t ssb = sbase + C::kOffSfb + stage * C::kSfBytes;
          const uint32_t tbuf = tmem + C::kColBuf + C::kBufCols * (uint32_t)tb;
          if constexpr (DENSE) {
            // four 64-wide K chunks: weight scales at tbuf + 4 j, token scales at tbuf + 16 + 4 j
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              tc_cp_32x128b_x4(tbuf + 4 * j, smem_desc(sa + kDTileScales + 512 * j, 16, 128, 0));
              tc_cp_32x128b_x4(tbuf + 16 + 4 * j, smem_desc(ssb + 512 * j, 16, 128, 0));
            }
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
              const uint64_t adesc = smem_desc(sa + kb * 32, 16, 1024, 2);    // 128-byte swizzle
              const uint64_t bdesc = smem_desc(sb + kb * 32, 16, 1024, 2);
              tc_mma_nvf4(d_tmem, adesc, bdesc, idesc, tbuf + 4 * kb, tbuf + 16 + 4 * kb + tl.q,
                          (kt | kb) != 0 ? 1u : 0u);
            }
          } else {
            tc_cp_128x128b(tbuf, smem_desc(sa + kKTileMeta, 16, 128, 0));
            tc_cp_32x128b_x4(tbuf + 4, smem_desc(sa + kKTileScales, 16, 128, 0));
            tc_cp_32x128b_x4(tbuf + 8, smem_desc(sa + kKTileScales + 512, 16, 128, 0));
            tc_cp_32x128b_x4(tbuf + 12, smem_desc(ssb, 16, 128, 0));
            tc_cp_32x128b_x4(tbuf + 16, smem_desc(ssb + 512, 16, 128, 0));
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
              const uint64_t adesc = smem_desc(sa + kb * 32, 16, 512, 4);     // 64-byte swizzle
              const uint64_t bdesc = smem_desc(sb + kb * 64, 16, 1024, 2);    // 128-byte swizzle
              tc_mma_sp_nvf4(d_tmem, adesc, bdesc, tbuf + 2 * kb, idesc, tbuf + 4 + 4 * kb,
                             tbuf + 12 + 4 * kb + tl.q, (kt | kb) != 0 ? 1u : 0u);
            }
          }
          any = true;
          tc_commit(empty_bar(stage));
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        if (ok) tc_commit(accf_bar(buf));
      }
      if (!ok && any) {                 // drain the MMAs in flight before TMEM is released
        int zero = 0;
        tc_commit(drain_bar);
        mbar_wait(drain_bar, 0, p.timeout_ns, &zero);
      }
    }
  } else if constexpr (SWIGLU) {
    // Warps 2..5 = TMEM lane quadrants 2, 3, 0, 1.  The tile's 128 weight
    // rows are gate features 64 mb + [0, 64) (quadrants 0, 1) and the up
    // rows of the same features (quadrants 2, 3).  The epilogue turns the
    // accumulator, rounded to bf16 as the unfused GEMM writes y, around in
    // shared memory 64 token rows at a time (a row: the 64 gate features,
    // then the 64 up features) and hands TMEM back once the second half is
    // in registers; thread (token tau, block b) then forms h = SiLU(g) u
    // for features 64 mb + 32 b + [0, 32) of its token and requantises it
    // with quantize_block32, the function the SwiGLU kernel uses, while the
    // MMA runs the next tile.
    const int quad = warp & 3, fb = quad & 1;
    const int half_off = (quad >= 2 ? 64 : 0) + fb * 32 + lane;   // feature slot of this lane in a row
    uint8_t* xbuf = smem + C::kOffX;
    const int ept = threadIdx.x - 64;               // 0..127
    const int tau = ept & 63, b = ept >> 6;
    const int I = p.M >> 1, KBH = I / 128;
    constexpr int kHalves = TN / 64;
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const Tile tl = decode_tile<TN>(t, MB, E, ntp, rstart, cnt);
      const int buf = it % C::kNAcc;
      const uint32_t aph = (uint32_t)(it / C::kNAcc) & 1u;
      const bool ok = mbar_wait(accf_bar(buf), aph, p.timeout_ns, abort_flag);
      if (!ok && lane == 0) { record_error(kWhereGemmEpilogue, kErrTimeout); *abort_flag = 1; }
      // every epilogue warp reaches this barrier once per tile, so all four
      // leave together; it also orders the previous tile's reads of the
      // transpose buffer before this tile's writes
      if (bar_red_or(1, 128, !ok)) break;
      tc_fence_after();
      const float alpha = __frcp_rn(__fmul_rn(p.gamma_w[tl.e], p.gamma_a[tl.e]));
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * TN);
      const int nch = tl.nmma >> 4;
      uint32_t hold[4][8];                          // second half (TN = 128): bf16 pairs, columns 64 + 16 c + 2 q, +1
#pragma unroll
      for (int c = 0; c < TN / 16; ++c) {
        if (c >= nch) break;
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr + 16 * c, r);
        tmem_ld_wait();
        if (c < 4) {
#pragma unroll
          for (int j = 0; j < 16; ++j)
            *reinterpret_cast<uint16_t*>(xbuf + (16 * c + j) * C::kXRow + 2 * half_off) =
                (uint16_t)f32_to_bf16_bits(__fmul_rn(alpha, __uint_as_float(r[j])));
        } else {
#pragma unroll
          for (int q = 0; q < 8; ++q)
            hold[c & 3][q] = f32_to_bf16_bits(__fmul_rn(alpha, __uint_as_float(r[2 * q]))) |
                             (f32_to_bf16_bits(__fmul_rn(alpha, __uint_as_float(r[2 * q + 1]))) << 16);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar(buf));    // the accumulator goes back to the MMA warp
      const float g_h = p.gamma_h[tl.e];
      const int blk = 2 * tl.mb + b;                  // 32-feature scale block of h
#pragma unroll
      for (int hf = 0; hf < kHalves; ++hf) {
        if (hf == 1) {
          bar_sync_named(1, 128);                   // the first half has been read
#pragma unroll
          for (int c = 4; c < 8; ++c) {
            if (c >= nch) break;
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              const uint32_t w2 = hold[c & 3][j >> 1];
              *reinterpret_cast<uint16_t*>(xbuf + (16 * (c - 4) + j) * C::kXRow + 2 * half_off) =
                  (uint16_t)((j & 1) ? (w2 >> 16) : (w2 & 0xFFFFu));
            }
          }
        }
        bar_sync_named(1, 128);                     // this half is in shared memory
        const int n = 64 * hf + tau;                // token column of this thread
        if (n < tl.nvalid) {
          const uint8_t* row = xbuf + tau * C::kXRow;
          float h[32];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint4 gw = *reinterpret_cast<const uint4*>(row + 64 * b + 16 * k);
            const uint4 uw = *reinterpret_cast<const uint4*>(row + 128 + 64 * b + 16 * k);
            const uint32_t g4[4] = {gw.x, gw.y, gw.z, gw.w}, u4[4] = {uw.x, uw.y, uw.z, uw.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              h[8 * k + 2 * q] = silu_mul(bf16lo(g4[q]), bf16lo(u4[q]));
              h[8 * k + 2 * q + 1] = silu_mul(bf16hi(g4[q]), bf16hi(u4[q]));
            }
          }
          const int64_t row_n = (int64_t)tl.row0 + n;
          const uint32_t code = quantize_block32(h, g_h, p.h_codes + row_n * (I / 2) + blk * 16);
          p.h_scales[mma_scale_offset(row_n, blk, KBH)] = (uint8_t)code;
        }
      }
    }
  } else {
    const int quad = warp & 3;          // warps 2..5: TMEM lanes 32*quad .. 32*quad+31
    int it = 0;
    for (int t = blockIdx.x; t < total; t += gridDim.x, ++it) {
      const Tile tl = decode_tile<TN>(t, MB, E, ntp, rstart, cnt);
      const int buf = it % C::kNAcc;
      const uint32_t aph = (uint32_t)(it / C::kNAcc) & 1u;
      if (!mbar_wait(accf_bar(buf), aph, p.timeout_ns, abort_flag)) {
        if (lane == 0) { record_error(kWhereGemmEpilogue, kErrTimeout); *abort_flag = 1; }
        break;
      }
      tc_fence_after();
      const float alpha = __frcp_rn(__fmul_rn(p.gamma_w[tl.e], p.gamma_a[tl.e]));
      const int m = tl.mb * 128 + quad * 32 + lane;
      const uint32_t taddr = tmem + ((uint32_t)(quad * 32) << 16) + (uint32_t)(buf * TN);
      uint16_t* yrow = p.y + (int64_t)tl.row0 * p.M + m;
      for (int c0 = 0; c0 < tl.nmma; c0 += 16) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr + c0, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c0 + j;
          if (n < tl.nvalid)
            yrow[(int64_t)n * p.M] = (uint16_t)f32_to_bf16_bits(__fmul_rn(alpha, __uint_as_float(r[j])));
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acce_bar(buf));
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

}  // namespace moesq
