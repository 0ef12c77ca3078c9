// Grouped sparse NVFP4 GEMM on SM pairs (tcgen05 cta_group::2).
//
// Same result as grouped_sparse_gemm_kernel (gemm.cuh) -- y[r][m] =
// bf16(alpha_e * sum_k deq(a[r][k]) deq(W_e[m][k])) -- with a 256-row weight
// tile per unit computed by a cluster of two CTAs on two SMs: one
// tcgen05.mma.sp.cta_group::2 (M = 256) takes the weight rows of the
// leader's 128-row block from the leader's shared memory and those of the
// next block from the peer's, and the tile's N token rows half from each
// (rows [0, N/2) in the leader, [N/2, N) in the peer); each CTA's TMEM holds
// the accumulator of its own 128 weight rows x N tokens.
//
// Why: in prefill the one-SM kernel moves about 57 KB through an SM's shared
// memory per 128 x 128 x 256 piece of work (the TMA writes of an 11 KB weight
// tile and a 16 KB token tile, the MMA reads of 8 KB of weights and 16 KB of
// tokens, the scale copies), near the bandwidth of shared memory; here each
// SM stages and serves only half of the token tile, about 40 KB for the same
// work.  Measured on the B200 it is nevertheless slower than the one-SM
// kernel (e.g. 2.6 vs 1.6 ms for 32 experts x 4096 rows of the Kimi gate_up
// shape): with one CTA per SM a single thread issues all of a pair's
// metadata / scale copies and MMAs and a single producer per SM issues the
// copies, each of which holds its thread for about a hundred cycles.  It is
// kept as a selectable variant (sm_mode 2) and tuning candidate.
//
// One CTA per SM (the shared memory of a CTA exceeds half an SM's), so the
// two CTAs of a cluster sit on two SMs; 192 threads: warp 0 producer,
// warp 1 TMEM allocator and (leader only) MMA issuer, warps 2-5 epilogue.
//   * Both CTAs' producers load their own stage (the weight tile of their
//     own 128-row block, their half of the token rows, the 1 KB of token
//     scales both need) with TMA tensor copies of the cta_group::2 form,
//     which complete on the leader's full barrier; the leader registers the
//     transaction bytes of both CTAs.
//   * The leader's MMA thread issues, per K step, the cta_group::2 copies of
//     metadata and scales (each CTA's shared memory into its own TMEM) and
//     two M = 256 sparse MMAs; tcgen05.commit with multicast frees the stage
//     in both CTAs and hands both accumulators to their epilogues.
//   * Each CTA's epilogue drains its own accumulator and arrives on the
//     leader's accumulator-empty barrier (the peer remotely).
// All waits are bounded as in the one-SM kernel; a cluster barrier after the
// barrier set-up and one before TMEM is released keep each CTA's barriers
// and shared memory alive while the other may still signal them.
#pragma once
#include <cuda.h>
#include "common.cuh"
#include "gemm.cuh"
#include "pack.cuh"

namespace moesq {

__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory offset in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" :: "r"(cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\t"
               "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
// Bounded wait with cluster-scope acquire (barriers the other CTA signals).
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                                  volatile int* abort) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((spin & 15u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > timeout_ns) return false;
    }
  }
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// TMA 2-D tile load whose completion is counted on an mbarrier of either CTA
// of the pair (no multicast).
__device__ __forceinline__ void tma_load_2d_pair(uint32_t dst, const void* tmap, uint32_t cluster_bar, int x, int y,
                                                 uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1, {%3, %4}], [%2], %5;"
      :: "r"(dst), "l"(tmap), "r"(cluster_bar), "r"(x), "r"(y), "l"(policy) : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" :: "r"(dst_smem), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" :: "r"(taddr), "r"(ncols) : "memory");
}
// Arrives on the mbarrier at this shared-memory offset in both CTAs of the
// pair once all prior tcgen05 operations of the thread have completed.
__device__ __forceinline__ void tc_commit_pair_mc(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               :: "r"(bar), "h"((uint16_t)3) : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" :: "r"(bar) : "memory");
}
__device__ __forceinline__ void tc_cp_pair_128x128b(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.128x128b [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_cp_pair_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" :: "r"(taddr), "l"(sdesc) : "memory");
}
__device__ __forceinline__ void tc_mma_sp_nvf4_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t e_tmem,
                                                    uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                                    uint32_t accumulate) {
  asm volatile("{\n\t.reg .pred p;\n\t"
               "setp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.sp.cta_group::2.kind::mxf4nvf4.block_scale.block16"
               " [%0], %1, %2, [%7], %3, [%5], [%6], p;\n\t}"
               :: "r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate),
                  "r"(sfa_tmem), "r"(sfb_tmem), "r"(e_tmem) : "memory");
}

struct PairCfg {
  static constexpr int TN = 128;                 // token rows per tile (N <= 128, N/2 per CTA)
  static constexpr int kStages = 10;
  static constexpr int kWBytes = kKTileBytes;    // this CTA's weight tile of one K step
  static constexpr int kBBytes = 64 * 128;       // this CTA's token rows (up to 64) of one K step
  static constexpr int kSfBytes = 1024;          // token scales of the tile's 128-row block, both halves of K
  static constexpr int kOffW = 0;
  static constexpr int kOffB = kOffW + kStages * kWBytes;
  static constexpr int kOffSfb = kOffB + kStages * kBBytes;
  static constexpr int kOffBar = kOffSfb + kStages * kSfBytes;
  // full[S], empty[S], acc_full[2], acc_empty[2], drain
  static constexpr int kNumBars = 2 * kStages + 5;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffTab = kOffMisc + 16;
  static constexpr int kSmemBytes = kOffTab + (3 * kGemmMaxE + 1) * 4 + 1024;
  static constexpr uint32_t kTmemCols = 512;
  static constexpr int kTBufs = 4;               // rotating TMEM buffers of metadata + scales
  static constexpr uint32_t kColBuf = 2 * TN;    // after the double-buffered accumulator
  static constexpr uint32_t kBufCols = 20;
  static_assert(kSmemBytes + 1024 > 114 * 1024, "one CTA per SM, so the two CTAs of a pair are on two SMs");
  static_assert(kSmemBytes + 1024 <= 227 * 1024, "shared memory");
  static_assert(kColBuf + kTBufs * kBufCols <= kTmemCols, "tensor memory");
};

// Token codes (2-D, 32-row boxes), the kernel-form weight tiles seen as
// rows of 128 B (box 128 B x 88 rows = one 11 KB tile) and the MMA-layout
// activation scales seen as rows of 256 B (box 256 B x 4 rows = the 1 KB of
// one K step of a 128-row block).
struct PairMaps {
  CUtensorMap tok, wt, sf;
};

// Unit t -> (expert, weight block pair, token block).
__device__ __forceinline__ Tile decode_pair_tile(int t, int MBP, int E, const int* ntp, const int* rstart,
                                                 const int* cnt) {
  Tile tl;
  const int g = t / MBP;
  tl.mb = t - g * MBP;                           // weight block pair
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (ntp[mid] <= g) lo = mid; else hi = mid - 1;
  }
  tl.e = lo;
  const int nb = g - ntp[lo];
  tl.row0 = rstart[lo] + nb * PairCfg::TN;
  tl.nvalid = min(PairCfg::TN, cnt[lo] - nb * PairCfg::TN);
  tl.nmma = (tl.nvalid + 15) & ~15;
  tl.q = 0;                                      // tiles start on 128-row boundaries
  return tl;
}

__global__ void __launch_bounds__(192, 1)
grouped_sparse_gemm_pair_kernel(const __grid_constant__ PairMaps maps, const GemmParams p) {
  using C = PairCfg;
  constexpr int TN = C::TN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  const uint32_t sbase = smem_u32(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int MB = p.M / 128, MBP = p.M / 256, KT = p.K / 256, KB = p.K / 128, E = p.E;
  const int cid = (int)blockIdx.x >> 1, ncl = (int)gridDim.x >> 1;

  uint32_t* misc = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 1);
  int* ntp = reinterpret_cast<int*>(smem + C::kOffTab);
  int* rstart = ntp + kGemmMaxE + 1;
  int* cnt = rstart + kGemmMaxE;
  auto bar = [&](int i) { return sbase + C::kOffBar + 8u * (uint32_t)i; };
  auto full_bar = [&](int s) { return bar(s); };
  auto empty_bar = [&](int s) { return bar(C::kStages + s); };
  auto accf_bar = [&](int b) { return bar(2 * C::kStages + b); };
  auto acce_bar = [&](int b) { return bar(2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = bar(2 * C::kStages + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) { mbar_init(full_bar(s), 1); mbar_init(empty_bar(s), 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(accf_bar(b), 1); mbar_init(acce_bar(b), 8); }
    mbar_init(drain_bar, 1);
    fence_barrier_init();
    misc[1] = 0;
    prefetch_tmap(&maps.tok);
    prefetch_tmap(&maps.wt);
    prefetch_tmap(&maps.sf);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(misc), C::kTmemCols);
    tmem_relinquish_pair();
  }
  pdl_trigger();
  pdl_wait();
  int local_bad = 0;
  for (int e = threadIdx.x; e < E; e += blockDim.x) {
    const int c = p.counts[e], r0 = p.row_offsets[e], r1 = p.row_offsets[e + 1];
    const bool ok = c >= 0 && r0 >= 0 && (r0 & 127) == 0 && r1 - r0 >= ((c + 127) & ~127) && r1 <= p.rows_cap;
    local_bad |= ok ? 0 : 1;
    cnt[e] = ok ? c : 0;
    rstart[e] = r0;
    ntp[e + 1] = ok ? (c + TN - 1) / TN : 0;
  }
  tc_fence_before();
  const int bad = __syncthreads_or(local_bad);
  tc_fence_after();
  if (warp == 0) {
    const int per = (E + 31) / 32, e0 = lane * per;
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
    __syncwarp();
    int run = inc - sum;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (i < per && e0 + i < E) { ntp[e0 + i] = run; run += vals[i]; }
    }
    if (lane == 31) ntp[E] = inc;
    if (lane == 0 && bad && blockIdx.x == 0) record_error(kWhereGemmCounts, kErrFault);
  }
  __syncthreads();
  // both CTAs' barriers are initialised before either signals the other's
  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem = misc[0];
  const int total = bad ? 0 : ntp[E] * MBP;
  bool aborted = false;

  if (warp == 0) {
    if (lane == 0) {
      const uint64_t pol_keep = policy_evict_last();
      const uint64_t pol_stream = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued = 0, issued_parity = 0;
      bool ok = true;
      for (int t = cid; t < total && ok; t += ncl) {
        const Tile tl = decode_pair_tile(t, MBP, E, ntp, rstart, cnt);
        const int half = tl.nmma >> 1;                        // token rows per CTA
        const int nbox = (half + 31) >> 5;
        // both CTAs' bytes are counted on the leader's barrier
        const uint32_t bytes = 2u * (uint32_t)(kKTileBytes + 1024 + nbox * 4096);
        const int mb = 2 * tl.mb + (int)rank;
        const int wrow0 = ((tl.e * MB + mb) * KT) * (kKTileBytes / 128);
        const uint64_t pol_w = (ntp[tl.e + 1] - ntp[tl.e] > 1) ? pol_keep : pol_stream;
        const int srow0 = ((tl.row0 >> 7) * KB) * 2;
        const int trow0 = tl.row0 + (int)rank * half;
        for (int kt = 0; kt < KT; ++kt) {
          if (!mbar_wait_cluster(empty_bar(stage), phase ^ 1u, p.timeout_ns, abort_flag)) {
            record_error(kWhereGemmProducer, kErrTimeout);
            *abort_flag = 1;
            ok = false;
            break;
          }
          // a copy of the peer that lands before the leader registered the
          // bytes only takes the transaction count below zero until then
          const uint32_t fb = mapa_shared(full_bar(stage), 0);
          if (leader) mbar_arrive_expect_tx(full_bar(stage), bytes);
          tma_load_2d_pair(sbase + C::kOffW + stage * C::kWBytes, &maps.wt, fb, 0,
                           wrow0 + kt * (kKTileBytes / 128), pol_w);
          tma_load_2d_pair(sbase + C::kOffSfb + stage * C::kSfBytes, &maps.sf, fb, 0, srow0 + kt * 4, pol_x);
          for (int i = 0; i < nbox; ++i)
            tma_load_2d_pair(sbase + C::kOffB + stage * C::kBBytes + i * 4096, &maps.tok, fb, kt * 128,
                             trow0 + 32 * i, pol_x);
          issued |= 1u << stage;
          issued_parity = (issued_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        aborted = true;
        if (leader) {                   // the leader's barriers count both CTAs' copies
          int zero = 0;
          for (int s = 0; s < C::kStages; ++s)
            if (issued >> s & 1u) mbar_wait(full_bar(s), (issued_parity >> s) & 1u, p.timeout_ns, &zero);
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t g = 0;
      bool ok = true, any = false;
      int it = 0;
      for (int t = cid; t < total && ok; t += ncl, ++it) {
        const Tile tl = decode_pair_tile(t, MBP, E, ntp, rstart, cnt);
        const int buf = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait_cluster(acce_bar(buf), aph ^ 1u, p.timeout_ns, abort_flag)) {
          record_error(kWhereGemmMma, kErrTimeout);
          *abort_flag = 1;
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(buf * TN);
        // M = 256 (both CTAs' weight rows), N = the tile's rows
        const uint32_t idesc = (idesc_sp_nvf4((uint32_t)tl.nmma) & ~(0x1Fu << 24)) | ((256u >> 4) << 24);
        for (int kt = 0; kt < KT; ++kt, ++g) {
          const int tb = (int)(g % C::kTBufs);
          if (!mbar_wait_cluster(full_bar(stage), phase, p.timeout_ns, abort_flag)) {
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
          tc_cp_pair_128x128b(tbuf, smem_desc(sa + kKTileMeta, 16, 128, 0));
          tc_cp_pair_32x128b_x4(tbuf + 4, smem_desc(sa + kKTileScales, 16, 128, 0));
          tc_cp_pair_32x128b_x4(tbuf + 8, smem_desc(sa + kKTileScales + 512, 16, 128, 0));
          tc_cp_pair_32x128b_x4(tbuf + 12, smem_desc(ssb, 16, 128, 0));
          tc_cp_pair_32x128b_x4(tbuf + 16, smem_desc(ssb + 512, 16, 128, 0));
#pragma unroll
          for (int kb = 0; kb < 2; ++kb) {
            const uint64_t adesc = smem_desc(sa + kb * 32, 16, 512, 4);
            const uint64_t bdesc = smem_desc(sb + kb * 64, 16, 1024, 2);
            tc_mma_sp_nvf4_pair(d_tmem, adesc, bdesc, tbuf + 2 * kb, idesc, tbuf + 4 + 4 * kb, tbuf + 12 + 4 * kb,
                                (kt | kb) != 0 ? 1u : 0u);
          }
          any = true;
          tc_commit_pair_mc(empty_bar(stage));
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
        if (ok) tc_commit_pair_mc(accf_bar(buf));
      }
      if (!ok) {
        aborted = true;
        if (any) {
          int zero = 0;
          tc_commit_pair(drain_bar);
          mbar_wait(drain_bar, 0, p.timeout_ns, &zero);
        }
      }
    }
  } else {
    const int quad = warp & 3;          // warps 2..5
    const uint32_t acce_leader0 = mapa_shared(acce_bar(0), 0), acce_leader1 = mapa_shared(acce_bar(1), 0);
    int it = 0;
    for (int t = cid; t < total; t += ncl, ++it) {
      const Tile tl = decode_pair_tile(t, MBP, E, ntp, rstart, cnt);
      const int buf = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      if (!mbar_wait_cluster(accf_bar(buf), aph, p.timeout_ns, abort_flag)) {
        if (lane == 0) { record_error(kWhereGemmEpilogue, kErrTimeout); *abort_flag = 1; }
        aborted = true;
        break;
      }
      tc_fence_after();
      const int mb = 2 * tl.mb + (int)rank;
      const float alpha = __frcp_rn(__fmul_rn(p.gamma_w[tl.e], p.gamma_a[tl.e]));
      const int m = mb * 128 + quad * 32 + lane;
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
      if (lane == 0) mbar_arrive_cluster(buf ? acce_leader1 : acce_leader0);
    }
  }

  __syncthreads();
  // neither CTA releases TMEM or exits while the other may still signal it
  tc_fence_before();
  cluster_sync();
  if (__syncthreads_or(aborted ? 1 : 0)) {
    // after an abort a copy issued by one CTA may still be landing in the
    // other's shared memory: give it time (bounded) before the CTAs exit
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 200000ull) {
    }
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::kTmemCols);
  }
}

}  // namespace moesq
