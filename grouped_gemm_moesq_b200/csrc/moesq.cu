// moesq C ABI (include/moesq.h): argument checks, launch configuration,
// tensor-map construction and the MoE layer composition.  Single
// translation unit so the device error word is shared by every kernel.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <utility>

#include <nvtx3/nvToolsExt.h>

#include "../../include/moesq.h"
#include "common.cuh"
#include "dense.cuh"
#include "gemm.cuh"
#include "gemm_pair.cuh"
#include "pack.cuh"
#include "peak.cuh"
#include "quant.cuh"
#include "route.cuh"

using namespace moesq;

namespace {

uint64_t g_timeout_ns = 2000000000ull;

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

thread_local cudaError_t t_last_cuda_error = cudaSuccess;

#define MOESQ_CUDA(call)                                   \
  do {                                                     \
    cudaError_t err_ = (call);                             \
    if (err_ != cudaSuccess) {                             \
      t_last_cuda_error = err_;                            \
      return MOESQ_ERR_CUDA;                               \
    }                                                      \
  } while (0)

#define MOESQ_TRY(call)                                    \
  do {                                                     \
    moesq_status st_ = (call);                             \
    if (st_ != MOESQ_OK) return st_;                       \
  } while (0)

// NVTX range named after the ABI call, around its host-side work (argument
// checks and launches), for timeline tools; a no-op without a tool attached.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};
#define MOESQ_NVTX_RANGE() NvtxRange nvtx_range_(__func__)

inline moesq_status last_launch() {
  const cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) return MOESQ_OK;
  t_last_cuda_error = e;
  return MOESQ_ERR_CUDA;
}

// Launch with programmatic stream serialisation: the grid may start while its
// predecessor in the stream finishes; every such kernel calls
// griddepcontrol.wait before it touches global memory.
template <typename... KArgs, typename... Args>
moesq_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                        Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  if (e == cudaSuccess) return MOESQ_OK;
  t_last_cuda_error = e;
  return MOESQ_ERR_CUDA;
}

struct DeviceInfo {
  int sms = 0;
  bool gemm_attr64 = false, gemm_attr128 = false, gemm_attr_pair = false, combine_attr = false;
  bool dense_attr64 = false, dense_attr128 = false;
  bool swiglu_attr64 = false, swiglu_attr128 = false;
  int pair_clusters = 0;     // co-resident clusters of the SM-pair GEMM
};

DeviceInfo& device_info() {
  static DeviceInfo info[64];
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  DeviceInfo& d = info[dev & 63];
  if (d.sms == 0) cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
  return d;
}

inline int grid_for(int64_t work_items, int per_block, int sms) {
  const int64_t want = (work_items + per_block - 1) / per_block;
  return (int)std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * 32));
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D uint8 tensor map: rows x row_bytes, box of box_rows x box_bytes.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_bytes,
               uint32_t box_rows, CUtensorMapSwizzle swz) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_bytes, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

moesq_status check_weights(const moesq_weights* w) {
  if (!w) return MOESQ_ERR_INVALID_ARG;
  if (w->E < 1 || w->E > kGemmMaxE || w->M < 128 || w->K < 256) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (w->M % 128 || w->K % 256) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (!w->values || !w->mask || !w->scales || !w->global_scale || !w->ktiles) return MOESQ_ERR_INVALID_ARG;
  if (!aligned(w->values, 16) || !aligned(w->ktiles, 16) || !aligned(w->mask, 2) || !aligned(w->global_scale, 4))
    return MOESQ_ERR_INVALID_ARG;
  if ((int64_t)w->E * w->M >= (int64_t)1 << 31) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (w->layout != MOESQ_LAYOUT_PLAIN && w->layout != MOESQ_LAYOUT_SWIGLU) return MOESQ_ERR_INVALID_ARG;
  if (w->layout == MOESQ_LAYOUT_SWIGLU && w->M % 256) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  return MOESQ_OK;
}

moesq_status check_routing(const moesq_routing* rt) {
  if (!rt) return MOESQ_ERR_INVALID_ARG;
  if (rt->T < 1 || rt->E < 1 || rt->E > kRouteMaxE || rt->k < 1 || rt->k > std::min(rt->E, 32))
    return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (!rt->topk_ids || !rt->topk_w || !rt->counts || !rt->offsets || !rt->row_offsets || !rt->sorted_to_slot ||
      !rt->slot_to_row)
    return MOESQ_ERR_INVALID_ARG;
  const void* arrays[7] = {rt->topk_ids, rt->topk_w, rt->counts, rt->offsets, rt->row_offsets, rt->sorted_to_slot,
                           rt->slot_to_row};
  for (const void* a : arrays)
    if (!aligned(a, 4)) return MOESQ_ERR_INVALID_ARG;
  if (rt->rows_cap % 128 || rt->rows_cap < moesq_rows_capacity(rt->T, rt->k, rt->E)) return MOESQ_ERR_INVALID_ARG;
  return MOESQ_OK;
}

// Output of a one-SM GEMM launch: y (bf16), or with SWIGLU the requantised
// h (codes, scales, gamma_h).
struct GemmOut {
  uint16_t* y;
  uint8_t* h_codes;
  uint8_t* h_scales;
  const float* gamma_h;
};

// One-SM grouped GEMM: the sparse kernel, (DENSE) the dense NVFP4 control,
// or (SWIGLU) the gate_up GEMM with the SwiGLU requantisation in its
// epilogue; `tiles` is the weights' kernel form.
template <int TN, bool DENSE, bool SWIGLU = false>
moesq_status launch_gemm_tiles(const uint8_t* tiles, const float* gamma_w, int E, int M, int K,
                               const uint8_t* a_codes, const uint8_t* a_scales, int rows_cap, const int32_t* counts,
                               const int32_t* row_offsets, const float* gamma_a, const GemmOut& out, int num_ctas,
                               cudaStream_t s) {
  using C = GemmCfg<TN, DENSE, SWIGLU>;
  DeviceInfo& di = device_info();
  bool& attr = SWIGLU  ? ((TN == 128) ? di.swiglu_attr128 : di.swiglu_attr64)
               : DENSE ? ((TN == 128) ? di.dense_attr128 : di.dense_attr64)
                       : ((TN == 128) ? di.gemm_attr128 : di.gemm_attr64);
  if (!attr) {
    MOESQ_CUDA(cudaFuncSetAttribute(grouped_sparse_gemm_kernel<TN, DENSE, SWIGLU>,
                                    cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes));
    attr = true;
  }
  CUtensorMap tmb;
  if (!make_tmap(&tmb, a_codes, (uint64_t)K / 2, (uint64_t)rows_cap, 128, 32, CU_TENSOR_MAP_SWIZZLE_128B))
    return MOESQ_ERR_CUDA;
  GemmParams p{};
  p.ktiles = tiles;
  p.a_scales = a_scales;
  p.gamma_w = gamma_w;
  p.gamma_a = gamma_a;
  p.counts = counts;
  p.row_offsets = row_offsets;
  p.y = out.y;
  p.h_codes = out.h_codes;
  p.h_scales = out.h_scales;
  p.gamma_h = out.gamma_h;
  p.E = E;
  p.M = M;
  p.K = K;
  p.rows_cap = rows_cap;
  p.timeout_ns = g_timeout_ns;
  const int grid = num_ctas > 0 ? num_ctas : di.sms * C::kCtasPerSm;
  return launch_pdl(grouped_sparse_gemm_kernel<TN, DENSE, SWIGLU>, dim3(grid), dim3(kGemmThreads),
                    (size_t)C::kSmemBytes, s, tmb, p);
}

template <int TN>
moesq_status launch_gemm(const moesq_weights* w, const uint8_t* a_codes, const uint8_t* a_scales, int rows_cap,
                         const int32_t* counts, const int32_t* row_offsets, const float* gamma_a, uint16_t* y,
                         int num_ctas, cudaStream_t s) {
  return launch_gemm_tiles<TN, false>(w->ktiles, w->global_scale, w->E, w->M, w->K, a_codes, a_scales, rows_cap,
                                      counts, row_offsets, gamma_a, GemmOut{y, nullptr, nullptr, nullptr}, num_ctas,
                                      s);
}

moesq_status check_dense_weights(const moesq_dense_weights* w) {
  if (!w) return MOESQ_ERR_INVALID_ARG;
  if (w->E < 1 || w->E > kGemmMaxE || w->M < 128 || w->K < 256) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (w->M % 128 || w->K % 256) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (!w->codes || !w->scales || !w->global_scale || !w->dtiles) return MOESQ_ERR_INVALID_ARG;
  if (!aligned(w->codes, 16) || !aligned(w->dtiles, 16) || !aligned(w->global_scale, 4))
    return MOESQ_ERR_INVALID_ARG;
  if ((int64_t)w->E * w->M >= (int64_t)1 << 31) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  return MOESQ_OK;
}

// SM-pair GEMM (cta_group::2): 256-row weight tiles, 128-row token tiles.
moesq_status launch_gemm_pair(const moesq_weights* w, const uint8_t* a_codes, const uint8_t* a_scales, int rows_cap,
                              const int32_t* counts, const int32_t* row_offsets, const float* gamma_a, uint16_t* y,
                              int num_ctas, cudaStream_t s) {
  using C = PairCfg;
  DeviceInfo& di = device_info();
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (!di.gemm_attr_pair) {
    MOESQ_CUDA(cudaFuncSetAttribute(grouped_sparse_gemm_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    C::kSmemBytes));
    cfg.gridDim = dim3(2 * di.sms);
    int ncl = 0;
    MOESQ_CUDA(cudaOccupancyMaxActiveClusters(&ncl, grouped_sparse_gemm_pair_kernel, &cfg));
    if (ncl < 1) return MOESQ_ERR_UNSUPPORTED_SHAPE;
    di.pair_clusters = ncl;
    di.gemm_attr_pair = true;
  }
  const int64_t KT = w->K / 256;
  PairMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  if (!make_tmap(&maps.tok, a_codes, (uint64_t)w->K / 2, (uint64_t)rows_cap, 128, 32, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap(&maps.wt, w->ktiles, 128, (uint64_t)w->E * (w->M / 128) * KT * (kKTileBytes / 128), 128,
                 kKTileBytes / 128, CU_TENSOR_MAP_SWIZZLE_NONE) ||
      !make_tmap(&maps.sf, a_scales, 256, (uint64_t)(rows_cap / 128) * (w->K / 128) * 2, 256, 4,
                 CU_TENSOR_MAP_SWIZZLE_NONE))
    return MOESQ_ERR_CUDA;
  GemmParams p{};
  p.ktiles = w->ktiles;
  p.a_scales = a_scales;
  p.gamma_w = w->global_scale;
  p.gamma_a = gamma_a;
  p.counts = counts;
  p.row_offsets = row_offsets;
  p.y = y;
  p.E = w->E;
  p.M = w->M;
  p.K = w->K;
  p.rows_cap = rows_cap;
  p.timeout_ns = g_timeout_ns;
  int ncl = di.pair_clusters;
  if (num_ctas > 0) ncl = std::max(1, std::min(ncl, num_ctas / 2));
  cfg.gridDim = dim3(2 * ncl);
  const cudaError_t e = cudaLaunchKernelEx(&cfg, grouped_sparse_gemm_pair_kernel, maps, p);
  if (e == cudaSuccess) return MOESQ_OK;
  t_last_cuda_error = e;
  return MOESQ_ERR_CUDA;
}

// Layer workspace carve-up.
struct LayerWs {
  int32_t *topk_ids, *counts, *offsets, *row_offsets, *sorted_to_slot, *slot_to_row, *route_ws;
  float* topk_w;
  uint8_t *a_codes, *a_scales, *h_codes, *h_scales;
  uint16_t *y_gu, *y_dn;
  uint16_t* x_in;    // host variant only
  float* logits_in;  // host variant only
  uint16_t* out;     // host variant only
  int rows_cap;
  size_t bytes;
};

LayerWs carve(void* base, int T, int k, int E, int H, int I, bool host_io) {
  LayerWs w;
  std::memset(&w, 0, sizeof(w));
  const int64_t R = (int64_t)T * k;
  const int64_t rc = moesq_rows_capacity(T, k, E);
  w.rows_cap = (int)rc;
  uint8_t* p = static_cast<uint8_t*>(base);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    uint8_t* q = p ? p + off : nullptr;
    off += align256(bytes);
    return q;
  };
  w.topk_ids = reinterpret_cast<int32_t*>(take(R * 4));
  w.topk_w = reinterpret_cast<float*>(take(R * 4));
  w.counts = reinterpret_cast<int32_t*>(take((size_t)E * 4));
  w.offsets = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
  w.row_offsets = reinterpret_cast<int32_t*>(take((size_t)(E + 1) * 4));
  w.sorted_to_slot = reinterpret_cast<int32_t*>(take(R * 4));
  w.slot_to_row = reinterpret_cast<int32_t*>(take(R * 4));
  w.route_ws = reinterpret_cast<int32_t*>(take(moesq_route_workspace_bytes(T, E)));
  w.a_codes = take((size_t)rc * H / 2);
  w.a_scales = take((size_t)rc * H / 32);
  w.y_gu = reinterpret_cast<uint16_t*>(take((size_t)rc * 2 * I * 2));
  w.h_codes = take((size_t)rc * I / 2);
  w.h_scales = take((size_t)rc * I / 32);
  w.y_dn = reinterpret_cast<uint16_t*>(take((size_t)rc * H * 2));
  if (host_io) {
    w.x_in = reinterpret_cast<uint16_t*>(take((size_t)T * H * 2));
    w.logits_in = reinterpret_cast<float*>(take((size_t)T * E * 4));
    w.out = reinterpret_cast<uint16_t*>(take((size_t)T * H * 2));
  }
  w.bytes = off;
  return w;
}

moesq_routing routing_of(const LayerWs& w, int T, int E, int k) {
  moesq_routing rt;
  rt.T = T;
  rt.E = E;
  rt.k = k;
  rt.rows_cap = w.rows_cap;
  rt.topk_ids = w.topk_ids;
  rt.topk_w = w.topk_w;
  rt.counts = w.counts;
  rt.offsets = w.offsets;
  rt.row_offsets = w.row_offsets;
  rt.sorted_to_slot = w.sorted_to_slot;
  rt.slot_to_row = w.slot_to_row;
  return rt;
}

// Launches the routing kernels for logits [T][E] into rt, with the per-block
// counts in bc (nblk x E int32).  PL = logits per lane of a token's warp.
template <int PL>
moesq_status route_launch_pl(const float* logits, const moesq_routing* rt, int32_t* bc, cudaStream_t s) {
  const int nblk = (rt->T + kRouteTPB - 1) / kRouteTPB;
  const size_t smem = (size_t)rt->E * kRouteWords * 4;
  MOESQ_TRY(launch_pdl(route_topk_kernel<PL>, dim3((rt->T + 7) / 8), dim3(256), 0, s, logits, rt->T, rt->E, rt->k,
                       rt->topk_ids, rt->topk_w));
  if (rt->T <= kRouteSmallMaxT) {       // few tokens: one CTA counts, scans and scatters
    const int words = (rt->T + 31) / 32;
    return launch_pdl(route_finish_kernel, dim3(1), dim3(1024), (size_t)rt->E * words * 4, s, rt->T, rt->E, rt->k,
                      (const int32_t*)rt->topk_ids, rt->counts, rt->offsets, rt->row_offsets, rt->sorted_to_slot,
                      rt->slot_to_row, words);
  }
  MOESQ_TRY(launch_pdl(route_count_kernel, dim3(nblk), dim3(256), smem, s, rt->T, rt->E, rt->k, rt->topk_ids, bc));
  MOESQ_TRY(launch_pdl(route_scan_kernel, dim3(1), dim3(1024), 0, s, bc, nblk, rt->E, rt->counts, rt->offsets,
                       rt->row_offsets));
  return launch_pdl(route_scatter_kernel, dim3(nblk), dim3(256), smem, s, rt->T, rt->E, rt->k, rt->topk_ids, bc,
                    rt->offsets, rt->row_offsets, rt->sorted_to_slot, rt->slot_to_row);
}

moesq_status route_launch(const float* logits, const moesq_routing* rt, int32_t* bc, cudaStream_t s) {
  const int pl = (rt->E + 31) / 32;
  if (pl <= 1) return route_launch_pl<1>(logits, rt, bc, s);
  if (pl <= 2) return route_launch_pl<2>(logits, rt, bc, s);
  if (pl <= 4) return route_launch_pl<4>(logits, rt, bc, s);
  if (pl <= 8) return route_launch_pl<8>(logits, rt, bc, s);
  if (pl <= 12) return route_launch_pl<12>(logits, rt, bc, s);
  return route_launch_pl<16>(logits, rt, bc, s);
}

moesq_status check_layer(int T, int k, const moesq_weights* w_gu, const moesq_weights* w_dn) {
  MOESQ_TRY(check_weights(w_gu));
  MOESQ_TRY(check_weights(w_dn));
  if (T < 1 || k < 1) return MOESQ_ERR_INVALID_ARG;
  if (w_gu->E != w_dn->E) return MOESQ_ERR_INVALID_ARG;
  const int H = w_gu->K, I2 = w_gu->M;
  if (I2 % 2 || w_dn->K != I2 / 2 || w_dn->M != H) return MOESQ_ERR_INVALID_ARG;
  if (k > std::min(w_gu->E, 32)) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if ((I2 / 2) % 256) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (w_dn->layout != MOESQ_LAYOUT_PLAIN) return MOESQ_ERR_INVALID_ARG;
  return MOESQ_OK;
}

moesq_status layer_body(const uint16_t* x, const float* logits, int T, int k, const moesq_weights* w_gu,
                        const moesq_weights* w_dn, const float* ga_gu, const float* ga_dn, uint16_t* out,
                        const LayerWs& ws, cudaStream_t s) {
  const int E = w_gu->E, H = w_gu->K, I = w_gu->M / 2;
  moesq_routing rt = routing_of(ws, T, E, k);
  MOESQ_TRY(moesq_route_permute(logits, &rt, ws.route_ws, moesq_route_workspace_bytes(T, E), s));
  MOESQ_TRY(moesq_quantize_act(x, T, H, &rt, ga_gu, rt.rows_cap, ws.a_codes, ws.a_scales, s));
  if (w_gu->layout == MOESQ_LAYOUT_SWIGLU) {
    // SwiGLU and its requantisation in the gate_up epilogue: y_gu is never written
    MOESQ_TRY(moesq_grouped_sparse_gemm_swiglu(w_gu, ws.a_codes, ws.a_scales, rt.rows_cap, rt.counts,
                                               rt.row_offsets, ga_gu, ga_dn, ws.h_codes, ws.h_scales, nullptr, s));
  } else {
    MOESQ_TRY(moesq_grouped_sparse_gemm(w_gu, ws.a_codes, ws.a_scales, rt.rows_cap, rt.counts, rt.row_offsets,
                                        ga_gu, ws.y_gu, nullptr, s));
    MOESQ_TRY(moesq_swiglu_quant(ws.y_gu, I, &rt, ga_dn, ws.h_codes, ws.h_scales, MOESQ_LAYOUT_PLAIN, s));
  }
  MOESQ_TRY(moesq_grouped_sparse_gemm(w_dn, ws.h_codes, ws.h_scales, rt.rows_cap, rt.counts, rt.row_offsets, ga_dn,
                                      ws.y_dn, nullptr, s));
  MOESQ_TRY(moesq_combine(ws.y_dn, H, &rt, out, s));
  return MOESQ_OK;
}

}  // namespace

// ----------------------------------------------------------------------------
// Scratch of moesq_route_permute_noalloc: the per-block expert counts of the
// routing kernels, for up to kNoAllocMaxT tokens and kRouteMaxE experts
// (128 blocks x 512 experts x 4 bytes = 256 KiB).  It lives in the module's
// global memory, so every GPU that loads the library holds it until the
// process exits.  The name below is only a host-side handle; kernels get the
// device address that cudaGetSymbolAddress returns for the current device.
constexpr int kNoAllocMaxT = 16384;
constexpr size_t kNoAllocScratchInts = (size_t)(kNoAllocMaxT / kRouteTPB) * kRouteMaxE;
static __device__ __align__(256) int32_t g_route_scratch[kNoAllocScratchInts];

namespace {

// Device address of g_route_scratch on the current device, looked up once per
// device (nullptr if the lookup fails).
int32_t* route_scratch_device_ptr() {
  static int32_t* ptrs[64] = {};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lk(mu);
  if (!ptrs[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_route_scratch);
    if (e != cudaSuccess) {
      t_last_cuda_error = e;
      return nullptr;
    }
    ptrs[dev] = static_cast<int32_t*>(p);
  }
  return ptrs[dev];
}

}  // namespace

extern "C" {

const char* moesq_status_str(moesq_status s) {
  switch (s) {
    case MOESQ_OK: return "ok";
    case MOESQ_ERR_INVALID_ARG: return "invalid argument";
    case MOESQ_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case MOESQ_ERR_CUDA: return "CUDA error";
    case MOESQ_ERR_TIMEOUT: return "device wait timed out";
    case MOESQ_ERR_DEVICE_FAULT: return "device-side validation failed";
    case MOESQ_ERR_WORKSPACE: return "workspace too small";
  }
  return "unknown status";
}

const char* moesq_version(void) { return "moesq 0.1 sm_100a"; }

const char* moesq_last_cuda_error(void) {
  return t_last_cuda_error == cudaSuccess ? "no error" : cudaGetErrorString(t_last_cuda_error);
}

moesq_status moesq_get_device_error(void* stream, int32_t* device_code) {
  cudaStream_t s = as_stream(stream);
  MOESQ_CUDA(cudaStreamSynchronize(s));
  int v = 0, zero = 0;
  MOESQ_CUDA(cudaMemcpyFromSymbol(&v, g_error_word, sizeof(int)));
  MOESQ_CUDA(cudaMemcpyToSymbol(g_error_word, &zero, sizeof(int)));
  if (device_code) *device_code = v;
  if (v == 0) return MOESQ_OK;
  return (v & 0xFF) == kErrTimeout ? MOESQ_ERR_TIMEOUT : MOESQ_ERR_DEVICE_FAULT;
}

void moesq_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns = ns ? ns : 1; }

size_t moesq_weights_bytes(int E, int M, int K, size_t* per_tensor) {
  const size_t emk = (size_t)E * M * K;
  size_t t[5] = {emk / 4, emk / 16, emk / 32, (size_t)E * 4, emk / 32 * 11};
  size_t sum = 0;
  for (int i = 0; i < 5; ++i) {
    if (per_tensor) per_tensor[i] = t[i];
    sum += align256(t[i]);
  }
  return sum;
}

moesq_status moesq_pack_weights(const uint16_t* w_bf16, int e_begin, int e_count, const moesq_weights* out,
                                void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_weights(out));
  if (!w_bf16 || !aligned(w_bf16, 16)) return MOESQ_ERR_INVALID_ARG;
  if (e_begin < 0 || e_count < 1 || e_begin + e_count > out->E) return MOESQ_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  const int sms = device_info().sms;
  const int M = out->M, K = out->K;
  float* gamma = out->global_scale + e_begin;
  MOESQ_CUDA(cudaMemsetAsync(gamma, 0, sizeof(float) * e_count, s));
  const int64_t groups_per_expert = (int64_t)M * K / 8;
  const int64_t n_groups = groups_per_expert * e_count;
  pack_amax_kernel<<<grid_for(n_groups, 256, sms), 256, 0, s>>>(w_bf16, n_groups, groups_per_expert,
                                                                 reinterpret_cast<unsigned int*>(gamma));
  MOESQ_TRY(last_launch());
  pack_gamma_kernel<<<(e_count + 255) / 256, 256, 0, s>>>(gamma, e_count);
  MOESQ_TRY(last_launch());
  PackOut po{out->values, out->mask, out->scales, out->global_scale, out->ktiles, out->layout};
  const int64_t n_blocks = (int64_t)e_count * M * (K / 32);
  pack_blocks_kernel<<<grid_for(n_blocks, 256, sms), 256, 0, s>>>(w_bf16, e_begin, n_blocks, M, K, po);
  return last_launch();
}

moesq_status moesq_import_dense_nvfp4(const uint8_t* codes, const uint8_t* scales, const float* global_scale,
                                      int e_begin, int e_count, const moesq_weights* out, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_weights(out));
  if (!codes || !scales || !global_scale || !aligned(codes, 16)) return MOESQ_ERR_INVALID_ARG;
  if (e_begin < 0 || e_count < 1 || e_begin + e_count > out->E) return MOESQ_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  const int M = out->M, K = out->K;
  PackOut po{out->values, out->mask, out->scales, out->global_scale, out->ktiles, out->layout};
  const int64_t n_blocks = (int64_t)e_count * M * (K / 32);
  import_dense_kernel<<<grid_for(n_blocks, 256, device_info().sms), 256, 0, s>>>(
      codes, scales, global_scale, e_begin, n_blocks, M, K, po, out->global_scale);
  return last_launch();
}

moesq_status moesq_export_dense_nvfp4(const moesq_weights* w, uint8_t* codes, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_weights(w));
  if (!codes || !aligned(codes, 16)) return MOESQ_ERR_INVALID_ARG;
  const int64_t n_blocks = (int64_t)w->E * w->M * (w->K / 32);
  export_dense_kernel<<<grid_for(n_blocks, 256, device_info().sms), 256, 0, as_stream(stream)>>>(
      w->values, w->mask, n_blocks, w->K, codes);
  return last_launch();
}

int64_t moesq_rows_capacity(int T, int k, int E) {
  if (T < 0 || k < 0 || E < 0) return 0;
  const int64_t R = (int64_t)T * k;
  const int64_t rc = R + 127 * std::min<int64_t>(E, R);
  return std::max<int64_t>(128, (rc + 127) / 128 * 128);
}

size_t moesq_route_workspace_bytes(int T, int E) {
  const size_t nblk = (size_t)(T + kRouteTPB - 1) / kRouteTPB;
  return align256(nblk * (size_t)E * 4);
}

moesq_status moesq_route_permute(const float* logits, const moesq_routing* rt, void* workspace,
                                 size_t workspace_bytes, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_routing(rt));
  if (!logits || !aligned(logits, 4)) return MOESQ_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < moesq_route_workspace_bytes(rt->T, rt->E)) return MOESQ_ERR_WORKSPACE;
  if (!aligned(workspace, 4)) return MOESQ_ERR_INVALID_ARG;
  return route_launch(logits, rt, static_cast<int32_t*>(workspace), as_stream(stream));
}

moesq_status moesq_quantize_act(const uint16_t* x_bf16, int T, int K, const moesq_routing* rt, const float* gamma,
                                int rows_cap, uint8_t* codes, uint8_t* scales, void* stream) {
  MOESQ_NVTX_RANGE();
  if (!x_bf16 || !gamma || !codes || !scales) return MOESQ_ERR_INVALID_ARG;
  if (T < 1 || K < 256 || K % 256) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(x_bf16, 16) || !aligned(codes, 16) || !aligned(gamma, 4)) return MOESQ_ERR_INVALID_ARG;
  if (rows_cap < 128 || rows_cap % 128) return MOESQ_ERR_INVALID_ARG;
  int k = 1, E = 1;
  const int32_t* ids = nullptr;
  const int32_t* s2r = nullptr;
  if (rt) {
    MOESQ_TRY(check_routing(rt));
    if (rt->T != T || rows_cap != rt->rows_cap) return MOESQ_ERR_INVALID_ARG;
    k = rt->k;
    E = rt->E;
    ids = rt->topk_ids;
    s2r = rt->slot_to_row;
  } else if (rows_cap < T) {
    return MOESQ_ERR_INVALID_ARG;
  }
  cudaStream_t s = as_stream(stream);
  const int sms = device_info().sms;
  const int64_t token_tasks = (int64_t)T * ((K + 1023) / 1024);
  // fewer (token, chunk) tasks than about 16 warps per SM: one warp per slot
  // instead of one per token, so that enough warps run
  const int slot_groups = token_tasks < (int64_t)16 * sms ? k : 1;
  const int64_t tasks = token_tasks * slot_groups;
  if (tasks >= ((int64_t)1 << 31) || (int64_t)T * k >= ((int64_t)1 << 31)) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  return launch_pdl(quantize_act_kernel, dim3(grid_for(tasks, 8, sms)), dim3(256), 0, s, x_bf16, T, K, k, ids, s2r,
                    E, gamma, rows_cap, codes, scales, slot_groups);
}

moesq_status moesq_act_global_scale(const uint16_t* x_bf16, int64_t n, float* gamma_out, void* stream) {
  MOESQ_NVTX_RANGE();
  if (!x_bf16 || !gamma_out || n < 1) return MOESQ_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  MOESQ_CUDA(cudaMemsetAsync(gamma_out, 0, sizeof(float), s));
  amax_bf16_kernel<<<grid_for(n, 256 * 8, device_info().sms), 256, 0, s>>>(
      x_bf16, n, reinterpret_cast<unsigned int*>(gamma_out));
  MOESQ_TRY(last_launch());
  amax_to_gamma_kernel<<<1, 32, 0, s>>>(gamma_out, 1, 0);
  return last_launch();
}

moesq_status moesq_grouped_sparse_gemm(const moesq_weights* w, const uint8_t* a_codes, const uint8_t* a_scales,
                                       int rows_cap, const int32_t* counts, const int32_t* row_offsets,
                                       const float* gamma_a, uint16_t* y_bf16, const moesq_gemm_config* cfg,
                                       void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_weights(w));
  if (!a_codes || !a_scales || !counts || !row_offsets || !gamma_a || !y_bf16) return MOESQ_ERR_INVALID_ARG;
  if (rows_cap < 128 || rows_cap % 128) return MOESQ_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(a_scales, 16) || !aligned(y_bf16, 2)) return MOESQ_ERR_INVALID_ARG;
  if (!aligned(counts, 4) || !aligned(row_offsets, 4) || !aligned(gamma_a, 4)) return MOESQ_ERR_INVALID_ARG;
  int tile_n = cfg ? cfg->tile_n : 0;
  const int num_ctas = cfg ? cfg->num_ctas : 0;
  const int sm_mode = cfg ? cfg->sm_mode : 0;
  if (tile_n != 0 && tile_n != 64 && tile_n != 128) return MOESQ_ERR_INVALID_ARG;
  if (num_ctas < 0 || sm_mode < 0 || sm_mode > 2) return MOESQ_ERR_INVALID_ARG;
  if (sm_mode == 2) {
    if (w->M % 256 || (tile_n != 0 && tile_n != 128)) return MOESQ_ERR_UNSUPPORTED_SHAPE;
    if (!aligned(a_scales, 16)) return MOESQ_ERR_INVALID_ARG;
    return launch_gemm_pair(w, a_codes, a_scales, rows_cap, counts, row_offsets, gamma_a, y_bf16, num_ctas,
                            as_stream(stream));
  }
  if (tile_n == 0) {
    // The counts stay on the device.  The aligned row capacity, less the
    // padding of at most 127 rows per expert, bounds the mean rows per expert.
    const int64_t rows_est = std::max<int64_t>(0, (int64_t)rows_cap - 127 * (int64_t)w->E);
    tile_n = rows_est / w->E > 64 ? 128 : 64;
  }
  cudaStream_t s = as_stream(stream);
  if (tile_n == 64)
    return launch_gemm<64>(w, a_codes, a_scales, rows_cap, counts, row_offsets, gamma_a, y_bf16, num_ctas, s);
  return launch_gemm<128>(w, a_codes, a_scales, rows_cap, counts, row_offsets, gamma_a, y_bf16, num_ctas, s);
}

moesq_status moesq_grouped_dense_gemm(const moesq_dense_weights* w, const uint8_t* a_codes,
                                      const uint8_t* a_scales16, int rows_cap, const int32_t* counts,
                                      const int32_t* row_offsets, const float* gamma_a, uint16_t* y_bf16,
                                      const moesq_gemm_config* cfg, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_dense_weights(w));
  if (!a_codes || !a_scales16 || !counts || !row_offsets || !gamma_a || !y_bf16) return MOESQ_ERR_INVALID_ARG;
  if (rows_cap < 128 || rows_cap % 128) return MOESQ_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(a_scales16, 16) || !aligned(y_bf16, 2)) return MOESQ_ERR_INVALID_ARG;
  if (!aligned(counts, 4) || !aligned(row_offsets, 4) || !aligned(gamma_a, 4)) return MOESQ_ERR_INVALID_ARG;
  int tile_n = cfg ? cfg->tile_n : 0;
  const int num_ctas = cfg ? cfg->num_ctas : 0;
  const int sm_mode = cfg ? cfg->sm_mode : 0;
  if (tile_n != 0 && tile_n != 64 && tile_n != 128) return MOESQ_ERR_INVALID_ARG;
  if (num_ctas < 0 || sm_mode < 0 || sm_mode > 2) return MOESQ_ERR_INVALID_ARG;
  if (sm_mode == 2) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (tile_n == 0) {
    const int64_t rows_est = std::max<int64_t>(0, (int64_t)rows_cap - 127 * (int64_t)w->E);
    tile_n = rows_est / w->E > 64 ? 128 : 64;
  }
  cudaStream_t s = as_stream(stream);
  if (tile_n == 64)
    return launch_gemm_tiles<64, true>(w->dtiles, w->global_scale, w->E, w->M, w->K, a_codes, a_scales16, rows_cap,
                                       counts, row_offsets, gamma_a, GemmOut{y_bf16, nullptr, nullptr, nullptr},
                                       num_ctas, s);
  return launch_gemm_tiles<128, true>(w->dtiles, w->global_scale, w->E, w->M, w->K, a_codes, a_scales16, rows_cap,
                                      counts, row_offsets, gamma_a, GemmOut{y_bf16, nullptr, nullptr, nullptr},
                                      num_ctas, s);
}

size_t moesq_dense_weights_bytes(int E, int M, int K, size_t* per_tensor) {
  const size_t emk = (size_t)E * M * K;
  size_t t[4] = {emk / 2, emk / 16, (size_t)E * 4, emk / 32768 * kDTileBytes};   // 18 KB per 128 x 256 tile
  size_t sum = 0;
  for (int i = 0; i < 4; ++i) {
    if (per_tensor) per_tensor[i] = t[i];
    sum += align256(t[i]);
  }
  return sum;
}

moesq_status moesq_pack_dense_nvfp4(const uint16_t* w_bf16, int e_begin, int e_count, const moesq_dense_weights* out,
                                    void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_dense_weights(out));
  if (!w_bf16 || !aligned(w_bf16, 16)) return MOESQ_ERR_INVALID_ARG;
  if (e_begin < 0 || e_count < 1 || e_begin + e_count > out->E) return MOESQ_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  const int sms = device_info().sms;
  const int M = out->M, K = out->K;
  float* gamma = out->global_scale + e_begin;
  MOESQ_CUDA(cudaMemsetAsync(gamma, 0, sizeof(float) * e_count, s));
  const int64_t groups_per_expert = (int64_t)M * K / 8;
  dense_amax_kernel<<<grid_for(groups_per_expert * e_count, 256, sms), 256, 0, s>>>(
      w_bf16, groups_per_expert * e_count, groups_per_expert, reinterpret_cast<unsigned int*>(gamma));
  MOESQ_TRY(last_launch());
  pack_gamma_kernel<<<(e_count + 255) / 256, 256, 0, s>>>(gamma, e_count);
  MOESQ_TRY(last_launch());
  DensePackOut po{out->codes, out->scales, out->global_scale, out->dtiles};
  const int64_t n_groups = (int64_t)e_count * M * (K / 16);
  dense_pack_kernel<<<grid_for(n_groups, 256, sms), 256, 0, s>>>(w_bf16, e_begin, n_groups, M, K, po);
  return last_launch();
}

moesq_status moesq_expand_scales16(const uint8_t* a_scales, int rows_cap, int K, uint8_t* a_scales16, void* stream) {
  MOESQ_NVTX_RANGE();
  if (!a_scales || !a_scales16 || !aligned(a_scales, 4) || !aligned(a_scales16, 4)) return MOESQ_ERR_INVALID_ARG;
  if (rows_cap < 128 || rows_cap % 128 || K < 256 || K % 256) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  const int64_t n_words = (int64_t)rows_cap * (K / 16) / 4;
  expand_scales16_kernel<<<grid_for(n_words, 256, device_info().sms), 256, 0, as_stream(stream)>>>(a_scales, n_words,
                                                                                                  K, a_scales16);
  return last_launch();
}

}  // extern "C"

namespace {

// Times `launch(cfg)` for every candidate (one warm-up launch, then `reps`
// launches between CUDA events on s) and keeps the fastest.
template <typename Launch>
moesq_status autotune_configs(const moesq_gemm_config* cands, int n, int reps, Launch&& launch,
                              moesq_gemm_config* best, float* best_ms, cudaStream_t s) {
  if (!best || !best_ms || reps < 1) return MOESQ_ERR_INVALID_ARG;
  cudaEvent_t ev[2];
  MOESQ_CUDA(cudaEventCreate(&ev[0]));
  if (cudaEventCreate(&ev[1]) != cudaSuccess) {
    cudaEventDestroy(ev[0]);
    return MOESQ_ERR_CUDA;
  }
  moesq_status st = MOESQ_OK;
  float best_t = -1.0f;
  for (int i = 0; i < n && st == MOESQ_OK; ++i) {
    const moesq_gemm_config& c = cands[i];
    st = launch(c);
    if (st != MOESQ_OK) break;
    if (cudaEventRecord(ev[0], s) != cudaSuccess) { st = MOESQ_ERR_CUDA; break; }
    for (int r = 0; r < reps && st == MOESQ_OK; ++r) st = launch(c);
    if (st != MOESQ_OK) break;
    float ms = 0.0f;
    if (cudaEventRecord(ev[1], s) != cudaSuccess || cudaEventSynchronize(ev[1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, ev[0], ev[1]) != cudaSuccess) {
      st = MOESQ_ERR_CUDA;
      break;
    }
    ms /= (float)reps;
    if (best_t < 0.0f || ms < best_t) {
      best_t = ms;
      *best = c;
    }
  }
  cudaEventDestroy(ev[0]);
  cudaEventDestroy(ev[1]);
  if (st == MOESQ_OK) *best_ms = best_t;
  return st;
}

}  // namespace

extern "C" {

moesq_status moesq_gemm_autotune(const moesq_weights* w, const uint8_t* a_codes, const uint8_t* a_scales,
                                 int rows_cap, const int32_t* counts, const int32_t* row_offsets,
                                 const float* gamma_a, uint16_t* y_bf16, int reps,
                                 moesq_gemm_config* best, float* best_ms, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_weights(w));
  if (!best || !best_ms || reps < 1) return MOESQ_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  const int sms = device_info().sms;
  const moesq_gemm_config cands[5] = {{64, 2 * sms, 1}, {128, 2 * sms, 1}, {64, sms, 1}, {128, sms, 1},
                                      {128, 2 * sms, 2}};
  const int n = (w->M % 256) ? 4 : 5;        // SM-pair tiles need M % 256 == 0
  return autotune_configs(
      cands, n, reps,
      [&](const moesq_gemm_config& c) {
        return moesq_grouped_sparse_gemm(w, a_codes, a_scales, rows_cap, counts, row_offsets, gamma_a, y_bf16, &c, s);
      },
      best, best_ms, s);
}

moesq_status moesq_grouped_sparse_gemm_swiglu(const moesq_weights* w, const uint8_t* a_codes,
                                              const uint8_t* a_scales, int rows_cap, const int32_t* counts,
                                              const int32_t* row_offsets, const float* gamma_a,
                                              const float* gamma_h, uint8_t* h_codes, uint8_t* h_scales,
                                              const moesq_gemm_config* cfg, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_weights(w));
  if (w->layout != MOESQ_LAYOUT_SWIGLU) return MOESQ_ERR_INVALID_ARG;
  if (!a_codes || !a_scales || !counts || !row_offsets || !gamma_a || !gamma_h || !h_codes || !h_scales)
    return MOESQ_ERR_INVALID_ARG;
  if (!aligned(counts, 4) || !aligned(row_offsets, 4) || !aligned(gamma_a, 4) || !aligned(gamma_h, 4))
    return MOESQ_ERR_INVALID_ARG;
  if (rows_cap < 128 || rows_cap % 128) return MOESQ_ERR_INVALID_ARG;
  // 16-byte code stores per (row, 32-feature block) in the epilogue
  if (!aligned(a_codes, 16) || !aligned(a_scales, 16) || !aligned(h_codes, 16)) return MOESQ_ERR_INVALID_ARG;
  int tile_n = cfg ? cfg->tile_n : 0;
  const int num_ctas = cfg ? cfg->num_ctas : 0;
  const int sm_mode = cfg ? cfg->sm_mode : 0;
  if (tile_n != 0 && tile_n != 64 && tile_n != 128) return MOESQ_ERR_INVALID_ARG;
  if (num_ctas < 0 || sm_mode < 0 || sm_mode > 2) return MOESQ_ERR_INVALID_ARG;
  if (sm_mode == 2) return MOESQ_ERR_UNSUPPORTED_SHAPE;     // one-SM tiles only
  if (tile_n == 0) {
    const int64_t rows_est = std::max<int64_t>(0, (int64_t)rows_cap - 127 * (int64_t)w->E);
    tile_n = rows_est / w->E > 64 ? 128 : 64;
  }
  cudaStream_t s = as_stream(stream);
  const GemmOut out{nullptr, h_codes, h_scales, gamma_h};
  if (tile_n == 64)
    return launch_gemm_tiles<64, false, true>(w->ktiles, w->global_scale, w->E, w->M, w->K, a_codes, a_scales,
                                              rows_cap, counts, row_offsets, gamma_a, out, num_ctas, s);
  return launch_gemm_tiles<128, false, true>(w->ktiles, w->global_scale, w->E, w->M, w->K, a_codes, a_scales,
                                             rows_cap, counts, row_offsets, gamma_a, out, num_ctas, s);
}

moesq_status moesq_gemm_swiglu_autotune(const moesq_weights* w, const uint8_t* a_codes, const uint8_t* a_scales,
                                        int rows_cap, const int32_t* counts, const int32_t* row_offsets,
                                        const float* gamma_a, const float* gamma_h, uint8_t* h_codes,
                                        uint8_t* h_scales, int reps, moesq_gemm_config* best, float* best_ms,
                                        void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_weights(w));
  if (w->layout != MOESQ_LAYOUT_SWIGLU) return MOESQ_ERR_INVALID_ARG;
  if (!best || !best_ms || reps < 1) return MOESQ_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  const int sms = device_info().sms;
  const moesq_gemm_config cands[4] = {{64, 2 * sms, 1}, {128, 2 * sms, 1}, {64, sms, 1}, {128, sms, 1}};
  return autotune_configs(
      cands, 4, reps,
      [&](const moesq_gemm_config& c) {
        return moesq_grouped_sparse_gemm_swiglu(w, a_codes, a_scales, rows_cap, counts, row_offsets, gamma_a,
                                                gamma_h, h_codes, h_scales, &c, s);
      },
      best, best_ms, s);
}

moesq_status moesq_swiglu_quant(const uint16_t* y_gu, int I, const moesq_routing* rt, const float* gamma_h,
                                uint8_t* h_codes, uint8_t* h_scales, int gu_layout, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_routing(rt));
  if (!y_gu || !gamma_h || !h_codes || !h_scales || !aligned(gamma_h, 4)) return MOESQ_ERR_INVALID_ARG;
  if (gu_layout != MOESQ_LAYOUT_PLAIN && gu_layout != MOESQ_LAYOUT_SWIGLU) return MOESQ_ERR_INVALID_ARG;
  if (I < 256 || I % 256) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  if (!aligned(y_gu, 16) || !aligned(h_codes, 16)) return MOESQ_ERR_INVALID_ARG;
  const int R = rt->T * rt->k;
  return launch_pdl(swiglu_quant_kernel, dim3(grid_for(R, 8, device_info().sms)), dim3(256), 0, as_stream(stream),
                    y_gu, I, R, rt->E, rt->topk_ids, rt->slot_to_row, rt->rows_cap, gamma_h, h_codes, h_scales,
                    (unsigned int*)nullptr, gu_layout);
}

moesq_status moesq_combine(const uint16_t* y, int H, const moesq_routing* rt, uint16_t* out, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_routing(rt));
  if (!y || !out || H < 8 || H % 8) return MOESQ_ERR_INVALID_ARG;
  if (!aligned(y, 16) || !aligned(out, 16)) return MOESQ_ERR_INVALID_ARG;
  const int64_t nch = (H + kCombineCols - 1) / kCombineCols;
  const int64_t blocks = (int64_t)rt->T * nch;
  if (blocks >= ((int64_t)1 << 31)) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  const size_t smem = (size_t)rt->k * kCombineCols * 2;
  DeviceInfo& di = device_info();
  if (!di.combine_attr) {
    MOESQ_CUDA(cudaFuncSetAttribute(combine_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 32 * kCombineCols * 2));
    di.combine_attr = true;
  }
  return launch_pdl(combine_kernel, dim3((unsigned)blocks), dim3(kCombineThreads), smem, as_stream(stream), y, H,
                    rt->T, rt->k, rt->topk_w, rt->slot_to_row, rt->rows_cap, out, g_timeout_ns);
}

size_t moesq_layer_workspace_bytes(int T, int k, int E, int H, int I) {
  return carve(nullptr, T, k, E, H, I, false).bytes;
}

size_t moesq_layer_host_workspace_bytes(int T, int k, int E, int H, int I) {
  return carve(nullptr, T, k, E, H, I, true).bytes;
}

moesq_status moesq_moe_layer(const uint16_t* x_bf16, const float* logits, int T, int k, const moesq_weights* w_gu,
                             const moesq_weights* w_dn, const float* gamma_a_gu, const float* gamma_a_dn,
                             uint16_t* out_bf16, void* workspace, size_t workspace_bytes, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_layer(T, k, w_gu, w_dn));
  if (!x_bf16 || !logits || !gamma_a_gu || !gamma_a_dn || !out_bf16) return MOESQ_ERR_INVALID_ARG;
  const int E = w_gu->E, H = w_gu->K, I = w_gu->M / 2;
  if (!workspace || !aligned(workspace, 256)) return MOESQ_ERR_INVALID_ARG;
  LayerWs ws = carve(workspace, T, k, E, H, I, false);
  if (workspace_bytes < ws.bytes) return MOESQ_ERR_WORKSPACE;
  return layer_body(x_bf16, logits, T, k, w_gu, w_dn, gamma_a_gu, gamma_a_dn, out_bf16, ws, as_stream(stream));
}

moesq_status moesq_moe_layer_host(const uint16_t* x_bf16_host, const float* logits_host, int T, int k,
                                  const moesq_weights* w_gu, const moesq_weights* w_dn, const float* gamma_a_gu,
                                  const float* gamma_a_dn, uint16_t* out_bf16_host, void* workspace,
                                  size_t workspace_bytes, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_layer(T, k, w_gu, w_dn));
  if (!x_bf16_host || !logits_host || !gamma_a_gu || !gamma_a_dn || !out_bf16_host) return MOESQ_ERR_INVALID_ARG;
  const int E = w_gu->E, H = w_gu->K, I = w_gu->M / 2;
  if (!workspace || !aligned(workspace, 256)) return MOESQ_ERR_INVALID_ARG;
  LayerWs ws = carve(workspace, T, k, E, H, I, true);
  if (workspace_bytes < ws.bytes) return MOESQ_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  MOESQ_CUDA(cudaMemcpyAsync(ws.x_in, x_bf16_host, (size_t)T * H * 2, cudaMemcpyHostToDevice, s));
  MOESQ_CUDA(cudaMemcpyAsync(ws.logits_in, logits_host, (size_t)T * E * 4, cudaMemcpyHostToDevice, s));
  MOESQ_TRY(layer_body(ws.x_in, ws.logits_in, T, k, w_gu, w_dn, gamma_a_gu, gamma_a_dn, ws.out, ws, s));
  MOESQ_CUDA(cudaMemcpyAsync(out_bf16_host, ws.out, (size_t)T * H * 2, cudaMemcpyDeviceToHost, s));
  MOESQ_CUDA(cudaStreamSynchronize(s));
  return MOESQ_OK;
}

moesq_status moesq_calibrate_layer(const uint16_t* x_bf16, const float* logits, int T, int k,
                                   const moesq_weights* w_gu, const moesq_weights* w_dn, float* gamma_a_gu,
                                   float* gamma_a_dn, void* workspace, size_t workspace_bytes, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_layer(T, k, w_gu, w_dn));
  if (!x_bf16 || !logits || !gamma_a_gu || !gamma_a_dn) return MOESQ_ERR_INVALID_ARG;
  const int E = w_gu->E, H = w_gu->K, I = w_gu->M / 2;
  if (!workspace || !aligned(workspace, 256)) return MOESQ_ERR_INVALID_ARG;
  LayerWs ws = carve(workspace, T, k, E, H, I, false);
  if (workspace_bytes < ws.bytes) return MOESQ_ERR_WORKSPACE;
  cudaStream_t s = as_stream(stream);
  const int sms = device_info().sms;
  moesq_routing rt = routing_of(ws, T, E, k);
  MOESQ_TRY(moesq_route_permute(logits, &rt, ws.route_ws, moesq_route_workspace_bytes(T, E), s));
  MOESQ_CUDA(cudaMemsetAsync(gamma_a_gu, 0, sizeof(float) * E, s));
  routed_amax_kernel<<<grid_for((int64_t)T * k, 8, sms), 256, 0, s>>>(x_bf16, T, H, k, rt.topk_ids, E,
                                                                       reinterpret_cast<unsigned int*>(gamma_a_gu));
  MOESQ_TRY(last_launch());
  amax_to_gamma_kernel<<<1, 1024, 0, s>>>(gamma_a_gu, E, 1);
  MOESQ_TRY(last_launch());
  MOESQ_TRY(moesq_quantize_act(x_bf16, T, H, &rt, gamma_a_gu, rt.rows_cap, ws.a_codes, ws.a_scales, s));
  MOESQ_TRY(moesq_grouped_sparse_gemm(w_gu, ws.a_codes, ws.a_scales, rt.rows_cap, rt.counts, rt.row_offsets,
                                      gamma_a_gu, ws.y_gu, nullptr, s));
  MOESQ_CUDA(cudaMemsetAsync(gamma_a_dn, 0, sizeof(float) * E, s));
  const int R = T * k;
  swiglu_quant_kernel<<<grid_for(R, 8, sms), 256, 0, s>>>(
      ws.y_gu, I, R, E, rt.topk_ids, rt.slot_to_row, rt.rows_cap, nullptr, nullptr, nullptr,
      reinterpret_cast<unsigned int*>(gamma_a_dn), w_gu->layout);
  MOESQ_TRY(last_launch());
  amax_to_gamma_kernel<<<1, 1024, 0, s>>>(gamma_a_dn, E, 1);
  return last_launch();
}

moesq_status moesq_debug_bounded_wait(uint64_t timeout_ns, void* stream) {
  debug_wait_kernel<<<1, 32, 0, as_stream(stream)>>>(timeout_ns ? timeout_ns : 1);
  return last_launch();
}

moesq_status moesq_mma_peak(int sparse, int n, int ctas_per_sm, int with_copies, int iters, double* tflops,
                            void* stream) {
  MOESQ_NVTX_RANGE();
  if (!tflops || iters < 1 || (sparse != 0 && sparse != 1)) return MOESQ_ERR_INVALID_ARG;
  if (with_copies != 0 && with_copies != 1) return MOESQ_ERR_INVALID_ARG;
  if (ctas_per_sm != 1 && ctas_per_sm != 2) return MOESQ_ERR_INVALID_ARG;
  if (n < 16 || n > 256 || n % 16 || (ctas_per_sm == 2 && n > 128)) return MOESQ_ERR_INVALID_ARG;
  cudaStream_t s = as_stream(stream);
  const int sms = device_info().sms;
  // dynamic shared memory sized so that exactly ctas_per_sm CTAs fit on an
  // SM: each then owns 512 / ctas_per_sm TMEM columns
  const size_t smem = ctas_per_sm == 1 ? (size_t)150 * 1024 : (size_t)100 * 1024;
  const uint32_t cols = ctas_per_sm == 1 ? 512u : 256u;
  auto kern = sparse ? (with_copies ? mma_peak_kernel<true, true> : mma_peak_kernel<true, false>)
                     : (with_copies ? mma_peak_kernel<false, true> : mma_peak_kernel<false, false>);
  MOESQ_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  cudaEvent_t ev[2];
  MOESQ_CUDA(cudaEventCreate(&ev[0]));
  if (cudaEventCreate(&ev[1]) != cudaSuccess) {
    cudaEventDestroy(ev[0]);
    return MOESQ_ERR_CUDA;
  }
  moesq_status st = MOESQ_OK;
  float ms = 0.0f;
  if (cudaEventRecord(ev[0], s) != cudaSuccess) st = MOESQ_ERR_CUDA;
  if (st == MOESQ_OK) {
    kern<<<sms * ctas_per_sm, kPeakThreads, smem, s>>>(n, iters, cols, g_timeout_ns, nullptr);
    st = last_launch();
  }
  if (st == MOESQ_OK && (cudaEventRecord(ev[1], s) != cudaSuccess || cudaEventSynchronize(ev[1]) != cudaSuccess ||
                         cudaEventElapsedTime(&ms, ev[0], ev[1]) != cudaSuccess))
    st = MOESQ_ERR_CUDA;
  cudaEventDestroy(ev[0]);
  cudaEventDestroy(ev[1]);
  if (st != MOESQ_OK) return st;
  const double k_dense = sparse ? 128.0 : 64.0;
  const double flops = (double)sms * ctas_per_sm * iters * 2.0 * 2.0 * 128.0 * n * k_dense;
  *tflops = flops / ((double)ms * 1e-3) / 1e12;
  return MOESQ_OK;
}

moesq_status moesq_route_permute_noalloc(const float* logits, const moesq_routing* rt, void* stream) {
  MOESQ_NVTX_RANGE();
  MOESQ_TRY(check_routing(rt));
  if (!logits || !aligned(logits, 4)) return MOESQ_ERR_INVALID_ARG;
  if (rt->T > kNoAllocMaxT) return MOESQ_ERR_UNSUPPORTED_SHAPE;   // beyond the static scratch
  const int nblk = (rt->T + kRouteTPB - 1) / kRouteTPB;
  if ((size_t)nblk * (size_t)rt->E > kNoAllocScratchInts) return MOESQ_ERR_UNSUPPORTED_SHAPE;
  int32_t* bc = route_scratch_device_ptr();
  if (!bc) return MOESQ_ERR_CUDA;
  // the counting kernel writes every [block][expert] count the later kernels
  // read, so the scratch needs no clearing between calls.
  return route_launch(logits, rt, bc, as_stream(stream));
}

}  // extern "C"
