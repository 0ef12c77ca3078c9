/*
 * moesq.h -- C ABI of the paired-4:8 NVFP4 grouped sparse GEMM for routed
 * Mixture-of-Experts layers on NVIDIA B200 (sm_100a).
 *
 * The operations follow "Hardware-Native Joint Sparse-Quantization for
 * Trillion-Scale Mixture-of-Experts" (arXiv 2610.02241; cited below as
 * "paper") and the storage layout of the model card
 * "Kimi-K2.5-P48NVFP4-MoESQ" (cited as "model card").
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor arguments are DEVICE pointers unless a comment says "host".
 *    The caller owns all memory; the library never allocates or frees.
 *  - Every call is asynchronous on the given stream (a cudaStream_t passed as
 *    void*, NULL = the legacy default stream), does no host synchronisation
 *    and reads no device data on the host, so a sequence of calls can be
 *    captured into a CUDA graph.  The exceptions are moesq_get_device_error
 *    (synchronises), moesq_moe_layer_host (synchronises at the end), the
 *    autotuners and moesq_mma_peak (time launches, synchronise).
 *  - Every call that launches work opens an NVTX range named after itself
 *    (host side, around its checks and launches) for timeline tools.
 *  - Shape and argument errors are detected on the host and returned at once;
 *    nothing is launched then.  Faults detected on the device (inconsistent
 *    routing counts, out-of-range expert ids, a bounded wait that ran out)
 *    set a device-side error word that moesq_get_device_error reports.
 *    No call aborts the process or traps the GPU.
 *  - bf16 tensors are passed as uint16_t bit patterns.  NVFP4 values are
 *    E2M1 codes, two per byte, the even (lower-K) element in the low nibble.
 *    Scales are UE4M3 codes (unsigned E4M3, one byte).
 *
 * Sizes: K (contraction) must be a multiple of 256, M (weight output rows) a
 * multiple of 128, 1 <= E <= 512 experts, 1 <= k <= min(E, 32).
 */
#ifndef MOESQ_H_
#define MOESQ_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOESQ_OK = 0,
  MOESQ_ERR_INVALID_ARG = 1,       /* null pointer, bad size, misaligned buffer */
  MOESQ_ERR_UNSUPPORTED_SHAPE = 2, /* K % 256, M % 128, E or k out of range */
  MOESQ_ERR_CUDA = 3,              /* a CUDA runtime call failed */
  MOESQ_ERR_TIMEOUT = 4,           /* a device wait ran past its limit */
  MOESQ_ERR_DEVICE_FAULT = 5,      /* device-side validation failed */
  MOESQ_ERR_WORKSPACE = 6          /* workspace smaller than required */
} moesq_status;

/* Rows of the expert-aligned row space start every MOESQ_ROW_ALIGN rows. */
#define MOESQ_ROW_ALIGN 128

/* Human-readable name of a status code (static string). */
const char* moesq_status_str(moesq_status s);

/* Library version string, e.g. "moesq 0.1 sm_100a" (static string). */
const char* moesq_version(void);

/* Text of the CUDA error behind the calling thread's most recent
 * MOESQ_ERR_CUDA ("no error" if none); static string. */
const char* moesq_last_cuda_error(void);

/* Synchronises `stream`, then reads and clears the device error word.
 * *device_code (host) receives the raw word: 0 = none; otherwise
 * (where << 8) | kind, kind 4 = wait timeout, 5 = validation fault;
 * where: 1-4 grouped GEMM, 5 routing, 6 activation quantisation, 8 SwiGLU,
 * 9 combine, 10 dense import / export.
 * Returns MOESQ_OK, MOESQ_ERR_TIMEOUT or MOESQ_ERR_DEVICE_FAULT. */
moesq_status moesq_get_device_error(void* stream, int32_t* device_code);

/* Limit, in nanoseconds, of every bounded wait inside the kernels launched
 * after this call (default 2e9).  Host-side setting, not thread-safe. */
void moesq_set_wait_timeout_ns(uint64_t ns);

/* ------------------------------------------------------------------ weights
 * One stack of E expert linears W_e [M, K] (swap-AB orientation: the weight is
 * the sparse left operand, paper Sec. 3.4), paired-4:8 sparse NVFP4.
 *
 * Storage form (model card, "Sparse storage layout (paired48_sparse,
 * pair-bitmask v1)"):
 *   values  [E][M][K/4]  the 2 kept bytes of every 4-byte chunk, in K order;
 *                        a byte is one kept pair (two adjacent K elements)
 *   mask    [E][M][K/16] 4 bits per chunk of 8 K elements, bit p = pair p
 *                        kept (exactly 2 set), low nibble = lower-K chunk
 *   scales  [E][M][K/32] UE4M3 block scale per 32 dense K (linear layout)
 *   global_scale [E]     float32 gamma_w, the tensor multiplier of paper
 *                        Eq. 5 (dequantised weight = code * scale / gamma)
 * Kernel form (derived at pack time, the "kernel's own layout" the model
 * card's loader builds; read only by moesq_grouped_sparse_gemm):
 *   ktiles  [E][M/128][K/256][11264]  one contiguous tile per 128 weight rows
 *           and 256 dense K, copied to shared memory as is:
 *     bytes [0, 8192)      the tile's 128 rows of `values` (64 B each), row r
 *                          at r*64 with its 16-byte chunk c stored in chunk
 *                          position c ^ ((r >> 1) & 3) (the 64-byte swizzle the
 *                          tensor-core descriptor reads)
 *     bytes [8192, 10240)  sparse-MMA metadata, 16 B per row: byte b holds
 *                          chunks 2b (low nibble) and 2b+1; a chunk's nibble
 *                          is i0 | i1 << 2, the indices i0 < i1 of its two
 *                          kept pairs
 *     bytes [10240, 11264) the UE4M3 scales of the two 128-wide K halves, 512 B
 *                          each: the scale of row 32a+b and K sub-block s at
 *                          byte b*16 + a*4 + s
 * The kernel form holds the same 11*M*K/32 bytes per expert as the storage
 * form, rearranged so that one K step of the GEMM is one sequential read.
 *
 * layout orders the rows of the kernel form (the storage form always keeps
 * the rows as given):
 *   MOESQ_LAYOUT_PLAIN   kernel row m = storage row m;
 *   MOESQ_LAYOUT_SWIGLU  for a gate_up linear (M = 2I: gate rows [0, I), up
 *                        rows [I, 2I)), the 128 kernel rows of block b are
 *                        gate rows [64 b, 64 b + 64) followed by up rows
 *                        I + [64 b, 64 b + 64), so that one 128-row weight
 *                        tile yields both halves of 64 SwiGLU features (the
 *                        fused SwiGLU + requantisation of App. D.1 "Serving
 *                        integration"); needs M % 256 == 0.
 * The grouped GEMM writes its output columns in kernel row order. */
#define MOESQ_LAYOUT_PLAIN 0
#define MOESQ_LAYOUT_SWIGLU 1

typedef struct {
  int32_t E, M, K;
  uint8_t* values;
  uint8_t* mask;
  uint8_t* scales;
  float* global_scale;
  uint8_t* ktiles;
  int32_t layout;      /* MOESQ_LAYOUT_PLAIN or MOESQ_LAYOUT_SWIGLU */
} moesq_weights;

/* Bytes of each weight tensor: per_tensor[0..4] (host, may be NULL) =
 * values, mask, scales, global_scale, ktiles.  Returns the sum (each tensor
 * rounded up to 256 bytes). */
size_t moesq_weights_bytes(int E, int M, int K, size_t* per_tensor);

/* moesq_pack_weights: bf16 expert weights -> paired-4:8 NVFP4, for experts
 * [e_begin, e_begin + e_count) of `out` (out->E, M, K give the full stack;
 * w_bf16 holds the e_count experts [e_count][M][K] contiguously).
 * Per group of 8 K elements the two pairs of largest w0^2 + w1^2 (binary32)
 * are kept, an exact tie keeping the lower pair index (magnitude pair
 * selection standing in for the learned support of paper Sec. 3.2; paper
 * App. A Eq. 6 and model card "Sparsity" fix the pattern set).  Scales are
 * computed on the masked weights (paper Sec. 3.4, Eq. 5):
 *   gamma = 448 / (amax_t / 6), amax_t = largest kept |w| of the expert,
 *   code_b = RNE_E4M3(gamma * amax_b / 6) saturating at 448,
 *   s_b = UE4M3(code_b) / gamma, value code = RNE_E2M1(w / s_b) (Eq. 3),
 * in binary32 with one rounding per operation; a block with code_b = 0 gets
 * value codes 0; a zero expert gets gamma = 1.  Writes all six tensors.
 * out->global_scale of the packed experts is used as scratch first. */
moesq_status moesq_pack_weights(const uint16_t* w_bf16, int e_begin, int e_count,
                                const moesq_weights* out, void* stream);

/* moesq_import_dense_nvfp4: weights already quantised to NVFP4 in the
 * paired 4:8 pattern, held densely, -> the storage and kernel forms of `out`
 * for experts [e_begin, e_begin + e_count) (model card "Kimi-K2.5-P48NVFP4-
 * MoESQ", pair-bitmask v1 layout).  Inputs (device, e_count experts
 * contiguous): codes [e_count][M][K/2] (two E2M1 codes per byte, even K in the
 * low nibble), scales [e_count][M][K/32] (UE4M3, one per 32 dense K,
 * row-major), global_scale [e_count] (the stored gamma).  Per 4-byte chunk
 * (4 pairs of K) the nonzero bytes are kept; a chunk with fewer than two
 * nonzero bytes keeps its lowest-index zero bytes as well (the model card's
 * canonical rule), so dense -> pair-bitmask -> dense is lossless.  A chunk
 * with more than two nonzero bytes is not in the pattern: the device error
 * word gets a validation fault (where 10) and the chunk keeps its lowest two
 * nonzero bytes.  codes must be 16-byte aligned. */
moesq_status moesq_import_dense_nvfp4(const uint8_t* codes, const uint8_t* scales, const float* global_scale,
                                      int e_begin, int e_count, const moesq_weights* out, void* stream);

/* moesq_export_dense_nvfp4: the storage form of all w->E experts -> dense
 * NVFP4 codes [E][M][K/2] (kept bytes at their chunk positions, zeros
 * elsewhere); the scales and global scales of the dense form are w->scales
 * and w->global_scale unchanged.  A mask nibble without exactly two bits set
 * sets a validation fault (where 10).  codes must be 16-byte aligned. */
moesq_status moesq_export_dense_nvfp4(const moesq_weights* w, uint8_t* codes, void* stream);

/* ------------------------------------------------------------------ routing
 * Router output for T tokens, top-k of E experts.  Rows of every activation
 * tensor handed to the grouped GEMM live in the "expert-aligned row space":
 * expert e owns rows [row_offsets[e], row_offsets[e] + counts[e]) and
 * row_offsets[e+1] - row_offsets[e] = counts[e] rounded up to
 * MOESQ_ROW_ALIGN (the paper's per-expert fixed stride, App. D.1, with the
 * capacity shrunk to the 128-row MMA tile).  Rows in the padding are never
 * read for a valid output and never written by the activation kernels.
 * rows_cap is the allocated number of rows (>= row_offsets[E]).          */
typedef struct {
  int32_t T, E, k;
  int32_t rows_cap;
  int32_t* topk_ids;       /* [T*k] expert of slot t*k + j, descending logit */
  float* topk_w;           /* [T*k] softmax(logits[t])[topk_ids[t*k + j]] */
  int32_t* counts;         /* [E] slots routed to each expert */
  int32_t* offsets;        /* [E+1] exclusive prefix of counts (compact order) */
  int32_t* row_offsets;    /* [E+1] expert-aligned row starts */
  int32_t* sorted_to_slot; /* [T*k] compact position -> slot, ordered by
                              (expert, token, slot) */
  int32_t* slot_to_row;    /* [T*k] slot -> row in the aligned row space */
} moesq_routing;

/* Rows of the aligned row space needed for any routing of T tokens, top-k of
 * E experts: T*k + 127 * min(E, T*k), rounded up to 128. */
int64_t moesq_rows_capacity(int T, int k, int E);

/* Scratch bytes moesq_route_permute needs. */
size_t moesq_route_workspace_bytes(int T, int E);

/* moesq_route_permute: logits float32 [T][E] -> top-k ids and softmax gate
 * weights, per-expert counts, compact and aligned offsets and the stable
 * token permutation (routing and dispatch planning, paper App. D.1).
 * Selection is by descending logit, an exact tie to the lower expert id;
 * the weight is the softmax over all E logits (binary32, not renormalised
 * over the k chosen).  Ids, counts, offsets and both permutations are
 * exact integers.  rt->rows_cap must be >= moesq_rows_capacity(T, k, E). */
moesq_status moesq_route_permute(const float* logits, const moesq_routing* rt,
                                 void* workspace, size_t workspace_bytes, void* stream);

/* moesq_route_permute_noalloc: the same routing as moesq_route_permute, for
 * callers that cannot provide scratch memory -- e.g. an op slot of an
 * inference runtime that hands the op only its inputs and outputs, or code
 * running where allocating device memory is not allowed (a tight serving
 * loop with a fixed memory budget).  The paper has no counterpart; this is a
 * calling convention of this library.  Its scratch (the per-block expert
 * counts) is a static device array inside the library, sized for at most
 * T = 16384 tokens and E = 512 experts (256 KiB on every GPU that loads the
 * library, held until the process exits); larger T returns
 * MOESQ_ERR_UNSUPPORTED_SHAPE.  No memory is allocated.
 * The first call on a device looks up the array's device address for that
 * device (cudaGetSymbolAddress); make that first call before any stream
 * capture.  All calls share the one array: calls that may overlap on the GPU
 * (different streams, or different host threads) race and must be
 * serialised by the caller.  Each call overwrites every scratch entry it
 * reads, so nothing needs clearing between calls. */
moesq_status moesq_route_permute_noalloc(const float* logits, const moesq_routing* rt, void* stream);

/* --------------------------------------------------------- activation quant
 * Scales of an activation tensor with R rows (R a multiple of 128) and K
 * columns use the MMA scale layout [R/128][K/128][32][4][4]: the scale of
 * row 128*r + 32*a + b for K elements [128*c + 32*s, 128*c + 32*s + 32) sits
 * at byte ((r * (K/128) + c) * 512) + b*16 + a*4 + s.
 * Codes are row-major [R][K/2].
 *
 * moesq_quantize_act: bf16 x [T][K] -> NVFP4 (paper Sec. 3.4 and App. D.1:
 * dynamic per-32 UE4M3 block scales under a stored float32 global scale;
 * model card "Activations").  Per 32-element block:
 *   code_b = RNE_E4M3(gamma * amax_b / 6) saturating at 448,
 *   s_b = UE4M3(code_b) / gamma, value code = RNE_E2M1(x / s_b) saturating at 6.
 * Dispatch form (rt != NULL): every slot (t, j) writes token t, quantised
 * with gamma[rt->topk_ids[t*k+j]], to row rt->slot_to_row[t*k+j] (the fused
 * dispatch-scatter + quantisation of App. D.1); rows_cap = rt->rows_cap.
 * Plain form (rt == NULL): token t goes to row t with gamma[0]; rows_cap is
 * the allocated row count (multiple of 128, >= T).
 * K is a multiple of 256; x_bf16 and codes are 16-byte aligned
 * (MOESQ_ERR_INVALID_ARG otherwise).                                      */
moesq_status moesq_quantize_act(const uint16_t* x_bf16, int T, int K,
                                const moesq_routing* rt, const float* gamma,
                                int rows_cap, uint8_t* codes, uint8_t* scales,
                                void* stream);

/* moesq_act_global_scale: *gamma_out (device float) = 448 / (amax / 6) over
 * the n bf16 values of x (paper Eq. 5 applied to a calibration batch; 1 if
 * all are zero).  Calibrates the static activation global scale. */
moesq_status moesq_act_global_scale(const uint16_t* x_bf16, int64_t n, float* gamma_out,
                                    void* stream);

/* -------------------------------------------------------------- grouped GEMM
 * moesq_grouped_sparse_gemm: for every expert e and every valid row r of e
 * (aligned row space, see moesq_routing)
 *   y[r][m] = bf16_RN( alpha_e * sum_k deq(a[r][k]) * deq(W_e[m][k]) ),
 *   alpha_e = 1 / (w->global_scale[e] * gamma_a[e])   (binary32),
 * where deq = E2M1 code value * UE4M3 scale value (paper Sec. 3.4: Y_e^T =
 * W_e X_e^T with the weight as the sparse operand, both block scales applied
 * in the MMA, the tensor scales folded into alpha_e in the epilogue).
 * a_codes [rows_cap][K/2], a_scales in the MMA scale layout, y [rows_cap][M]
 * bf16 (only valid rows are written).  counts [E] and row_offsets [E+1]
 * (device) give expert e the rows row_offsets[e] + [0, counts[e]); each
 * row_offsets[e] is a multiple of 128 and each span row_offsets[e+1] -
 * row_offsets[e] holds at least counts[e] rounded up to 128, so both the
 * compact aligned layout of moesq_routing and a fixed capacity N per expert
 * (row_offsets[e] = e * N, N a multiple of 128: the paper's App. D.1
 * batched layout) qualify.  They are validated on the device (validation
 * fault, where 4, and no output otherwise).
 * cfg may be NULL (defaults).                                            */
typedef struct {
  int32_t tile_n;      /* token rows per tile: 0 = auto, 64 or 128 */
  int32_t num_ctas;    /* persistent CTAs: 0 = two per SM (two independent
                          tensor-core issue streams per SM) */
  int32_t sm_mode;     /* 0 = auto; 1 = one SM per 128-row weight tile;
                          2 = a pair of SMs (a cluster of two CTAs, one
                          tcgen05 cta_group::2 MMA per 256-row weight tile,
                          each SM staging half of the 128-row token tile);
                          needs M % 256 == 0 and tile_n 0 or 128
                          (MOESQ_ERR_UNSUPPORTED_SHAPE otherwise); num_ctas
                          then caps twice the number of clusters */
} moesq_gemm_config;

moesq_status moesq_grouped_sparse_gemm(const moesq_weights* w, const uint8_t* a_codes,
                                       const uint8_t* a_scales, int rows_cap,
                                       const int32_t* counts, const int32_t* row_offsets,
                                       const float* gamma_a, uint16_t* y_bf16,
                                       const moesq_gemm_config* cfg, void* stream);

/* moesq_gemm_autotune: times moesq_grouped_sparse_gemm on these inputs for
 * each candidate configuration (token tile 64 or 128 rows x one or two
 * persistent CTAs per SM, and the SM-pair variant when M % 256 == 0), one
 * warm-up launch and `reps` timed launches each
 * (CUDA events on `stream`), and writes the fastest to *best and its mean
 * time in milliseconds to *best_ms (the paper freezes one kernel variant
 * per problem geometry before CUDA-graph capture, App. D.1).  Writes y_bf16
 * as the GEMM does; synchronises the stream, so call it before a capture.
 * reps >= 1. */
moesq_status moesq_gemm_autotune(const moesq_weights* w, const uint8_t* a_codes, const uint8_t* a_scales,
                                 int rows_cap, const int32_t* counts, const int32_t* row_offsets,
                                 const float* gamma_a, uint16_t* y_bf16, int reps,
                                 moesq_gemm_config* best, float* best_ms, void* stream);

/* ------------------------------------------------------- dense NVFP4 control
 * The dense NVFP4 grouped GEMM the paper measures its sparse kernel against
 * (App. D.2: "Dense (transposed)", the same kernel orientation, differing
 * only in sparsity; Tables 8 and 9, Fig. 1a).  Every weight is kept:
 * one UE4M3 scale per 16 K elements (the NVFP4 group), Eq. 5's gamma over
 * the whole expert linear, value codes by Eq. 3 -- 4.5 bits per weight
 * against the sparse form's 2.75 (Eq. 7).                                  */
typedef struct {
  int32_t E, M, K;       /* E <= 512, M % 128 == 0, K % 256 == 0 */
  uint8_t* codes;        /* [E][M][K/2] E2M1, element 2i in the low nibble of byte i */
  uint8_t* scales;       /* [E][M][K/16] UE4M3, row-major */
  float* global_scale;   /* [E] gamma */
  uint8_t* dtiles;       /* kernel form [E][M/128][K/256][18432]: per tile 128 rows x 128 B of
                            codes in the 128-byte swizzle (16-byte chunk c of row r at
                            chunk c ^ (r & 7)), then the scales of the four 64-wide K
                            chunks in the MMA scale layout */
} moesq_dense_weights;

/* Bytes of each dense tensor: per_tensor[0..3] (host, may be NULL) = codes,
 * scales, global_scale, dtiles; returns the sum (each rounded up to 256). */
size_t moesq_dense_weights_bytes(int E, int M, int K, size_t* per_tensor);

/* moesq_pack_dense_nvfp4: bf16 expert weights [e_count][M][K] -> the dense
 * NVFP4 form of experts [e_begin, e_begin + e_count) of `out`:
 * gamma = 448 / (amax / 6) over all weights of the expert linear,
 * per 16-element group code = RNE_E4M3(gamma * amax_16 / 6) saturating at
 * 448, s = UE4M3(code) / gamma, value code = RNE_E2M1(w / s) (binary32, one
 * rounding per operation; a zero group gets codes 0).  w_bf16 is 16-byte
 * aligned. */
moesq_status moesq_pack_dense_nvfp4(const uint16_t* w_bf16, int e_begin, int e_count,
                                    const moesq_dense_weights* out, void* stream);

/* moesq_expand_scales16: activation scales in the MMA scale layout with one
 * code per 32 K ([rows_cap/128][K/128][512], as moesq_quantize_act writes
 * them) -> one code per 16 K in the layout the dense MMA reads
 * ([rows_cap/128][K/64][512]: 64-wide K chunk j, row 32 a + b, 16-group s
 * at b * 16 + a * 4 + s); each 32-block's code serves both of its halves,
 * which leaves every dequantised value unchanged. */
moesq_status moesq_expand_scales16(const uint8_t* a_scales, int rows_cap, int K, uint8_t* a_scales16,
                                   void* stream);

/* moesq_grouped_dense_gemm: the result moesq_grouped_sparse_gemm defines,
 * for dense weights: y[r][m] = bf16_RN(alpha_e * sum_k deq(a[r][k]) *
 * deq(W_e[m][k])), alpha_e = 1 / (w->global_scale[e] * gamma_a[e]), with
 * the token scales one per 16 K (moesq_expand_scales16).  Same row space,
 * validation and cfg as the sparse GEMM; sm_mode 2 is not offered
 * (MOESQ_ERR_UNSUPPORTED_SHAPE). */
moesq_status moesq_grouped_dense_gemm(const moesq_dense_weights* w, const uint8_t* a_codes,
                                      const uint8_t* a_scales16, int rows_cap, const int32_t* counts,
                                      const int32_t* row_offsets, const float* gamma_a, uint16_t* y_bf16,
                                      const moesq_gemm_config* cfg, void* stream);

/* ------------------------------------------------------------- layer parts
 * moesq_swiglu_quant: h = SiLU(g) * u for every valid row of the gate_up
 * output y_gu [rows_cap][2I] bf16 (gu_layout MOESQ_LAYOUT_PLAIN: g = columns
 * [0, I), u = [I, 2I); MOESQ_LAYOUT_SWIGLU: the kernel row order of weights
 * packed with that layout, feature f at column 128 (f / 64) + f % 64 and its
 * up half 64 columns later; SiLU(g) = g / (1 + e^-g) in binary32 with the
 * hardware exponential and divide, a few ulp from the exact value),
 * requantised to NVFP4 with gamma_h[e] of the row's expert into h_codes
 * [rows_cap][I/2] and h_scales (MMA scale layout) -- the SwiGLU +
 * requantisation of App. D.1 as a kernel of its own.
 * I is a multiple of 256; y_gu and h_codes are 16-byte aligned. */
moesq_status moesq_swiglu_quant(const uint16_t* y_gu, int I, const moesq_routing* rt,
                                const float* gamma_h, uint8_t* h_codes, uint8_t* h_scales,
                                int gu_layout, void* stream);

/* moesq_grouped_sparse_gemm_swiglu: the gate_up GEMM with SwiGLU and the
 * NVFP4 requantisation of h fused into its epilogue (App. D.1 "Serving
 * integration": "fused SwiGLU with requantization").  w is a gate_up stack
 * (M = 2I) packed with layout MOESQ_LAYOUT_SWIGLU.  For every valid row r
 * of expert e the result equals moesq_grouped_sparse_gemm followed by
 * moesq_swiglu_quant (gu_layout MOESQ_LAYOUT_SWIGLU) bit for bit: g and u
 * are the bf16-rounded GEMM outputs, h = SiLU(g) * u as there, each 32-wide
 * block of h gets scale code RNE_E4M3(gamma_h[e] * amax / 6) and the E2M1
 * codes of the correctly rounded quotients; written to h_codes
 * [rows_cap][I/2] (row r) and h_scales (MMA scale layout, I / 32 scales per
 * row).  The bf16 gate_up output never reaches memory.  Same row space,
 * validation and cfg as moesq_grouped_sparse_gemm, except that sm_mode 2
 * is not offered (MOESQ_ERR_UNSUPPORTED_SHAPE) and weights of another
 * layout are rejected (MOESQ_ERR_INVALID_ARG).  a_codes, a_scales and
 * h_codes are 16-byte aligned. */
moesq_status moesq_grouped_sparse_gemm_swiglu(const moesq_weights* w, const uint8_t* a_codes,
                                              const uint8_t* a_scales, int rows_cap, const int32_t* counts,
                                              const int32_t* row_offsets, const float* gamma_a,
                                              const float* gamma_h, uint8_t* h_codes, uint8_t* h_scales,
                                              const moesq_gemm_config* cfg, void* stream);

/* moesq_gemm_swiglu_autotune: moesq_gemm_autotune for the fused gate_up
 * GEMM (token tile 64 or 128 rows x one or two CTAs per SM); writes h_codes
 * and h_scales as the GEMM does; synchronises the stream. */
moesq_status moesq_gemm_swiglu_autotune(const moesq_weights* w, const uint8_t* a_codes, const uint8_t* a_scales,
                                        int rows_cap, const int32_t* counts, const int32_t* row_offsets,
                                        const float* gamma_a, const float* gamma_h, uint8_t* h_codes,
                                        uint8_t* h_scales, int reps, moesq_gemm_config* best, float* best_ms,
                                        void* stream);

/* moesq_combine: out[t][h] = bf16( sum_{j<k} topk_w[t][j] * y[slot_to_row[t*k+j]][h] )
 * with binary32 accumulation in slot order (router-weighted token
 * combination, App. D.1).  y [rows_cap][H], out [T][H] bf16. */
moesq_status moesq_combine(const uint16_t* y, int H, const moesq_routing* rt,
                           uint16_t* out, void* stream);

/* ------------------------------------------------------------------- layer
 * moesq_moe_layer: one routed-expert MoE layer on T tokens (App. D.1):
 * route + permute -> dispatch-quantise (gamma_a_gu) -> gate_up grouped GEMM
 * (w_gu: M = 2I, K = H) -> SwiGLU + requantise (gamma_a_dn) -> down grouped
 * GEMM (w_dn: M = H, K = I) -> router-weighted combine into out [T][H].
 * When w_gu has layout MOESQ_LAYOUT_SWIGLU the gate_up GEMM and the SwiGLU
 * requantisation are one kernel (moesq_grouped_sparse_gemm_swiglu); the
 * result is the same bit for bit.  w_dn must have layout MOESQ_LAYOUT_PLAIN.
 * x [T][H] bf16, logits [T][E] float32; gamma_a_* [E] float32 (device).
 * All intermediates live in `workspace` (moesq_layer_workspace_bytes).    */
size_t moesq_layer_workspace_bytes(int T, int k, int E, int H, int I);

moesq_status moesq_moe_layer(const uint16_t* x_bf16, const float* logits, int T, int k,
                             const moesq_weights* w_gu, const moesq_weights* w_dn,
                             const float* gamma_a_gu, const float* gamma_a_dn,
                             uint16_t* out_bf16, void* workspace, size_t workspace_bytes,
                             void* stream);

/* moesq_moe_layer_host: the same layer with x, logits and out in HOST memory
 * (pinned memory gives asynchronous copies); the inputs are copied into the
 * workspace, the layer runs, the output is copied back and the stream is
 * synchronised before returning.  Weights and gamma_* stay on the device.
 * Needs moesq_layer_host_workspace_bytes. */
size_t moesq_layer_host_workspace_bytes(int T, int k, int E, int H, int I);

moesq_status moesq_moe_layer_host(const uint16_t* x_bf16_host, const float* logits_host,
                                  int T, int k, const moesq_weights* w_gu,
                                  const moesq_weights* w_dn, const float* gamma_a_gu,
                                  const float* gamma_a_dn, uint16_t* out_bf16_host,
                                  void* workspace, size_t workspace_bytes, void* stream);

/* moesq_calibrate_layer: static activation global scales of a layer from a
 * calibration batch: gamma_a_gu[e] = 448 / (amax_e / 6) with amax_e the
 * largest |x| over the tokens routed to e, and gamma_a_dn[e] likewise over
 * the SwiGLU output rows of e (computed with the calibrated gamma_a_gu).
 * Experts that receive no token take the largest amax over all experts.
 * Uses the layer workspace. */
moesq_status moesq_calibrate_layer(const uint16_t* x_bf16, const float* logits, int T, int k,
                                   const moesq_weights* w_gu, const moesq_weights* w_dn,
                                   float* gamma_a_gu, float* gamma_a_dn,
                                   void* workspace, size_t workspace_bytes, void* stream);

/* ------------------------------------------------------------------- debug
 * moesq_debug_bounded_wait: launches one CTA that waits on a barrier nothing
 * ever signals, with a limit of timeout_ns; the wait gives up, records
 * MOESQ_ERR_TIMEOUT in the device error word and the kernel exits.  Exists
 * to test the watchdog path of the kernels without faulting the GPU. */
moesq_status moesq_debug_bounded_wait(uint64_t timeout_ns, void* stream);

/* --------------------------------------------------------- tensor-core peak
 * Throughput of the block-scaled FP4 MMA this library's GEMM is built on
 * (tcgen05.mma kind::mxf4nvf4 with UE4M3 scales; the sparse form is the
 * paper's SpTC path, Sec. 3.4 and App. D.1; the 18 PFLOP/s sparse peak the
 * paper quotes for B200 in its introduction is the nominal counterpart):
 * ctas_per_sm (1 or 2) CTAs on every SM each issue `iters` x 2 back-to-back
 * MMAs of M = 128, N = n (16 <= n <= 256, a multiple of 16; n <= 128 with
 * 2 CTAs per SM), K = 64 (dense, sparse = 0) or K = 128 dense-equivalent
 * (sparse = 1), on operands resident in shared and tensor memory, so no
 * memory traffic limits it.  with_copies = 1 adds, before every two MMAs,
 * the shared-to-tensor-memory copies of metadata and scales that the
 * grouped GEMM issues per 256-wide K step, so the rate then includes their
 * share of the tensor pipe.  *tflops (host) receives the dense-equivalent
 * TFLOP/s of the whole GPU (2 M N K per MMA over the launch's event-timed
 * duration).  Synchronises `stream`; about iters x 0.14 us of device time.
 * Errors: MOESQ_ERR_INVALID_ARG for sizes outside the above. */
moesq_status moesq_mma_peak(int sparse, int n, int ctas_per_sm, int with_copies, int iters, double* tflops,
                            void* stream);

#ifdef __cplusplus
}
#endif
#endif /* MOESQ_H_ */
