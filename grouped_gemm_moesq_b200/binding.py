"""Python binding of libmoesq.so (include/moesq.h).

Argument marshalling only: every function below hands device pointers,
sizes and the current CUDA stream to the C ABI function of the same name.
PyTorch provides device memory and streams.  There is no fallback: if the
compiled library is missing, `load()` raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoesq.so")

ROW_ALIGN = 128

# Kernel row order of a weight stack (moesq_weights.layout)
LAYOUT_PLAIN = 0
LAYOUT_SWIGLU = 1     # gate_up rows interleaved by 64 for the fused SwiGLU epilogue

_c = ctypes
_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t

STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "CUDA error",
          4: "device wait timed out", 5: "device-side validation failed", 6: "workspace too small"}


class MoesqError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__("%s: %s (status %d)" % (where, STATUS.get(status, "unknown"), status))
        self.status = status


class moesq_weights(ctypes.Structure):
    _fields_ = [("E", _i32), ("M", _i32), ("K", _i32), ("values", _vp), ("mask", _vp), ("scales", _vp),
                ("global_scale", _vp), ("ktiles", _vp), ("layout", _i32)]


class moesq_routing(ctypes.Structure):
    _fields_ = [("T", _i32), ("E", _i32), ("k", _i32), ("rows_cap", _i32), ("topk_ids", _vp), ("topk_w", _vp),
                ("counts", _vp), ("offsets", _vp), ("row_offsets", _vp), ("sorted_to_slot", _vp),
                ("slot_to_row", _vp)]


class moesq_dense_weights(ctypes.Structure):
    _fields_ = [("E", _i32), ("M", _i32), ("K", _i32), ("codes", _vp), ("scales", _vp), ("global_scale", _vp),
                ("dtiles", _vp)]


class moesq_gemm_config(ctypes.Structure):
    _fields_ = [("tile_n", _i32), ("num_ctas", _i32), ("sm_mode", _i32)]


_lib = None
_P = ctypes.POINTER


def load():
    """Load libmoesq.so and declare the ABI; raises if the library is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError("libmoesq.so is not built (run grouped_gemm_moesq_b200/build.py); "
                           "there is no fallback path")
    L = ctypes.CDLL(LIB_PATH)
    sig = {
        "moesq_status_str": (_c.c_char_p, [_c.c_int]),
        "moesq_version": (_c.c_char_p, []),
        "moesq_last_cuda_error": (_c.c_char_p, []),
        "moesq_get_device_error": (_c.c_int, [_vp, _P(_i32)]),
        "moesq_set_wait_timeout_ns": (None, [_c.c_uint64]),
        "moesq_weights_bytes": (_sz, [_c.c_int, _c.c_int, _c.c_int, _P(_sz)]),
        "moesq_pack_weights": (_c.c_int, [_vp, _c.c_int, _c.c_int, _P(moesq_weights), _vp]),
        "moesq_gemm_autotune": (_c.c_int, [_P(moesq_weights), _vp, _vp, _c.c_int, _vp, _vp, _vp, _vp, _c.c_int,
                                           _P(moesq_gemm_config), _P(_c.c_float), _vp]),
        "moesq_import_dense_nvfp4": (_c.c_int, [_vp, _vp, _vp, _c.c_int, _c.c_int, _P(moesq_weights), _vp]),
        "moesq_export_dense_nvfp4": (_c.c_int, [_P(moesq_weights), _vp, _vp]),
        "moesq_rows_capacity": (_i64, [_c.c_int, _c.c_int, _c.c_int]),
        "moesq_route_workspace_bytes": (_sz, [_c.c_int, _c.c_int]),
        "moesq_route_permute": (_c.c_int, [_vp, _P(moesq_routing), _vp, _sz, _vp]),
        "moesq_route_permute_noalloc": (_c.c_int, [_vp, _P(moesq_routing), _vp]),
        "moesq_dense_weights_bytes": (_sz, [_c.c_int, _c.c_int, _c.c_int, _P(_sz)]),
        "moesq_pack_dense_nvfp4": (_c.c_int, [_vp, _c.c_int, _c.c_int, _P(moesq_dense_weights), _vp]),
        "moesq_expand_scales16": (_c.c_int, [_vp, _c.c_int, _c.c_int, _vp, _vp]),
        "moesq_grouped_dense_gemm": (_c.c_int, [_P(moesq_dense_weights), _vp, _vp, _c.c_int, _vp, _vp, _vp, _vp,
                                                _P(moesq_gemm_config), _vp]),
        "moesq_mma_peak": (_c.c_int, [_c.c_int, _c.c_int, _c.c_int, _c.c_int, _c.c_int, _P(_c.c_double), _vp]),
        "moesq_quantize_act": (_c.c_int, [_vp, _c.c_int, _c.c_int, _P(moesq_routing), _vp, _c.c_int, _vp, _vp,
                                          _vp]),
        "moesq_act_global_scale": (_c.c_int, [_vp, _i64, _vp, _vp]),
        "moesq_grouped_sparse_gemm": (_c.c_int, [_P(moesq_weights), _vp, _vp, _c.c_int, _vp, _vp, _vp, _vp,
                                                 _P(moesq_gemm_config), _vp]),
        "moesq_swiglu_quant": (_c.c_int, [_vp, _c.c_int, _P(moesq_routing), _vp, _vp, _vp, _c.c_int, _vp]),
        "moesq_grouped_sparse_gemm_swiglu": (_c.c_int, [_P(moesq_weights), _vp, _vp, _c.c_int, _vp, _vp, _vp, _vp,
                                                        _vp, _vp, _P(moesq_gemm_config), _vp]),
        "moesq_gemm_swiglu_autotune": (_c.c_int, [_P(moesq_weights), _vp, _vp, _c.c_int, _vp, _vp, _vp, _vp, _vp,
                                                  _vp, _c.c_int, _P(moesq_gemm_config), _P(_c.c_float), _vp]),
        "moesq_combine": (_c.c_int, [_vp, _c.c_int, _P(moesq_routing), _vp, _vp]),
        "moesq_layer_workspace_bytes": (_sz, [_c.c_int] * 5),
        "moesq_layer_host_workspace_bytes": (_sz, [_c.c_int] * 5),
        "moesq_moe_layer": (_c.c_int, [_vp, _vp, _c.c_int, _c.c_int, _P(moesq_weights), _P(moesq_weights), _vp,
                                       _vp, _vp, _vp, _sz, _vp]),
        "moesq_moe_layer_host": (_c.c_int, [_vp, _vp, _c.c_int, _c.c_int, _P(moesq_weights), _P(moesq_weights),
                                            _vp, _vp, _vp, _vp, _sz, _vp]),
        "moesq_calibrate_layer": (_c.c_int, [_vp, _vp, _c.c_int, _c.c_int, _P(moesq_weights), _P(moesq_weights),
                                             _vp, _vp, _vp, _sz, _vp]),
        "moesq_debug_bounded_wait": (_c.c_int, [_c.c_uint64, _vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


def _check(status: int, where: str):
    if status != 0:
        if status == 3:
            where = "%s [%s]" % (where, load().moesq_last_cuda_error().decode())
        raise MoesqError(status, where)


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return _vp(s.cuda_stream)


def _ptr(t):
    return None if t is None else _vp(t.data_ptr())


# ------------------------------------------------------------------ buffers
class PackedWeights:
    """Device tensors of one expert stack (storage form + kernel form) and
    the moesq_weights struct that points at them.  layout: LAYOUT_PLAIN, or
    LAYOUT_SWIGLU for a gate_up stack feeding the fused SwiGLU GEMM."""

    def __init__(self, E: int, M: int, K: int, device="cuda", layout: int = LAYOUT_PLAIN):
        import torch
        self.E, self.M, self.K, self.layout = E, M, K, layout
        u8 = dict(dtype=torch.uint8, device=device)
        self.values = torch.empty(E, M, K // 4, **u8)
        self.mask = torch.empty(E, M, K // 16, **u8)
        self.scales = torch.empty(E, M, K // 32, **u8)
        self.global_scale = torch.empty(E, dtype=torch.float32, device=device)
        self.ktiles = torch.empty(E * M * K // 32 * 11, **u8)
        self.struct = moesq_weights(E, M, K, self.values.data_ptr(), self.mask.data_ptr(), self.scales.data_ptr(),
                                    self.global_scale.data_ptr(), self.ktiles.data_ptr(), layout)

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.values, self.mask, self.scales, self.global_scale, self.ktiles))


class DenseWeights:
    """Device tensors of one dense NVFP4 expert stack (the dense control:
    storage form + kernel form) and the moesq_dense_weights struct."""

    def __init__(self, E: int, M: int, K: int, device="cuda"):
        import torch
        self.E, self.M, self.K = E, M, K
        u8 = dict(dtype=torch.uint8, device=device)
        self.codes = torch.empty(E, M, K // 2, **u8)
        self.scales = torch.empty(E, M, K // 16, **u8)
        self.global_scale = torch.empty(E, dtype=torch.float32, device=device)
        self.dtiles = torch.empty(E * M * K // 32768 * 18432, **u8)   # 18 KB per 128 x 256 tile
        self.struct = moesq_dense_weights(E, M, K, self.codes.data_ptr(), self.scales.data_ptr(),
                                          self.global_scale.data_ptr(), self.dtiles.data_ptr())


class RoutingBuffers:
    """Device arrays of one routing (moesq_routing)."""

    def __init__(self, T: int, E: int, k: int, device="cuda", rows_cap: int | None = None):
        import torch
        self.T, self.E, self.k = T, E, k
        self.rows_cap = int(rows_cap if rows_cap is not None else moesq_rows_capacity(T, k, E))
        i32 = dict(dtype=torch.int32, device=device)
        R = T * k
        self.topk_ids = torch.empty(R, **i32)
        self.topk_w = torch.empty(R, dtype=torch.float32, device=device)
        self.counts = torch.empty(E, **i32)
        self.offsets = torch.empty(E + 1, **i32)
        self.row_offsets = torch.empty(E + 1, **i32)
        self.sorted_to_slot = torch.empty(R, **i32)
        self.slot_to_row = torch.empty(R, **i32)
        self.workspace = torch.empty(max(1, moesq_route_workspace_bytes(T, E)), dtype=torch.uint8, device=device)
        self.struct = moesq_routing(T, E, k, self.rows_cap, self.topk_ids.data_ptr(), self.topk_w.data_ptr(),
                                    self.counts.data_ptr(), self.offsets.data_ptr(), self.row_offsets.data_ptr(),
                                    self.sorted_to_slot.data_ptr(), self.slot_to_row.data_ptr())


def act_buffers(rows_cap: int, K: int, device="cuda"):
    """(codes [rows_cap, K/2], scales [rows_cap * K / 32]) uint8 tensors."""
    import torch
    return (torch.empty(rows_cap, K // 2, dtype=torch.uint8, device=device),
            torch.empty(rows_cap * K // 32, dtype=torch.uint8, device=device))


# ------------------------------------------------------------------ ABI calls
def moesq_version() -> str:
    return load().moesq_version().decode()


def moesq_get_device_error(stream=None):
    """(status, raw device word); synchronises the stream.  A CUDA failure
    (status 3) raises with the CUDA error text."""
    code = _i32(0)
    st = load().moesq_get_device_error(_stream(stream), ctypes.byref(code))
    if st == 3:
        _check(st, "moesq_get_device_error")
    return st, code.value


def moesq_set_wait_timeout_ns(ns: int):
    load().moesq_set_wait_timeout_ns(int(ns))


def moesq_weights_bytes(E: int, M: int, K: int) -> int:
    return load().moesq_weights_bytes(E, M, K, None)


def moesq_rows_capacity(T: int, k: int, E: int) -> int:
    return load().moesq_rows_capacity(T, k, E)


def moesq_route_workspace_bytes(T: int, E: int) -> int:
    return load().moesq_route_workspace_bytes(T, E)


def moesq_layer_workspace_bytes(T: int, k: int, E: int, H: int, I: int) -> int:
    return load().moesq_layer_workspace_bytes(T, k, E, H, I)


def moesq_layer_host_workspace_bytes(T: int, k: int, E: int, H: int, I: int) -> int:
    return load().moesq_layer_host_workspace_bytes(T, k, E, H, I)


def moesq_pack_weights(w_bf16, e_begin: int, e_count: int, out: PackedWeights, stream=None):
    _check(load().moesq_pack_weights(_ptr(w_bf16), e_begin, e_count, ctypes.byref(out.struct), _stream(stream)),
           "moesq_pack_weights")


def moesq_gemm_autotune(w: PackedWeights, a_codes, a_scales, rows_cap: int, counts, row_offsets, gamma_a, y_bf16,
                        reps: int = 5, stream=None):
    """Fastest (tile_n, num_ctas, sm_mode) for these inputs and its mean time in ms."""
    cfg = moesq_gemm_config(0, 0)
    ms = _c.c_float(0.0)
    _check(load().moesq_gemm_autotune(ctypes.byref(w.struct), _ptr(a_codes), _ptr(a_scales), rows_cap, _ptr(counts),
                                      _ptr(row_offsets), _ptr(gamma_a), _ptr(y_bf16), reps, ctypes.byref(cfg),
                                      ctypes.byref(ms), _stream(stream)), "moesq_gemm_autotune")
    return (cfg.tile_n, cfg.num_ctas, cfg.sm_mode), ms.value


def moesq_import_dense_nvfp4(codes, scales, global_scale, e_begin: int, e_count: int, out: PackedWeights,
                             stream=None):
    _check(load().moesq_import_dense_nvfp4(_ptr(codes), _ptr(scales), _ptr(global_scale), e_begin, e_count,
                                           ctypes.byref(out.struct), _stream(stream)), "moesq_import_dense_nvfp4")


def moesq_export_dense_nvfp4(w: PackedWeights, codes, stream=None):
    _check(load().moesq_export_dense_nvfp4(ctypes.byref(w.struct), _ptr(codes), _stream(stream)),
           "moesq_export_dense_nvfp4")


def moesq_route_permute(logits, rt: RoutingBuffers, stream=None):
    _check(load().moesq_route_permute(_ptr(logits), ctypes.byref(rt.struct), _ptr(rt.workspace),
                                      rt.workspace.numel(), _stream(stream)), "moesq_route_permute")


def moesq_route_permute_noalloc(logits, rt: RoutingBuffers, stream=None):
    """Routing without a caller-provided workspace (static scratch inside the
    library; T <= 16384)."""
    _check(load().moesq_route_permute_noalloc(_ptr(logits), ctypes.byref(rt.struct), _stream(stream)),
           "moesq_route_permute_noalloc")


def moesq_quantize_act(x_bf16, T: int, K: int, rt, gamma, rows_cap: int, codes, scales, stream=None):
    rts = ctypes.byref(rt.struct) if rt is not None else None
    _check(load().moesq_quantize_act(_ptr(x_bf16), T, K, rts, _ptr(gamma), rows_cap, _ptr(codes), _ptr(scales),
                                     _stream(stream)), "moesq_quantize_act")


def moesq_act_global_scale(x_bf16, gamma_out, stream=None):
    _check(load().moesq_act_global_scale(_ptr(x_bf16), x_bf16.numel(), _ptr(gamma_out), _stream(stream)),
           "moesq_act_global_scale")


def moesq_grouped_sparse_gemm(w: PackedWeights, a_codes, a_scales, rows_cap: int, counts, row_offsets, gamma_a,
                              y_bf16, tile_n: int = 0, num_ctas: int = 0, sm_mode: int = 0, stream=None):
    cfg = moesq_gemm_config(tile_n, num_ctas, sm_mode)
    _check(load().moesq_grouped_sparse_gemm(ctypes.byref(w.struct), _ptr(a_codes), _ptr(a_scales), rows_cap,
                                            _ptr(counts), _ptr(row_offsets), _ptr(gamma_a), _ptr(y_bf16),
                                            ctypes.byref(cfg), _stream(stream)), "moesq_grouped_sparse_gemm")


def moesq_swiglu_quant(y_gu, I: int, rt: RoutingBuffers, gamma_h, h_codes, h_scales, gu_layout: int = LAYOUT_PLAIN,
                       stream=None):
    _check(load().moesq_swiglu_quant(_ptr(y_gu), I, ctypes.byref(rt.struct), _ptr(gamma_h), _ptr(h_codes),
                                     _ptr(h_scales), gu_layout, _stream(stream)), "moesq_swiglu_quant")


def moesq_grouped_sparse_gemm_swiglu(w: PackedWeights, a_codes, a_scales, rows_cap: int, counts, row_offsets,
                                     gamma_a, gamma_h, h_codes, h_scales, tile_n: int = 0, num_ctas: int = 0,
                                     sm_mode: int = 0, stream=None):
    cfg = moesq_gemm_config(tile_n, num_ctas, sm_mode)
    _check(load().moesq_grouped_sparse_gemm_swiglu(ctypes.byref(w.struct), _ptr(a_codes), _ptr(a_scales), rows_cap,
                                                   _ptr(counts), _ptr(row_offsets), _ptr(gamma_a), _ptr(gamma_h),
                                                   _ptr(h_codes), _ptr(h_scales), ctypes.byref(cfg),
                                                   _stream(stream)), "moesq_grouped_sparse_gemm_swiglu")


def moesq_gemm_swiglu_autotune(w: PackedWeights, a_codes, a_scales, rows_cap: int, counts, row_offsets, gamma_a,
                               gamma_h, h_codes, h_scales, reps: int = 5, stream=None):
    """Fastest (tile_n, num_ctas, sm_mode) of the fused gate_up GEMM and its mean time in ms."""
    cfg = moesq_gemm_config(0, 0)
    ms = _c.c_float(0.0)
    _check(load().moesq_gemm_swiglu_autotune(ctypes.byref(w.struct), _ptr(a_codes), _ptr(a_scales), rows_cap,
                                             _ptr(counts), _ptr(row_offsets), _ptr(gamma_a), _ptr(gamma_h),
                                             _ptr(h_codes), _ptr(h_scales), reps, ctypes.byref(cfg),
                                             ctypes.byref(ms), _stream(stream)), "moesq_gemm_swiglu_autotune")
    return (cfg.tile_n, cfg.num_ctas, cfg.sm_mode), ms.value


def moesq_combine(y, H: int, rt: RoutingBuffers, out, stream=None):
    _check(load().moesq_combine(_ptr(y), H, ctypes.byref(rt.struct), _ptr(out), _stream(stream)), "moesq_combine")


def moesq_moe_layer(x_bf16, logits, T: int, k: int, w_gu: PackedWeights, w_dn: PackedWeights, gamma_a_gu,
                    gamma_a_dn, out_bf16, workspace, stream=None):
    _check(load().moesq_moe_layer(_ptr(x_bf16), _ptr(logits), T, k, ctypes.byref(w_gu.struct),
                                  ctypes.byref(w_dn.struct), _ptr(gamma_a_gu), _ptr(gamma_a_dn), _ptr(out_bf16),
                                  _ptr(workspace), workspace.numel(), _stream(stream)), "moesq_moe_layer")


def moesq_moe_layer_host(x_host, logits_host, T: int, k: int, w_gu: PackedWeights, w_dn: PackedWeights,
                         gamma_a_gu, gamma_a_dn, out_host, workspace, stream=None):
    """x_host / logits_host / out_host are CPU tensors (pinned for async copies)."""
    _check(load().moesq_moe_layer_host(_ptr(x_host), _ptr(logits_host), T, k, ctypes.byref(w_gu.struct),
                                       ctypes.byref(w_dn.struct), _ptr(gamma_a_gu), _ptr(gamma_a_dn),
                                       _ptr(out_host), _ptr(workspace), workspace.numel(), _stream(stream)),
           "moesq_moe_layer_host")


def moesq_calibrate_layer(x_bf16, logits, T: int, k: int, w_gu: PackedWeights, w_dn: PackedWeights,
                          gamma_a_gu, gamma_a_dn, workspace, stream=None):
    _check(load().moesq_calibrate_layer(_ptr(x_bf16), _ptr(logits), T, k, ctypes.byref(w_gu.struct),
                                        ctypes.byref(w_dn.struct), _ptr(gamma_a_gu), _ptr(gamma_a_dn),
                                        _ptr(workspace), workspace.numel(), _stream(stream)),
           "moesq_calibrate_layer")


def moesq_debug_bounded_wait(timeout_ns: int, stream=None):
    _check(load().moesq_debug_bounded_wait(int(timeout_ns), _stream(stream)), "moesq_debug_bounded_wait")


def moesq_mma_peak(sparse: bool, n: int, ctas_per_sm: int = 1, with_copies: bool = False, iters: int = 20000,
                   stream=None) -> float:
    """Dense-equivalent TFLOP/s of back-to-back block-scaled FP4 MMAs on every SM."""
    out = ctypes.c_double(0.0)
    _check(load().moesq_mma_peak(int(bool(sparse)), n, ctas_per_sm, int(bool(with_copies)), iters,
                                 ctypes.byref(out), _stream(stream)),
           "moesq_mma_peak")
    return out.value


def scales16_buffer(rows_cap: int, K: int, device="cuda"):
    """Token scales, one per 16 K, in the dense MMA's layout (uint8, flat)."""
    import torch
    return torch.empty(rows_cap * K // 16, dtype=torch.uint8, device=device)


def moesq_dense_weights_bytes(E: int, M: int, K: int) -> int:
    return load().moesq_dense_weights_bytes(E, M, K, None)


def moesq_pack_dense_nvfp4(w_bf16, e_begin: int, e_count: int, out: DenseWeights, stream=None):
    _check(load().moesq_pack_dense_nvfp4(_ptr(w_bf16), e_begin, e_count, ctypes.byref(out.struct), _stream(stream)),
           "moesq_pack_dense_nvfp4")


def moesq_expand_scales16(a_scales, rows_cap: int, K: int, a_scales16, stream=None):
    _check(load().moesq_expand_scales16(_ptr(a_scales), rows_cap, K, _ptr(a_scales16), _stream(stream)),
           "moesq_expand_scales16")


def moesq_grouped_dense_gemm(w: DenseWeights, a_codes, a_scales16, rows_cap: int, counts, row_offsets, gamma_a,
                             y_bf16, tile_n: int = 0, num_ctas: int = 0, sm_mode: int = 0, stream=None):
    cfg = moesq_gemm_config(tile_n, num_ctas, sm_mode)
    _check(load().moesq_grouped_dense_gemm(ctypes.byref(w.struct), _ptr(a_codes), _ptr(a_scales16), rows_cap,
                                           _ptr(counts), _ptr(row_offsets), _ptr(gamma_a), _ptr(y_bf16),
                                           ctypes.byref(cfg), _stream(stream)), "moesq_grouped_dense_gemm")
