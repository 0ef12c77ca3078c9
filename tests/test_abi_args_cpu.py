"""Host-side argument checking of the C ABI, on CPU: every case here is
refused by the library's checks before any CUDA call, so the pointers are
never dereferenced (they are stand-in addresses with the alignment each
case needs).  No case is ever valid, so nothing is launched on any machine."""
import ctypes

import pytest

from grouped_gemm_moesq_b200 import binding as B

OK, INVALID, SHAPE, WORKSPACE = 0, 1, 2, 6
P = 0x100000                       # 1 MiB-aligned stand-in address (never used)


def ptr(off=0):
    return ctypes.c_void_p(P + off)


@pytest.fixture(scope="module")
def L():
    from grouped_gemm_moesq_b200 import build
    build.build()
    return B.load()


def weights(E=4, M=256, K=512, layout=0, **kw):
    f = dict(values=P, mask=P, scales=P, global_scale=P, ktiles=P)
    f.update(kw)
    return B.moesq_weights(E, M, K, f["values"], f["mask"], f["scales"], f["global_scale"], f["ktiles"], layout)


def routing(T=8, E=4, k=2, rows_cap=None, **kw):
    if rows_cap is None:
        rows_cap = B.load().moesq_rows_capacity(T, k, E)
    f = dict(topk_ids=P, topk_w=P, counts=P, offsets=P, row_offsets=P, sorted_to_slot=P, slot_to_row=P)
    f.update(kw)
    return B.moesq_routing(T, E, k, rows_cap, f["topk_ids"], f["topk_w"], f["counts"], f["offsets"],
                           f["row_offsets"], f["sorted_to_slot"], f["slot_to_row"])


def gemm(L, w, a_codes=ptr(), a_scales=ptr(), rows_cap=256, counts=ptr(), row_offsets=ptr(), gamma=ptr(),
         y=ptr(), cfg=None):
    c = ctypes.byref(cfg) if cfg is not None else None
    return L.moesq_grouped_sparse_gemm(ctypes.byref(w), a_codes, a_scales, rows_cap, counts, row_offsets, gamma, y,
                                       c, None)


def test_gemm_refuses_bad_weights(L):
    assert L.moesq_grouped_sparse_gemm(None, ptr(), ptr(), 256, ptr(), ptr(), ptr(), ptr(), None, None) == INVALID
    assert gemm(L, weights(M=100)) == SHAPE                        # M not a multiple of 128
    assert gemm(L, weights(K=384)) == SHAPE                        # K not a multiple of 256
    assert gemm(L, weights(E=0)) == SHAPE
    assert gemm(L, weights(E=513)) == SHAPE                        # above 512 experts
    assert gemm(L, weights(values=0)) == INVALID                   # missing tensor
    assert gemm(L, weights(values=P + 8)) == INVALID               # values not 16-byte aligned


def test_gemm_refuses_bad_activations_and_config(L):
    w = weights()
    assert gemm(L, w, a_codes=None) == INVALID
    assert gemm(L, w, rows_cap=100) == INVALID                     # not a multiple of 128
    assert gemm(L, w, a_codes=ptr(4)) == INVALID                   # codes not 16-byte aligned
    assert gemm(L, w, y=ptr(1)) == INVALID                         # bf16 output misaligned
    assert gemm(L, w, cfg=B.moesq_gemm_config(32, 0)) == INVALID   # token tile 32 is not offered
    assert gemm(L, w, cfg=B.moesq_gemm_config(64, -1)) == INVALID
    assert gemm(L, w, cfg=B.moesq_gemm_config(64, 0, 3)) == INVALID      # sm_mode 0, 1 or 2
    assert gemm(L, w, cfg=B.moesq_gemm_config(64, 0, -1)) == INVALID


def test_autotune_refuses_bad_arguments(L):
    w = weights()
    best = B.moesq_gemm_config(0, 0)
    ms = ctypes.c_float(0)
    args = (ctypes.byref(w), ptr(), ptr(), 256, ptr(), ptr(), ptr(), ptr())
    assert L.moesq_gemm_autotune(*args, 0, ctypes.byref(best), ctypes.byref(ms), None) == INVALID
    assert L.moesq_gemm_autotune(*args, 3, None, ctypes.byref(ms), None) == INVALID


def test_routing_checks(L):
    rt = routing()
    assert L.moesq_route_permute(ptr(), ctypes.byref(routing(k=0)), ptr(), 1 << 20, None) == SHAPE
    assert L.moesq_route_permute(ptr(), ctypes.byref(routing(E=4, k=5)), ptr(), 1 << 20, None) == SHAPE
    assert L.moesq_route_permute(ptr(), ctypes.byref(routing(rows_cap=100)), ptr(), 1 << 20,
                                 None) == INVALID
    assert L.moesq_route_permute(ptr(), ctypes.byref(routing(topk_ids=0)), ptr(), 1 << 20, None) == INVALID
    assert L.moesq_route_permute(None, ctypes.byref(rt), ptr(), 1 << 20, None) == INVALID
    need = L.moesq_route_workspace_bytes(8, 4)
    assert L.moesq_route_permute(ptr(), ctypes.byref(rt), ptr(), max(0, need - 1), None) == WORKSPACE
    assert L.moesq_route_permute(ptr(), ctypes.byref(rt), None, need, None) == WORKSPACE
    assert L.moesq_route_permute(ptr(), ctypes.byref(routing(T=0)), ptr(), 1 << 20, None) == SHAPE
    assert L.moesq_route_permute(ptr(), ctypes.byref(routing(E=513, k=8)), ptr(), 1 << 30, None) == SHAPE
    assert L.moesq_route_permute(ptr(), ctypes.byref(routing(E=64, k=33)), ptr(), 1 << 30, None) == SHAPE
    # the allocation-free variant: the same checks, and tokens beyond its static scratch
    assert L.moesq_route_permute_noalloc(ptr(), ctypes.byref(routing(k=0)), None) == SHAPE
    assert L.moesq_route_permute_noalloc(None, ctypes.byref(rt), None) == INVALID
    assert L.moesq_route_permute_noalloc(ptr(), ctypes.byref(routing(T=16385, E=8, k=2)), None) == SHAPE


def test_misaligned_index_arrays_are_refused(L):
    """Arrays read with 4-byte loads (routing, counts, global scales) must be
    4-byte aligned; the calls refuse them on the host."""
    for field in ("topk_ids", "topk_w", "counts", "offsets", "row_offsets", "sorted_to_slot", "slot_to_row"):
        rt = routing(**{field: P + 2})
        assert L.moesq_route_permute(ptr(), ctypes.byref(rt), ptr(), 1 << 20, None) == INVALID, field
    rt = routing()
    assert L.moesq_route_permute(ptr(2), ctypes.byref(rt), ptr(), 1 << 20, None) == INVALID        # logits
    assert L.moesq_route_permute(ptr(), ctypes.byref(rt), ptr(2), 1 << 20, None) == INVALID        # workspace
    assert L.moesq_route_permute_noalloc(ptr(2), ctypes.byref(rt), None) == INVALID
    assert gemm(L, weights(), counts=ptr(2)) == INVALID
    assert gemm(L, weights(), row_offsets=ptr(2)) == INVALID
    assert gemm(L, weights(), gamma=ptr(2)) == INVALID
    assert L.moesq_quantize_act(ptr(), 8, 512, ctypes.byref(rt), ptr(2), rt.rows_cap, ptr(), ptr(), None) == INVALID
    assert L.moesq_swiglu_quant(ptr(), 256, ctypes.byref(rt), ptr(2), ptr(), ptr(), 0, None) == INVALID


def test_quantise_swiglu_combine_checks(L):
    rt = routing()
    rc = rt.rows_cap
    assert L.moesq_quantize_act(ptr(), 8, 100, ctypes.byref(rt), ptr(), rc, ptr(), ptr(), None) == SHAPE
    assert L.moesq_quantize_act(ptr(), 8, 512, ctypes.byref(rt), ptr(), rc, ptr(4), ptr(), None) == INVALID
    assert L.moesq_quantize_act(ptr(2), 8, 512, ctypes.byref(rt), ptr(), rc, ptr(), ptr(), None) == INVALID
    assert L.moesq_quantize_act(ptr(), 9, 512, ctypes.byref(rt), ptr(), rc, ptr(), ptr(), None) == INVALID
    assert L.moesq_quantize_act(ptr(), 8, 512, None, ptr(), 100, ptr(), ptr(), None) == INVALID
    assert L.moesq_swiglu_quant(ptr(), 100, ctypes.byref(rt), ptr(), ptr(), ptr(), 0, None) == SHAPE
    assert L.moesq_swiglu_quant(ptr(), 256, ctypes.byref(rt), ptr(), ptr(8), ptr(), 0, None) == INVALID
    assert L.moesq_swiglu_quant(ptr(), 256, ctypes.byref(rt), ptr(), ptr(), ptr(), 2, None) == INVALID
    assert L.moesq_combine(ptr(), 7, ctypes.byref(rt), ptr(), None) == INVALID
    assert L.moesq_combine(ptr(2), 256, ctypes.byref(rt), ptr(), None) == INVALID


def test_layer_checks(L):
    E, H, I = 4, 512, 256
    wgu, wdn = weights(E, 2 * I, H), weights(E, H, I)
    args = lambda ws, n, T=8, k=2, wd=wdn: L.moesq_moe_layer(ptr(), ptr(), T, k, ctypes.byref(wgu),   # noqa: E731
                                                              ctypes.byref(wd), ptr(), ptr(), ptr(), ws, n, None)
    need = L.moesq_layer_workspace_bytes(8, 2, E, H, I)
    assert need > 0
    assert args(ptr(), need - 1) == WORKSPACE
    assert args(ptr(128), need) == INVALID                          # workspace not 256-byte aligned
    assert args(ptr(), need, T=0) == INVALID
    assert args(ptr(), need, k=5) == SHAPE                          # top-k above the expert count
    assert args(ptr(), need, wd=weights(E, H, 512)) == INVALID     # down K != I
    assert args(ptr(), need, wd=weights(E, H, I, layout=1)) == INVALID   # down stack in the SwiGLU order


def test_weight_layout_and_fused_gemm_checks(L):
    def fused(w, cfg=None, h_codes=ptr(), a_scales=ptr()):
        return L.moesq_grouped_sparse_gemm_swiglu(ctypes.byref(w), ptr(), a_scales, 256, ptr(), ptr(), ptr(), ptr(),
                                                  h_codes, ptr(), ctypes.byref(cfg) if cfg else None, None)
    assert gemm(L, weights(layout=2)) == INVALID                    # unknown layout
    assert gemm(L, weights(M=384, layout=1)) == SHAPE               # SwiGLU order needs M % 256 == 0
    assert L.moesq_pack_weights(ptr(), 0, 4, ctypes.byref(weights(M=384, layout=1)), None) == SHAPE
    assert fused(weights()) == INVALID                              # plain order: not a fused gate_up stack
    assert fused(weights(layout=1), h_codes=None) == INVALID
    assert fused(weights(layout=1), a_scales=ptr(8)) == INVALID
    assert fused(weights(layout=1), h_codes=ptr(8)) == INVALID      # 16-byte code stores
    assert fused(weights(layout=1), B.moesq_gemm_config(96, 0, 0)) == INVALID
    assert fused(weights(layout=1), B.moesq_gemm_config(128, 0, 2)) == SHAPE   # no SM-pair form
    best, ms = B.moesq_gemm_config(0, 0, 0), ctypes.c_float(0)
    tune = lambda w, reps: L.moesq_gemm_swiglu_autotune(  # noqa: E731
        ctypes.byref(w), ptr(), ptr(), 256, ptr(), ptr(), ptr(), ptr(), ptr(), ptr(), reps, ctypes.byref(best),
        ctypes.byref(ms), None)
    assert tune(weights(), 3) == INVALID                            # plain order
    assert tune(weights(layout=1), 0) == INVALID


def test_dense_converter_checks(L):
    w = weights()
    assert L.moesq_import_dense_nvfp4(ptr(4), ptr(), ptr(), 0, 4, ctypes.byref(w), None) == INVALID
    assert L.moesq_import_dense_nvfp4(ptr(), ptr(), ptr(), 0, 0, ctypes.byref(w), None) == INVALID
    assert L.moesq_import_dense_nvfp4(ptr(), ptr(), ptr(), 3, 2, ctypes.byref(w), None) == INVALID
    assert L.moesq_export_dense_nvfp4(ctypes.byref(w), ptr(8), None) == INVALID
    assert L.moesq_export_dense_nvfp4(ctypes.byref(weights(M=64)), ptr(), None) == SHAPE


def test_mma_peak_checks(L):
    out = ctypes.c_double(0)
    assert L.moesq_mma_peak(1, 128, 1, 0, 100, None, None) == INVALID
    assert L.moesq_mma_peak(2, 128, 1, 0, 100, ctypes.byref(out), None) == INVALID     # sparse is 0 or 1
    assert L.moesq_mma_peak(1, 8, 1, 0, 100, ctypes.byref(out), None) == INVALID       # n below 16
    assert L.moesq_mma_peak(1, 264, 1, 0, 100, ctypes.byref(out), None) == INVALID     # n above 256
    assert L.moesq_mma_peak(1, 200, 1, 0, 100, ctypes.byref(out), None) == INVALID     # not a multiple of 16
    assert L.moesq_mma_peak(1, 256, 2, 0, 100, ctypes.byref(out), None) == INVALID     # two CTAs: n <= 128
    assert L.moesq_mma_peak(1, 128, 3, 0, 100, ctypes.byref(out), None) == INVALID
    assert L.moesq_mma_peak(1, 128, 1, 0, 0, ctypes.byref(out), None) == INVALID
    assert L.moesq_mma_peak(1, 128, 1, 2, 100, ctypes.byref(out), None) == INVALID   # with_copies is 0 or 1


def dense(E=4, M=256, K=512, **kw):
    f = dict(codes=P, scales=P, global_scale=P, dtiles=P)
    f.update(kw)
    return B.moesq_dense_weights(E, M, K, f["codes"], f["scales"], f["global_scale"], f["dtiles"])


def test_dense_control_checks(L):
    d = dense()
    args = lambda w, cfg=None: L.moesq_grouped_dense_gemm(ctypes.byref(w), ptr(), ptr(), 256, ptr(), ptr(),  # noqa
                                                          ptr(), ptr(), ctypes.byref(cfg) if cfg else None, None)
    assert args(dense(M=100)) == SHAPE
    assert args(dense(K=384)) == SHAPE
    assert args(dense(codes=0)) == INVALID
    assert args(dense(dtiles=P + 8)) == INVALID
    assert args(d, B.moesq_gemm_config(32, 0, 0)) == INVALID
    assert args(d, B.moesq_gemm_config(128, 0, 2)) == SHAPE                # no SM-pair form of the control
    assert L.moesq_pack_dense_nvfp4(ptr(4), 0, 4, ctypes.byref(d), None) == INVALID
    assert L.moesq_pack_dense_nvfp4(ptr(), 3, 2, ctypes.byref(d), None) == INVALID
    assert L.moesq_expand_scales16(ptr(), 100, 512, ptr(), None) == SHAPE
    assert L.moesq_expand_scales16(ptr(), 128, 384, ptr(), None) == SHAPE
    assert L.moesq_expand_scales16(None, 128, 512, ptr(), None) == INVALID
    sizes = (ctypes.c_size_t * 4)()
    L.moesq_dense_weights_bytes(2, 256, 512, sizes)
    assert list(sizes) == [2 * 256 * 256, 2 * 256 * 32, 8, 2 * 2 * 2 * 18432]
