"""Pins of the oracle's grouped GEMM (Sec. 3.4: Y_e = X_e W_e^T per expert,
swap-AB form Y_e^T = W_e X_e^T, epilogue factor alpha_e) and of the layer
composition (App. D.1), against numpy matmul over dequantised operands."""
import numpy as np
import pytest
import scipy.special

import oracle as O
import synthetic as S
from conftest import golden_dict


def _case(E=4, M=32, K=256, T=24, k=2, seed=21):
    w = np.stack([S.expert_weights_bf16_np(seed, 0, e, M, K) for e in range(E)])
    pk = O.pack_weights(w)
    x = S.activations_bf16_np(seed, T, K)
    rt = O.route(S.uniform_logits_np(seed, T, E), k)
    ga = np.full(E, O.act_global_scale(x), np.float32)
    ga[1] *= np.float32(0.5)                     # distinct per-expert scales
    a_c, a_s = O.permute_quantize(x, rt, ga)
    return pk, rt, a_c, a_s, ga


def _deq_act(codes, scales, gamma):
    R, K2 = codes.shape
    c = np.stack([codes & 15, codes >> 4], -1).reshape(R, 2 * K2)
    return np.vectorize(O.e2m1_value)(c) * np.repeat(np.vectorize(O.ue4m3_value)(scales), 32, 1) / gamma


def test_grouped_equals_per_expert_matmul():
    pk, rt, a_c, a_s, ga = _case()
    E, M, K = pk.values.shape[0], pk.values.shape[1], pk.values.shape[2] * 4
    y, basis, exact = O.grouped_gemm(pk, a_c, a_s, rt.offsets, ga, want_exact=True)
    for e in range(E):
        r0, r1 = rt.offsets[e], rt.offsets[e + 1]
        if r1 == r0:
            continue
        W = O.unpack_weights(pk.values[e], pk.mask[e], pk.scales[e], pk.gamma[e], M, K)
        X = _deq_act(a_c[r0:r1], a_s[r0:r1], ga[e])
        ref = X @ W.T                                 # Y_e = X_e W_e^T
        assert np.allclose(exact[r0:r1], ref, rtol=1e-6, atol=1e-6 * np.abs(ref).max())
        # swap-AB: (W_e X_e^T)^T is the same matrix
        assert np.allclose((W @ X.T).T, ref, rtol=1e-12, atol=1e-12)
        # tolerance basis is sum |a w|
        assert np.allclose(basis[r0:r1], np.abs(X) @ np.abs(W).T, rtol=1e-6)
        # bf16 output is the once-rounded exact value
        yb = S.bf16_bits_to_f32_np(y[r0:r1]).astype(np.float64)
        assert (np.abs(yb - exact[r0:r1]) <= np.abs(exact[r0:r1]) * 2.0 ** -8 + 1e-30).all()


def test_brute_force_tiny():
    """Element-by-element triple loop in Python on a tiny case."""
    pk, rt, a_c, a_s, ga = _case(E=2, M=8, K=64, T=3, k=1, seed=5)
    y, basis, exact = O.grouped_gemm(pk, a_c, a_s, rt.offsets, ga, want_exact=True)
    M, K = 8, 64
    for e in range(2):
        W = O.unpack_weights(pk.values[e], pk.mask[e], pk.scales[e], pk.gamma[e], M, K)
        for r in range(rt.offsets[e], rt.offsets[e + 1]):
            X = _deq_act(a_c[r:r + 1], a_s[r:r + 1], ga[e])[0]
            for m in range(M):
                s, sa = 0.0, 0.0
                for kk in range(K):
                    s += float(X[kk]) * float(W[m, kk])
                    sa += abs(float(X[kk]) * float(W[m, kk]))
                # alpha_e is one binary32 rounding of 1 / (gamma_w * gamma_a)
                assert abs(exact[r, m] - s) <= 2.0 ** -22 * sa + 1e-300
                assert abs(basis[r, m] - sa) <= 2.0 ** -22 * sa + 1e-300


def test_empty_experts_leave_rows_untouched():
    pk, rt, a_c, a_s, ga = _case(E=8, T=3, k=1)
    assert (rt.counts == 0).any()
    y, _ = O.grouped_gemm(pk, a_c, a_s, rt.offsets, ga)
    assert y.shape == (3, pk.values.shape[1])


def test_swiglu_matches_library():
    rng = np.random.default_rng(0)
    g = rng.normal(size=(5, 16)).astype(np.float32)
    u = rng.normal(size=(5, 16)).astype(np.float32)
    y = S.f32_to_bf16_bits_np(np.concatenate([g, u], 1))
    h = O.swiglu(y)
    gb = S.bf16_bits_to_f32_np(y[:, :16]).astype(np.float64)
    ub = S.bf16_bits_to_f32_np(y[:, 16:]).astype(np.float64)
    ref = gb * scipy.special.expit(gb) * ub
    assert np.allclose(h, ref, rtol=1e-6, atol=1e-7)


def test_combine_matches_einsum():
    rng = np.random.default_rng(2)
    T, k, H = 6, 3, 32
    R = T * k
    y = S.f32_to_bf16_bits_np(rng.normal(size=(R, H)).astype(np.float32))
    perm = rng.permutation(R).astype(np.int32)
    w = rng.uniform(size=(T, k)).astype(np.float32)
    out = O.combine(y, w, perm, T, k)
    yf = S.bf16_bits_to_f32_np(y).astype(np.float64)
    ref = np.einsum("tj,tjh->th", w.astype(np.float64), yf[perm.reshape(T, k)])
    got = S.bf16_bits_to_f32_np(out)
    assert np.allclose(got, ref, rtol=2 ** -8, atol=1e-6)


def test_layer_single_expert_chain():
    """E = 1, k = 1: the router weight is 1 and the layer is the plain
    gate_up -> SiLU*up -> down chain of that expert (numpy matmul)."""
    H, I, T = 128, 64, 8
    wgu = S.expert_weights_bf16_np(8, 0, 0, 2 * I, H)[None]
    wdn = S.expert_weights_bf16_np(8, 1, 0, H, I)[None]
    pgu, pdn = O.pack_weights(wgu), O.pack_weights(wdn)
    x = S.activations_bf16_np(8, T, H)
    logits = np.zeros((T, 1), np.float32)
    ga = np.array([O.act_global_scale(x)], np.float32)
    out, st = O.moe_layer(x, logits, 1, pgu, pdn, ga, np.array([1.0], np.float32), keep=True)
    gh = np.array([O.global_scale(np.abs(st["h"]).max())], np.float32)
    out, st = O.moe_layer(x, logits, 1, pgu, pdn, ga, gh, keep=True)
    assert (st["rt"].topk_w == 1.0).all()
    Wg = O.unpack_weights(pgu.values[0], pgu.mask[0], pgu.scales[0], pgu.gamma[0], 2 * I, H)
    Wd = O.unpack_weights(pdn.values[0], pdn.mask[0], pdn.scales[0], pdn.gamma[0], H, I)
    X = _deq_act(*O.quantize_rows_bf16(x, ga[0]), ga[0])
    gu = X @ Wg.T
    gu = S.bf16_bits_to_f32_np(S.f32_to_bf16_bits_np(gu.astype(np.float32))).astype(np.float64)
    hh = gu[:, :I] * scipy.special.expit(gu[:, :I]) * gu[:, I:]
    Hq = _deq_act(*O.quantize_rows(hh.astype(np.float32), gh[0]), gh[0])
    ref = Hq @ Wd.T
    got = S.bf16_bits_to_f32_np(out).astype(np.float64)
    assert np.abs(got - ref).max() / np.abs(ref).max() < 1e-2


def test_layer_identical_experts_reduce_to_weighted_single_expert():
    """E identical experts with equal global scales compute the same function
    of a token, so routing, dispatch, grouped GEMMs and combine must give
    out[t] = bf16((sum_j w_tj) * y[t]), y[t] the single-expert layer's output
    row (exact in bf16), for every token: a token row landing in another
    token's slot, a dropped or doubled slot, or a wrong router weight breaks
    it."""
    E, k, H, I, T = 6, 3, 128, 64, 16
    w1gu = S.expert_weights_bf16_np(9, 0, 0, 2 * I, H)[None]
    w1dn = S.expert_weights_bf16_np(9, 1, 0, H, I)[None]
    p1gu, p1dn = O.pack_weights(w1gu), O.pack_weights(w1dn)
    pEgu, pEdn = O.pack_weights(np.repeat(w1gu, E, axis=0)), O.pack_weights(np.repeat(w1dn, E, axis=0))
    x = S.activations_bf16_np(9, T, H)
    ga1 = np.array([O.act_global_scale(x)], np.float32)
    _, st = O.moe_layer(x, np.zeros((T, 1), np.float32), 1, p1gu, p1dn, ga1, np.ones(1, np.float32), keep=True)
    gh1 = np.array([O.global_scale(np.abs(st["h"]).max())], np.float32)
    y1 = O.moe_layer(x, np.zeros((T, 1), np.float32), 1, p1gu, p1dn, ga1, gh1)
    logits = S.uniform_logits_np(9, T, E)
    outE = O.moe_layer(x, logits, k, pEgu, pEdn, np.repeat(ga1, E), np.repeat(gh1, E))
    wsum = O.route(logits, k).topk_w.reshape(T, k).astype(np.float64).sum(axis=1)
    y1f = S.bf16_bits_to_f32_np(y1).astype(np.float64)
    want = np.array([[O.bf16_round(wsum[t] * y1f[t, h]) for h in range(H)] for t in range(T)], np.uint16)
    assert (wsum > 0.3).all() and (wsum <= 1.0 + 1e-6).all()
    assert (outE == want).all()


def test_effective_tflops_formula_table10():
    """App. D.2's TFLOP/s_eff with Table 10's setting reproduces the printed
    2627 TFLOP/s from the printed 0.687 ms (to the printed precision)."""
    from grouped_gemm_moesq_b200.metrics import effective_tflops, token_pattern
    g = golden_dict("table10_throughput.txt")
    counts = token_pattern(int(g["N"]), int(g["G"]))
    assert sum(counts) == 30720
    tf = effective_tflops(int(g["M"]), int(g["K"]), counts, g["latency_ms"] * 1e-3)
    assert abs(tf - g["tflops_printed"]) / g["tflops_printed"] < 1e-3
