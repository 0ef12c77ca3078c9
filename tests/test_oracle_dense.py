"""Pins of the oracle's dense NVFP4 control (the paper's dense W4A4
baseline, App. D.2): every weight kept, one UE4M3 scale per 16 K elements,
the Eq. 5 global scale.  The codes are restated here with ml_dtypes
rounding, and the GEMM against numpy matmul of the decoded operands."""
import ml_dtypes
import numpy as np

import oracle as O
import synthetic as S


def _f32(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32)


def _restated_pack(w_bf16):
    """Eq. 5 / Eq. 3 per 16-element group in binary32 with library rounding:
    code_b = RNE_E4M3(gamma * amax_b / 6) (saturating at 448), s_b =
    UE4M3(code_b) / gamma, value code = RNE_E2M1(w / s_b) (saturating at 6,
    -0 written as +0, zero-scale blocks all zero)."""
    M, K = w_bf16.shape
    w = _f32(w_bf16)
    amax_t = np.float32(np.abs(w).max())
    gamma = np.float32(448.0) / np.float32(amax_t / np.float32(6.0)) if amax_t > 0 else np.float32(1.0)
    blocks = np.abs(w).reshape(M, K // 16, 16).max(-1)
    sc = (np.float32(gamma) * blocks).astype(np.float32) / np.float32(6.0)
    sc = np.minimum(sc.astype(np.float32), np.float32(448.0))
    code = sc.astype(ml_dtypes.float8_e4m3fn)
    code_bits = code.view(np.uint8) & 0x7F
    val = code.astype(np.float32)
    step = (val / gamma).astype(np.float32)
    q = np.where(step[..., None] > 0, w.reshape(M, K // 16, 16) / np.where(step > 0, step, 1)[..., None], 0)
    q = np.clip(q.astype(np.float32), -6.0, 6.0)
    c4 = q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    c4 = np.where(c4 == 8, 0, c4).reshape(M, K)                       # -0 -> +0
    codes = (c4[:, 0::2] | (c4[:, 1::2] << 4)).astype(np.uint8)
    return codes, code_bits.astype(np.uint8), gamma


def test_dense_pack_matches_library_rounding():
    w = np.stack([S.expert_weights_bf16_np(5, 0, e, 64, 256) for e in range(3)])
    w[1, :, :16] = 0                                                    # a zero block
    w[2, 3, 32:48] = S.f32_to_bf16_bits_np(np.full(16, 3.0, np.float32))   # a block at the tensor amax
    dp = O.pack_dense_nvfp4(w)
    for e in range(3):
        codes, scales, gamma = _restated_pack(w[e])
        assert dp.gamma[e] == gamma
        assert (dp.scales[e] == scales).all()
        assert (dp.codes[e] == codes).all()
    assert dp.scales[2, 3, 2] == 0x7E                                   # 448: the amax block


def _deq(codes, scales, group):
    R, K2 = codes.shape
    c = np.stack([codes & 15, codes >> 4], -1).reshape(R, 2 * K2).astype(np.uint8)
    v = c.view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    s = scales.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return v * np.repeat(s, group, 1)


def test_dense_grouped_gemm_is_the_dequantised_matmul():
    E, M, K, T, k = 3, 32, 256, 12, 2
    w = np.stack([S.expert_weights_bf16_np(6, 0, e, M, K) for e in range(E)])
    dp = O.pack_dense_nvfp4(w)
    x = S.activations_bf16_np(6, T, K)
    rt = O.route(S.uniform_logits_np(6, T, E), k)
    ga = np.full(E, O.act_global_scale(x), np.float32)
    a_c, a_s = O.permute_quantize(x, rt, ga)
    y, basis, exact = O.dense_grouped_gemm(dp, a_c, a_s, rt.offsets, ga, want_exact=True)
    for e in range(E):
        r0, r1 = rt.offsets[e], rt.offsets[e + 1]
        if r1 == r0:
            continue
        Wq = _deq(dp.codes[e], dp.scales[e], 16)
        Xq = _deq(a_c[r0:r1], a_s[r0:r1], 32)
        alpha = np.float64(np.float32(1.0) / np.float32(dp.gamma[e] * ga[e]))
        ref = alpha * (Xq @ Wq.T)
        assert np.allclose(exact[r0:r1], ref, rtol=1e-12, atol=1e-300)
        assert np.allclose(basis[r0:r1], np.abs(alpha) * (np.abs(Xq) @ np.abs(Wq).T), rtol=1e-12)


def test_dense_reconstruction_within_one_step():
    w = S.expert_weights_bf16_np(7, 0, 0, 64, 512)[None]
    dp = O.pack_dense_nvfp4(w)
    wf = _f32(w[0]).astype(np.float64)
    deq = _deq(dp.codes[0], dp.scales[0], 16) / np.float64(dp.gamma[0])
    step = np.repeat(dp.scales[0].view(ml_dtypes.float8_e4m3fn).astype(np.float64), 16, 1) / dp.gamma[0]
    # E2M1 spacing is at most 2 steps (between 4 and 6), so |error| <= 1 step
    assert (np.abs(deq - wf) <= step * (1 + 1e-6) + 1e-30).all()


def test_storage_bits_dense_vs_paired():
    """Dense NVFP4: 4 bits per value + 8 bits per 16 = 4.5 bits per weight;
    the paired format stores 2.75 (App. A, Eq. 7)."""
    M, K = 128, 2048
    dense_bits = 8 * (M * K // 2 + M * K // 16) / (M * K)
    paired_bits = 8 * (M * K // 4 + M * K // 16 + M * K // 32) / (M * K)
    assert dense_bits == 4.5 and paired_bits == 2.75
