"""Pins of the oracle's activation quantiser (Sec. 3.4 Eq. 5 with a stored
per-expert-linear global scale, model card "Activations") and of its top-k
routing / expert grouping."""
import ml_dtypes
import numpy as np
import pytest
import scipy.special

import oracle as O
import synthetic as S


def test_power_of_two_scale_reduces_to_plain_e2m1():
    """With gamma = 448 (amax_t = 6) a block of amax 6 gets scale 448 -> s_b = 1
    and a block of amax 3 gets scale 224 -> s_b = 1/2: the codes are then plain
    E2M1 rounding of x and 2x, checked against the library's float4."""
    rng = np.random.default_rng(1)
    x = rng.uniform(-6, 6, size=(4, 64)).astype(np.float32)
    x[:, 0] = 6.0
    x[:, 32] = 3.0
    x[:, 33:64] = np.clip(x[:, 33:64], -3, 3)
    codes, scales = O.quantize_rows(x, 448.0)
    assert (scales[:, 0] == 0x7E).all() and (scales[:, 1] == 0x76).all()
    assert O.ue4m3_value(0x76) == 224.0
    lo = np.stack([codes & 15, codes >> 4], -1).reshape(4, 64)
    ref0 = x[:, :32].astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    ref1 = (2 * x[:, 32:]).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    ref = np.concatenate([ref0, ref1], 1)
    ref = np.where(ref == 8, 0, ref)
    assert (lo == ref).all()


def test_saturation_when_gamma_underestimates():
    # gamma fitted to amax 1 while the block reaches 10: scale clips at 448,
    # values clip at +-6
    x = np.zeros((1, 32), np.float32)
    x[0, 0], x[0, 1], x[0, 2] = 10.0, -10.0, 0.5
    g = O.global_scale(1.0)
    codes, scales = O.quantize_rows(x, g)
    assert scales[0, 0] == 0x7E
    assert codes[0, 0] == (0x7 | (0xF << 4))
    s_b = 448.0 / g
    assert O.e2m1_value(codes[0, 1] & 15) == O.e2m1_value(O.e2m1_encode(np.float32(0.5) / np.float32(s_b)))


def test_zero_rows_and_blocks():
    x = np.zeros((2, 64), np.float32)
    x[1, 40] = 1.0
    codes, scales = O.quantize_rows(x, 100.0)
    assert (codes[0] == 0).all() and (scales[0] == 0).all()
    assert scales[1, 0] == 0 and scales[1, 1] != 0


def test_quantize_error_bound():
    """Dequantised values lie within one scale step of x (largest grid gap 2
    between 4 and 6) unless saturated; average error is well below that."""
    xb = S.activations_bf16_np(2, 16, 512)
    x = S.bf16_bits_to_f32_np(xb)
    g = O.act_global_scale(xb)
    codes, scales = O.quantize_rows(x, g)
    c = np.stack([codes & 15, codes >> 4], -1).reshape(16, 512)
    vals = np.vectorize(O.e2m1_value)(c)
    s = np.vectorize(O.ue4m3_value)(scales) / g
    deq = vals * np.repeat(s, 32, 1)
    err = np.abs(deq - x)
    assert (err <= np.repeat(s, 32, 1) + 1e-12).all()
    assert err.mean() / np.abs(x).mean() < 0.15


def test_bf16_path_equals_float_path():
    xb = S.activations_bf16_np(4, 3, 256)
    a = O.quantize_rows_bf16(xb, 37.5)
    b = O.quantize_rows(S.bf16_bits_to_f32_np(xb), 37.5)
    assert (a[0] == b[0]).all() and (a[1] == b[1]).all()


# ---------------------------------------------------------------- routing
@pytest.mark.parametrize("T,E,k", [(64, 8, 2), (37, 128, 8), (5, 384, 8), (1, 8, 8)])
def test_route_brute_force(T, E, k):
    lg = S.uniform_logits_np(7, T, E)
    lg[0, 1] = lg[0, 0]                          # an exact tie
    rt = O.route(lg, k)
    # ids: descending logit, ties to the lower index (numpy lexsort)
    for t in range(T):
        order = np.lexsort((np.arange(E), -lg[t].astype(np.float64)))[:k]
        assert (rt.topk_ids[t] == order).all()
    # weights: softmax over all E (scipy, float64)
    sm = scipy.special.softmax(lg.astype(np.float64), axis=1)
    want = np.take_along_axis(sm, rt.topk_ids.astype(np.int64), 1)
    assert np.allclose(rt.topk_w, want, rtol=2e-6, atol=1e-9)
    # grouping: counts, offsets, a bijection sorted by (expert, token, slot)
    assert (rt.counts == np.bincount(rt.topk_ids.ravel(), minlength=E)).all()
    assert rt.offsets[0] == 0 and (np.diff(rt.offsets) == rt.counts).all()
    assert sorted(rt.sorted_to_slot.tolist()) == list(range(T * k))
    ex = rt.topk_ids.ravel()[rt.sorted_to_slot]
    assert (np.diff(ex) >= 0).all()
    for e in range(E):
        seg = rt.sorted_to_slot[rt.offsets[e]:rt.offsets[e + 1]]
        assert (np.diff(seg) > 0).all()
        assert (ex[rt.offsets[e]:rt.offsets[e + 1]] == e).all()


def test_zipf_routing_is_skewed():
    lg = S.zipf_logits_np(1234, 2048, 384)
    rt = O.route(lg, 8)
    c = np.sort(rt.counts)
    assert c[-1] / max(c[0], 1) > 50
