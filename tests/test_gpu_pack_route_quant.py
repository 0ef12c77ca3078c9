"""GPU parity: weight packing, routing and activation quantisation must match
the oracle bit for bit (codes, scales, masks, ids, offsets, permutations);
gate weights and SwiGLU outputs within the stated tolerances."""
import numpy as np
import pytest

import layouts as L
import oracle as O
import synthetic as S
from gpu_cases import (pack_gpu_from_np, pack_gpu_generated, requant_mismatches, to_dev, to_np, weights_np)

pytestmark = pytest.mark.gpu


def _check_pack(pw, pk, E, M, K):
    assert (to_np(pw.values) == pk.values).all()
    assert (to_np(pw.mask) == pk.mask).all()
    assert (to_np(pw.scales) == pk.scales).all()
    assert (to_np(pw.global_scale).view(np.uint32) == pk.gamma.view(np.uint32)).all()
    assert (to_np(pw.ktiles) == L.storage_to_ktiles(pk.values, pk.mask, pk.scales)).all()
    v, mk, sc = L.ktiles_to_storage(to_np(pw.ktiles), E, M, K)
    assert (v == pk.values).all() and (mk == pk.mask).all() and (sc == pk.scales).all()


@pytest.mark.parametrize("E,M,K", [(8, 256, 512), (3, 128, 256)])
def test_pack_bit_exact(cuda_lib, E, M, K):
    w = weights_np(31, 0, E, M, K)
    if E == 3:                      # a zero expert, a zero block and tied pairs
        w[1] = 0
        w[2, :, :32] = 0
        w[2, 5, 64:72] = S.f32_to_bf16_bits_np(np.full(8, 0.01, np.float32))
    pw = pack_gpu_from_np(cuda_lib, w)
    _check_pack(pw, O.pack_weights(w), E, M, K)


def test_pack_30b_class_sampled_experts(cuda_lib):
    E, M, K = 128, 1536, 2048
    pw = pack_gpu_generated(cuda_lib, 77, 0, E, M, K)
    for e in (0, 63, 127):
        w = S.expert_weights_bf16_np(77, 0, e, M, K)[None]
        pk = O.pack_weights(w)
        assert (to_np(pw.values[e]) == pk.values[0]).all()
        assert (to_np(pw.mask[e]) == pk.mask[0]).all()
        assert (to_np(pw.scales[e]) == pk.scales[0]).all()
        assert to_np(pw.global_scale)[e] == pk.gamma[0]
        per = M * K // 32 * 11
        assert (to_np(pw.ktiles[e * per:(e + 1) * per]) == L.storage_to_ktiles(pk.values, pk.mask, pk.scales)).all()


# ---------------------------------------------------------------- routing
ROUTE_CASES = [
    ("tiny", 64, 8, 2, "uniform"),
    ("one_token", 1, 384, 8, "uniform"),
    ("30b", 256, 128, 8, "uniform"),
    ("kimi_t16", 16, 384, 8, "uniform"),
    ("kimi_t256", 256, 384, 8, "uniform"),
    ("ragged_blocks", 300, 64, 4, "uniform"),
    ("kimi_prefill_zipf", 8192, 384, 8, "zipf"),
    ("k_equals_e", 5, 8, 8, "uniform"),
]


@pytest.mark.parametrize("name,T,E,k,dist", ROUTE_CASES)
def test_route_permute_bit_exact(cuda_lib, name, T, E, k, dist):
    m = cuda_lib
    lg = S.zipf_logits_np(1234, T, E) if dist == "zipf" else S.uniform_logits_np(42, T, E)
    if T > 2:
        lg[1, 3] = lg[1, 5]          # exact ties
        lg[2, :] = 0.25
    rt = O.route(lg, k)
    rb = m.RoutingBuffers(T, E, k)
    m.moesq_route_permute(to_dev(lg), rb)
    assert (to_np(rb.topk_ids).reshape(T, k) == rt.topk_ids).all()
    assert (to_np(rb.counts) == rt.counts).all()
    assert (to_np(rb.offsets) == rt.offsets).all()
    assert (to_np(rb.sorted_to_slot) == rt.sorted_to_slot).all()
    assert (to_np(rb.row_offsets) == L.aligned_rows(rt.counts)).all()
    rows = L.compact_to_rows(rt.counts)
    assert (to_np(rb.slot_to_row)[rt.sorted_to_slot] == rows).all()
    w = to_np(rb.topk_w).reshape(T, k)
    assert np.allclose(w, rt.topk_w, rtol=4e-6, atol=1e-12)


# ---------------------------------------------------------------- quantisation
def test_quantize_plain_bit_exact(cuda_lib):
    m = cuda_lib
    T, K = 200, 1024
    x = S.activations_bf16_np(5, T, K)
    g = np.float32(O.act_global_scale(x))
    rc = 256
    codes, scales = m.act_buffers(rc, K)
    m.moesq_quantize_act(to_dev(x), T, K, None, to_dev(np.array([g], np.float32)), rc, codes, scales)
    oc, os_ = O.quantize_rows_bf16(x, g)
    assert (to_np(codes)[:T] == oc).all()
    assert (L.mma_to_scales(to_np(scales), rc, K)[:T] == os_).all()


def test_act_global_scale_bit_exact(cuda_lib):
    torch = pytest.importorskip("torch")
    x = S.activations_bf16_np(6, 33, 512)
    out = torch.empty(1, dtype=torch.float32, device="cuda")
    cuda_lib.moesq_act_global_scale(to_dev(x), out)
    assert to_np(out)[0] == np.float32(O.act_global_scale(x))


@pytest.mark.parametrize("T,E,k,K", [(64, 8, 2, 512), (37, 128, 8, 2048)])
def test_quantize_dispatch_bit_exact(cuda_lib, T, E, k, K):
    m = cuda_lib
    x = S.activations_bf16_np(8, T, K)
    lg = S.uniform_logits_np(8, T, E)
    rt = O.route(lg, k)
    ga = (np.float32(O.act_global_scale(x)) * (1 + np.arange(E, dtype=np.float32) / 7)).astype(np.float32)
    oc, os_ = O.permute_quantize(x, rt, ga)
    rb = m.RoutingBuffers(T, E, k)
    m.moesq_route_permute(to_dev(lg), rb)
    codes, scales = m.act_buffers(rb.rows_cap, K)
    m.moesq_quantize_act(to_dev(x), T, K, rb, to_dev(ga), rb.rows_cap, codes, scales)
    rows = L.compact_to_rows(rt.counts)
    assert (to_np(codes)[rows] == oc).all()
    assert (L.mma_to_scales(to_np(scales), rb.rows_cap, K)[rows] == os_).all()


@pytest.mark.parametrize("I,sigma", [(512, 2.0), (2048, 6.0)])
def test_swiglu_quant_matches_oracle(cuda_lib, I, sigma):
    """SwiGLU + requantisation against the oracle, complete: every scale code
    equal unless the block's gamma * amax / 6 lies within SWIGLU_BAND of a
    UE4M3 decision point; under an equal scale code every E2M1 code equal
    unless h / s_b lies within SWIGLU_BAND of an E2M1 decision point; no
    other difference is allowed (gpu_cases.requant_mismatches)."""
    m = cuda_lib
    T, E, k = 48, 8, 2
    lg = S.uniform_logits_np(9, T, E)
    rt = O.route(lg, k)
    R = T * k
    rng = np.random.default_rng(9 + I)
    y_c = S.f32_to_bf16_bits_np(rng.normal(0, sigma, size=(R, 2 * I)).astype(np.float32))
    h = O.swiglu(y_c)
    gh = np.full(E, O.global_scale(np.abs(h).max()), np.float32)
    gh[3] *= np.float32(0.5)
    gh[5] *= np.float32(3.0)
    oc, os_ = O.requantize_rows(h, rt, gh)
    rb = m.RoutingBuffers(T, E, k)
    m.moesq_route_permute(to_dev(lg), rb)
    rows = L.compact_to_rows(rt.counts)
    y_rows = np.zeros((rb.rows_cap, 2 * I), np.uint16)
    y_rows[rows] = y_c
    hc, hs = m.act_buffers(rb.rows_cap, I)
    m.moesq_swiglu_quant(to_dev(y_rows), I, rb, to_dev(gh), hc, hs)
    assert m.moesq_get_device_error()[0] == 0
    gc = to_np(hc)[rows]
    gs = L.mma_to_scales(to_np(hs), rb.rows_cap, I)[rows]

    bad_scale, bad_code, scale_diff, code_diff = requant_mismatches(h, gh[rt.expert_of_sorted()], os_, oc, gs, gc)
    assert not bad_scale.any(), np.argwhere(bad_scale)[:5]
    assert not bad_code.any(), (np.argwhere(bad_code)[:5], int(bad_code.sum()))
    # the allowance is rare: the band covers a tiny part of the value range
    assert scale_diff.mean() < 1e-2 and code_diff.mean() < 1e-3


# ---------------------------------------------------------------- quantiser near the E2M1 decision points
E2M1_DECISIONS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)   # midpoints of the E2M1 grid (App. A, Fig. 3)


def _bf16_neighbours(t: np.ndarray):
    """The bf16 numbers just below-or-at and just above t > 0 (exact in float64)."""
    e = np.floor(np.log2(t))
    ulp = 2.0 ** (e - 7)
    lo = np.floor(t / ulp) * ulp
    return lo, lo + ulp


def _boundary_rows(gamma: float, T: int, K: int, rng):
    """Rows whose blocks hold an amax A and, for every decision point tau, the
    bf16 values nearest tau * s_b (both signs), s_b = UE4M3(code_b) / gamma."""
    nb = K // 32
    amax = rng.uniform(1.0, 2.0, size=(T, nb)) * 2.0 ** rng.integers(-3, 6, size=(T, nb))
    a_bits = S.f32_to_bf16_bits_np(amax.astype(np.float32))
    only_a = np.zeros((T, K), np.uint16)
    only_a[:, ::32] = a_bits
    _, sc = O.quantize_rows_bf16(only_a, gamma)
    s = (np.array([O.ue4m3_value(int(c)) for c in sc.ravel()], np.float32).reshape(T, nb)
         / np.float32(gamma)).astype(np.float64)
    vals = np.zeros((T, nb, 32), np.float64)
    taus = np.zeros((T, nb, 32), np.float64)
    j = 1
    for tau in E2M1_DECISIONS:
        lo, hi = _bf16_neighbours(tau * s)
        for v in (lo, hi):
            vals[:, :, j], taus[:, :, j] = v, tau
            vals[:, :, j + 1], taus[:, :, j + 1] = -v, tau
            j += 2
    x = S.f32_to_bf16_bits_np(vals.astype(np.float32)).reshape(T, nb, 32)
    x[:, :, 0] = a_bits
    rel = np.abs(np.abs(vals[:, :, 1:j]) / (s[:, :, None] * taus[:, :, 1:j]) - 1.0)
    return x.reshape(T, K), rel


@pytest.mark.parametrize("gamma", [1.0, 0.125, 32.0, 3.7, 259.1])
def test_quantize_near_decision_points_bit_exact(cuda_lib, gamma):
    """Every value within one bf16 step of an E2M1 decision point (exact ties
    when the step is a power of two): the GPU codes equal the oracle's, which
    rounds the correctly rounded quotient."""
    m = cuda_lib
    T, K = 64, 512
    rng = np.random.default_rng(int(gamma * 1000) + 7)
    x, rel = _boundary_rows(np.float32(gamma), T, K, rng)
    g = np.float32(gamma)
    oc, os_ = O.quantize_rows_bf16(x, g)
    rc = 128
    codes, scales = m.act_buffers(rc, K)
    m.moesq_quantize_act(to_dev(x), T, K, None, to_dev(np.array([g], np.float32)), rc, codes, scales)
    assert (L.mma_to_scales(to_np(scales), rc, K)[:T] == os_).all()
    assert (to_np(codes)[:T] == oc).all()
    if gamma in (1.0, 0.125, 32.0):
        assert (rel == 0).sum() > 100                      # exact ties on the decision points


def _near_miss_case(rng):
    """A global scale gamma, block amax A and bf16 value v with v / s_b within
    2^-21 (relative, nonzero) of a decision point, s_b = UE4M3(code) / gamma."""
    while True:
        c = int(rng.integers(40, 110))
        tau = float(rng.choice(E2M1_DECISIONS))
        v = float(np.frombuffer((np.uint32(S.f32_to_bf16_bits_np(np.float32([rng.uniform(1, 2)]))[0]) << 16).tobytes(),
                                np.float32)[0])
        val = O.ue4m3_value(c)
        g0 = np.float32(tau * val / v)
        want_above = bool(rng.integers(0, 2))
        for step in range(-64, 65):
            g = np.float32(g0 * (1.0 + step * 2.0 ** -23))
            sb = np.float32(np.float32(val) / g)
            d = (v / float(sb)) / tau - 1.0
            if d != 0 and abs(d) < 2.0 ** -21 and (d > 0) == want_above:
                amax = float(np.float32(6.0 * val / float(g)))
                a_bits = S.f32_to_bf16_bits_np(np.float32([amax]))[0]
                _, sc = O.quantize_rows_bf16(np.array([[a_bits] + [0] * 31], np.uint16), g)
                if int(sc[0, 0]) == c:
                    return g, a_bits, v
                break


def test_quantize_guard_band_bit_exact(cuda_lib):
    """Quotients within 2^-21 of a decision point (above and below), where the
    fast reciprocal path must defer to the exact quotient."""
    m = cuda_lib
    rng = np.random.default_rng(2024)
    T, K = 8, 256
    for _ in range(24):
        g, a_bits, v = _near_miss_case(rng)
        vb = S.f32_to_bf16_bits_np(np.float32([v, -v]))
        x = np.zeros((T, K), np.uint16)
        x[:, ::32] = a_bits
        for j in range(1, 32, 2):
            x[:, j::32] = vb[0]
            x[:, j + 1::32] = vb[1] if j + 1 < 32 else 0
        oc, os_ = O.quantize_rows_bf16(x, g)
        codes, scales = m.act_buffers(128, K)
        m.moesq_quantize_act(to_dev(x), T, K, None, to_dev(np.array([g], np.float32)), 128, codes, scales)
        assert (L.mma_to_scales(to_np(scales), 128, K)[:T] == os_).all()
        assert (to_np(codes)[:T] == oc).all()
