"""The gate_up GEMM with SwiGLU and the NVFP4 requantisation of h in its
epilogue (paper App. D.1, "Serving integration": the backend's fused SwiGLU
with requantization), on the GPU:

- the gate/up-interleaved kernel row order of the packed weights against
  the oracle's storage form and the layout's definition;
- the fused kernel bit for bit against the unfused pair (the same grouped
  GEMM, then the SwiGLU kernel reading y_gu in that order), over ragged
  expert sizes, both token tiles and one or two CTAs per SM;
- the fused h codes and scales against the oracle's SwiGLU and
  requantisation of the same bf16 gate_up output, with the complete check
  of gpu_cases.requant_mismatches;
- whole layers (30B-A3B and Kimi-K2.5 shapes) with and without the fusion:
  outputs identical."""
import numpy as np
import pytest

import layouts as L
import oracle as O
import synthetic as S
from gpu_cases import requant_mismatches, to_dev, to_np, weights_np
from layouts import swiglu_kernel_rows

pytestmark = pytest.mark.gpu


def test_pack_swiglu_layout(cuda_lib):
    m = cuda_lib
    E, M, K = 3, 512, 512
    w = weights_np(61, 0, E, M, K)
    pk = O.pack_weights(w)
    p0 = m.PackedWeights(E, M, K)
    p1 = m.PackedWeights(E, M, K, layout=m.LAYOUT_SWIGLU)
    m.moesq_pack_weights(to_dev(w), 0, E, p0)
    m.moesq_pack_weights(to_dev(w), 0, E, p1)
    assert m.moesq_get_device_error()[0] == 0
    for name in ("values", "mask", "scales"):                # the storage form keeps the rows as given
        assert (to_np(getattr(p1, name)) == getattr(pk, name)).all(), name
    assert (to_np(p1.global_scale) == pk.gamma).all()
    perm = swiglu_kernel_rows(M)
    want = L.storage_to_ktiles(pk.values[:, perm], pk.mask[:, perm], pk.scales[:, perm])
    assert (to_np(p1.ktiles) == want).all()
    assert (to_np(p0.ktiles) == L.storage_to_ktiles(pk.values, pk.mask, pk.scales)).all()


def _fixed_routing(m, counts, I):
    """Routing buffers of one slot per row (T = sum(counts), k = 1): slot s
    is compact row s, its expert's aligned row; as the SwiGLU kernel reads
    them."""
    torch = pytest.importorskip("torch")
    counts = np.asarray(counts, np.int64)
    E, R = counts.size, int(counts.sum())
    rb = m.RoutingBuffers(max(R, 1), E, 1)
    ro = L.aligned_rows(counts)
    assert ro[-1] <= rb.rows_cap
    rows = L.compact_to_rows(counts)
    ex = np.repeat(np.arange(E), counts)
    rb.counts.copy_(torch.from_numpy(counts.astype(np.int32)))
    rb.row_offsets.copy_(torch.from_numpy(ro.astype(np.int32)))
    if R:
        rb.topk_ids[:R].copy_(torch.from_numpy(ex.astype(np.int32)))
        rb.slot_to_row[:R].copy_(torch.from_numpy(rows.astype(np.int32)))
    return rb, rows, ex


def _fused_case(m, counts, I, K, seed, tile_n, num_ctas=0):
    """Runs the unfused pair and the fused kernel on the same inputs.
    Returns (fused codes, fused scales, unfused codes, unfused scales, y in
    natural column order, rows, experts of the rows, gamma_h, rows_cap)."""
    torch = pytest.importorskip("torch")
    E, M = len(counts), 2 * I
    w = weights_np(seed, 0, E, M, K)
    pw = m.PackedWeights(E, M, K, layout=m.LAYOUT_SWIGLU)
    m.moesq_pack_weights(to_dev(w), 0, E, pw)
    rb, rows, ex = _fixed_routing(m, counts, I)
    R = len(rows)
    x = S.activations_bf16_np(seed + 1, max(R, 1), K)
    ga = np.array([np.float32(O.act_global_scale(x)) * np.float32(1 + e % 3) for e in range(E)], np.float32)
    codes = np.zeros((rb.rows_cap, K // 2), np.uint8)
    scales = np.zeros((rb.rows_cap, K // 32), np.uint8)
    for e in range(E):
        sel = np.nonzero(ex == e)[0]
        if sel.size:
            c, s = O.quantize_rows_bf16(x[sel], ga[e])
            codes[rows[sel]], scales[rows[sel]] = c, s
    a_codes, a_scales = to_dev(codes), to_dev(L.scales_to_mma(scales))
    y = torch.full((rb.rows_cap, M), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.moesq_grouped_sparse_gemm(pw, a_codes, a_scales, rb.rows_cap, rb.counts, rb.row_offsets, to_dev(ga), y,
                                tile_n=tile_n, num_ctas=num_ctas)
    assert m.moesq_get_device_error()[0] == 0
    # y in kernel row order -> natural [gate | up] order for the oracle
    y_nat = np.zeros((R, M), np.uint16)
    y_nat[:, swiglu_kernel_rows(M)] = to_np(y)[rows]
    h = O.swiglu(y_nat) if R else np.zeros((0, I))
    amax = np.array([np.abs(h[ex == e]).max() if (ex == e).any() else 1.0 for e in range(E)])
    gh = np.array([O.global_scale(a) for a in amax], np.float32) * np.array([1.0, 0.5, 3.0])[np.arange(E) % 3]
    gh = gh.astype(np.float32)
    hc0, hs0 = m.act_buffers(rb.rows_cap, I)
    hc0.fill_(0xAB)
    hs0.fill_(0xAB)
    m.moesq_swiglu_quant(y, I, rb, to_dev(gh), hc0, hs0, gu_layout=m.LAYOUT_SWIGLU)
    hc1, hs1 = m.act_buffers(rb.rows_cap, I)
    hc1.fill_(0xAB)
    hs1.fill_(0xAB)
    m.moesq_grouped_sparse_gemm_swiglu(pw, a_codes, a_scales, rb.rows_cap, rb.counts, rb.row_offsets, to_dev(ga),
                                       to_dev(gh), hc1, hs1, tile_n=tile_n, num_ctas=num_ctas)
    st, word = m.moesq_get_device_error()
    assert st == 0, "device error word %#x" % word
    return (to_np(hc1), to_np(hs1), to_np(hc0), to_np(hs0), h, rows, ex, gh, rb.rows_cap)


@pytest.mark.parametrize("tile_n", [64, 128])
@pytest.mark.parametrize("counts", [
    [0, 1, 0, 5, 0, 0, 0, 2],
    [129, 0, 31, 33, 1, 16, 17, 300],
    [128, 256, 32, 64, 96, 160, 192, 224],
])
def test_fused_equals_unfused(cuda_lib, tile_n, counts):
    """Every valid row's h codes and scales equal the unfused pair's; rows
    outside the experts' valid rows are left as they were."""
    I, K = 256, 512
    hc1, hs1, hc0, hs0, _, rows, _, _, rc = _fused_case(cuda_lib, counts, I, K, 71, tile_n)
    assert (hc1[rows] == hc0[rows]).all()
    s1, s0 = L.mma_to_scales(hs1, rc, I), L.mma_to_scales(hs0, rc, I)
    assert (s1[rows] == s0[rows]).all()
    pad = np.ones(rc, bool)
    pad[rows] = False
    assert (hc1[pad] == 0xAB).all() and (s1[pad] == 0xAB).all()


@pytest.mark.parametrize("I,K,tile_n,num_ctas", [(768, 2048, 64, 148), (2048, 1024, 128, 0), (2048, 1024, 64, 0)])
def test_fused_equals_unfused_wide(cuda_lib, I, K, tile_n, num_ctas):
    """30B-A3B and Kimi-K2.5 intermediate sizes (12 and 32 weight blocks of
    64 features), multi-K steps, one CTA per SM in the first case."""
    counts = [200, 0, 77, 129, 5, 256]
    hc1, hs1, hc0, hs0, _, rows, _, _, rc = _fused_case(cuda_lib, counts, I, K, 73, tile_n, num_ctas)
    assert (hc1[rows] == hc0[rows]).all()
    assert (L.mma_to_scales(hs1, rc, I)[rows] == L.mma_to_scales(hs0, rc, I)[rows]).all()


@pytest.mark.parametrize("tile_n", [64, 128])
def test_fused_matches_oracle(cuda_lib, tile_n):
    """Fused h codes and scales against the oracle's SwiGLU (binary64) and
    requantisation of the same bf16 gate_up output: the complete check
    (differences only next to a decision point, within SWIGLU_BAND)."""
    I, K = 512, 512
    counts = [64, 130, 0, 17, 255, 1]
    hc1, hs1, _, _, h, rows, ex, gh, rc = _fused_case(cuda_lib, counts, I, K, 75, tile_n)
    oc = np.zeros((len(rows), I // 2), np.uint8)
    os_ = np.zeros((len(rows), I // 32), np.uint8)
    for e in np.unique(ex):
        sel = ex == e
        oc[sel], os_[sel] = O.quantize_rows(h[sel], gh[e])
    gc = hc1[rows]
    gs = L.mma_to_scales(hs1, rc, I)[rows]
    bad_scale, bad_code, scale_diff, code_diff = requant_mismatches(h, gh[ex], os_, oc, gs, gc)
    assert not bad_scale.any(), np.argwhere(bad_scale)[:5]
    assert not bad_code.any(), (np.argwhere(bad_code)[:5], int(bad_code.sum()))
    assert scale_diff.mean() < 1e-2 and code_diff.mean() < 1e-3


def _layer_both_layouts(m, E, k, H, I, T, routing, seed):
    torch = pytest.importorskip("torch")
    from gpu_cases import pack_gpu_generated
    w_plain = pack_gpu_generated(m, seed, 0, E, 2 * I, H)
    w_dn = pack_gpu_generated(m, seed, 1, E, H, I)
    w_fused = m.PackedWeights(E, 2 * I, H, layout=m.LAYOUT_SWIGLU)
    for e0 in range(0, E, 8):
        n = min(8, E - e0)
        w = torch.stack([S.expert_weights_bf16_torch(seed, 0, e, 2 * I, H, "cuda") for e in range(e0, e0 + n)])
        m.moesq_pack_weights(w, e0, n, w_fused)
        del w
    x = S.activations_bf16_torch(seed, T, H, "cuda")
    lg_np = S.zipf_logits_np(seed, T, E) if routing == "zipf" else S.uniform_logits_np(seed, T, E)
    lg = torch.from_numpy(lg_np).cuda()
    ws = torch.empty(m.moesq_layer_workspace_bytes(T, k, E, H, I), dtype=torch.uint8, device="cuda")
    outs, gammas = [], []
    for w_gu in (w_plain, w_fused):
        ga = torch.empty(E, dtype=torch.float32, device="cuda")
        gh = torch.empty(E, dtype=torch.float32, device="cuda")
        m.moesq_calibrate_layer(x, lg, T, k, w_gu, w_dn, ga, gh, ws)
        out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        m.moesq_moe_layer(x, lg, T, k, w_gu, w_dn, ga, gh, out, ws)
        st, word = m.moesq_get_device_error()
        assert st == 0, "device error word %#x" % word
        outs.append(to_np(out))
        gammas.append((to_np(ga), to_np(gh)))
    return outs, gammas


@pytest.mark.parametrize("E,k,H,I,T,routing", [
    (128, 8, 2048, 768, 256, "uniform"),          # 30B-A3B shapes
    (384, 8, 7168, 2048, 4096, "zipf"),           # Kimi-K2.5 shapes
])
def test_layer_fused_equals_unfused(cuda_lib, E, k, H, I, T, routing):
    outs, gammas = _layer_both_layouts(cuda_lib, E, k, H, I, T, routing, 77)
    assert (gammas[0][0] == gammas[1][0]).all() and (gammas[0][1] == gammas[1][1]).all()
    assert (outs[0] == outs[1]).all()
