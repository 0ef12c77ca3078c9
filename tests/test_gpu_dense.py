"""GPU parity of the dense NVFP4 control (the paper's "Dense (transposed)"
baseline of App. D.2): the dense pack bit-exact against the oracle's
(storage form and the kernel form decoded back), the per-32 -> per-16 token
scale expansion exact, and the dense grouped GEMM within the GEMM tolerance
(|y - y_ref| <= 1e-3 * sum|a w| + one bf16 spacing) of
oracle_dense_grouped_gemm."""
import numpy as np
import pytest

import layouts as L
import oracle as O
import synthetic as S
from gpu_cases import gemm_tolerance_ok, to_dev, to_np, weights_np

pytestmark = pytest.mark.gpu


def _dense_from_oracle(m, dp):
    torch = pytest.importorskip("torch")
    E, M, K2 = dp.codes.shape
    K = 2 * K2
    dw = m.DenseWeights(E, M, K)
    dw.codes.copy_(torch.from_numpy(dp.codes))
    dw.scales.copy_(torch.from_numpy(dp.scales))
    dw.global_scale.copy_(torch.from_numpy(dp.gamma))
    dw.dtiles.copy_(torch.from_numpy(L.dense_storage_to_dtiles(dp.codes, dp.scales)))
    torch.cuda.synchronize()
    return dw


@pytest.mark.parametrize("E,M,K", [(3, 256, 512), (2, 1536, 2048)])
def test_dense_pack_bit_exact(cuda_lib, E, M, K):
    m = cuda_lib
    w = weights_np(41, 0, E, M, K)
    dp = O.pack_dense_nvfp4(w)
    dw = m.DenseWeights(E, M, K)
    m.moesq_pack_dense_nvfp4(to_dev(w), 0, E, dw)
    assert m.moesq_get_device_error()[0] == 0
    assert (to_np(dw.codes) == dp.codes).all()
    assert (to_np(dw.scales) == dp.scales).all()
    assert (to_np(dw.global_scale) == dp.gamma).all()
    codes, scales = L.dtiles_to_dense_storage(to_np(dw.dtiles), E, M, K)
    assert (codes == dp.codes).all() and (scales == dp.scales).all()


def test_expand_scales16_exact(cuda_lib):
    m = cuda_lib
    R, K = 256, 1024
    rng = np.random.default_rng(5)
    s32 = rng.integers(0, 127, size=(R, K // 32), dtype=np.uint8)
    out = m.scales16_buffer(R, K)
    m.moesq_expand_scales16(to_dev(L.scales_to_mma(s32)), R, K, out)
    assert (to_np(out) == L.scales32_to_scales16_mma(s32)).all()


def _run_dense(m, dp, counts, K, seed, tile_n):
    torch = pytest.importorskip("torch")
    E = counts.size
    R = int(counts.sum())
    x = S.activations_bf16_np(seed, max(R, 1), K)
    ga = np.array([np.float32(O.act_global_scale(x)) * np.float32(1 + e % 3) for e in range(E)], np.float32)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    codes = np.zeros((R, K // 2), np.uint8)
    scales = np.zeros((R, K // 32), np.uint8)
    for e in range(E):
        if counts[e]:
            c, s = O.quantize_rows_bf16(x[offs[e]:offs[e + 1]], ga[e])
            codes[offs[e]:offs[e + 1]], scales[offs[e]:offs[e + 1]] = c, s
    y_ref, basis = O.dense_grouped_gemm(dp, codes, scales, offs, ga)
    dw = _dense_from_oracle(m, dp)
    rows = L.compact_to_rows(counts)
    rc = max(128, int(L.aligned_rows(counts)[-1]))
    c_rows = np.zeros((rc, K // 2), np.uint8)
    s_rows = np.zeros((rc, K // 32), np.uint8)
    c_rows[rows], s_rows[rows] = codes, scales
    s16 = m.scales16_buffer(rc, K)
    m.moesq_expand_scales16(to_dev(L.scales_to_mma(s_rows)), rc, K, s16)
    M = dp.codes.shape[1]
    y = torch.full((rc, M), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.moesq_grouped_dense_gemm(dw, to_dev(c_rows), s16, rc, to_dev(counts.astype(np.int32)),
                               to_dev(L.aligned_rows(counts)), to_dev(ga), y, tile_n=tile_n)
    st, word = m.moesq_get_device_error()
    assert st == 0, "device error word %#x" % word
    ok, err, bound, bad = gemm_tolerance_ok(to_np(y)[rows], y_ref, basis)
    return ok, (err.max(), np.argwhere(bad)[:5])


@pytest.mark.parametrize("tile_n", [64, 128])
@pytest.mark.parametrize("counts", [
    [0, 1, 0, 5, 0, 0, 0, 2],
    [129, 0, 31, 33, 1, 16, 17, 300],
    [128, 256, 32, 64, 96, 160, 192, 224],
])
def test_dense_gemm_edge_counts(cuda_lib, tile_n, counts):
    E, M, K = 8, 256, 512
    dp = O.pack_dense_nvfp4(weights_np(43, 0, E, M, K))
    ok, info = _run_dense(cuda_lib, dp, np.array(counts, np.int64), K, 44, tile_n)
    assert ok, info


@pytest.mark.parametrize("K", [768, 2048])
@pytest.mark.parametrize("tile_n", [64, 128])
def test_dense_gemm_k_steps(cuda_lib, K, tile_n):
    """K = 768 (three K steps) and 2048 (eight: the ring wraps), M = 1536."""
    E, M = 3, 1536
    dp = O.pack_dense_nvfp4(weights_np(45, 0, E, M, K))
    ok, info = _run_dense(cuda_lib, dp, np.array([7, 0, 200]), K, 46, tile_n)
    assert ok, info


def test_dense_full_path_30b_class(cuda_lib):
    """30B-class gate_up (E=128, K=2048, M=1536, T=256, top-8): dense pack,
    route, quantise, scale expansion and dense GEMM on the GPU, checked on
    the rows of 4 experts against the oracle."""
    torch = pytest.importorskip("torch")
    m = cuda_lib
    E, M, K, T, k = 128, 1536, 2048, 256, 8
    dw = m.DenseWeights(E, M, K)
    for e0 in range(0, E, 16):
        w = torch.stack([S.expert_weights_bf16_torch(47, 0, e, M, K, "cuda") for e in range(e0, e0 + 16)])
        m.moesq_pack_dense_nvfp4(w, e0, 16, dw)
    x = S.activations_bf16_np(47, T, K)
    lg = S.uniform_logits_np(47, T, E)
    rt = O.route(lg, k)
    ga = np.full(E, O.act_global_scale(x), np.float32)
    rb = m.RoutingBuffers(T, E, k)
    m.moesq_route_permute(to_dev(lg), rb)
    codes, scales = m.act_buffers(rb.rows_cap, K)
    m.moesq_quantize_act(to_dev(x), T, K, rb, to_dev(ga), rb.rows_cap, codes, scales)
    s16 = m.scales16_buffer(rb.rows_cap, K)
    m.moesq_expand_scales16(scales, rb.rows_cap, K, s16)
    y = torch.full((rb.rows_cap, M), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.moesq_grouped_dense_gemm(dw, codes, s16, rb.rows_cap, rb.counts, rb.row_offsets, to_dev(ga), y)
    assert m.moesq_get_device_error()[0] == 0
    yg = to_np(y)
    ro = L.aligned_rows(rt.counts)
    used = np.nonzero(rt.counts)[0]
    for e in (int(used[0]), int(used[len(used) // 2]), int(used[-1]), int(used[np.argmax(rt.counts[used])])):
        n = int(rt.counts[e])
        dp = O.pack_dense_nvfp4(S.expert_weights_bf16_np(47, 0, e, M, K)[None])
        s0 = rt.offsets[e]
        toks = rt.sorted_to_slot[s0:s0 + n] // k
        c, s = O.quantize_rows_bf16(x[toks], ga[e])
        y_ref, basis = O.dense_grouped_gemm(dp, c, s, np.array([0, n], np.int32), ga[e:e + 1])
        ok, err, bound, bad = gemm_tolerance_ok(yg[ro[e]:ro[e] + n], y_ref, basis)
        assert ok, (e, n, err.max())
