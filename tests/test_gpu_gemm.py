"""GPU parity of the grouped sparse GEMM against the oracle:
|y - y_ref| <= 1e-3 * sum_k |a_k w_k| + one bf16 spacing, per element."""
import numpy as np
import pytest

import layouts as L
import oracle as O
import synthetic as S
from gpu_cases import (act_rows_from_compact, expert_weights_host, gemm_tolerance_ok, pack_gpu_from_np,
                       pack_gpu_generated, packed_from_oracle, to_dev, to_np, weights_np)

pytestmark = pytest.mark.gpu


def _run_isolated(m, pk, counts, K, seed, tile_n, ga_scale=1.0, mode=0):
    """Oracle weights + oracle-quantised activations, laid out on the host,
    through the CUDA GEMM; returns (ok, detail)."""
    torch = pytest.importorskip("torch")
    E = counts.size
    R = int(counts.sum())
    x = S.activations_bf16_np(seed, max(R, 1), K)
    ga = np.array([np.float32(O.act_global_scale(x)) * np.float32(ga_scale * (1 + e % 3))
                   for e in range(E)], np.float32)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    ex = np.repeat(np.arange(E), counts)
    codes = np.zeros((R, K // 2), np.uint8)
    scales = np.zeros((R, K // 32), np.uint8)
    for e in range(E):
        if counts[e]:
            c, s = O.quantize_rows_bf16(x[offs[e]:offs[e + 1]], ga[e])
            codes[offs[e]:offs[e + 1]], scales[offs[e]:offs[e + 1]] = c, s
    y_ref, basis = O.grouped_gemm(pk, codes, scales, offs, ga)
    pw = packed_from_oracle(m, pk)
    c_rows, s_mma, rc = act_rows_from_compact(codes, scales, counts, K)
    M = pk.values.shape[1]
    y = torch.full((rc, M), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.moesq_grouped_sparse_gemm(pw, to_dev(c_rows), to_dev(s_mma), rc, to_dev(counts.astype(np.int32)),
                                to_dev(L.aligned_rows(counts)), to_dev(ga), y, tile_n=tile_n, sm_mode=mode)
    st, word = m.moesq_get_device_error()
    assert st == 0, "device error word %#x" % word
    rows = L.compact_to_rows(counts)
    yg = to_np(y)[rows]
    ok, err, bound, bad = gemm_tolerance_ok(yg, y_ref, basis)
    return ok, (err.max(), np.argwhere(bad)[:5], ex)


@pytest.mark.parametrize("tile_n", [64, 128])
def test_gemm_tiny_config(cuda_lib, tile_n):
    """E=8, K=512, M=256 with the token counts of 64 tokens routed top-2."""
    E, M, K, T, k = 8, 256, 512, 64, 2
    pk = O.pack_weights(weights_np(1, 0, E, M, K))
    counts = O.route(S.uniform_logits_np(1, T, E), k).counts
    ok, info = _run_isolated(cuda_lib, pk, counts, K, 2, tile_n)
    assert ok, info[:2]


@pytest.mark.parametrize("tile_n,mode", [(64, 1), (128, 1), (128, 2)])
@pytest.mark.parametrize("counts", [
    [0, 1, 0, 5, 0, 0, 0, 2],              # empty experts, single rows
    [129, 0, 31, 33, 1, 16, 17, 300],      # ragged: several token blocks, partial last blocks
    [0, 0, 0, 0, 0, 0, 0, 512],            # all rows on one expert
    [128, 256, 32, 64, 96, 160, 192, 224], # exact multiples of the token block
])
def test_gemm_edge_counts(cuda_lib, tile_n, mode, counts):
    E, M, K = 8, 256, 512
    pk = O.pack_weights(weights_np(3, 0, E, M, K))
    ok, info = _run_isolated(cuda_lib, pk, np.array(counts, np.int64), K, 4, tile_n, mode=mode)
    assert ok, info[:2]


@pytest.mark.parametrize("tile_n,mode", [(0, 0), (64, 1), (128, 1), (128, 2)])
def test_gemm_multi_k_tiles_and_m_blocks(cuda_lib, tile_n, mode):
    """K = 7168 (28 K steps: every ring wraps several times), M = 1536."""
    E, M, K = 3, 1536, 7168
    pk = O.pack_weights(weights_np(5, 0, E, M, K))
    ok, info = _run_isolated(cuda_lib, pk, np.array([7, 0, 200]), K, 6, tile_n, mode=mode)
    assert ok, info[:2]


@pytest.mark.parametrize("K", [256, 768])
@pytest.mark.parametrize("tile_n,mode", [(64, 1), (128, 1), (128, 2)])
def test_gemm_odd_k_steps(cuda_lib, K, tile_n, mode):
    """K = 256 and 768: one and three 256-wide K steps, fewer than a ring
    holds, and a count that does not divide it."""
    E, M = 4, 256
    pk = O.pack_weights(weights_np(15, 0, E, M, K))
    ok, info = _run_isolated(cuda_lib, pk, np.array([33, 0, 130, 64]), K, 16, tile_n, mode=mode)
    assert ok, info[:2]


def test_gemm_saturating_activation_scale(cuda_lib):
    """gamma_a too large: scales clip at 448 and codes at 6; still exact math."""
    E, M, K = 2, 128, 256
    pk = O.pack_weights(weights_np(7, 0, E, M, K))
    ok, info = _run_isolated(cuda_lib, pk, np.array([20, 3]), K, 8, 64, ga_scale=64.0)
    assert ok, info[:2]


def test_gemm_full_path_30b_class(cuda_lib):
    """30B-class gate_up (E=128, top-8, K=2048, M=1536, T=256): CUDA pack,
    route, dispatch-quantise and GEMM, checked on the rows of 6 experts."""
    torch = pytest.importorskip("torch")
    m = cuda_lib
    E, M, K, T, k = 128, 1536, 2048, 256, 8
    pw = pack_gpu_generated(m, 11, 0, E, M, K)
    x = S.activations_bf16_np(11, T, K)
    lg = S.uniform_logits_np(11, T, E)
    rt = O.route(lg, k)
    ga = np.full(E, O.act_global_scale(x), np.float32)
    rb = m.RoutingBuffers(T, E, k)
    m.moesq_route_permute(to_dev(lg), rb)
    codes, scales = m.act_buffers(rb.rows_cap, K)
    m.moesq_quantize_act(to_dev(x), T, K, rb, to_dev(ga), rb.rows_cap, codes, scales)
    y = torch.full((rb.rows_cap, M), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.moesq_grouped_sparse_gemm(pw, codes, scales, rb.rows_cap, rb.counts, rb.row_offsets, to_dev(ga), y)
    assert m.moesq_get_device_error()[0] == 0
    yg_all = to_np(y)
    ro = L.aligned_rows(rt.counts)
    for e in (0, 17, 64, 101, 126, 127):
        n = int(rt.counts[e])
        if n == 0:
            continue
        pk = O.pack_weights(S.expert_weights_bf16_np(11, 0, e, M, K)[None])
        s0 = rt.offsets[e]
        toks = rt.sorted_to_slot[s0:s0 + n] // k
        c, s = O.quantize_rows_bf16(x[toks], ga[e])
        y_ref, basis = O.grouped_gemm(pk, c, s, np.array([0, n], np.int32), ga[e:e + 1])
        ok, err, bound, bad = gemm_tolerance_ok(yg_all[ro[e]:ro[e] + n], y_ref, basis)
        assert ok, (e, err.max())


@pytest.fixture(scope="module")
def kimi_gate_up(cuda_lib):
    """Kimi-shaped gate_up weights (E=384, M=4096, K=7168), drawn and packed on
    the GPU once for the decode tests of this module."""
    return pack_gpu_generated(cuda_lib, 21, 0, 384, 4096, 7168, chunk=4)


@pytest.mark.parametrize("T", [1, 16, 64, 256])
def test_gemm_kimi_decode_full_size_sampled(cuda_lib, kimi_gate_up, T):
    """Kimi-shaped gate_up at full size (E=384, K=7168, M=4096), the decode
    token counts: CUDA route, dispatch-quantise and GEMM; every output of four
    sampled experts (the heaviest, the lightest and two others) against the
    oracle, and their packed values bit for bit."""
    torch = pytest.importorskip("torch")
    m = cuda_lib
    E, M, K, k = 384, 4096, 7168, 8
    pw = kimi_gate_up
    x = S.activations_bf16_np(21 + T, T, K)
    lg = S.uniform_logits_np(21 + T, T, E)
    rt = O.route(lg, k)
    ga = np.full(E, O.act_global_scale(x), np.float32)
    rb = m.RoutingBuffers(T, E, k)
    m.moesq_route_permute(to_dev(lg), rb)
    codes, scales = m.act_buffers(rb.rows_cap, K)
    m.moesq_quantize_act(to_dev(x), T, K, rb, to_dev(ga), rb.rows_cap, codes, scales)
    y = torch.full((rb.rows_cap, M), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.moesq_grouped_sparse_gemm(pw, codes, scales, rb.rows_cap, rb.counts, rb.row_offsets, to_dev(ga), y)
    assert m.moesq_get_device_error()[0] == 0
    yg_all = to_np(y)
    ro = L.aligned_rows(rt.counts)
    used = np.nonzero(rt.counts)[0]
    rng = np.random.default_rng(T)
    pick = {int(used[np.argmax(rt.counts[used])]), int(used[np.argmin(rt.counts[used])])}
    pick.update(int(e) for e in rng.choice(used, size=min(2, used.size), replace=False))
    for e in sorted(pick):
        n = int(rt.counts[e])
        pk = O.pack_weights(expert_weights_host(21, 0, e, M, K)[None])
        assert (to_np(pw.values[e]) == pk.values[0]).all()
        s0 = rt.offsets[e]
        toks = rt.sorted_to_slot[s0:s0 + n] // k
        c, s = O.quantize_rows_bf16(x[toks], ga[e])
        y_ref, basis = O.grouped_gemm(pk, c, s, np.array([0, n], np.int32), ga[e:e + 1])
        ok, err, bound, bad = gemm_tolerance_ok(yg_all[ro[e]:ro[e] + n], y_ref, basis)
        assert ok, (T, e, n, err.max())


def test_gemm_rejects_inconsistent_counts(cuda_lib):
    """Counts that do not fit the aligned row offsets are refused on the
    device (error word), nothing is written, and the context stays usable."""
    torch = pytest.importorskip("torch")
    m = cuda_lib
    E, M, K = 2, 128, 256
    pk = O.pack_weights(weights_np(9, 0, E, M, K))
    pw = packed_from_oracle(m, pk)
    codes, scales = m.act_buffers(256, K)
    codes.zero_()
    scales.zero_()
    y = torch.zeros((256, M), dtype=torch.bfloat16, device="cuda")
    bad_counts = to_dev(np.array([200, 5], np.int32))          # 200 rows need 256 aligned rows
    m.moesq_grouped_sparse_gemm(pw, codes, scales, 256, bad_counts, to_dev(np.array([0, 128, 256], np.int32)),
                                to_dev(np.ones(E, np.float32)), y)
    st, word = m.moesq_get_device_error()
    assert st == 5 and (word & 0xFF) == 5
    assert float(y.float().abs().max()) == 0.0
    ok, info = _run_isolated(m, pk, np.array([3, 4]), K, 10, 0)
    assert ok


@pytest.mark.parametrize("tile_n", [64, 128])
def test_gemm_fixed_capacity_layout(cuda_lib, tile_n):
    """The paper's batched layout (App. D.1): expert e's rows start at e * N
    for a fixed capacity N; the GEMM reads and writes those rows only."""
    torch = pytest.importorskip("torch")
    m = cuda_lib
    E, M, K, cap = 5, 256, 512, 256
    counts = np.array([3, 0, 130, 64, 1])
    pk = O.pack_weights(weights_np(17, 0, E, M, K))
    R = int(counts.sum())
    x = S.activations_bf16_np(18, R, K)
    ga = np.full(E, np.float32(O.act_global_scale(x)), np.float32)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    codes, scales = O.quantize_rows_bf16(x, ga[0])
    y_ref, basis = O.grouped_gemm(pk, codes, scales, offs, ga)
    rows = np.concatenate([e * cap + np.arange(counts[e]) for e in range(E)]).astype(np.int64)
    rc = E * cap
    c_rows = np.zeros((rc, K // 2), np.uint8)
    s_rows = np.zeros((rc, K // 32), np.uint8)
    c_rows[rows], s_rows[rows] = codes, scales
    y = torch.full((rc, M), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.moesq_grouped_sparse_gemm(packed_from_oracle(m, pk), to_dev(c_rows), to_dev(L.scales_to_mma(s_rows)), rc,
                                to_dev(counts.astype(np.int32)), to_dev((np.arange(E + 1) * cap).astype(np.int32)),
                                to_dev(ga), y, tile_n=tile_n)
    st, word = m.moesq_get_device_error()
    assert st == 0, "device error word %#x" % word
    yn = to_np(y)
    ok, err, bound, bad = gemm_tolerance_ok(yn[rows], y_ref, basis)
    assert ok, err.max()
    untouched = np.setdiff1d(np.arange(rc), rows)
    assert np.isnan(S.bf16_bits_to_f32_np(yn[untouched])).all()       # gaps are not written


def test_gemm_autotune_picks_a_candidate_and_stays_correct(cuda_lib):
    """moesq_gemm_autotune returns one of its candidate configurations with a
    positive time, and the GEMM under that configuration matches the oracle."""
    torch = pytest.importorskip("torch")
    m = cuda_lib
    E, M, K = 6, 256, 512
    counts = np.array([5, 70, 0, 130, 1, 17])
    pk = O.pack_weights(weights_np(23, 0, E, M, K))
    R = int(counts.sum())
    x = S.activations_bf16_np(24, R, K)
    ga = np.full(E, np.float32(O.act_global_scale(x)), np.float32)
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    codes, scales = O.quantize_rows_bf16(x, ga[0])
    y_ref, basis = O.grouped_gemm(pk, codes, scales, offs, ga)
    c_rows, s_mma, rc = act_rows_from_compact(codes, scales, counts, K)
    pw = packed_from_oracle(m, pk)
    args = (to_dev(c_rows), to_dev(s_mma), rc, to_dev(counts.astype(np.int32)), to_dev(L.aligned_rows(counts)),
            to_dev(ga))
    y = torch.zeros((rc, M), dtype=torch.bfloat16, device="cuda")
    (tile_n, num_ctas, mode), ms = m.moesq_gemm_autotune(pw, *args, y, reps=2)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert tile_n in (64, 128) and num_ctas in (sms, 2 * sms) and mode in (1, 2) and ms > 0
    y.fill_(float("nan"))
    m.moesq_grouped_sparse_gemm(pw, *args, y, tile_n=tile_n, num_ctas=num_ctas, sm_mode=mode)
    assert m.moesq_get_device_error()[0] == 0
    ok, err, bound, bad = gemm_tolerance_ok(to_np(y)[L.compact_to_rows(counts)], y_ref, basis)
    assert ok, err.max()


def _prefill_rows(n):
    """Row indices checked in an expert with n rows: the first 32, 32 that
    straddle a 128-row token-tile boundary, and the last tile's rows."""
    idx = set(range(min(n, 32)))
    if n > 160:
        idx.update(range(112, 144))
    last = (n - 1) // 128 * 128
    idx.update(range(last, n))
    return np.array(sorted(idx), np.int64)


def test_gemm_kimi_prefill_down_full_size_sampled(cuda_lib):
    """Kimi-shaped down projection at full size (E=384, M=7168, K=2048),
    T=8192 with Zipf(1.1) routing, as the prefill bench runs it: sampled rows
    of the heaviest expert (several token tiles, a partial last tile) and all
    rows of the lightest, against the oracle."""
    torch = pytest.importorskip("torch")
    m = cuda_lib
    E, M, K, T, k = 384, 7168, 2048, 8192, 8
    pw = pack_gpu_generated(m, 31, 1, E, M, K, chunk=8)
    x = S.activations_bf16_np(31, T, K)
    lg = S.zipf_logits_np(1234, T, E)
    rt = O.route(lg, k)
    ga = np.full(E, O.act_global_scale(x), np.float32)
    rb = m.RoutingBuffers(T, E, k)
    m.moesq_route_permute(to_dev(lg), rb)
    assert (to_np(rb.counts) == rt.counts).all()
    codes, scales = m.act_buffers(rb.rows_cap, K)
    m.moesq_quantize_act(to_dev(x), T, K, rb, to_dev(ga), rb.rows_cap, codes, scales)
    y = torch.full((rb.rows_cap, M), float("nan"), dtype=torch.bfloat16, device="cuda")
    m.moesq_grouped_sparse_gemm(pw, codes, scales, rb.rows_cap, rb.counts, rb.row_offsets, to_dev(ga), y)
    assert m.moesq_get_device_error()[0] == 0
    yg_all = to_np(y)
    ro = L.aligned_rows(rt.counts)
    used = np.nonzero(rt.counts)[0]
    heavy, light = int(np.argmax(rt.counts)), int(used[np.argmin(rt.counts[used])])
    for e in (heavy, light):
        n = int(rt.counts[e])
        idx = _prefill_rows(n) if e == heavy else np.arange(n)
        pk = O.pack_weights(expert_weights_host(31, 1, e, M, K)[None])
        s0 = rt.offsets[e]
        toks = rt.sorted_to_slot[s0:s0 + n][idx] // k
        c, s = O.quantize_rows_bf16(x[toks], ga[e])
        y_ref, basis = O.grouped_gemm(pk, c, s, np.array([0, idx.size], np.int32), ga[e:e + 1])
        ok, err, bound, bad = gemm_tolerance_ok(yg_all[ro[e] + idx], y_ref, basis)
        assert ok, (e, n, err.max())
