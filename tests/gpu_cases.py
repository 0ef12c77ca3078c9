"""Shared builders for the GPU parity tests: seeded inputs from `synthetic`,
oracle results from `oracle`, CUDA results through the C ABI binding."""
import numpy as np

import layouts as L
import oracle as O
import synthetic as S


def torch_mod():
    import torch
    return torch


def to_dev(a: np.ndarray):
    torch = torch_mod()
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16).copy()).cuda().view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def to_np(t, dtype=None):
    torch = torch_mod()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    a = t.cpu().numpy()
    return a.astype(dtype) if dtype is not None else a


def weights_np(seed, linear, E, M, K, experts=None):
    experts = range(E) if experts is None else experts
    return np.stack([S.expert_weights_bf16_np(seed, linear, e, M, K) for e in experts])


def pack_gpu_from_np(m, w_np):
    """Upload bf16 weights [E, M, K] and pack them with the CUDA library."""
    E, M, K = w_np.shape
    pw = m.PackedWeights(E, M, K)
    m.moesq_pack_weights(to_dev(w_np), 0, E, pw)
    return pw


def pack_gpu_generated(m, seed, linear, E, M, K, chunk=8):
    """Draw the weights on the GPU (same bits as weights_np) and pack them,
    `chunk` experts at a time."""
    torch = torch_mod()
    pw = m.PackedWeights(E, M, K)
    for e0 in range(0, E, chunk):
        n = min(chunk, E - e0)
        w = torch.stack([S.expert_weights_bf16_torch(seed, linear, e, M, K, "cuda") for e in range(e0, e0 + n)])
        m.moesq_pack_weights(w, e0, n, pw)
        del w
    torch.cuda.synchronize()
    return pw


def packed_from_oracle(m, pk):
    """CUDA-side weights built on the host from the oracle's storage form
    (kernel form derived with the layout definitions): isolates the GEMM."""
    torch = torch_mod()
    E, M, K4 = pk.values.shape
    K = K4 * 4
    pw = m.PackedWeights(E, M, K)
    pw.values.copy_(torch.from_numpy(pk.values))
    pw.mask.copy_(torch.from_numpy(pk.mask))
    pw.scales.copy_(torch.from_numpy(pk.scales))
    pw.global_scale.copy_(torch.from_numpy(pk.gamma))
    pw.ktiles.copy_(torch.from_numpy(L.storage_to_ktiles(pk.values, pk.mask, pk.scales)))
    torch.cuda.synchronize()
    return pw


def act_rows_from_compact(codes, scales, counts, K):
    """Oracle compact activation rows -> aligned-row-space codes / MMA-layout scales."""
    rows = L.compact_to_rows(counts)
    rc = max(128, int(L.aligned_rows(counts)[-1]))
    c = np.zeros((rc, K // 2), np.uint8)
    s = np.zeros((rc, K // 32), np.uint8)
    c[rows] = codes
    s[rows] = scales
    return c, L.scales_to_mma(s), rc


def gemm_tolerance_ok(y_gpu_bits, y_ref_bits, basis):
    """|y_gpu - y_ref| <= 1e-3 * sum|a w| + one bf16 spacing of y_ref."""
    g = S.bf16_bits_to_f32_np(y_gpu_bits).astype(np.float64)
    r = S.bf16_bits_to_f32_np(y_ref_bits).astype(np.float64)
    err = np.abs(g - r)
    bound = 1e-3 * basis + L.bf16_ulp(r) + 1e-30
    bad = err > bound
    return (not bad.any()), err, bound, bad


def expert_weights_host(seed, linear, e, M, K):
    """One expert's bf16 weight bits on the host, drawn by the seeded
    generator's torch path on the GPU (same bits as the numpy path, which
    takes seconds per Kimi-sized expert on the host)."""
    torch = torch_mod()
    w = S.expert_weights_bf16_torch(seed, linear, int(e), M, K, "cuda")
    return w.view(torch.int16).cpu().numpy().view(np.uint16)


def oracle_pack_experts(seed, linear, E, M, K, experts):
    """Oracle storage form of an E-expert stack in which only `experts` hold
    their seeded weights (the other experts' tensors stay zero and unread):
    the oracle side of a token sample at full size."""
    import oracle as O
    experts = [int(e) for e in experts]
    pk = O.pack_weights(np.stack([expert_weights_host(seed, linear, e, M, K) for e in experts]))
    full = O.Packed(np.zeros((E, M, K // 4), np.uint8), np.zeros((E, M, K // 16), np.uint8),
                    np.zeros((E, M, K // 32), np.uint8), np.ones(E, np.float32))
    full.values[experts], full.mask[experts], full.scales[experts], full.gamma[experts] = \
        pk.values, pk.mask, pk.scales, pk.gamma
    return full


# ---------------------------------------------------------------- requantisation check with a decision band
E2M1_DECISION_POINTS = (0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0)   # midpoints of the App. A, Fig. 3 grid

# Relative band around a decision point inside which a binary32 SiLU with
# the hardware exponential and divide (a few tens of ulp for |g| <= 16, below
# 2^-18 relative) may put h on the other side of the oracle's binary64 h;
# 2^-16 leaves a factor of 4 over that.
SWIGLU_BAND = 2.0 ** -16


def _ue4m3_decisions():
    """Midpoints between consecutive UE4M3 values (codes 0..126): the points
    where Eq. 5's scale code changes."""
    import oracle as O
    v = np.array([O.ue4m3_value(c) for c in range(127)], np.float64)
    return (v[:-1] + v[1:]) / 2


def _near(x, points, band):
    """|x - p| <= band * p for the decision point p nearest x (x >= 0)."""
    pts = np.asarray(points, np.float64)
    i = np.clip(np.searchsorted(pts, x), 1, pts.size - 1)
    d = np.minimum(np.abs(x - pts[i - 1]) / pts[i - 1], np.abs(x - pts[i]) / pts[i])
    return d <= band


def requant_mismatches(h, gamma_rows, os_, oc, gs, gc, band=SWIGLU_BAND):
    """Compares a requantisation (gs scale codes [R, I/32], gc code bytes
    [R, I/2]) with the oracle's (os_, oc) of h (binary32 [R, I]) under the
    per-row global scales gamma_rows [R].  A scale code may differ only where
    gamma * amax_b / 6 lies within `band` of a UE4M3 decision point (a
    changed scale then frees its whole block); under an equal scale a value
    code may differ only where |h| / s_b lies within `band` of an E2M1
    decision point.  Returns (bad_scale [R, I/32], bad_code [R, I/32, 32],
    scale_diff, code_diff)."""
    import oracle as O
    R, I = h.shape
    hb = h.astype(np.float64).reshape(R, I // 32, 32)
    g = np.asarray(gamma_rows, np.float32)
    x_s = g.astype(np.float64)[:, None] * np.abs(hb).max(-1) / 6.0
    scale_diff = gs != os_
    bad_scale = scale_diff & ~_near(x_s, _ue4m3_decisions(), band)
    sv = np.vectorize(O.ue4m3_value)(os_).astype(np.float32)
    s_b = (sv / g[:, None]).astype(np.float64)
    q = np.abs(hb) / np.where(s_b > 0, s_b, np.inf)[..., None]
    code_free = _near(q, E2M1_DECISION_POINTS, band)
    nib = lambda c: np.stack([c & 15, c >> 4], -1).reshape(R, I // 32, 32)   # noqa: E731
    code_diff = nib(gc) != nib(oc)
    bad_code = code_diff & ~code_free & ~scale_diff[..., None]
    return bad_scale, bad_code, scale_diff, code_diff
