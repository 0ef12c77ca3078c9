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
