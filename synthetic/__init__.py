"""Seeded synthetic inputs for the paired-4:8 NVFP4 MoE hot path.

This module holds no step of the method: it only draws numbers. Both the
oracle-side tests and the CUDA-side harness take their inputs from here, so a
tensor drawn on the host (numpy) and the same tensor drawn on a GPU (torch)
are bit-identical.

Generator
---------
* Counter-based SplitMix64 (Steele, Lea and Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): output ``i`` of a stream with
  key ``k`` is ``mix64(k + (i + 1) * 0x9E3779B97F4A7C15)`` with the published
  finaliser ``mix64``.  Every element is a pure function of (key, index).
* Normal deviates by the Irwin-Hall construction: the sum of 12 uniforms on
  [0, 1) minus 6 has mean 0 and variance 1.  Each 64-bit output supplies two
  24-bit uniforms, so one deviate takes 6 outputs.  The 12 uniforms are summed
  as integers, so the deviate is exact in float64 on every backend; it is then
  scaled in float64, rounded to float32 (IEEE round-to-nearest-even) and, for
  bf16 tensors, to bf16 with round-to-nearest-even on the bit pattern.
* Router logits with a Zipf(s) expert popularity use Gumbel-top-k:
  ``logit[t, e] = log p[pi(e)] + G[t, e]``, ``p[r] ~ r^-s``, ``G ~ Gumbel(0,1)``,
  ``pi`` a seeded permutation.  These are drawn on the host only.

Workload shapes (sizes, distributions) are documented where they are used.
"""
from __future__ import annotations

import numpy as np

GOLDEN = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
M64 = (1 << 64) - 1


def _mix64_int(z: int) -> int:
    z &= M64
    z = ((z ^ (z >> 30)) * MIX1) & M64
    z = ((z ^ (z >> 27)) * MIX2) & M64
    return z ^ (z >> 31)


def stream_key(seed: int, *labels: int) -> int:
    """Key of the stream named by (seed, labels...); a chain of mix64 calls."""
    k = _mix64_int(seed * GOLDEN + 0x1234567)
    for lab in labels:
        k = _mix64_int(k ^ ((lab + 1) * GOLDEN))
    return k


# ---------------------------------------------------------------- numpy side
def _mix64_np(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX2)
    return z ^ (z >> np.uint64(31))


def raw_u64_np(key: int, start: int, count: int) -> np.ndarray:
    """Outputs start..start+count-1 of stream `key` as uint64."""
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(key) + idx * np.uint64(GOLDEN)
        return _mix64_np(z)


def _irwin_hall_sum_np(key: int, start: int, count: int) -> np.ndarray:
    """Integer sum of 12 24-bit uniforms for deviates start..start+count-1."""
    s = np.zeros(count, dtype=np.int64)
    with np.errstate(over="ignore"):
        base = (np.arange(start, start + count, dtype=np.uint64) * np.uint64(6))
        for j in range(6):
            z = np.uint64(key) + (base + np.uint64(j + 1)) * np.uint64(GOLDEN)
            u = _mix64_np(z)
            s += (u >> np.uint64(40)).astype(np.int64)
            s += ((u >> np.uint64(16)) & np.uint64(0xFFFFFF)).astype(np.int64)
    return s


def normal_f64_np(key: int, start: int, count: int) -> np.ndarray:
    """Standard normal deviates (Irwin-Hall, 12 uniforms), exact in float64."""
    s = _irwin_hall_sum_np(key, start, count)
    return (s - 6 * (1 << 24)).astype(np.float64) * (2.0 ** -24)


def f32_to_bf16_bits_np(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit pattern (uint16), round to nearest even."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounding = ((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    return ((u + rounding) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32_np(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16_np(key: int, shape, sigma: float, start: int = 0) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(0, sigma^2) deviates, C order."""
    n = int(np.prod(shape))
    v = normal_f64_np(key, start, n) * sigma
    return f32_to_bf16_bits_np(v.astype(np.float32)).reshape(shape)


def outlier_channels(key: int, K: int, count: int = 4) -> np.ndarray:
    """`count` distinct channel indices in [0, K) drawn from stream `key`."""
    chans = []
    i = 0
    while len(chans) < count:
        c = int(raw_u64_np(key, i, 1)[0] % np.uint64(K))
        if c not in chans:
            chans.append(c)
        i += 1
    return np.array(sorted(chans), dtype=np.int64)


def activations_bf16_np(seed: int, T: int, K: int, n_outliers: int = 4,
                        outlier_gain: float = 20.0, label: int = 0, rows: int = None) -> np.ndarray:
    """Hidden states X [T, K] ~ N(0, 1) with `n_outliers` channels scaled by
    `outlier_gain`, as bf16 bit patterns.  rows < T draws only the first
    `rows` rows (the same values as the first rows of the full batch)."""
    key = stream_key(seed, 1, label)
    n = T if rows is None else min(rows, T)
    v = normal_f64_np(key, 0, n * K).reshape(n, K)
    if n_outliers:
        ch = outlier_channels(stream_key(seed, 2, label), K, n_outliers)
        v[:, ch] *= outlier_gain
    return f32_to_bf16_bits_np(v.astype(np.float32))


def expert_weight_key(seed: int, linear: int, e: int) -> int:
    """Stream key of expert `e`'s weight for linear `linear` (0 gate_up, 1 down)."""
    return stream_key(seed, 10 + linear, e)


def expert_weights_bf16_np(seed: int, linear: int, e: int, M: int, K: int,
                           sigma: float = 0.02) -> np.ndarray:
    """Expert weight W_e [M, K] ~ N(0, sigma^2) as bf16 bit patterns."""
    return normal_bf16_np(expert_weight_key(seed, linear, e), (M, K), sigma)


def uniform_logits_np(seed: int, T: int, E: int, label: int = 0) -> np.ndarray:
    """Router logits [T, E] ~ N(0, 1), float32 (near-balanced expert loads)."""
    return normal_f64_np(stream_key(seed, 3, label), 0, T * E).reshape(T, E).astype(np.float32)


def zipf_logits_np(seed: int, T: int, E: int, s: float = 1.1, label: int = 0) -> np.ndarray:
    """Router logits [T, E] whose top-k follows a Zipf(s) expert popularity
    (Gumbel-top-k sampling without replacement), float32."""
    perm_key = stream_key(seed, 4, label)
    order = np.argsort(raw_u64_np(perm_key, 0, E), kind="stable")  # pi: rank -> expert
    rank_of = np.empty(E, dtype=np.int64)
    rank_of[order] = np.arange(E)
    logp = -s * np.log(rank_of.astype(np.float64) + 1.0)
    u = (raw_u64_np(stream_key(seed, 5, label), 0, T * E) >> np.uint64(11)).astype(np.float64)
    u = (u + 0.5) * (2.0 ** -53)                       # open interval (0, 1)
    g = -np.log(-np.log(u))
    return (logp[None, :] + g.reshape(T, E)).astype(np.float32)


# ---------------------------------------------------------------- torch side
def _torch_consts():
    import torch

    def s64(v):  # reinterpret an unsigned 64-bit constant as int64
        return v - (1 << 64) if v >= (1 << 63) else v
    return torch, s64(GOLDEN), s64(MIX1), s64(MIX2)


def _srl(torch, x, s):
    """Logical right shift of an int64 tensor."""
    return (x >> s) & ((1 << (64 - s)) - 1)


def _mix64_torch(torch, z, m1, m2):
    z = (z ^ _srl(torch, z, 30)) * m1
    z = (z ^ _srl(torch, z, 27)) * m2
    return z ^ _srl(torch, z, 31)


def normal_bf16_torch(key: int, shape, sigma: float, device, start: int = 0):
    """Same bits as `normal_bf16_np`, drawn on `device` with torch (uint16 view
    returned as torch.int16 holding the bf16 bit pattern)."""
    torch, g, m1, m2 = _torch_consts()
    n = 1
    for d in shape:
        n *= int(d)
    skey = key - (1 << 64) if key >= (1 << 63) else key
    idx = torch.arange(start, start + n, dtype=torch.int64, device=device) * 6
    s = torch.zeros(n, dtype=torch.int64, device=device)
    for j in range(6):
        z = (idx + (j + 1)) * g + skey
        u = _mix64_torch(torch, z, m1, m2)
        s += _srl(torch, u, 40)
        s += _srl(torch, u, 16) & 0xFFFFFF
        del z, u
    v = (s - 6 * (1 << 24)).to(torch.float64) * (2.0 ** -24) * sigma
    del s
    f = v.to(torch.float32)
    del v
    u32 = f.view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    rounding = ((u32 >> 16) & 1) + 0x7FFF
    bits = ((u32 + rounding) >> 16) & 0xFFFF
    out = bits.to(torch.int32)
    out = torch.where(out >= 32768, out - 65536, out).to(torch.int16)
    return out.view(torch.bfloat16).reshape(*shape)


def expert_weights_bf16_torch(seed: int, linear: int, e: int, M: int, K: int, device,
                              sigma: float = 0.02):
    return normal_bf16_torch(expert_weight_key(seed, linear, e), (M, K), sigma, device)



def _normal_f64_torch(key: int, start: int, count: int, device):
    """Same values as `normal_f64_np`, as a torch float64 tensor on `device`."""
    torch, g, m1, m2 = _torch_consts()
    skey = key - (1 << 64) if key >= (1 << 63) else key
    idx = torch.arange(start, start + count, dtype=torch.int64, device=device) * 6
    s = torch.zeros(count, dtype=torch.int64, device=device)
    for j in range(6):
        z = (idx + (j + 1)) * g + skey
        u = _mix64_torch(torch, z, m1, m2)
        s += _srl(torch, u, 40)
        s += _srl(torch, u, 16) & 0xFFFFFF
        del z, u
    del idx
    return (s - 6 * (1 << 24)).to(torch.float64) * (2.0 ** -24)


def _f32_to_bf16_torch(f):
    """float32 tensor -> bf16 tensor with round-to-nearest-even on the bit
    pattern (the same bits as `f32_to_bf16_bits_np`)."""
    import torch
    u32 = f.contiguous().view(torch.int32).to(torch.int64) & 0xFFFFFFFF
    bits = ((u32 + ((u32 >> 16) & 1) + 0x7FFF) >> 16) & 0xFFFF
    out = bits.to(torch.int32)
    out = torch.where(out >= 32768, out - 65536, out).to(torch.int16)
    return out.view(torch.bfloat16)


def activations_bf16_torch(seed: int, T: int, K: int, device, n_outliers: int = 4,
                           outlier_gain: float = 20.0, label: int = 0, chunk_rows: int = 2048):
    """Same bits as `activations_bf16_np`, drawn on `device` (a bf16 tensor
    [T, K]), `chunk_rows` rows at a time."""
    import torch
    key = stream_key(seed, 1, label)
    ch = outlier_channels(stream_key(seed, 2, label), K, n_outliers) if n_outliers else None
    out = torch.empty((T, K), dtype=torch.bfloat16, device=device)
    for r0 in range(0, T, chunk_rows):
        n = min(chunk_rows, T - r0)
        v = _normal_f64_torch(key, r0 * K, n * K, device).reshape(n, K)
        if ch is not None:
            idx = torch.as_tensor(ch, device=device)
            v[:, idx] *= outlier_gain
        out[r0:r0 + n] = _f32_to_bf16_torch(v.to(torch.float32))
        del v
    return out
