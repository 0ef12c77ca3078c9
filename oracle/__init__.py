"""CPU oracle for the paired-4:8 NVFP4 MoE expert path.

TEST INFRASTRUCTURE ONLY.  The tests, ``__graft_entry__.smoke()`` and the CPU
baseline of ``bench.py`` may import this package; the library and its Python
binding never do.

The arithmetic lives in plain C (``moesq_oracle.c``, built with gcc into
``liboracle.so`` next to it); this module marshals numpy arrays, composes
the C steps into the MoE layer in the order the paper gives (arXiv
2610.02241, Sec. 3.4 and App. D.1), and holds the two byte-layout converters
between dense NVFP4 codes and the pair-bitmask form (integer rearrangement
only, in numpy).  Every C function cites its passage.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moesq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_u8 = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_u16 = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_i32 = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_f32 = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64 = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_c = ctypes


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (no fused multiply-add, IEEE binary32)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-fexcess-precision=standard", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        L.oracle_e2m1_value.restype = _c.c_double
        L.oracle_e2m1_value.argtypes = [_c.c_int]
        L.oracle_e2m1_encode.restype = _c.c_int
        L.oracle_e2m1_encode.argtypes = [_c.c_float]
        L.oracle_ue4m3_value.restype = _c.c_double
        L.oracle_ue4m3_value.argtypes = [_c.c_int]
        L.oracle_ue4m3_encode.restype = _c.c_int
        L.oracle_ue4m3_encode.argtypes = [_c.c_float]
        L.oracle_bf16_round.restype = _c.c_uint16
        L.oracle_bf16_round.argtypes = [_c.c_double]
        L.oracle_global_scale.restype = _c.c_float
        L.oracle_global_scale.argtypes = [_c.c_float]
        L.oracle_pack_weights.restype = None
        L.oracle_pack_weights.argtypes = [_u16, _c.c_int, _c.c_int, _u8, _u8, _u8, _f32]
        L.oracle_unpack_weights.restype = None
        L.oracle_unpack_weights.argtypes = [_u8, _u8, _u8, _c.c_float, _c.c_int, _c.c_int, _f64]
        L.oracle_quantize_rows.restype = None
        L.oracle_quantize_rows.argtypes = [_f32, _c.c_int, _c.c_int, _c.c_float, _u8, _u8]
        L.oracle_quantize_rows_bf16.restype = None
        L.oracle_quantize_rows_bf16.argtypes = [_u16, _c.c_int, _c.c_int, _c.c_float, _u8, _u8]
        L.oracle_act_global_scale.restype = _c.c_float
        L.oracle_act_global_scale.argtypes = [_u16, _c.c_longlong]
        L.oracle_route.restype = None
        L.oracle_route.argtypes = [_f32, _c.c_int, _c.c_int, _c.c_int, _i32, _f32, _i32, _i32, _i32]
        L.oracle_grouped_gemm.restype = None
        L.oracle_grouped_gemm.argtypes = [_u8, _u8, _u8, _f32, _c.c_int, _c.c_int, _c.c_int,
                                          _u8, _u8, _i32, _f32, _u16, _c.c_void_p, _c.c_void_p]
        L.oracle_pack_dense_nvfp4.restype = None
        L.oracle_pack_dense_nvfp4.argtypes = [_u16, _c.c_int, _c.c_int, _u8, _u8, _f32]
        L.oracle_dense_grouped_gemm.restype = None
        L.oracle_dense_grouped_gemm.argtypes = [_u8, _u8, _f32, _c.c_int, _c.c_int, _c.c_int,
                                                _u8, _u8, _i32, _f32, _u16, _c.c_void_p, _c.c_void_p]
        L.oracle_swiglu.restype = None
        L.oracle_swiglu.argtypes = [_u16, _c.c_int, _c.c_int, _f32]
        L.oracle_combine.restype = None
        L.oracle_combine.argtypes = [_u16, _c.c_int, _f32, _i32, _c.c_int, _c.c_int, _u16]
        _lib = L
    return _lib


# ---------------------------------------------------------------- codecs
def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e2m1_encode(x: float) -> int:
    return lib().oracle_e2m1_encode(float(x))


def ue4m3_value(code: int) -> float:
    return lib().oracle_ue4m3_value(int(code))


def ue4m3_encode(x: float) -> int:
    return lib().oracle_ue4m3_encode(float(x))


def global_scale(amax: float) -> float:
    """Eq. 5's tensor multiplier gamma = 448 / (amax / 6) (binary32)."""
    return lib().oracle_global_scale(float(amax))


def bf16_round(v: float) -> int:
    return lib().oracle_bf16_round(float(v))


# ---------------------------------------------------------------- packing
class Packed:
    """Storage form of one expert stack (model card, pair-bitmask v1)."""

    def __init__(self, values, mask, scales, gamma):
        self.values = values      # uint8 [E, M, K/4]
        self.mask = mask          # uint8 [E, M, K/16]
        self.scales = scales      # uint8 [E, M, K/32] UE4M3 codes
        self.gamma = gamma        # float32 [E]

    @property
    def E(self):
        return self.values.shape[0]


def pack_weights(w_bf16: np.ndarray) -> Packed:
    """w_bf16: uint16 [E, M, K] bf16 bit patterns -> storage form."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    E, M, K = w.shape
    values = np.zeros((E, M, K // 4), np.uint8)
    mask = np.zeros((E, M, K // 16), np.uint8)
    scales = np.zeros((E, M, K // 32), np.uint8)
    gamma = np.zeros(E, np.float32)
    g1 = np.zeros(1, np.float32)
    for e in range(E):
        v = np.zeros((M, K // 4), np.uint8)
        m = np.zeros((M, K // 16), np.uint8)
        s = np.zeros((M, K // 32), np.uint8)
        lib().oracle_pack_weights(np.ascontiguousarray(w[e]), M, K, v, m, s, g1)
        values[e], mask[e], scales[e], gamma[e] = v, m, s, g1[0]
    return Packed(values, mask, scales, gamma)


def unpack_weights(values, mask, scales, gamma, M, K) -> np.ndarray:
    """Dequantised dense weight [M, K] of one expert (pruned entries zero)."""
    out = np.zeros((M, K), np.float64)
    lib().oracle_unpack_weights(np.ascontiguousarray(values), np.ascontiguousarray(mask),
                                np.ascontiguousarray(scales), float(gamma), M, K, out)
    return out


def dense_from_sparse(values: np.ndarray, mask: np.ndarray) -> np.ndarray:
    """Pair-bitmask storage -> dense NVFP4 codes (model card
    "Kimi-K2.5-P48NVFP4-MoESQ", pair-bitmask v1): values [..., K/4] hold the 2
    kept bytes of every 4-byte chunk in K order, mask [..., K/16] one nibble
    per chunk (bit i = byte i kept, low nibble = lower-K chunk).  The kept
    bytes go to the positions their nibble marks, zeros elsewhere."""
    v = np.ascontiguousarray(values, dtype=np.uint8)
    m = np.ascontiguousarray(mask, dtype=np.uint8)
    lead = v.shape[:-1]
    G = v.shape[-1] // 2                                   # 4-byte chunks per row
    nib = np.stack([m & 15, m >> 4], axis=-1).reshape(lead + (G,)).astype(np.int64)
    kept = v.reshape(lead + (G, 2))
    lowest = np.array([(n & -n).bit_length() - 1 if n else 0 for n in range(16)])
    highest = np.array([n.bit_length() - 1 if n else 1 for n in range(16)])
    dense = np.zeros(lead + (G, 4), np.uint8)
    np.put_along_axis(dense, lowest[nib][..., None], kept[..., 0:1], axis=-1)
    np.put_along_axis(dense, highest[nib][..., None], kept[..., 1:2], axis=-1)
    return dense.reshape(lead + (4 * G,))


def sparse_from_dense(dense: np.ndarray):
    """Dense NVFP4 codes [..., K/2] of a tensor in the paired pattern ->
    (values [..., K/4], mask [..., K/16]) by the model card's canonical rule:
    per 4-byte chunk the nonzero bytes are kept; with fewer than 2, its
    lowest-index zero bytes are kept too.  Chunks with more than 2 nonzero
    bytes are outside the pattern (ValueError)."""
    d = np.ascontiguousarray(dense, dtype=np.uint8)
    lead = d.shape[:-1]
    G = d.shape[-1] // 4
    ch = d.reshape(lead + (G, 4))
    nz = ch != 0
    cnt = nz.sum(-1)
    if (cnt > 2).any():
        raise ValueError("a 4-byte chunk has more than two nonzero bytes")
    zero_rank = np.cumsum(~nz, axis=-1) - 1                # order of each zero byte within its chunk
    keep = nz | (~nz & (zero_rank < (2 - cnt)[..., None]))
    pos = np.argsort(~keep, axis=-1, kind="stable")[..., :2]   # the two kept positions, ascending
    values = np.take_along_axis(ch, pos, axis=-1).reshape(lead + (2 * G,))
    nib = (keep * (1 << np.arange(4))).sum(-1).astype(np.uint8)   # [..., G]
    mask = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    return values, mask


# ---------------------------------------------------------------- activations
def quantize_rows(x: np.ndarray, gamma: float):
    """x: float32 [rows, K] -> (codes uint8 [rows, K/2], scales uint8 [rows, K/32])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    rows, K = x.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 32), np.uint8)
    lib().oracle_quantize_rows(x, rows, K, float(gamma), codes, scales)
    return codes, scales


def quantize_rows_bf16(x_bf16: np.ndarray, gamma: float):
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    rows, K = x.shape
    codes = np.zeros((rows, K // 2), np.uint8)
    scales = np.zeros((rows, K // 32), np.uint8)
    lib().oracle_quantize_rows_bf16(x, rows, K, float(gamma), codes, scales)
    return codes, scales


def act_global_scale(x_bf16: np.ndarray) -> float:
    """Eq. 5's gamma over a calibration batch (largest |x|)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16).ravel()
    return lib().oracle_act_global_scale(x, x.size)


# ---------------------------------------------------------------- routing
class Routing:
    def __init__(self, topk_ids, topk_w, counts, offsets, sorted_to_slot, k):
        self.topk_ids = topk_ids            # int32 [T, k]
        self.topk_w = topk_w                # float32 [T, k]
        self.counts = counts                # int32 [E]
        self.offsets = offsets              # int32 [E+1] compact
        self.sorted_to_slot = sorted_to_slot  # int32 [R]
        self.k = k
        R = sorted_to_slot.size
        self.slot_to_sorted = np.zeros(R, np.int32)
        self.slot_to_sorted[sorted_to_slot] = np.arange(R, dtype=np.int32)

    def expert_of_sorted(self):
        return np.repeat(np.arange(self.counts.size, dtype=np.int32), self.counts)


def route(logits: np.ndarray, k: int) -> Routing:
    lg = np.ascontiguousarray(logits, dtype=np.float32)
    T, E = lg.shape
    ids = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    counts = np.zeros(E, np.int32)
    offsets = np.zeros(E + 1, np.int32)
    s2s = np.zeros(T * k, np.int32)
    lib().oracle_route(lg, T, E, k, ids, w, counts, offsets, s2s)
    return Routing(ids, w, counts, offsets, s2s, k)


# ---------------------------------------------------------------- GEMM
def grouped_gemm(pk: Packed, a_codes, a_scales, offsets, gamma_a, want_exact=False):
    """Compact expert-sorted rows -> (y bf16 bits uint16 [R, M], abs-sum basis
    float64 [R, M][, exact float64 [R, M]])."""
    E, M, K4 = pk.values.shape
    K = K4 * 4
    R = a_codes.shape[0]
    y = np.zeros((R, M), np.uint16)
    basis = np.zeros((R, M), np.float64)
    exact = np.zeros((R, M), np.float64) if want_exact else None
    lib().oracle_grouped_gemm(pk.values, pk.mask, pk.scales, np.ascontiguousarray(pk.gamma, np.float32),
                              E, M, K, np.ascontiguousarray(a_codes), np.ascontiguousarray(a_scales),
                              np.ascontiguousarray(offsets, np.int32),
                              np.ascontiguousarray(gamma_a, np.float32), y,
                              exact.ctypes.data if want_exact else None, basis.ctypes.data)
    return (y, basis, exact) if want_exact else (y, basis)


class DensePacked:
    """Dense NVFP4 weights of E expert linears: codes [E, M, K/2] (two E2M1
    codes per byte, even K low), scales [E, M, K/16] UE4M3, gamma [E]."""

    def __init__(self, codes, scales, gamma):
        self.codes, self.scales, self.gamma = codes, scales, gamma


def pack_dense_nvfp4(w_bf16: np.ndarray) -> DensePacked:
    """The dense W4A4 control (no pruning, one scale per 16 K), per expert."""
    w = np.ascontiguousarray(w_bf16, dtype=np.uint16)
    E, M, K = w.shape
    codes = np.zeros((E, M, K // 2), np.uint8)
    scales = np.zeros((E, M, K // 16), np.uint8)
    gamma = np.zeros(E, np.float32)
    g1 = np.zeros(1, np.float32)
    for e in range(E):
        c = np.zeros((M, K // 2), np.uint8)
        sc = np.zeros((M, K // 16), np.uint8)
        lib().oracle_pack_dense_nvfp4(np.ascontiguousarray(w[e]), M, K, c, sc, g1)
        codes[e], scales[e], gamma[e] = c, sc, g1[0]
    return DensePacked(codes, scales, gamma)


def dense_grouped_gemm(dp: DensePacked, a_codes, a_scales, offsets, gamma_a, want_exact=False):
    """grouped_gemm for the dense control weights (same activations)."""
    E, M, K2 = dp.codes.shape
    K = K2 * 2
    R = a_codes.shape[0]
    y = np.zeros((R, M), np.uint16)
    basis = np.zeros((R, M), np.float64)
    exact = np.zeros((R, M), np.float64) if want_exact else None
    lib().oracle_dense_grouped_gemm(np.ascontiguousarray(dp.codes), np.ascontiguousarray(dp.scales),
                                    np.ascontiguousarray(dp.gamma, np.float32), E, M, K,
                                    np.ascontiguousarray(a_codes), np.ascontiguousarray(a_scales),
                                    np.ascontiguousarray(offsets, np.int32),
                                    np.ascontiguousarray(gamma_a, np.float32), y,
                                    exact.ctypes.data if want_exact else None, basis.ctypes.data)
    return (y, basis, exact) if want_exact else (y, basis)


def swiglu(y_gu_bf16: np.ndarray) -> np.ndarray:
    y = np.ascontiguousarray(y_gu_bf16, np.uint16)
    rows, I2 = y.shape
    h = np.zeros((rows, I2 // 2), np.float32)
    lib().oracle_swiglu(y, rows, I2 // 2, h)
    return h


def combine(y_dn_bf16: np.ndarray, topk_w: np.ndarray, slot_to_sorted: np.ndarray, T: int, k: int):
    y = np.ascontiguousarray(y_dn_bf16, np.uint16)
    H = y.shape[1]
    out = np.zeros((T, H), np.uint16)
    lib().oracle_combine(y, H, np.ascontiguousarray(topk_w, np.float32),
                         np.ascontiguousarray(slot_to_sorted, np.int32), T, k, out)
    return out


# ---------------------------------------------------------------- layer
def permute_quantize(x_bf16: np.ndarray, rt: Routing, gamma_a: np.ndarray):
    """Fused dispatch + activation quantisation, oracle form: sorted row s
    holds token sorted_to_slot[s] // k quantised with its expert's gamma."""
    K = x_bf16.shape[1]
    R = rt.sorted_to_slot.size
    codes = np.zeros((R, K // 2), np.uint8)
    scales = np.zeros((R, K // 32), np.uint8)
    ex = rt.expert_of_sorted()
    for s in range(R):
        t = rt.sorted_to_slot[s] // rt.k
        c, sc = quantize_rows_bf16(x_bf16[t:t + 1], gamma_a[ex[s]])
        codes[s], scales[s] = c[0], sc[0]
    return codes, scales


def requantize_rows(h: np.ndarray, rt: Routing, gamma_h: np.ndarray):
    R, I = h.shape
    codes = np.zeros((R, I // 2), np.uint8)
    scales = np.zeros((R, I // 32), np.uint8)
    ex = rt.expert_of_sorted()
    for e in np.unique(ex):
        rows = np.nonzero(ex == e)[0]
        c, sc = quantize_rows(h[rows], gamma_h[e])
        codes[rows], scales[rows] = c, sc
    return codes, scales


def moe_layer(x_bf16, logits, k, pk_gu: Packed, pk_dn: Packed, gamma_a_gu, gamma_a_dn,
              keep=False):
    """Route -> dispatch + quantise -> gate_up GEMM -> SiLU(gate)*up ->
    requantise -> down GEMM -> router-weighted combine (paper, App. D.1)."""
    T = x_bf16.shape[0]
    rt = route(logits, k)
    a_c, a_s = permute_quantize(x_bf16, rt, gamma_a_gu)
    y_gu, _ = grouped_gemm(pk_gu, a_c, a_s, rt.offsets, gamma_a_gu)
    h = swiglu(y_gu)
    h_c, h_s = requantize_rows(h, rt, gamma_a_dn)
    y_dn, _ = grouped_gemm(pk_dn, h_c, h_s, rt.offsets, gamma_a_dn)
    out = combine(y_dn, rt.topk_w, rt.slot_to_sorted, T, k)
    if keep:
        return out, dict(rt=rt, a_codes=a_c, a_scales=a_s, y_gu=y_gu, h=h, h_codes=h_c,
                         h_scales=h_s, y_dn=y_dn)
    return out


def calibrate_layer(x_bf16, logits, k, pk_gu: Packed, pk_dn: Packed):
    """Static activation global scales from a calibration batch (the
    definition moesq_calibrate_layer implements): per expert, Eq. 5's gamma
    of the largest |x| over its routed tokens, then of the largest |h| over
    its SwiGLU rows computed with those gammas; an expert without tokens
    takes the largest amax over all experts."""
    E = pk_gu.E
    rt = route(logits, k)
    ex = rt.expert_of_sorted()
    toks = rt.sorted_to_slot // k
    xf = np.abs((np.asarray(x_bf16, np.uint16).astype(np.uint32) << 16).view(np.float32))
    amax = np.zeros(E, np.float32)
    for s in range(toks.size):
        amax[ex[s]] = max(amax[ex[s]], xf[toks[s]].max())
    amax[amax == 0] = amax.max()
    ga = np.array([global_scale(a) for a in amax], np.float32)
    a_c, a_s = permute_quantize(x_bf16, rt, ga)
    y_gu, _ = grouped_gemm(pk_gu, a_c, a_s, rt.offsets, ga)
    h = np.abs(swiglu(y_gu))
    amax_h = np.zeros(E, np.float32)
    for s in range(toks.size):
        amax_h[ex[s]] = max(amax_h[ex[s]], h[s].max())
    amax_h[amax_h == 0] = amax_h.max()
    gh = np.array([global_scale(a) for a in amax_h], np.float32)
    return ga, gh
