"""Host-side transforms between the storage form and the kernel layouts that
include/moesq.h defines (test helpers; numpy only).

* ktiles  [E][M/128][K/256][11264]: per tile the 128 rows of values (64 B
          each, 16-byte chunk c of row r at chunk c ^ ((r >> 1) & 3)), then
          the metadata [128][16] (byte b of row i holds chunks 2b, 2b+1; a chunk
          nibble is i0 | i1 << 2 of its two kept pair indices), then the
          scales of the two 128-wide K halves in the MMA scale layout.
* MMA scale layout (weights per tile, activations [R/128][K/128][512]):
          scale of row 32a+b (of a 128-row block), sub-block s of a 128-wide K
          block, at byte b*16 + a*4 + s.
* aligned row space: expert e owns rows row_offsets[e] + [0, counts[e]).
"""
import numpy as np


def mask_to_kmeta(mask: np.ndarray) -> np.ndarray:
    """mask uint8 [E, M, K/16] (pair bitmask) -> kmeta bytes (flat)."""
    E, M, K16 = mask.shape
    K = K16 * 16
    nib = np.stack([mask & 15, mask >> 4], -1).reshape(E, M, K // 8)          # per chunk bitmask
    i0 = np.zeros_like(nib)
    i1 = np.zeros_like(nib)
    for p in range(3, -1, -1):
        hit = (nib >> p) & 1 == 1
        i0 = np.where(hit, p, i0)          # ends with the lowest set bit
    for p in range(4):
        hit = (nib >> p) & 1 == 1
        i1 = np.where(hit, p, i1)          # ends with the highest set bit
    code = (i0 | (i1 << 2)).astype(np.uint8)                                   # [E, M, K/8]
    byte = (code[..., 0::2] | (code[..., 1::2] << 4)).astype(np.uint8)         # [E, M, K/16]
    # [E, MB, 128, KT, 16] -> [E, MB, KT, 128, 16]
    b = byte.reshape(E, M // 128, 128, K // 256, 16).transpose(0, 1, 3, 2, 4)
    return np.ascontiguousarray(b).reshape(-1)


def kmeta_to_mask(kmeta: np.ndarray, E: int, M: int, K: int) -> np.ndarray:
    b = kmeta.reshape(E, M // 128, K // 256, 128, 16).transpose(0, 1, 3, 2, 4).reshape(E, M, K // 16)
    code = np.stack([b & 15, b >> 4], -1).reshape(E, M, K // 8)
    i0, i1 = code & 3, code >> 2
    nib = ((1 << i0) | (1 << i1)).astype(np.uint8)
    return (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)


def scales_to_mma(sc: np.ndarray) -> np.ndarray:
    """Row-major scales [R, K/32] (R multiple of 128) -> MMA scale layout (flat)."""
    R, S = sc.shape
    # [R/128, 4(a), 32(b), K/128, 4(s)] -> [R/128, K/128, 32(b), 4(a), 4(s)]
    t = sc.reshape(R // 128, 4, 32, S // 4, 4).transpose(0, 3, 2, 1, 4)
    return np.ascontiguousarray(t).reshape(-1)


def storage_to_ktiles(values: np.ndarray, mask: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """Storage form [E, M, *] -> kernel-form tiles (flat uint8)."""
    E, M, K4 = values.shape
    K = 4 * K4
    MB, KT = M // 128, K // 256
    v = values.reshape(E, MB, 128, KT, 4, 16).transpose(0, 1, 3, 2, 4, 5)   # [E,MB,KT,r,c,16]
    r = np.arange(128)[:, None]
    c = np.arange(4)[None, :]
    img = np.empty_like(v)
    img[:, :, :, r, c ^ ((r >> 1) & 3), :] = v[:, :, :, r, c, :]
    meta = mask_to_kmeta(mask).reshape(E, MB, KT, 128 * 16)
    sc = weight_scales_to_kscales(scales).reshape(E, MB, KT, 1024)
    out = np.concatenate([img.reshape(E, MB, KT, 8192), meta, sc], axis=-1)
    return np.ascontiguousarray(out).reshape(-1)


def ktiles_to_storage(flat: np.ndarray, E: int, M: int, K: int):
    """Kernel-form tiles -> (values, mask, scales) of the storage form."""
    MB, KT = M // 128, K // 256
    t = flat.reshape(E, MB, KT, 11264)
    img = t[..., :8192].reshape(E, MB, KT, 128, 4, 16)
    r = np.arange(128)[:, None]
    c = np.arange(4)[None, :]
    v = img[:, :, :, r, c ^ ((r >> 1) & 3), :]                              # [E,MB,KT,r,c,16]
    values = v.transpose(0, 1, 3, 2, 4, 5).reshape(E, M, K // 4)
    meta = t[..., 8192:10240].reshape(-1)
    mask = kmeta_to_mask(np.ascontiguousarray(meta), E, M, K)
    sc = np.ascontiguousarray(t[..., 10240:]).reshape(-1)
    scales = kscales_to_weight_scales(sc, E, M, K)
    return np.ascontiguousarray(values), mask, scales


def mma_to_scales(flat: np.ndarray, R: int, K: int) -> np.ndarray:
    t = flat.reshape(R // 128, K // 128, 32, 4, 4).transpose(0, 3, 2, 1, 4)
    return np.ascontiguousarray(t).reshape(R, K // 32)


def weight_scales_to_kscales(scales: np.ndarray) -> np.ndarray:
    E, M, S = scales.shape
    return np.concatenate([scales_to_mma(scales[e]) for e in range(E)])


def kscales_to_weight_scales(flat: np.ndarray, E: int, M: int, K: int) -> np.ndarray:
    per = M * K // 32
    return np.stack([mma_to_scales(flat[e * per:(e + 1) * per], M, K) for e in range(E)])


def aligned_rows(counts: np.ndarray):
    """row_offsets [E+1] of the expert-aligned row space."""
    pad = (counts + 127) // 128 * 128
    return np.concatenate([[0], np.cumsum(pad)]).astype(np.int32)


def compact_to_rows(counts: np.ndarray) -> np.ndarray:
    """row of every compact (expert-sorted) position."""
    offs = np.concatenate([[0], np.cumsum(counts)])
    ro = aligned_rows(counts)
    rows = np.empty(int(offs[-1]), np.int64)
    for e in range(counts.size):
        rows[offs[e]:offs[e + 1]] = ro[e] + np.arange(counts[e])
    return rows


def bf16_ulp(y: np.ndarray) -> np.ndarray:
    """Spacing of bf16 numbers at |y| (for y != 0)."""
    a = np.abs(np.asarray(y, np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    return np.where(a > 0, 2.0 ** (e - 7), 0.0)


# ---------------------------------------------------------------- dense control
def dense_storage_to_dtiles(codes: np.ndarray, scales16: np.ndarray) -> np.ndarray:
    """Dense storage form (codes [E, M, K/2], per-16 scales [E, M, K/16]) ->
    kernel-form tiles (flat uint8): per (e, 128-row block, 256-wide K step)
    128 rows x 128 B of codes with 16-byte chunk c of row r at c ^ (r & 7),
    then the scales of the four 64-wide K chunks in the MMA scale layout."""
    E, M, K2 = codes.shape
    K = 2 * K2
    MB, KT = M // 128, K // 256
    v = codes.reshape(E, MB, 128, KT, 8, 16).transpose(0, 1, 3, 2, 4, 5)     # [E,MB,KT,r,c,16]
    r = np.arange(128)[:, None]
    c = np.arange(8)[None, :]
    img = np.empty_like(v)
    img[:, :, :, r, c ^ (r & 7), :] = v[:, :, :, r, c, :]
    sc = np.stack([np.stack([scales_to_mma(scales16[e, mb * 128:(mb + 1) * 128]) for mb in range(MB)])
                   for e in range(E)]).reshape(E, MB, KT, 2048)
    out = np.concatenate([img.reshape(E, MB, KT, 16384), sc], axis=-1)
    return np.ascontiguousarray(out).reshape(-1)


def dtiles_to_dense_storage(flat: np.ndarray, E: int, M: int, K: int):
    MB, KT = M // 128, K // 256
    t = flat.reshape(E, MB, KT, 18432)
    img = t[..., :16384].reshape(E, MB, KT, 128, 8, 16)
    r = np.arange(128)[:, None]
    c = np.arange(8)[None, :]
    v = img[:, :, :, r, c ^ (r & 7), :]
    codes = v.transpose(0, 1, 3, 2, 4, 5).reshape(E, M, K // 2)
    sc = t[..., 16384:].reshape(E, MB, KT * 2048)
    scales = np.stack([np.concatenate([mma_to_scales(np.ascontiguousarray(sc[e, mb]), 128, 2 * K)
                                       for mb in range(MB)]) for e in range(E)])
    return np.ascontiguousarray(codes), np.ascontiguousarray(scales)


def scales32_to_scales16_mma(scales32: np.ndarray) -> np.ndarray:
    """Row-major per-32 scales [R, K/32] -> per-16 scales (each twice) in the
    dense MMA layout (flat)."""
    return scales_to_mma(np.repeat(scales32, 2, axis=1))


def swiglu_kernel_rows(M: int) -> np.ndarray:
    """perm[p] = storage row held by kernel row p in the SwiGLU order: block
    b of 128 kernel rows = gate rows 64 b + [0, 64), then up rows
    M/2 + 64 b + [0, 64)."""
    I = M // 2
    p = np.arange(M)
    b, r = p // 128, p % 128
    return np.where(r < 64, 64 * b + r, I + 64 * b + r - 64)
