"""CPU checks of the host-side layout transforms the GPU tests rely on
(tests/layouts.py): each kernel layout round-trips to the storage form, and
the metadata nibbles encode the mask's two kept pair indices."""
import numpy as np

import layouts as L
import oracle as O
from gpu_cases import weights_np


def test_kernel_form_round_trip():
    E, M, K = 2, 256, 768
    pk = O.pack_weights(weights_np(3, 0, E, M, K))
    tiles = L.storage_to_ktiles(pk.values, pk.mask, pk.scales)
    assert tiles.size == E * M * K * 11 // 32              # Eq. 7 bytes, tiled
    v, m, s = L.ktiles_to_storage(tiles, E, M, K)
    assert (v == pk.values).all() and (m == pk.mask).all() and (s == pk.scales).all()


def test_metadata_nibbles_are_the_kept_pair_indices():
    rng = np.random.default_rng(0)
    pats = [(0, 1), (0, 2), (0, 3), (1, 2), (1, 3), (2, 3)]
    E, M, K = 1, 128, 256
    pick = rng.integers(0, 6, size=(E, M, K // 8))
    nib = np.array([(1 << a) | (1 << b) for a, b in pats], np.uint8)[pick]
    mask = (nib[..., 0::2] | (nib[..., 1::2] << 4)).astype(np.uint8)
    meta = L.mask_to_kmeta(mask).reshape(E, M // 128, K // 256, 128, 16)
    code = np.array([a | (b << 2) for a, b in pats], np.uint8)[pick]      # i0 | i1 << 2, i0 < i1
    want = (code[..., 0::2] | (code[..., 1::2] << 4)).astype(np.uint8)   # [E, M, K/16]
    assert (meta[0, 0, 0] == want[0, :, :16]).all()
    assert (L.kmeta_to_mask(L.mask_to_kmeta(mask), E, M, K) == mask).all()


def test_mma_scale_layout_round_trip_and_position():
    R, K = 256, 512
    sc = np.arange(R * K // 32, dtype=np.int64).reshape(R, K // 32).astype(np.uint8)
    flat = L.scales_to_mma(sc)
    assert (L.mma_to_scales(flat, R, K) == sc).all()
    # row 128*r + 32*a + b, sub-block s of 128-wide block c at ((r*(K/128)+c)*512) + b*16 + a*4 + s
    r, a, b, c, s = 1, 2, 5, 3, 1
    row, col = 128 * r + 32 * a + b, 4 * c + s
    assert flat[(r * (K // 128) + c) * 512 + b * 16 + a * 4 + s] == sc[row, col]


def test_aligned_rows_and_compact_positions():
    counts = np.array([0, 1, 128, 129, 5])
    ro = L.aligned_rows(counts)
    assert list(ro) == [0, 0, 128, 256, 512, 640]
    rows = L.compact_to_rows(counts)
    assert rows.size == counts.sum() and rows[0] == 0 and rows[1] == 128 and rows[-1] == 512 + 4


def test_dense_tile_layout_round_trip_and_swizzle():
    """Dense kernel form: storage -> tiles -> storage is the identity, row r's
    16-byte chunk c sits at chunk c ^ (r & 7), and the per-16 scales of a
    64-wide K chunk land in the MMA scale layout."""
    import layouts as L
    rng = np.random.default_rng(3)
    E, M, K = 2, 256, 512
    codes = rng.integers(0, 256, size=(E, M, K // 2), dtype=np.uint8)
    sc = rng.integers(0, 127, size=(E, M, K // 16), dtype=np.uint8)
    t = L.dense_storage_to_dtiles(codes, sc)
    assert t.size == E * (M // 128) * (K // 256) * 18432
    c2, s2 = L.dtiles_to_dense_storage(t, E, M, K)
    assert (c2 == codes).all() and (s2 == sc).all()
    tile = t[:18432]                                  # e 0, row block 0, K step 0
    r, c = 5, 3
    assert (tile[r * 128 + (c ^ (r & 7)) * 16:][:16] == codes[0, r, c * 16:(c + 1) * 16]).all()
    r, j, s = 70, 2, 1                                # row 70 = 32 * 2 + 6, 64-chunk 2, 16-group 1
    assert tile[16384 + j * 512 + 6 * 16 + 2 * 4 + s] == sc[0, r, 4 * j + s]
    s32 = rng.integers(0, 127, size=(128, K // 32), dtype=np.uint8)
    s16 = L.mma_to_scales(L.scales32_to_scales16_mma(s32), 128, 2 * K)
    assert (s16[:, 0::2] == s32).all() and (s16[:, 1::2] == s32).all()


def test_swiglu_order_is_a_pairing_permutation():
    perm = L.swiglu_kernel_rows(1536)
    assert sorted(perm.tolist()) == list(range(1536))
    # kernel rows 128 b + j and 128 b + 64 + j hold gate and up of feature 64 b + j
    for b in range(12):
        for j in (0, 17, 63):
            assert perm[128 * b + j] == 64 * b + j and perm[128 * b + 64 + j] == 768 + 64 * b + j
