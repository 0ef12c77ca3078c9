"""Pins of the oracle's weight packing against what the pages fix: the
paired-4:8 feasible set (App. A, Eq. 6), the storage cost (Eq. 7), the
pair-bitmask storage layout and its lossless dense round trip (model card),
the scale rule (Sec. 3.4, Eq. 5) and magnitude pair selection."""
import ml_dtypes
import numpy as np
import pytest

import oracle as O
import synthetic as S
from conftest import golden_dict


def _weights(E=2, M=32, K=256, seed=3, sigma=0.02):
    return np.stack([S.expert_weights_bf16_np(seed, 0, e, M, K, sigma) for e in range(E)])


def _f32(bits):
    return S.bf16_bits_to_f32_np(bits).astype(np.float64)


@pytest.fixture(scope="module")
def packed():
    w = _weights()
    return w, O.pack_weights(w)


def test_storage_cost_eq7(packed):
    w, pk = packed
    c = golden_dict("format_constants.txt")
    E, M, K = w.shape
    assert pk.values.shape == (E, M, K // int(c["packed_div"]))
    assert pk.mask.shape == (E, M, K // int(c["mask_div"]))
    assert pk.scales.shape == (E, M, K // int(c["scale_div"]))
    bits = 8 * (pk.values[0].size + pk.mask[0].size + pk.scales[0].size) / (M * K)
    assert bits == c["bits_per_weight"]
    # versus dense NVFP4 with the same per-32 scales: values K/2 + scales K/32
    assert (pk.values[0].size + pk.mask[0].size + pk.scales[0].size) * 32 == 11 * M * K


def test_every_chunk_keeps_exactly_two_pairs(packed):
    _, pk = packed
    lo, hi = pk.mask & 15, pk.mask >> 4
    pop = np.vectorize(lambda v: bin(int(v)).count("1"))
    assert (pop(lo) == 2).all() and (pop(hi) == 2).all()
    # the six admissible patterns of App. A
    pats = set(np.unique(np.concatenate([lo.ravel(), hi.ravel()])).tolist())
    assert pats <= {0b0011, 0b0101, 0b1001, 0b0110, 0b1010, 0b1100}


def _dense_codes(pk, e):
    """Dense NVFP4 bytes [M][K/2] rebuilt from the pair-bitmask form (model
    card): kept bytes go back to their pair slot, the other bytes are zero."""
    v, m = pk.values[e], pk.mask[e]
    M, K4 = v.shape
    dense = np.zeros((M, 2 * K4), np.uint8)
    for g in range(2 * m.shape[1]):
        nib = (m[:, g // 2] >> (4 * (g % 2))) & 15
        slot = np.zeros(M, np.int64)
        for p in range(4):
            kept = (nib >> p) & 1 == 1
            dense[kept, 4 * g + p] = v[kept, 2 * g + slot[kept]]
            slot += kept
    return dense


def _sparse_from_dense(dense):
    """Dense NVFP4 -> pair-bitmask, the model card's canonical rule: keep the
    nonzero bytes of each 4-byte chunk; if fewer than 2, mark the
    lowest-index zero bytes as kept."""
    M, K2 = dense.shape
    values = np.zeros((M, K2 // 2), np.uint8)
    mask = np.zeros((M, K2 // 8), np.uint8)
    for r in range(M):
        for g in range(K2 // 4):
            chunk = dense[r, 4 * g:4 * g + 4]
            nz = [i for i in range(4) if chunk[i] != 0]
            assert len(nz) <= 2
            z = [i for i in range(4) if chunk[i] == 0]
            keep = sorted(nz + z[:2 - len(nz)])
            values[r, 2 * g:2 * g + 2] = chunk[keep]
            mask[r, g // 2] |= (sum(1 << i for i in keep)) << (4 * (g % 2))
    return values, mask


def test_dense_roundtrip_is_lossless(packed):
    _, pk = packed
    for e in range(pk.E):
        dense = _dense_codes(pk, e)
        v2, m2 = _sparse_from_dense(dense)
        # dense -> pair-bitmask -> dense reproduces every byte
        pk2 = O.Packed(v2[None], m2[None], pk.scales[e:e + 1], pk.gamma[e:e + 1])
        assert (_dense_codes(pk2, 0) == dense).all()


def test_kept_pairs_have_the_largest_l2(packed):
    w, pk = packed
    for e in range(pk.E):
        wf = _f32(w[e]).astype(np.float32)
        M, K = wf.shape
        sc = (wf[:, 0::2] * wf[:, 0::2] + wf[:, 1::2] * wf[:, 1::2]).reshape(M, K // 8, 4)
        nib = np.stack([pk.mask[e] & 15, pk.mask[e] >> 4], axis=-1).reshape(M, K // 8)
        kept = ((nib[..., None] >> np.arange(4)) & 1).astype(bool)
        kmin = np.where(kept, sc, np.inf).min(-1)
        dmax = np.where(~kept, sc, -np.inf).max(-1)
        assert (kmin >= dmax).all()
        # ties keep the lower pair index: a dropped pair never beats a kept
        # lower-indexed... i.e. among equal scores the kept ones come first
        for r, g in zip(*np.nonzero(kmin == dmax)):
            ks = [p for p in range(4) if kept[r, g, p] and sc[r, g, p] == kmin[r, g]]
            ds = [p for p in range(4) if not kept[r, g, p] and sc[r, g, p] == dmax[r, g]]
            assert max(ks) < min(ds)


def test_tie_break_and_zero_groups():
    M, K = 1, 64
    w = np.zeros((1, M, K), np.float32)
    w[0, 0, 8:16] = [1, 1, 1, 1, 1, 1, 1, 1]          # four equal pairs -> pairs 0 and 1
    w[0, 0, 16:24] = [0, 0, 0, 0, 2, 0, 0, 3]         # pairs 2 and 3
    w[0, 0, 24:32] = [0, 0.5, 0, 0, 0, 0, 0, 0]       # pair 0 and the lowest zero pair 1
    pk = O.pack_weights(S.f32_to_bf16_bits_np(w))
    nib = [(pk.mask[0, 0, g // 2] >> (4 * (g % 2))) & 15 for g in range(K // 8)]
    assert nib[0] == 0b0011                            # all-zero group
    assert nib[1] == 0b0011
    assert nib[2] == 0b1100
    assert nib[3] == 0b0011


def test_scale_rule_eq5_closed_forms():
    # the block holding the tensor's largest kept |w| gets scale 448 exactly
    w = _weights(E=3, M=16, K=256, seed=9)
    pk = O.pack_weights(w)
    for e in range(3):
        deq = O.unpack_weights(pk.values[e], pk.mask[e], pk.scales[e], pk.gamma[e], 16, 256)
        wf = _f32(w[e])
        kept = deq != 0
        amax = np.abs(np.where(kept | (wf == 0), wf, 0)).max()
        assert pk.scales[e].max() == 0x7E
        r, k = np.unravel_index(np.argmax(np.abs(np.where(kept, wf, 0))), wf.shape)
        assert pk.scales[e][r, k // 32] == 0x7E
        assert abs(pk.gamma[e] * amax / 6 - 448) <= 448 * 2 ** -22
    # a zero block gets scale code 0; a zero tensor gets gamma 1
    z = np.zeros((1, 8, 64), np.uint16)
    pkz = O.pack_weights(z)
    assert pkz.gamma[0] == 1.0 and (pkz.scales == 0).all() and (pkz.values == 0).all()


def test_reconstruction_lies_in_S_cap_Q_and_is_close(packed):
    """Eq. 6: decode(pack(W)) is paired-4:8 sparse and every block is
    s_b * (E2M1 grid) with s_b = UE4M3 / gamma; each kept weight is within
    half a grid step (times s_b) of its original value."""
    w, pk = packed
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    for e in range(pk.E):
        M, K = w.shape[1], w.shape[2]
        deq = O.unpack_weights(pk.values[e], pk.mask[e], pk.scales[e], pk.gamma[e], M, K)
        nz = (deq.reshape(M, K // 8, 4, 2) != 0).any(-1).sum(-1)
        assert (nz <= 2).all()
        s = np.array([[O.ue4m3_value(c) for c in row] for row in pk.scales[e]]) / pk.gamma[e]
        q = np.abs(deq) / np.repeat(s, 32, axis=1)
        assert np.isin(np.round(q, 9), grid).all()
        wf = _f32(w[e])
        kept = np.repeat(np.stack([pk.mask[e] & 15, pk.mask[e] >> 4], -1).reshape(M, K // 8), 8, 1)
        pair = (np.arange(K) % 8) // 2
        kept = ((kept >> pair) & 1).astype(bool)
        err = np.abs(np.where(kept, wf, 0) - deq)
        step = np.repeat(s, 32, axis=1)
        # the largest grid gap is 2 (between 4 and 6): error <= 1 * s_b
        assert (err <= 1.0 * step + 1e-12).all()
        # and relative to the block scale it is small on average
        assert np.mean(err[kept] / step[kept]) < 0.3


def test_pack_is_deterministic_and_expert_independent():
    w = _weights(E=3, M=16, K=128, seed=11)
    a = O.pack_weights(w)
    b = O.pack_weights(w[1:2])
    assert (a.values[1] == b.values[0]).all() and (a.mask[1] == b.mask[0]).all()
    assert (a.scales[1] == b.scales[0]).all() and a.gamma[1] == b.gamma[0]


def test_oracle_converters_match_the_chunk_loops(packed):
    """oracle.dense_from_sparse / sparse_from_dense (vectorised) against the
    chunk-by-chunk restatement above, including chunks left with 0 or 1
    nonzero bytes (the canonical rule's lowest-index zero bytes)."""
    _, pk = packed
    for e in range(pk.E):
        dense = _dense_codes(pk, e)
        assert (O.dense_from_sparse(pk.values[e], pk.mask[e]) == dense).all()
        d = dense.copy()
        d[:, 0:4] = 0                        # an empty chunk
        d[:, 4:8] = 0
        d[:, 6] = 0x31                       # a chunk with one nonzero byte
        v_loop, m_loop = _sparse_from_dense(d)
        v, m = O.sparse_from_dense(d)
        assert (v == v_loop).all() and (m == m_loop).all()
        assert (O.dense_from_sparse(v, m) == d).all()
        nib = np.stack([m & 15, m >> 4], -1)
        assert (np.vectorize(lambda x: bin(int(x)).count("1"))(nib) == 2).all()


def test_oracle_sparse_from_dense_rejects_three_nonzero_bytes():
    d = np.zeros((1, 8), np.uint8)
    d[0, :3] = 0x11
    with pytest.raises(ValueError):
        O.sparse_from_dense(d)
