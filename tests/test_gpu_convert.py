"""GPU parity of the dense NVFP4 <-> pair-bitmask converters (model card
"Kimi-K2.5-P48NVFP4-MoESQ", pair-bitmask v1 and its canonical rule): bit
exact against the oracle's converters, the kernel form against the host
layout transform, and the lossless round trip."""
import numpy as np
import pytest

import layouts as L
import oracle as O
from gpu_cases import pack_gpu_from_np, to_dev, to_np, weights_np

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def packed_case():
    E, M, K = 3, 256, 512
    w = weights_np(41, 0, E, M, K)
    w[1, :, 64:96] = 0                       # whole zero chunks and blocks
    return w, O.pack_weights(w), (E, M, K)


def test_export_matches_oracle(cuda_lib, packed_case):
    w, pk, (E, M, K) = packed_case
    pw = pack_gpu_from_np(cuda_lib, w)
    torch = pytest.importorskip("torch")
    dense = torch.empty(E, M, K // 2, dtype=torch.uint8, device="cuda")
    cuda_lib.moesq_export_dense_nvfp4(pw, dense)
    assert (to_np(dense) == O.dense_from_sparse(pk.values, pk.mask)).all()
    assert cuda_lib.moesq_get_device_error()[0] == 0


def _with_sparse_chunks(dense):
    """Chunks left with 0 and 1 nonzero bytes, for the canonical rule."""
    d = dense.copy()
    d[:, :, 0:8] = 0
    d[:, :, 8:12] = 0
    d[:, :, 11] = 0x2A
    d[:, 5, :] = 0
    return d


def test_import_matches_oracle_and_kernel_form(cuda_lib, packed_case):
    w, pk, (E, M, K) = packed_case
    torch = pytest.importorskip("torch")
    dense = _with_sparse_chunks(O.dense_from_sparse(pk.values, pk.mask))
    v_ref, m_ref = O.sparse_from_dense(dense)
    pw = cuda_lib.PackedWeights(E, M, K)
    g = torch.tensor(pk.gamma, device="cuda")
    # two calls, experts [0, 2) and [2, 3), as a loader streaming experts would
    cuda_lib.moesq_import_dense_nvfp4(to_dev(np.ascontiguousarray(dense[:2])), to_dev(pk.scales[:2].copy()),
                                      g[:2], 0, 2, pw)
    cuda_lib.moesq_import_dense_nvfp4(to_dev(np.ascontiguousarray(dense[2:])), to_dev(pk.scales[2:].copy()),
                                      g[2:], 2, 1, pw)
    assert cuda_lib.moesq_get_device_error()[0] == 0
    assert (to_np(pw.values) == v_ref).all()
    assert (to_np(pw.mask) == m_ref).all()
    assert (to_np(pw.scales) == pk.scales).all()
    assert (to_np(pw.global_scale).view(np.uint32) == pk.gamma.view(np.uint32)).all()
    assert (to_np(pw.ktiles) == L.storage_to_ktiles(v_ref, m_ref, pk.scales)).all()
    # and back: dense -> pair-bitmask -> dense is lossless
    back = torch.empty(E, M, K // 2, dtype=torch.uint8, device="cuda")
    cuda_lib.moesq_export_dense_nvfp4(pw, back)
    assert (to_np(back) == dense).all()


def test_import_flags_chunks_outside_the_pattern(cuda_lib):
    E, M, K = 1, 128, 256
    dense = np.zeros((E, M, K // 2), np.uint8)
    dense[0, 7, 4:7] = 0x11                  # three nonzero bytes in one chunk
    pw = cuda_lib.PackedWeights(E, M, K)
    torch = pytest.importorskip("torch")
    cuda_lib.moesq_import_dense_nvfp4(to_dev(dense), to_dev(np.zeros((E, M, K // 32), np.uint8)),
                                      torch.ones(E, device="cuda"), 0, E, pw)
    st, word = cuda_lib.moesq_get_device_error()
    assert st == 5 and word == (10 << 8) | 5
    assert cuda_lib.moesq_get_device_error()[0] == 0      # read and cleared
