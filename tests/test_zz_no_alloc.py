"""moesq_route_permute_noalloc: routing for callers that cannot hand the
library a scratch buffer (an op slot that only receives inputs and outputs,
or code that must not allocate device memory).  Its result must equal the
workspace-taking moesq_route_permute, call after call, although every call
reuses the same static scratch array inside the library.

This file is collected last on purpose; it passes alone and after the rest."""
import numpy as np
import pytest

import synthetic as S
from gpu_cases import to_dev, to_np

pytestmark = pytest.mark.gpu


def _route_both(m, lg, T, E, k):
    ref = m.RoutingBuffers(T, E, k)
    new = m.RoutingBuffers(T, E, k)
    m.moesq_route_permute(to_dev(lg), ref)
    m.moesq_route_permute_noalloc(to_dev(lg), new)
    st, word = m.moesq_get_device_error()
    assert st == 0, hex(word)
    return ref, new


# Both cases take the multi-kernel routing path (T > 512 tokens), the one
# that keeps per-block expert counts in the static scratch; the second fills
# the scratch to its limit (16384 tokens = 128 blocks, 512 experts).
@pytest.mark.parametrize("T,E,k", [(4096, 384, 8), (16384, 512, 8)])
def test_noalloc_routing_equals_workspace_routing_twice(cuda_lib, T, E, k):
    m = cuda_lib
    # two calls in a row with different logits: the second must not see the
    # first call's scratch contents
    for call, seed in enumerate((101, 202)):
        lg = S.uniform_logits_np(seed, T, E) if call == 0 else S.zipf_logits_np(seed, T, E)
        ref, new = _route_both(m, lg, T, E, k)
        for name in ("topk_ids", "counts", "offsets", "row_offsets", "sorted_to_slot", "slot_to_row"):
            assert (to_np(getattr(new, name)) == to_np(getattr(ref, name))).all(), (call, name)
        # gate weights: the tolerance the routing tests use against the oracle
        assert np.allclose(to_np(new.topk_w), to_np(ref.topk_w), rtol=4e-6, atol=1e-12)


def test_noalloc_rejects_more_tokens_than_its_scratch(cuda_lib):
    m = cuda_lib
    T, E, k = 16385, 8, 1
    rb = m.RoutingBuffers(T, E, k)
    lg = to_dev(np.zeros((T, E), np.float32))
    with pytest.raises(m.MoesqError) as ei:
        m.moesq_route_permute_noalloc(lg, rb)
    assert ei.value.status == 2
