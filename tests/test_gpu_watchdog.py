"""Failure detection without a GPU fault: a bounded wait on a barrier that
nothing signals gives up, the error word reports a timeout, and the context
keeps working."""
import numpy as np
import pytest

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_survives(cuda_lib):
    torch = pytest.importorskip("torch")
    m = cuda_lib
    assert m.moesq_get_device_error()[0] == 0
    m.moesq_debug_bounded_wait(20_000_000)            # 20 ms
    st, word = m.moesq_get_device_error()
    assert st == 4 and (word & 0xFF) == 4 and (word >> 8) == 7
    assert m.moesq_get_device_error()[0] == 0         # read clears the word
    a = torch.arange(1000, device="cuda", dtype=torch.float32)
    assert float(a.sum()) == 499500.0


def test_host_side_argument_errors(cuda_lib):
    torch = pytest.importorskip("torch")
    m = cuda_lib
    pw = m.PackedWeights(2, 128, 256)
    bad = m.PackedWeights(2, 128, 256)
    bad.struct.K = 100                                  # not a multiple of 256
    w = torch.zeros(2, 128, 256, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(m.MoesqError) as ei:
        m.moesq_pack_weights(w, 0, 2, bad)
    assert ei.value.status == 2
    with pytest.raises(m.MoesqError) as ei:
        m.moesq_pack_weights(w, 1, 2, pw)               # experts out of range
    assert ei.value.status == 1
    # a NULL routing struct is refused before any launch
    assert m.load().moesq_route_permute(None, None, None, 0, None) == 1
    rb = m.RoutingBuffers(4, 8, 2)
    with pytest.raises(m.MoesqError) as ei:               # NULL logits
        m.moesq_route_permute(None, rb)
    assert ei.value.status == 1
    assert m.moesq_get_device_error()[0] == 0
