"""The FP4 tensor-core throughput benchmark (moesq_mma_peak) runs, completes
without a device error, and gives rates in the range of the part: below the
nominal B200 dense-equivalent peaks (9 PFLOP/s dense FP4, 18 PFLOP/s with
2:4 sparsity) by no more than the clock's headroom, and well above the
bf16 rate."""
import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("copies", [False, True])
@pytest.mark.parametrize("sparse,n,ctas", [(1, 256, 1), (1, 128, 2), (0, 256, 1), (0, 128, 2)])
def test_mma_peak_runs_and_is_plausible(cuda_lib, sparse, n, ctas, copies):
    m = cuda_lib
    t = m.moesq_mma_peak(sparse, n, ctas, with_copies=copies, iters=4000)
    st, word = m.moesq_get_device_error()
    assert st == 0, hex(word)
    nominal = 18000.0 if sparse else 9000.0
    assert (0.05 if copies else 0.2) * nominal < t < 1.15 * nominal, t
