"""Every wait of the kernels that copy with TMA (the GEMMs) is bounded: on
running out the waiting warp records FP4_ERR_TIMEOUT in the status word and
the kernel returns.  fp4_test_bounded_wait runs that wait on a barrier that
nothing arrives on, so the test makes it run out without any fault: the
status must say TIMEOUT, the wait must have taken finite time, and the
context must still work afterwards (a quantisation matches the oracle)."""
import pytest
import torch

import block_scaled_fp4_reduce_b200 as fp4
import oracle
import workloads
from test_gpu_parity import assert_same, odata

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("tries", [1, 1000, 1 << 18])
def test_bounded_wait_runs_out_and_reports_timeout(tries):
    st = fp4.new_status(DEV)
    elapsed = torch.zeros(1, dtype=torch.int64, device=DEV)
    assert fp4.fp4_test_bounded_wait(tries, st, elapsed) == fp4.OK
    torch.cuda.synchronize()
    assert st.item() == fp4.ERR_TIMEOUT
    assert 0 < elapsed.item() < 10e9  # it ran out and returned (the full 2^18 polls: about a second)
    # the context is still usable
    x = workloads.generate(workloads.with_shape(workloads.WEIGHT_4K, 64, 1024))
    q = fp4.nvfp4_quantize(x.to(DEV))
    torch.cuda.synchronize()
    assert q.status.item() == fp4.OK
    p, s, g = oracle.nvfp4_quantize(odata(x))
    assert_same(q.packed, p, "packed after a timed-out wait")
    assert_same(q.scales, s, "scales after a timed-out wait")


def test_bounded_wait_argument_errors():
    st = fp4.new_status(DEV)
    elapsed = torch.zeros(1, dtype=torch.int64, device=DEV)
    assert fp4.fp4_test_bounded_wait(0, st, elapsed) == fp4.ERR_INVALID_ARG
    assert fp4.fp4_test_bounded_wait((1 << 18) + 1, st, elapsed) == fp4.ERR_INVALID_ARG
    assert fp4.lib().fp4_test_bounded_wait(10, None, elapsed.data_ptr(), None) == fp4.ERR_INVALID_ARG
