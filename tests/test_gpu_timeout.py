"""The device timeout path, forced without a fault or a hang.

Every pipeline wait in the library's kernels is bounded; when a wait runs out the
kernel records MXC_ERR_TIMEOUT in the device error word and winds down.  Here a
self-test kernel runs that same bounded wait on a barrier that nothing completes,
with a limit of about half a millisecond: the host must read MXC_ERR_TIMEOUT, the
read must clear it, and the context must stay usable (a linear layer right after
runs clean and matches the oracle).
"""
import numpy as np
import pytest
import torch

from oracle import mxcode_oracle as O
from vector_quantized_mx_b200 import mxc, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mxc.lib()


def test_bounded_wait_runs_out_and_reports_timeout():
    assert mxc.get_device_error() == 0
    mxc.selftest_wait_timeout(1_000_000)             # ~0.5 ms at the B200's clocks
    assert mxc.get_device_error() == 7               # MXC_ERR_TIMEOUT
    assert mxc.get_device_error() == 0               # cleared by the read
    # the context is still usable
    w, x = synth.config1()
    pw = mxc.pack_weight(w)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16)
    y = mxc.linear(mxc.quantize_act(xd, w.fmt), pw).cpu().numpy()
    assert mxc.get_device_error() == 0
    ref, sabs = O.w4a4_linear(x, w)
    assert np.all(np.abs(y - ref) <= 1e-4 * sabs)


def test_selftest_rejects_out_of_range_limits():
    with pytest.raises(mxc.MxcError):
        mxc.selftest_wait_timeout(0)
    with pytest.raises(mxc.MxcError):
        mxc.selftest_wait_timeout(3_000_000_000)
