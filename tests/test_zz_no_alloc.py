"""mxc_moe_linear_noalloc: the grouped-expert layer for callers that cannot allocate
device memory (plugins whose host owns all device memory, real-time serving loops
that forbid allocator calls because an allocation may block or synchronize mid-step,
C callers without a device allocator).  It must give the same result as mxc_moe_linear, which takes a
caller workspace, on consecutive calls that reuse the library's fixed scratch
array.  This file runs last so that a failure here never hides the others.
"""
import numpy as np
import pytest
import torch

from oracle import mxcode_oracle as O
from vector_quantized_mx_b200 import mxc, synth

pytestmark = pytest.mark.gpu

TOL = 1e-4   # |gpu - oracle| <= TOL * sum_k |a_k w_k|, as in the other parity tests


def _dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def _case(seed, counts, fmt, strat, distinct_weights=True):
    E, N, K = len(counts), 256, 512
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    M = int(offsets[-1])
    n_w = E if distinct_weights else 1           # one shared weight keeps a 256-expert case small
    weights = [synth.make_weight(seed, fmt, strat, N, K, 256, 256, sub=e) for e in range(n_w)]
    x = synth.make_activations(seed, M, K, outliers=False)
    off_d = torch.from_numpy(offsets.astype(np.int32)).cuda()
    a = mxc.quantize_act_grouped(_dev_bf16(x), fmt, off_d)
    packed_w = [mxc.pack_weight(w) for w in weights]
    packed = [packed_w[e % n_w] for e in range(E)]
    # tolerance scale from the oracle: sum_k |a_k w_k| per output element
    codes, sf, s = O.quantize_act(x, fmt)
    a_hat = O.dequant_act(codes, sf, fmt, s)
    w_hats = [O.dequant_weight(w) for w in weights]
    sabs = np.zeros((M, N))
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 > r0:
            sabs[r0:r1] = O.abs_linear(a_hat[r0:r1], w_hats[e % n_w])
    return a, off_d, packed, sabs


def _compare(a, off_d, packed, sabs):
    y_ref = mxc.moe_linear(a, off_d, packed)
    y_new = mxc.moe_linear_noalloc(a, off_d, packed)
    assert mxc.get_device_error() == 0
    diff = (y_new - y_ref).abs().cpu().numpy()
    assert np.all(diff <= TOL * sabs), f"max diff/bound {np.max(diff / np.maximum(TOL * sabs, 1e-300)):.3g}"
    # same kernels on the same inputs: the results are the same bits
    assert torch.equal(y_new, y_ref)


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mxc.lib()


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    cases = [_case(81, [3, 0, 140, 17, 260, 1], "e4m3_b16", "prescale_plus"),
             _case(82, [129, 2, 0, 64], "e8m0_b32", "prescale")]
    for case in cases:                                # two calls in a row share the scratch array
        _compare(*case)


def test_noalloc_at_its_limit_of_256_experts():
    """E = 256, the largest table the fixed array holds: tiny per-expert row counts
    (zeros included), one packed weight shared by every expert; then a smaller call
    right after it on the same array."""
    counts = [(e * 7) % 5 for e in range(256)]       # 0..4 rows per expert
    _compare(*_case(84, counts, "e4m3_b16", "prescale", distinct_weights=False))
    _compare(*_case(85, [2, 0, 3], "e4m3_b16", "prescale"))


def test_noalloc_rejects_too_many_experts():
    a, off_d, packed, _ = _case(83, [4, 4], "e8m0_b32", "prescale")
    table = (mxc._Weight * 257)(*([packed[0]._c()] * 257))
    at = a._c()
    y = torch.empty((8, 256), device="cuda")
    status = mxc.lib().mxc_moe_linear_noalloc(mxc.ctypes.byref(at), off_d.data_ptr(), table, 257, y.data_ptr(), 256,
                                              0, torch.cuda.current_stream().cuda_stream)
    assert status == 2   # MXC_ERR_UNSUPPORTED: beyond the fixed scratch size, nothing enqueued
