"""MoE gate/up fused with SwiGLU and the down projection's activation quantization.

The fused kernel computes g and u exactly as mxc_moe_linear does (same tiles, same
K order, same FP32 scaling), so the oracle is applied to mxc_moe_linear's FP32
gate/up output: its SwiGLU (FP32, one operation per step, the fixed FP32 exp) and
MX quantization must give the fused kernel's FP4 codes and block scales bit for
bit, padding rows of each expert tile must carry zero scales, and the down
projection on the fused activation must match the oracle's down projection of the
oracle's activation within |gpu - oracle| <= 1e-4 * sum |a w|.
"""
import numpy as np
import pytest
import torch

from oracle import mxcode_oracle as O
from vector_quantized_mx_b200 import mxc, synth

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mxc.lib()


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def tile_prefix(offsets):
    counts = np.diff(offsets)
    return np.concatenate([[0], np.cumsum((counts + 127) // 128)]).astype(np.int64)


def check_fused(x, offsets, gu_weights, down_weights, fmt, row_chunk=2048, experts_to_check=None):
    E = len(gu_weights)
    F = gu_weights[0].N // 2
    B = O.BLOCK[fmt]
    off_d = torch.from_numpy(offsets.astype(np.int32)).cuda()
    a = mxc.quantize_act_grouped(dev_bf16(x), fmt, off_d)
    gu = [mxc.pack_weight(w) for w in gu_weights]
    y = mxc.moe_linear(a, off_d, gu)                         # FP32 gate/up output
    assert mxc.get_device_error() == 0
    yh = y.cpu().numpy()
    # the oracle's SwiGLU of the GPU's own gate/up output, chunk by chunk
    h_tscale = None
    if fmt == "e4m3_b16":                                   # a calibrated scale for h
        hmax = max(float(np.abs(O.swiglu_fp32(yh[r:r + row_chunk, :F], yh[r:r + row_chunk, F:])).max())
                   for r in range(0, len(yh), row_chunk))
        h_tscale = np.float32(hmax) / np.float32(2688.0)
    codes = np.zeros((len(yh), F), np.uint8)
    sfs = np.zeros((len(yh), F // B), np.uint8)
    for r in range(0, len(yh), row_chunk):
        codes[r:r + row_chunk], sfs[r:r + row_chunk] = O.swiglu_quantize(yh[r:r + row_chunk], fmt, h_tscale)
    ts_d = None if h_tscale is None else torch.tensor([h_tscale], dtype=torch.float32, device="cuda")
    h = mxc.moe_gate_up_swiglu(a, off_d, gu, h_tscale=ts_d)
    assert mxc.get_device_error() == 0
    got_q = h.q.cpu().numpy()
    ref_q = O.pack_fp4(codes)
    assert np.array_equal(got_q, ref_q), f"FP4 codes of h differ at {np.argwhere(got_q != ref_q)[:5]}"
    # scales: grouped SF layout, each expert's rows from tile_prefix[e] * 128
    tp = tile_prefix(offsets)
    rows_sf = int(tp[-1]) * 128
    sf_rows = mxc.sf_to_rows(h.sf.cpu().numpy(), rows_sf, F, fmt)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        base = int(tp[e]) * 128
        assert np.array_equal(sf_rows[base:base + r1 - r0], sfs[r0:r1]), f"scales of h, expert {e}"
        pad_end = int(tp[e + 1]) * 128
        assert not sf_rows[base + r1 - r0:pad_end].any(), f"padding scales of expert {e}"
    # the down projection on the fused activation against the oracle's
    dn = [mxc.pack_weight(w) for w in down_weights]
    yd = mxc.moe_linear(h, off_d, dn).cpu().numpy()
    assert mxc.get_device_error() == 0
    s_h = 1.0 if h_tscale is None else float(h_tscale)
    for e in (range(E) if experts_to_check is None else experts_to_check):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r1 == r0:
            continue
        rows = slice(r0, min(r1, r0 + 64))
        a_hat = O.dequant_act(codes[rows], sfs[rows], fmt, s_h)
        w_hat = O.dequant_weight(down_weights[e])
        ref, sabs = O.linear(a_hat, w_hat), O.abs_linear(a_hat, w_hat)
        err = np.abs(yd[rows] - ref)
        assert np.all(err <= TOL * sabs), f"down projection, expert {e}: max err/bound {np.max(err / (TOL * sabs)):.3g}"


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("strat", ["prescale", "prescale_plus", "postscale_qb"])
def test_swiglu_small(fmt, strat):
    counts = [0, 5, 130, 1, 257, 0]
    E, F, K = len(counts), 256, 512
    offsets = np.concatenate([[0], np.cumsum(counts)])
    gu = [synth.make_weight(91, fmt, strat, 2 * F, K, 256, 256, sub=e) for e in range(E)]
    dn = [synth.make_weight(92, fmt, strat, 256, F, 256, 256, sub=e) for e in range(E)]
    x = synth.make_activations(91, int(offsets[-1]), K, outliers=True)
    check_fused(x, offsets, gu, dn, fmt)


def test_swiglu_config4_full_size():
    """Config 4 (PreScale+ E4M3-B16, 128 experts, gate/up [3072, 4096], down
    [4096, 1536], 2048 tokens top-8 Zipf(1.1)): every code and scale of h for all
    16384 rows, and the down projection for four experts."""
    row_tok, off = synth.config4_routing()
    x = synth.config4_activations("gate_up", row_tok)
    gu = [synth.config4_expert(e, "gate_up") for e in range(synth.MOE_EXPERTS)]
    dn = [synth.config4_expert(e, "down") for e in range(synth.MOE_EXPERTS)]
    counts = np.diff(off)
    nonempty = np.flatnonzero(counts)
    check = sorted({int(counts.argmax()), int(nonempty[counts[nonempty].argmin()]), 0, 127})
    check_fused(x, off, gu, dn, "e4m3_b16", experts_to_check=check)
