"""The offline MXCode quantizer (vector_quantized_mx_b200/quantize.py).

Its k-means has no reference values on the pages (they report SQNR of trained
model tensors, Table 4), so what is checked is: its rounding helpers against the
oracle's pinned encoders; that what it emits is exactly the weight the oracle
(and so the kernels) reconstruct, with the storage the BPE accounting predicts;
and SQNR sanity on Gaussian tensors (about 2 bits a weight at d = 4, K = 256:
near the 10 dB design point of Figure 2, far below native FP4, better with
smaller QBlocks).
"""
import numpy as np
import pytest
import torch

from oracle import mxcode_oracle as O
from vector_quantized_mx_b200 import mxc
from vector_quantized_mx_b200 import quantize as Q

FMTS = ("e8m0_b32", "e4m3_b16")


def test_e2m1_rounding_matches_oracle():
    grid = np.concatenate([np.linspace(-8, 8, 4001), [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -0.75, -2.5, 7.0]])
    assert np.array_equal(Q.e2m1_codes(grid) & 7, O.e2m1_encode_rne(grid))
    assert np.array_equal(Q.e2m1_values(Q.e2m1_codes(grid)),
                          np.sign(grid) * O.E2M1_MAG[O.e2m1_encode_rne(grid)])


def test_e4m3_rounding_matches_oracle():
    rng = np.random.default_rng(0)
    v = np.concatenate([np.exp2(rng.uniform(-12, 10, 20000)), O.e4m3_value(np.arange(127)), [0.0, 500.0, 1e6]])
    mids = (O.e4m3_value(np.arange(126)) + O.e4m3_value(np.arange(1, 127))) / 2   # exact ties
    v = np.concatenate([v, mids])
    assert np.array_equal(Q.e4m3_byte(v), O.e4m3_encode_rne_satfinite(v))
    assert np.array_equal(Q.e4m3_value(np.arange(127)), O.e4m3_value(np.arange(127)))


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("strategy", Q.STRATEGIES)
def test_output_is_the_weight_the_oracle_reads(fmt, strategy):
    W = np.random.default_rng(1).normal(size=(256, 512)) * 0.02
    w = Q.quantize_weight(W, fmt, strategy, 128, 256, iters=6, seed=1)
    assert w.idx.shape == (256, 128) and w.cb.shape == (2, 2, 256)
    assert np.array_equal(Q.dequantize(w), O.dequant_weight(w))
    bpw = O.bits_per_weight(fmt, strategy, 256, 512, 128, 256)
    assert O.storage_bytes(w) * 8 / (256 * 512) == pytest.approx(bpw)
    assert Q.quality(W, w)["bits_per_weight"] == pytest.approx(bpw)
    # the C ABI accepts it as it is
    h = mxc.pack_weight_host(w)
    assert h["idx"].size == 256 * 128


def test_sqnr_sanity_on_gaussian_weights():
    W = np.random.default_rng(2).normal(size=(256, 1024))
    for fmt in FMTS:
        for strategy in Q.STRATEGIES:
            s = [Q.quality(W, Q.quantize_weight(W, fmt, strategy, qb, qb, iters=8, seed=2)) for qb in (0, 128)]
            full, small = s[0]["sqnr_db"], s[1]["sqnr_db"]
            assert 8.0 < full < 13.0 and 8.0 < small < 13.0, (fmt, strategy, full, small)
            assert small > full, (fmt, strategy, full, small)           # more codebooks, less error
            assert s[0]["native_fp4_sqnr_db"] > full + 6.0                # 4.25 / 4.5 bits vs ~2


def test_zero_and_constant_tensors():
    for fmt in FMTS:
        Z = np.zeros((128, 256))
        w = Q.quantize_weight(Z, fmt, "prescale", 128, 256, iters=2)
        assert not Q.dequantize(w).any()
        C = np.full((128, 256), 1.5)
        w = Q.quantize_weight(C, fmt, "postscale_qb", 128, 256, iters=2)
        assert np.allclose(Q.dequantize(w), C)                          # 1.5 is on the FP4 grid


@pytest.mark.gpu
def test_quantized_weight_runs_through_the_gpu_path():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    from vector_quantized_mx_b200 import synth
    W = np.random.default_rng(3).normal(size=(512, 1024)) * 0.05
    x = synth.make_activations(3, 16, 1024, outliers=True)
    for strategy in ("prescale", "postscale_qb"):
        w = Q.quantize_weight(W, "e4m3_b16", strategy, 256, 256, iters=6, seed=3)
        a = mxc.quantize_act(torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16),
                             w.fmt)
        y = mxc.linear(a, mxc.pack_weight(w)).cpu().numpy()
        assert mxc.get_device_error() == 0
        ref, sabs = O.w4a4_linear(x, w)
        assert np.all(np.abs(y - ref) <= 1e-4 * sabs)


def test_command_line_report(capsys):
    Q.main(["--n", "128", "--k", "256", "--qb", "128", "--iters", "2", "--strategy", "postscale_qb"])
    out = capsys.readouterr().out
    assert out.startswith("postscale_qb e4m3_b16 QBlock 128: SQNR") and "bits/weight" in out
