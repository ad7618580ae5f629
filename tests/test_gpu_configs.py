"""Full-size workload points against the oracle: the MoE down projection, and the
K = N = 8192 sweep across QBlocks, strategies, formats and token counts.

The oracle runs on seeded output tiles computed densely and on row and column
checksums (linearity), both computed in row chunks so that an 8192 x 8192 weight
or a 16384-row activation never has to be dequantized in one piece.  Bars as in
the other parity tests: |gpu - oracle| <= 1e-4 * sum |a w| per element (and per
checksum), MXCode bit-identical to native FP4 on the decoded weight.
"""
import numpy as np
import pytest
import torch

from oracle import mxcode_oracle as O
from vector_quantized_mx_b200 import mxc, synth

pytestmark = pytest.mark.gpu

TOL = 1e-4
CHUNK = 512


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mxc.lib()


def dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def assert_close(y, ref, sabs, what):
    err = np.abs(np.asarray(y, dtype=np.float64) - ref)
    bad = err > TOL * sabs
    assert not bad.any(), (f"{what}: {bad.sum()} of {bad.size} outside tolerance, max err/bound "
                           f"{np.max(err / np.maximum(TOL * sabs, 1e-300)):.3g}")


def act_chunks(x_bits, fmt):
    """Yields (r0, a_hat[r0:r0+CHUNK]) with the tensor scale of the whole activation."""
    s = O.tensor_scale_e4m3(x_bits) if fmt == "e4m3_b16" else None
    for r0 in range(0, x_bits.shape[0], CHUNK):
        codes, sf, ts = O.quantize_act(x_bits[r0:r0 + CHUNK], fmt, s)
        yield r0, O.dequant_act(codes, sf, fmt, ts)


def check_layer(y, x_bits, w, tile_rows, tile_cols, what):
    """y (device, [M, N] FP32) against the oracle: a dense tile, then all row and
    column sums, everything in row chunks."""
    M, N, K = x_bits.shape[0], w.N, w.K
    # activation side: the tile's rows, sum_m a and sum_m |a| over all rows
    a_tile = np.zeros((len(tile_rows), K))
    a_sum, a_abs = np.zeros(K), np.zeros(K)
    a_rows = {}
    for r0, ah in act_chunks(x_bits, w.fmt):
        a_sum += ah.sum(axis=0)
        a_abs += np.abs(ah).sum(axis=0)
        a_rows[r0] = ah
        for i, r in enumerate(tile_rows):
            if r0 <= r < r0 + CHUNK:
                a_tile[i] = ah[r - r0]
    # weight side: the tile's columns, column sums of Y, sum_n w and sum_n |w|
    w_sum, w_abs = np.zeros(K), np.zeros(K)
    col, abs_col = np.zeros(N), np.zeros(N)
    w_tile = np.zeros((len(tile_cols), K))
    for n0 in range(0, N, CHUNK):
        wh = O.dequant_weight(synth.weight_rows(w, n0, min(N, n0 + CHUNK)))
        w_sum += wh.sum(axis=0)
        w_abs += np.abs(wh).sum(axis=0)
        col[n0:n0 + len(wh)] = wh @ a_sum
        abs_col[n0:n0 + len(wh)] = np.abs(wh) @ a_abs
        for i, c in enumerate(tile_cols):
            if n0 <= c < n0 + CHUNK:
                w_tile[i] = wh[c - n0]
    row = np.concatenate([a_rows[r0] @ w_sum for r0 in sorted(a_rows)])
    abs_row = np.concatenate([np.abs(a_rows[r0]) @ w_abs for r0 in sorted(a_rows)])
    yt = y[torch.as_tensor(tile_rows, device=y.device)][:, torch.as_tensor(tile_cols, device=y.device)]
    assert_close(yt.cpu().numpy(), O.linear(a_tile, w_tile), O.abs_linear(a_tile, w_tile), f"{what} tile")
    assert_close(y.double().sum(dim=1).cpu().numpy(), row, abs_row, f"{what} row sums")
    assert_close(y.double().sum(dim=0).cpu().numpy(), col, abs_col, f"{what} column sums")


def run_point(w, x, with_native=True):
    pw = mxc.pack_weight(w)
    a = mxc.quantize_act(dev_bf16(x), w.fmt)
    y = mxc.linear(a, pw)
    assert mxc.get_device_error() == 0
    if with_native:
        yn = mxc.native_linear(a, mxc.decode_weight(pw))
        assert mxc.get_device_error() == 0
        assert torch.equal(y, yn)
    return y


# ---------------------------------------------------------------------------
# K = N = 8192 sweep points
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("strat", ["postscale", "prescale", "prescale_plus", "postscale_qb"])
def test_config5_qblock_1024(fmt, strat):
    """QBlock 1024 x 1024 (four 256-channel stages share a codebook) at M = 16."""
    w = synth.make_weight(5, fmt, strat, 8192, 8192, 1024, 1024, sub=200 + 2 * ["postscale", "prescale",
                          "prescale_plus", "postscale_qb"].index(strat) + ["e8m0_b32", "e4m3_b16"].index(fmt))
    x = synth.config5_activations(16)
    y = run_point(w, x)
    check_layer(y, x, w, np.arange(16), np.arange(3072, 3328), f"1024^2 {strat} {fmt}")


@pytest.mark.parametrize("M,qb,strat,fmt", [
    (1, 0, "postscale", "e4m3_b16"),        # decode, one codebook for the whole tensor
    (128, 128, "prescale", "e8m0_b32"),     # 128-token tile, two codebooks per stage
    (128, 256, "prescale_plus", "e4m3_b16"),
])
def test_config5_small_and_mid_m(M, qb, strat, fmt):
    w = synth.config5_weight(qb, strat, fmt)
    x = synth.config5_activations(M)
    y = run_point(w, x)
    check_layer(y, x, w, np.arange(M), np.arange(0, 256), f"M={M} qb={qb} {strat} {fmt}")


def test_config5_m16384_prefill():
    """M = 16384 prefill (decode once, then the native GEMM) on a PreScale+ E8M0-B32
    weight with 1024 x 1024 QBlocks: a seeded 256 x 256 tile plus all checksums."""
    w = synth.config5_weight(1024, "prescale_plus", "e8m0_b32")
    x = synth.config5_activations(16384)
    y = run_point(w, x, with_native=False)
    rng = np.random.default_rng(16384)
    rows = np.sort(rng.choice(16384, 256, replace=False))
    c0 = int(rng.integers(0, 8192 - 256))
    check_layer(y, x, w, rows, np.arange(c0, c0 + 256), "M=16384")


# ---------------------------------------------------------------------------
# MoE down projection at full size (1536 -> 4096 per expert)
# ---------------------------------------------------------------------------

def test_config4_down_projection_full_size():
    """The down projection of the MoE workload: 16384 expert-sorted rows of the
    1536-wide SwiGLU output (synthetic N(0,1)), 128 PreScale+ E4M3-B16 experts of
    [4096, 1536] with 256 x 256 QBlocks.  For the largest, the smallest and two fixed
    experts: up to 64 rows x 256 columns densely plus the expert's row and column sums."""
    row_tok, off = synth.config4_routing()
    xd = synth.config4_activations("down", row_tok)
    experts = [synth.config4_expert(e, "down") for e in range(synth.MOE_EXPERTS)]
    packed = [mxc.pack_weight(w) for w in experts]
    offd = torch.from_numpy(off.astype(np.int32)).cuda()
    a = mxc.quantize_act_grouped(dev_bf16(xd), "e4m3_b16", offd)
    y = mxc.moe_linear(a, offd, packed)
    assert mxc.get_device_error() == 0
    s = O.tensor_scale_e4m3(xd)
    assert a.tscale.item() == np.float32(s)
    counts = np.diff(off)
    nonempty = np.flatnonzero(counts)
    for e in sorted({int(counts.argmax()), int(nonempty[counts[nonempty].argmin()]), 0, 127}):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        codes, sf, _ = O.quantize_act(xd[r0:r1], "e4m3_b16", s)
        a_hat = O.dequant_act(codes, sf, "e4m3_b16", s)
        w_hat = O.dequant_weight(experts[e])
        rows = np.arange(min(64, r1 - r0))
        ye = y[r0:r1].double()
        assert_close(ye[:len(rows), 2048:2304].cpu().numpy(), O.linear(a_hat[rows], w_hat[2048:2304]),
                     O.abs_linear(a_hat[rows], w_hat[2048:2304]), f"expert {e} tile")
        row, colsum, abs_row, abs_col = O.checksums(a_hat, w_hat)
        assert_close(ye.sum(dim=1).cpu().numpy(), row, abs_row, f"expert {e} row sums")
        assert_close(ye.sum(dim=0).cpu().numpy(), colsum, abs_col, f"expert {e} column sums")
