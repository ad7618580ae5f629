"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Bars (from the method's W4A4 contract and the oracle's definitions):
* quantized activations (FP4 codes, scale bytes, tensor scale) and decoded
  weights (FP4 codes, scale bytes): bit-exact;
* linear outputs: |gpu - oracle| <= 1e-4 * sum_k |a_k w_k| per element (FP32
  output); BF16 output additionally allows the BF16 rounding of the result;
* MXCode and native FP4 on the same decoded weights: bit-identical outputs
  (same operands, same tensor-core K order).
"""
import numpy as np
import pytest
import torch

from oracle import mxcode_oracle as O
from vector_quantized_mx_b200 import mxc, synth

pytestmark = pytest.mark.gpu

TOL = 1e-4


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    mxc.lib()
    assert torch.cuda.get_device_capability()[0] == 10


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def assert_close(y, ref, sabs, tol=TOL, what=""):
    y = np.asarray(y, dtype=np.float64)
    err = np.abs(y - ref)
    bound = tol * sabs
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; first at {tuple(i)}: "
                             f"gpu={y[tuple(i)]!r} ref={ref[tuple(i)]!r} bound={bound[tuple(i)]!r} "
                             f"max err/bound={np.max(err / np.maximum(bound, 1e-300)):.3g}")


def oracle_act(x_bits, fmt, tscale=None):
    codes, sf, s = O.quantize_act(x_bits, fmt, tscale)
    return O.pack_fp4(codes), sf, s


def check_act(mx, x_bits, fmt, tscale=None):
    M, K = x_bits.shape
    q_ref, sf_ref, s_ref = oracle_act(x_bits, fmt, tscale)
    q = mx.q.cpu().numpy()
    assert np.array_equal(q, q_ref), f"FP4 codes differ at {np.argwhere(q != q_ref)[:5]}"
    sf_all = mx.sf.cpu().numpy()
    rows_pad = (M + 127) // 128 * 128
    sf_rows = mxc.sf_to_rows(sf_all, rows_pad, K, fmt)
    assert np.array_equal(sf_rows[:M], sf_ref), f"scales differ at {np.argwhere(sf_rows[:M] != sf_ref)[:5]}"
    assert not sf_rows[M:].any(), "padding rows must have zero scales"
    if fmt == "e4m3_b16":
        assert mx.tscale.item() == np.float32(s_ref)


# ---------------------------------------------------------------------------
# Activation quantization: bit-exact
# ---------------------------------------------------------------------------

def special_activations(M, K, seed):
    rng = np.random.default_rng(seed)
    z = rng.normal(size=(M, K)) * np.exp(rng.uniform(-8, 8, size=(M, 1)))
    x = torch.from_numpy(z).to(torch.bfloat16)
    bits = x.view(torch.int16).numpy().view(np.uint16).copy()
    # exact E2M1 midpoints after a power-of-two scale, zeros, negative zeros, subnormals, big values
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 7.0, -0.25, -2.5, -5.0])
    for r in range(0, M, 3):
        row = torch.from_numpy(mids * 2.0 ** rng.integers(-20, 20)).to(torch.bfloat16)
        bits[r, 32:32 + len(mids)] = row.view(torch.int16).numpy().view(np.uint16)
    specials = [(slice(0, 64), 0),           # +0 blocks
                (slice(64, 96), 0x8000),     # -0 block
                (slice(96, 128), 0x0001),    # smallest BF16 subnormal
                (slice(128, 160), 0x7F7F),   # largest finite BF16
                (slice(160, 176), 0x8080)]   # negative subnormal
    for i, (cols, val) in enumerate(specials):
        bits[(i + 1) % M, cols] = val
    return bits


ACT_CASES = {
    "config1": lambda: synth.config1()[1],
    "config2": lambda: synth.config2(16)[1],
    "special_300x1024": lambda: special_activations(300, 1024, 1),
    "one_row": lambda: special_activations(1, 512, 2),
}


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("case", list(ACT_CASES))
def test_quantize_act_bitexact(fmt, case):
    x = ACT_CASES[case]()
    mx = mxc.quantize_act(dev_bf16(x), fmt)
    torch.cuda.synchronize()
    check_act(mx, x, fmt)


def every_bf16_value_blocks(e, K=1024):
    """Rows of 32-element blocks that hold every finite BF16 value v with |v| below the
    block maximum 1.5 * 2^(e+2), which every block also holds (first element): the
    E8M0 block exponent of every block is e."""
    amax = np.array([1.5 * 2.0 ** (e + 2)], dtype=np.float32)
    amax_bits = (amax.view(np.uint32) >> 16).astype(np.uint16)
    allb = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = (allb.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(vals) & (np.abs(vals) <= amax[0])
    vb = allb[keep]
    n_blocks = -(-len(vb) // 31)
    blocks = np.zeros((n_blocks, 32), dtype=np.uint16)
    blocks[:, 0] = amax_bits[0]
    flat = blocks[:, 1:].reshape(-1)
    flat[:len(vb)] = vb
    blocks[:, 1:] = flat.reshape(n_blocks, 31)
    per_row = K // 32
    rows = -(-n_blocks // per_row)
    out = np.zeros((rows * per_row, 32), dtype=np.uint16)
    out[:n_blocks] = blocks
    out[n_blocks:, 0] = amax_bits[0]
    return out.reshape(rows, K)


@pytest.mark.parametrize("e", [-127, -100, -30, -2, 0, 3, 40, 125])
def test_quantize_e8m0_every_bf16_value(e):
    """E8M0-B32 codes (by the tensor-core format conversion of x * 2^-e) for every BF16
    value below the block maximum, at block exponents across the E8M0 range:
    bit-exact against the oracle."""
    x = every_bf16_value_blocks(e)
    mx = mxc.quantize_act(dev_bf16(x), "e8m0_b32")
    torch.cuda.synchronize()
    check_act(mx, x, "e8m0_b32")


def test_quantize_act_given_tensor_scale():
    x = synth.config2(16)[1]
    ts = torch.tensor([0.0123], dtype=torch.float32, device="cuda")
    mx = mxc.quantize_act(dev_bf16(x), "e4m3_b16", tscale_in=ts)
    check_act(mx, x, "e4m3_b16", tscale=np.float32(0.0123))


# ---------------------------------------------------------------------------
# Weight decode: bit-exact
# ---------------------------------------------------------------------------

def check_decode(w):
    pw = mxc.pack_weight(w)
    d = mxc.decode_weight(pw)
    assert mxc.get_device_error() == 0
    codes_ref = O.pack_fp4(O.weight_codes(w))
    q = d.q.cpu().numpy()
    assert np.array_equal(q, codes_ref), f"decoded FP4 differ at {np.argwhere(q != codes_ref)[:5]}"
    sf = mxc.sf_to_rows(d.sf.cpu().numpy(), w.N, w.K, w.fmt)
    assert np.array_equal(sf, O.weight_scale_bytes(w))
    return pw, d


DECODE_CASES = [
    ("e8m0_b32", "prescale", 256, 1024, 0, 0),
    ("e8m0_b32", "postscale", 512, 1024, 256, 256),
    ("e8m0_b32", "prescale_plus", 384, 1536, 128, 128),
    ("e4m3_b16", "prescale", 256, 1024, 128, 128),
    ("e4m3_b16", "postscale", 256, 2048, 256, 1024),
    ("e4m3_b16", "prescale_plus", 512, 1024, 256, 256),
    ("e4m3_b16", "prescale_plus", 256, 768, 0, 0),
    ("e4m3_b16", "postscale_qb", 512, 1024, 256, 256),
    ("e8m0_b32", "postscale_qb", 256, 1024, 128, 128),
    ("e8m0_b32", "postscale_qb", 256, 1536, 128, 512),
    ("e4m3_b16", "postscale_qb", 384, 768, 0, 0),
]


@pytest.mark.parametrize("case", DECODE_CASES, ids=lambda c: "-".join(map(str, c)))
def test_decode_weight_bitexact(case):
    fmt, strat, N, K, qn, qk = case
    check_decode(synth.make_weight(11, fmt, strat, N, K, qn, qk))


def test_decode_config1_config2_full():
    check_decode(synth.config1()[0])
    check_decode(synth.config2(16)[0])


# ---------------------------------------------------------------------------
# Linear layers
# ---------------------------------------------------------------------------

def run_mxcode(w, x_bits, out_dtype=torch.float32):
    pw = mxc.pack_weight(w)
    a = mxc.quantize_act(dev_bf16(x_bits), w.fmt)
    y = mxc.linear(a, pw, out_dtype)
    assert mxc.get_device_error() == 0
    return y, pw, a


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("M", [1, 4, 16, 200])
def test_native_linear(fmt, M):
    w = synth.make_weight(21, fmt, "prescale", 256, 1024, 256, 256)
    x = synth.make_activations(21, M, 1024, outliers=True)
    pw = mxc.pack_weight(w)
    wn = mxc.decode_weight(pw)
    a = mxc.quantize_act(dev_bf16(x), fmt)
    y = mxc.native_linear(a, wn).cpu().numpy()
    assert mxc.get_device_error() == 0
    ref, sabs = O.w4a4_linear(x, w)
    assert_close(y, ref, sabs, what=f"native {fmt} M={M}")


def test_config1_mxcode():
    w, x = synth.config1()
    y, _, _ = run_mxcode(w, x)
    ref, sabs = O.w4a4_linear(x, w)
    assert_close(y.cpu().numpy(), ref, sabs, what="config1")


@pytest.mark.parametrize("M", [1, 4, 16])
def test_config2_decode_gemv(M):
    w, x = synth.config2(M)
    y, _, _ = run_mxcode(w, x)
    ref, sabs = O.w4a4_linear(x, w)
    assert_close(y.cpu().numpy(), ref, sabs, what=f"config2 M={M}")


SWEEP = [(f, s, qb) for f in ("e8m0_b32", "e4m3_b16")
         for s in ("postscale", "prescale", "prescale_plus", "postscale_qb") for qb in (0, 256, 128)]


@pytest.mark.parametrize("case", SWEEP, ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("M", [16, 130])
def test_mxcode_linear_sweep(case, M):
    fmt, strat, qb = case
    w = synth.make_weight(31, fmt, strat, 512, 1024, qb, qb)
    x = synth.make_activations(31, M, 1024, outliers=True)
    y, _, _ = run_mxcode(w, x)
    ref, sabs = O.w4a4_linear(x, w)
    assert_close(y.cpu().numpy(), ref, sabs, what=f"{case} M={M}")


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("M", [16, 300])
@pytest.mark.parametrize("strat", ["prescale_plus", "postscale_qb"])
def test_mxcode_equals_native_on_decoded_weights(fmt, M, strat):
    w = synth.make_weight(41, fmt, strat, 384, 2048, 128, 256)
    x = synth.make_activations(41, M, 2048, outliers=True)
    y, pw, a = run_mxcode(w, x)
    wn = mxc.decode_weight(pw)
    yn = mxc.native_linear(a, wn)
    assert torch.equal(y, yn)


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("M", [17, 77, 128])
@pytest.mark.parametrize("strat", ["prescale_plus", "postscale"])
def test_mid_m_split_k_through_the_workspace(fmt, M, strat):
    """17..128 tokens run the fused kernel on 128-token tiles; with the workspace given,
    each tile's K is split over CTAs (N = 512: 4 tiles x 4 ranks of 2 stages) whose
    scaled partials the last rank adds in rank order.  Checked against the oracle with
    FP32 and BF16 output, ragged token tiles included; MXCode and native FP4 on the same
    decoded operands take the same split and agree bit for bit; without a workspace the
    one-CTA-per-tile path runs and agrees within the bound."""
    w = synth.make_weight(71, fmt, strat, 512, 2048, 256, 256)
    x = synth.make_activations(71, M, 2048, outliers=True)
    assert mxc.lib().mxc_linear_workspace_bytes(M, 512, 2048, 1) == 4096 + 4 * 4 * 128 * 128 * 4
    y, pw, a = run_mxcode(w, x)
    ref, sabs = O.w4a4_linear(x, w)
    assert_close(y.cpu().numpy(), ref, sabs, what=f"split {strat} {fmt} M={M}")
    yb = mxc.linear(a, pw, torch.bfloat16)
    assert torch.equal(yb, y.to(torch.bfloat16))                  # BF16 = RNE of the same FP32 sum
    wn = mxc.decode_weight(pw)
    assert torch.equal(mxc.native_linear(a, wn), y)
    y1 = mxc.linear(a, pw, ws=torch.zeros(16, dtype=torch.uint8, device="cuda"))   # no room: no split
    assert mxc.get_device_error() == 0
    assert_close(y1.cpu().numpy(), ref, sabs, what=f"no split {strat} {fmt} M={M}")


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("M,K", [(129, 256), (300, 1536), (700, 1024), (1000, 4096)])
@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
def test_pair_gemm_equals_one_cta(fmt, M, K, out):
    """Native weights with 256-token tiles and N a multiple of 256 run on CTA pairs
    (cta_group::2, persistent); with N = 384 the one-CTA kernel runs.  On the same
    decoded operands the first 384 output channels must agree bit for bit, ragged
    token tiles included (a pair's second half past M), one stage (K = 256) included,
    and lie within the oracle's bound."""
    w = synth.make_weight(61, fmt, "prescale", 512, K, 256, 256)
    x = synth.make_activations(61, M, K, outliers=True)
    pw = mxc.pack_weight(w)
    wn = mxc.decode_weight(pw)
    a = mxc.quantize_act(dev_bf16(x), fmt)
    y = mxc.native_linear(a, wn, out)                              # N = 512: CTA pairs
    B = 32 if fmt == "e8m0_b32" else 16
    rows = 384                                                      # 128-row scale blocks are contiguous
    w384 = mxc.MXTensor(wn.q[:rows].contiguous(), wn.sf.view(-1)[: rows * K // B].contiguous(), wn.tscale,
                        rows, K, fmt)
    y384 = mxc.native_linear(a, w384, out)                          # N = 384: one CTA per tile
    assert mxc.get_device_error() == 0
    assert torch.equal(y[:, :rows], y384)
    ref, sabs = O.w4a4_linear(x, w)
    yy = y.float().cpu().numpy()
    bound = sabs if out == torch.float32 else sabs + np.abs(ref) * 2.0 ** -8 / TOL
    assert_close(yy, ref, bound, what=f"pair {fmt} M={M} K={K}")


def test_bf16_output():
    w = synth.make_weight(51, "e4m3_b16", "prescale", 256, 1024, 256, 256)
    x = synth.make_activations(51, 40, 1024, outliers=True)
    y, pw, a = run_mxcode(w, x, torch.bfloat16)
    y32 = mxc.linear(a, pw, torch.float32)
    ref_bf16 = y32.to(torch.bfloat16)               # RNE of the FP32 result
    assert torch.equal(y, ref_bf16)
    ref, sabs = O.w4a4_linear(x, w)
    yy = y.float().cpu().numpy()
    assert_close(yy, ref, sabs + np.abs(ref) * 2.0 ** -8 / TOL, what="bf16")


# ---------------------------------------------------------------------------
# Grouped experts (MoE)
# ---------------------------------------------------------------------------

def run_moe(fmt, strat, E, N, K, counts, seed, qn=256, qk=256):
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    M = int(offsets[-1])
    ws = [synth.make_weight(seed, fmt, strat, N, K, qn, qk, sub=e) for e in range(E)]
    x = synth.make_activations(seed, M, K, outliers=False)
    off_d = torch.from_numpy(offsets.astype(np.int32)).cuda()
    a = mxc.quantize_act_grouped(dev_bf16(x), fmt, off_d)
    packed = [mxc.pack_weight(w) for w in ws]
    y = mxc.moe_linear(a, off_d, packed).cpu().numpy()
    assert mxc.get_device_error() == 0
    # the activation tensor scale is shared by all rows
    codes, sf, s = O.quantize_act(x, fmt)
    a_hat = O.dequant_act(codes, sf, fmt, s)
    # grouped quantization must equal the dense one, row for row
    assert np.array_equal(a.q.cpu().numpy(), O.pack_fp4(codes))
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 == r0:
            continue
        w_hat = O.dequant_weight(ws[e])
        ref = O.linear(a_hat[r0:r1], w_hat)
        sabs = O.abs_linear(a_hat[r0:r1], w_hat)
        assert_close(y[r0:r1], ref, sabs, what=f"expert {e}")


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("strat", ["prescale", "prescale_plus", "postscale_qb"])
def test_moe_small(fmt, strat):
    run_moe(fmt, strat, 6, 256, 512, [0, 5, 130, 1, 257, 0], seed=61)


@pytest.mark.parametrize("fmt,strat,qn,qk", [("e4m3_b16", "prescale_plus", 128, 128),
                                              ("e8m0_b32", "postscale_qb", 256, 128),
                                              ("e4m3_b16", "prescale", 256, 512),
                                              ("e8m0_b32", "prescale_plus", 0, 0),
                                              ("e4m3_b16", "postscale", 512, 256)])
def test_moe_rounds(fmt, strat, qn, qk):
    """K = 1536: a full round of four 256-channel stages and a ragged one of two;
    QBlocks 128 wide along K (two codebooks a stage), 512 wide (one codebook for two
    stages) and the whole tensor; experts of 1 to 3 token tiles (a chunk of two
    tiles, a chunk of one, a ragged tile)."""
    run_moe(fmt, strat, 6, 512, 1536, [300, 0, 17, 129, 256, 1], seed=63, qn=qn, qk=qk)


def test_moe_bad_offsets_sets_device_error():
    E, N, K = 3, 128, 256
    ws = [mxc.pack_weight(synth.make_weight(71, "e8m0_b32", "prescale", N, K, 0, 0, sub=e)) for e in range(E)]
    x = synth.make_activations(71, 10, K, outliers=False)
    good = torch.tensor([0, 4, 7, 10], dtype=torch.int32, device="cuda")
    a = mxc.quantize_act_grouped(dev_bf16(x), "e8m0_b32", good)
    assert mxc.get_device_error() == 0
    bad = torch.tensor([0, 6, 3, 10], dtype=torch.int32, device="cuda")     # decreasing
    y = torch.full((10, N), 7.0, device="cuda")
    mxc.moe_linear(a, bad, ws, y=y)
    assert mxc.get_device_error() == 6                                       # MXC_ERR_DEVICE_INVALID
    assert torch.all(y == 7.0)                                               # nothing written
    assert mxc.get_device_error() == 0                                       # cleared by the read


# ---------------------------------------------------------------------------
# Decode GEMV (M <= 16): stage counts 1..8 per CTA, ragged last split, both
# codebook widths along K, cluster sizes 1..4, and the long-K fallback
# ---------------------------------------------------------------------------

GEMV_CASES = [
    (1024, 2048, 128, "e8m0_b32", "prescale_plus", 16),   # 2 stages per CTA, two codebooks per stage
    (256, 3072, 128, "e4m3_b16", "prescale", 7),          # 3 stages per CTA
    (2048, 5120, 256, "e8m0_b32", "prescale", 3),         # 5 stages per CTA
    (128, 7936, 0, "e4m3_b16", "postscale", 16),          # one tensor codebook, splits 8/8/8/7
    (9216, 4096, 128, "e4m3_b16", "postscale", 16),       # 8 stages, two codebooks per stage
    (18944, 1024, 256, "e4m3_b16", "prescale_plus", 2),   # 148 tiles: no split (cluster of 1)
    (256, 12288, 256, "e8m0_b32", "postscale", 5),        # 12 stages per CTA: pipelined kernel
    (9216, 4096, 256, "e4m3_b16", "postscale_qb", 16),    # PostScale-QB on the fused-QKV shape
    (1024, 2048, 128, "e8m0_b32", "postscale_qb", 1),     # PostScale-QB, two QBlocks per stage
]


@pytest.mark.parametrize("case", GEMV_CASES, ids=lambda c: "-".join(map(str, c)))
def test_decode_gemv_shapes(case):
    N, K, qb, fmt, strat, M = case
    w = synth.make_weight(61, fmt, strat, N, K, qb, qb)
    x = synth.make_activations(61, M, K, outliers=True)
    y, pw, a = run_mxcode(w, x)
    assert mxc.get_device_error() == 0
    ref, sabs = O.w4a4_linear(x, w)
    assert_close(y.cpu().numpy(), ref, sabs, what=f"{case}")
    yn = mxc.native_linear(a, mxc.decode_weight(pw))
    assert torch.equal(y, yn)


# ---------------------------------------------------------------------------
# Full-size workloads: sampled outputs and checksums (linearity) against the oracle
# ---------------------------------------------------------------------------

def _tile_and_checksums(y, a_hat, w_hat, rows, cols, what):
    yc = y.cpu().numpy().astype(np.float64)
    assert_close(yc[rows][:, cols], O.linear(a_hat[rows], w_hat[cols]), O.abs_linear(a_hat[rows], w_hat[cols]),
                 what=f"{what} tile")
    row, col, abs_row, abs_col = O.checksums(a_hat, w_hat)
    assert_close(yc.sum(axis=1), row, abs_row, what=f"{what} row sums")
    assert_close(yc.sum(axis=0), col, abs_col, what=f"{what} column sums")


def test_config3_full_size_prefill():
    """M=8192, K=4096, N=9216 (PreScale E8M0-B32): the decode-once path (workspace
    given) and the fused path (no workspace) are bit-identical; a seeded 256 x 256
    output tile and all row and column sums match the oracle."""
    w, x = synth.config3()
    pw = mxc.pack_weight(w)
    a = mxc.quantize_act(dev_bf16(x), w.fmt)
    y = mxc.linear(a, pw)
    y_fused = mxc.linear(a, pw, ws=torch.empty((16,), dtype=torch.uint8, device="cuda"))
    assert mxc.get_device_error() == 0
    assert torch.equal(y, y_fused)
    codes, sf, s = O.quantize_act(x, w.fmt)
    a_hat = O.dequant_act(codes, sf, w.fmt, s)
    w_hat = O.dequant_weight(w)
    rng = np.random.default_rng(3)
    r0, c0 = int(rng.integers(0, 8192 - 256)), int(rng.integers(0, 9216 - 256))
    _tile_and_checksums(y, a_hat, w_hat, np.arange(r0, r0 + 256), np.arange(c0, c0 + 256), "config 3")


@pytest.mark.parametrize("M", [16, 1024])
def test_config5_full_size_point(M):
    """K = N = 8192, PreScale E4M3-B16 with 256 x 256 QBlocks: M=16 (decode, pipelined
    kernel: 16 stages per split) and M=1024 (decode-once); oracle tile + checksums, and
    equality with native FP4 on the decoded weight."""
    w = synth.config5_weight(256, "prescale", "e4m3_b16")
    x = synth.config5_activations(M)
    pw = mxc.pack_weight(w)
    a = mxc.quantize_act(dev_bf16(x), w.fmt)
    y = mxc.linear(a, pw)
    yn = mxc.native_linear(a, mxc.decode_weight(pw))
    assert mxc.get_device_error() == 0
    assert torch.equal(y, yn)
    codes, sf, s = O.quantize_act(x, w.fmt)
    a_hat = O.dequant_act(codes, sf, w.fmt, s)
    w_hat = O.dequant_weight(w)
    rows = np.arange(M) if M <= 256 else np.random.default_rng(5).choice(M, 256, replace=False)
    _tile_and_checksums(y, a_hat, w_hat, rows, np.arange(8192 - 256, 8192), f"config 5 M={M}")


def test_config4_full_size_moe():
    """MoE gate/up at full size: 2048 tokens routed top-8 (Zipf 1.1) over 128 experts of
    [3072, 4096] (PreScale+ E4M3-B16) = 16384 expert-sorted rows.  The tensor scale is
    the oracle's; for the largest, the smallest and two fixed experts, up to 64 of
    their rows x 256 columns densely and the expert's row and column sums."""
    row_tok, off = synth.config4_routing()
    xg = synth.config4_activations("gate_up", row_tok)
    experts = [synth.config4_expert(e, "gate_up") for e in range(synth.MOE_EXPERTS)]
    packed = [mxc.pack_weight(w) for w in experts]
    offd = torch.from_numpy(off.astype(np.int32)).cuda()
    a = mxc.quantize_act_grouped(dev_bf16(xg), "e4m3_b16", offd)
    y = mxc.moe_linear(a, offd, packed)
    assert mxc.get_device_error() == 0
    s = O.tensor_scale_e4m3(xg)
    assert a.tscale.item() == np.float32(s)
    counts = np.diff(off)
    nonempty = np.flatnonzero(counts)
    for e in sorted({int(counts.argmax()), int(nonempty[counts[nonempty].argmin()]), 0, 127}):
        r0, r1 = int(off[e]), int(off[e + 1])
        if r1 == r0:
            continue
        codes, sf, _ = O.quantize_act(xg[r0:r1], "e4m3_b16", s)
        a_hat = O.dequant_act(codes, sf, "e4m3_b16", s)
        w_hat = O.dequant_weight(experts[e])
        rows = np.arange(min(64, r1 - r0))
        _tile_and_checksums(y[r0:r1], a_hat, w_hat, rows, np.arange(1024, 1280), f"expert {e}")


@pytest.mark.parametrize("M", [5, 16])
def test_decode_gemv_bf16_output(M):
    """Decode shape (N=9216, K=4096: two split-K ranks) with BF16 output, where the
    ranks hand their partial tiles over through distributed shared memory: equal to
    the RNE of the FP32 path (which adds the same two scaled partials in global
    memory), to native FP4, and within the oracle's bound plus BF16 rounding."""
    w = synth.make_weight(71, "e4m3_b16", "postscale", 9216, 4096, 256, 256)
    x = synth.make_activations(71, M, 4096, outliers=True)
    y16, pw, a = run_mxcode(w, x, torch.bfloat16)
    y32 = mxc.linear(a, pw, torch.float32)
    yn = mxc.native_linear(a, mxc.decode_weight(pw), torch.bfloat16)
    assert mxc.get_device_error() == 0
    assert torch.equal(y16, y32.to(torch.bfloat16))
    assert torch.equal(y16, yn)
    ref, sabs = O.w4a4_linear(x, w)
    assert_close(y16.float().cpu().numpy(), ref, sabs + np.abs(ref) * 2.0 ** -8 / TOL, what=f"bf16 M={M}")


# ---------------------------------------------------------------------------
# PreScale+ with larger scale groups (ds = 16, 32: Figure 3's higher scale
# compression ratios), through every kernel path
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("ds", [16, 32])
@pytest.mark.parametrize("M", [16, 130, 1024])
def test_prescale_plus_scale_groups(fmt, ds, M):
    """Decoded weight bit-exact; decode GEMV (M=16), fused GEMM (M=130) and decode-once
    (M=1024) within the oracle bound and equal to native FP4 on the decoded weight."""
    N, K = 512, 2048
    w = synth.make_weight(101, fmt, "prescale_plus", N, K, 256, 256, ds=ds)
    pw, d = check_decode(w)
    x = synth.make_activations(101, M, K, outliers=True)
    a = mxc.quantize_act(dev_bf16(x), fmt)
    y = mxc.linear(a, pw)
    yn = mxc.native_linear(a, d)
    assert mxc.get_device_error() == 0
    assert torch.equal(y, yn)
    rows = np.arange(M) if M <= 130 else np.arange(0, M, 7)
    codes, sf, s = O.quantize_act(x, fmt)
    a_hat = O.dequant_act(codes, sf, fmt, s)[rows]
    w_hat = O.dequant_weight(w)
    assert_close(y.cpu().numpy()[rows], O.linear(a_hat, w_hat), O.abs_linear(a_hat, w_hat),
                 what=f"ds={ds} {fmt} M={M}")


@pytest.mark.parametrize("ds", [16, 32])
def test_moe_prescale_plus_scale_groups(ds):
    E, N, K = 4, 256, 1024
    counts = [3, 0, 140, 20]
    offsets = np.concatenate([[0], np.cumsum(counts)])
    ws = [synth.make_weight(102, "e8m0_b32", "prescale_plus", N, K, 256, 256, sub=e, ds=ds) for e in range(E)]
    x = synth.make_activations(102, int(offsets[-1]), K, outliers=False)
    off_d = torch.from_numpy(offsets.astype(np.int32)).cuda()
    a = mxc.quantize_act_grouped(dev_bf16(x), "e8m0_b32", off_d)
    y = mxc.moe_linear(a, off_d, [mxc.pack_weight(w) for w in ws]).cpu().numpy()
    assert mxc.get_device_error() == 0
    codes, sf, s = O.quantize_act(x, "e8m0_b32")
    a_hat = O.dequant_act(codes, sf, "e8m0_b32", s)
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 > r0:
            w_hat = O.dequant_weight(ws[e])
            assert_close(y[r0:r1], O.linear(a_hat[r0:r1], w_hat), O.abs_linear(a_hat[r0:r1], w_hat),
                         what=f"moe ds={ds} expert {e}")


# ---------------------------------------------------------------------------
# QBlocks of 64 rows or 64 input channels (down to 64 x 64: Figure 3's sweep),
# decoded once per call by the direct-lookup decode kernel
# ---------------------------------------------------------------------------

SMALL_QB = [("e8m0_b32", "prescale", 64, 64), ("e4m3_b16", "postscale", 64, 64),
            ("e4m3_b16", "prescale_plus", 64, 256), ("e8m0_b32", "postscale_qb", 64, 64),
            ("e4m3_b16", "postscale_qb", 128, 64), ("e8m0_b32", "prescale_plus", 128, 64),
            ("e4m3_b16", "prescale", 64, 128)]


@pytest.mark.parametrize("case", SMALL_QB, ids=lambda c: "-".join(map(str, c)))
def test_small_qblock_decode_bitexact(case):
    fmt, strat, qn, qk = case
    check_decode(synth.make_weight(111, fmt, strat, 384, 1024, qn, qk))


@pytest.mark.parametrize("case", SMALL_QB[:4], ids=lambda c: "-".join(map(str, c)))
@pytest.mark.parametrize("M", [1, 16, 77, 130])
def test_small_qblock_linear(case, M):
    fmt, strat, qn, qk = case
    w = synth.make_weight(112, fmt, strat, 512, 1024, qn, qk)
    x = synth.make_activations(112, M, 1024, outliers=True)
    y, pw, a = run_mxcode(w, x)
    ref, sabs = O.w4a4_linear(x, w)
    assert_close(y.cpu().numpy(), ref, sabs, what=f"{case} M={M}")
    assert torch.equal(y, mxc.native_linear(a, mxc.decode_weight(pw)))
    # without the decode workspace the call refuses, and enqueues nothing
    yy = torch.full_like(y, 3.0)
    with pytest.raises(mxc.MxcError) as e:
        mxc.linear(a, pw, y=yy, ws=torch.empty((16,), dtype=torch.uint8, device="cuda"))
    assert e.value.status == 4                       # MXC_ERR_WORKSPACE
    assert torch.all(yy == 3.0)


def test_small_qblock_moe_is_refused():
    w = mxc.pack_weight(synth.make_weight(113, "e8m0_b32", "prescale", 256, 512, 64, 64))
    x = synth.make_activations(113, 8, 512, outliers=False)
    off = torch.tensor([0, 8], dtype=torch.int32, device="cuda")
    a = mxc.quantize_act_grouped(dev_bf16(x), "e8m0_b32", off)
    with pytest.raises(mxc.MxcError) as e:
        mxc.moe_linear(a, off, [w])
    assert e.value.status == 2                       # MXC_ERR_UNSUPPORTED


# ---------------------------------------------------------------------------
# Decode GEMV with split-K through the workspace (more than two ranks, or slices
# past 8 stages): no cluster, the last rank to arrive sums the partials in rank order
# ---------------------------------------------------------------------------

def _splitk_ws_layout(N, K, M=16):
    n = mxc.lib().mxc_linear_workspace_bytes(M, N, K, 1)
    return n, 4096                                   # the counter area leads every linear workspace


@pytest.mark.parametrize("fmt,strat,N,K,M", [
    ("e4m3_b16", "postscale", 512, 4096, 16),      # 4 ranks of 4 stages (cluster path: same split)
    ("e8m0_b32", "prescale", 256, 8192, 1),        # 4 ranks of 8 stages (cluster path: same split)
    ("e4m3_b16", "prescale_plus", 256, 9216, 16),  # 5 ranks, the last one 4 stages (cluster path: none)
    ("e8m0_b32", "postscale_qb", 256, 12288, 7),   # 6 ranks of 8 stages
    ("e4m3_b16", "native", 512, 2048, 16),         # native FP4 weights, 4 ranks of 2 stages
])
def test_gemv_splitk_through_workspace(fmt, strat, N, K, M):
    native = strat == "native"
    w = synth.make_weight(131, fmt, "prescale" if native else strat, N, K, 256, 256)
    x = synth.make_activations(131, M, K, outliers=True)
    a = mxc.quantize_act(dev_bf16(x), fmt)
    pw = mxc.pack_weight(w)
    wt = mxc.decode_weight(pw) if native else pw
    call = mxc.native_linear if native else mxc.linear
    n, ctr = _splitk_ws_layout(N, K, M)
    assert n > ctr
    ws = mxc.linear_workspace(M, N, K, fmt, "cuda")
    y = call(a, wt, ws=ws)
    assert mxc.get_device_error() == 0
    assert torch.count_nonzero(ws[:ctr]).item() == 0          # every counter back at zero
    ref, sabs = O.w4a4_linear(x, w)
    assert_close(y.cpu().numpy(), ref, sabs, what=f"{fmt} {strat} N={N} K={K} M={M}")
    # deterministic: the same bits again, and BF16 output is the rounding of FP32
    y2 = call(a, wt, ws=ws)
    yb = call(a, wt, out_dtype=torch.bfloat16, ws=ws)
    assert mxc.get_device_error() == 0
    assert torch.equal(y, y2)
    assert torch.equal(yb, y.to(torch.bfloat16))
    assert torch.count_nonzero(ws[:ctr]).item() == 0
    if not native:
        assert torch.equal(y, mxc.native_linear(a, mxc.decode_weight(pw)))
    # without the workspace the split-K cluster path runs; where it splits K the same
    # way (at most 4 ranks of at most 8 stages) it gives the same bits
    yc = call(a, wt, ws=torch.zeros((16,), dtype=torch.uint8, device="cuda"))
    assert mxc.get_device_error() == 0
    if K // 256 <= 32 and (K // 256) % 4 == 0:
        assert torch.equal(y, yc)
    else:
        assert_close(yc.cpu().numpy(), ref, sabs, what=f"{fmt} {strat} N={N} K={K} M={M} (no workspace)")


# ---------------------------------------------------------------------------
# Decode GEMV slices of 9 to 32 stages: rounds of 8 resident stages per CTA
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("fmt,strat,N,K,qk,M,out,ws", [
    ("e4m3_b16", "postscale", 6400, 4608, 256, 16, torch.float32, True),       # 2 ranks of 9: red.global.add
    ("e8m0_b32", "prescale", 4864, 7680, 128, 5, torch.bfloat16, True),        # 3 ranks of 10: cluster sum, 2 codebooks a stage
    ("e4m3_b16", "prescale_plus", 256, 10240, 256, 16, torch.float32, False),  # 4 ranks of 10 (no workspace)
    ("e8m0_b32", "postscale_qb", 256, 9216, 256, 1, torch.float32, False),     # 4 ranks of 9, one stage in the second round of 8
    ("e4m3_b16", "native", 6400, 4608, 256, 16, torch.bfloat16, True),         # native FP4 weights
    ("e4m3_b16", "postscale", 6400, 12288, 256, 16, torch.float32, True),      # 2 ranks of 24: three rounds
    ("e8m0_b32", "prescale_plus", 256, 32768, 256, 3, torch.bfloat16, False),  # 4 ranks of 32: four rounds
    ("e4m3_b16", "prescale_plus", 256, 10240, 128, 16, torch.float32, False),  # two codebooks a stage, scale VQ
    ("e8m0_b32", "postscale_qb", 512, 8704, 128, 9, torch.float32, False),     # two codebooks a stage, QBlock scales
])
def test_gemv_rounds(fmt, strat, N, K, qk, M, out, ws):
    native = strat == "native"
    w = synth.make_weight(141, fmt, "prescale" if native else strat, N, K, 256, qk)
    x = synth.make_activations(141, M, K, outliers=True)
    a = mxc.quantize_act(dev_bf16(x), fmt)
    pw = mxc.pack_weight(w)
    nat = mxc.decode_weight(pw)
    wsb = mxc.linear_workspace(M, N, K, fmt, "cuda") if ws else torch.zeros((16,), dtype=torch.uint8, device="cuda")
    y = (mxc.native_linear(a, nat, out, ws=wsb) if native else mxc.linear(a, pw, out, ws=wsb))
    assert mxc.get_device_error() == 0
    ref, sabs = O.w4a4_linear(x, w)
    if out == torch.float32:
        assert_close(y.cpu().numpy(), ref, sabs, what=f"{fmt} {strat} N={N} K={K} M={M}")
    else:
        # BF16 output: one more rounding of at most half an ulp of the FP32 value
        y32 = (mxc.native_linear(a, nat, ws=wsb) if native else mxc.linear(a, pw, ws=wsb))
        assert torch.equal(y, y32.to(torch.bfloat16))
        assert_close(y32.cpu().numpy(), ref, sabs, what=f"{fmt} {strat} N={N} K={K} M={M}")
    if not native:                                   # the same MMAs on the decoded weight
        assert torch.equal(y, mxc.native_linear(a, nat, out, ws=wsb))
    assert torch.equal(y, (mxc.native_linear(a, nat, out, ws=wsb) if native else mxc.linear(a, pw, out, ws=wsb)))
    assert mxc.get_device_error() == 0


def test_linear_workspace_shared_by_decode_once_and_split_k():
    """One workspace, zeroed once, serves a decode call that reduces through its arrival
    counters, a decode-once call (which writes the decoded weight past the counter area)
    and the decode call again: the counters stay valid and the results do not change."""
    fmt, N, K = "e4m3_b16", 512, 4096                # 4 output tiles: 4 split-K ranks at M <= 16
    w = synth.make_weight(151, fmt, "postscale", N, K, 256, 256)
    pw = mxc.pack_weight(w)
    x = synth.make_activations(151, 256, K, outliers=True)
    a16 = mxc.quantize_act(dev_bf16(x[:16]), fmt)
    a256 = mxc.quantize_act(dev_bf16(x), fmt)
    ws = mxc.linear_workspace(256, N, K, fmt, "cuda")
    assert ws.numel() >= mxc.lib().mxc_linear_workspace_bytes(16, N, K, 1) > 4096
    y1 = mxc.linear(a16, pw, ws=ws)
    y256 = mxc.linear(a256, pw, ws=ws)               # decode once into the same workspace
    y2 = mxc.linear(a16, pw, ws=ws)
    assert mxc.get_device_error() == 0
    assert torch.count_nonzero(ws[:4096]).item() == 0
    assert torch.equal(y1, y2)
    ref, sabs = O.w4a4_linear(x[:16], w)
    assert_close(y2.cpu().numpy(), ref, sabs, what="decode after decode once")
    ref256, sabs256 = O.w4a4_linear(x, w)
    assert_close(y256.cpu().numpy(), ref256, sabs256, what="decode once")
