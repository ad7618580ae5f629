"""Pins for the CPU oracle: each check ties an oracle function to something other
than itself -- the pages' printed numbers, closed forms of the formats, library
casts, exact-rational brute force, round trips and exact integer arithmetic.

Citations name "MXCode: Vector Quantization for MX-Native Inference at Scale"
(the method's paper) by table or caption.
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import mxcode_oracle as O
from vector_quantized_mx_b200 import synth


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


def bf16_bits(vals):
    return torch.tensor(vals, dtype=torch.float64).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ---------------------------------------------------------------------------
# Formats (Table 1)
# ---------------------------------------------------------------------------

def test_e2m1_values_match_bitfield_closed_form():
    # E2M1: sign s, exponent e (2 bits, bias 1), mantissa m (1 bit); e = 0 is subnormal.
    for c in range(16):
        s, e, m = c >> 3, (c >> 1) & 3, c & 1
        ref = (0.5 * m) if e == 0 else (2.0 ** (e - 1)) * (1 + m / 2)
        ref = -ref if s else ref
        assert O.e2m1_value(c) == ref


def test_e8m0_scale_range_table1(golden_dir):
    t1 = _load(golden_dir, "table1_formats.json")["formats"]["E8M0-B32-FP4"]
    assert O.e8m0_value(0) == 2.0 ** t1["min_positive_scale_log2"]
    mx = float(O.e8m0_value(254))
    assert float(f"{mx:.2e}") == t1["max_finite_scale"]
    # library decode: torch's float8_e8m0fnu cast, every non-NaN byte
    b = np.arange(255, dtype=np.uint8)
    lib = torch.from_numpy(b).view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    assert np.array_equal(O.e8m0_value(b), lib)
    with pytest.raises(ValueError):
        O.e8m0_value(255)


def test_e4m3_decode_vs_torch_and_table1(golden_dir):
    t1 = _load(golden_dir, "table1_formats.json")["formats"]["E4M3-B16-FP4"]
    b = np.array([x for x in range(256) if x not in (0x7F, 0xFF)], dtype=np.uint8)
    lib = torch.from_numpy(b).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(O.e4m3_value(b), lib)
    pos = O.e4m3_value(np.arange(1, 127))
    assert pos.min() == 2.0 ** t1["min_positive_scale_log2"]
    assert pos.max() == t1["max_finite_scale"]


def test_e4m3_encode_vs_torch_cast():
    rng = np.random.default_rng(7)
    vals = list(rng.uniform(0, 448, 20000).astype(np.float32))
    vals += list((rng.uniform(0, 2.0 ** -6, 5000)).astype(np.float32))  # subnormal range
    grid = O.e4m3_value(np.arange(0, 127))
    mids = ((grid[1:] + grid[:-1]) / 2).astype(np.float32)                # exact ties
    assert np.array_equal(mids.astype(np.float64), (grid[1:] + grid[:-1]) / 2)
    vals += list(mids) + list(grid.astype(np.float32))
    v = np.array(vals, dtype=np.float32)
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(O.e4m3_encode_rne_satfinite(v.astype(np.float64)), lib)


def test_e4m3_encode_saturates_at_table1_max():
    big = np.array([448.0, 449.0, 464.0, 465.0, 1e6, np.inf])
    assert np.all(O.e4m3_encode_rne_satfinite(big) == 0x7E)


def test_bf16_decode_vs_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    ok = ~np.isnan(lib)
    assert np.array_equal(O.bf16_value(bits)[ok], lib[ok])


# ---------------------------------------------------------------------------
# E2M1 round-to-nearest-even: exact rational brute force + worked examples
# ---------------------------------------------------------------------------

_E2M1_FR = [Fraction(0), Fraction(1, 2), Fraction(1), Fraction(3, 2), Fraction(2), Fraction(3), Fraction(4), Fraction(6)]


def _rne_e2m1_fraction(q: Fraction) -> int:
    """Nearest E2M1 magnitude by exact rational distance; a tie keeps the code whose mantissa bit is 0."""
    q = abs(q)
    best = None
    for c, v in enumerate(_E2M1_FR):
        d = abs(q - v)
        if best is None or d < best[0] or (d == best[0] and (c & 1) == 0):
            best = (d, c)
    return best[1]


def test_e2m1_rne_worked_examples(golden_dir):
    for ex in _load(golden_dir, "act_quant_worked_examples.json")["e2m1_rne"]:
        assert int(O.e2m1_encode_rne(ex["q"])) == ex["code"], ex


def test_e2m1_rne_bruteforce_rational():
    qs = [Fraction(i, 64) for i in range(0, 64 * 9)]
    qs += [Fraction(v) for v in (1e-30, 5.999999, 6.000001, 1e9)]
    got = O.e2m1_encode_rne(np.array([float(q) for q in qs]))
    ref = [_rne_e2m1_fraction(q) for q in qs]
    assert list(got) == ref


# ---------------------------------------------------------------------------
# Activation quantization
# ---------------------------------------------------------------------------

def test_e8m0_act_quant_worked_examples(golden_dir):
    for ex in _load(golden_dir, "act_quant_worked_examples.json")["e8m0_blocks"]:
        x = np.zeros((1, 32))
        x[0, 0] = ex["block_amax_element"]
        codes, sf = O.quantize_act_e8m0(bf16_bits(x))
        assert int(sf[0, 0]) == ex["scale_byte"], ex
        assert int(codes[0, 0]) == ex["code"], ex


def test_e8m0_act_quant_every_bf16_amax():
    """Every finite BF16 value v as a block's amax element (with a companion
    element w = v * 0.37 rounded to BF16).  Independent characterisation of the
    OCP MX shared scale: the exponent e is the unique integer with
    |v| / 2^e in [4, 8), clamped to [-127, 127]; codes by exact rational RNE."""
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    vals = O.bf16_value(bits)
    keep = np.isfinite(vals) & (vals != 0)
    bits, vals = bits[keep], vals[keep]
    comp = bf16_bits(vals * 0.37)
    x = np.zeros((len(bits), 32), dtype=np.uint16)
    x[:, 0] = bits
    x[:, 5] = comp
    codes, sf = O.quantize_act_e8m0(x)
    compv = O.bf16_value(comp)
    for i in range(0, len(bits), 7):   # every 7th value keeps the loop at a few seconds
        v = Fraction(float(vals[i]))
        e = 0
        while abs(v) / Fraction(2) ** e >= 8:
            e += 1
        while abs(v) / Fraction(2) ** e < 4:
            e -= 1
        e = max(-127, min(127, e))
        assert int(sf[i, 0]) == e + 127
        for col, val in ((0, v), (5, Fraction(float(compv[i])))):
            mag = _rne_e2m1_fraction(val / Fraction(2) ** e)
            sign = 8 if (val < 0 or (val == 0 and np.signbit(O.bf16_value(x[i, col])))) else 0
            assert int(codes[i, col]) == (mag | sign), (i, col)


def test_e8m0_all_zero_block_and_signed_zero():
    x = bf16_bits(np.array([[0.0] * 16 + [-0.0] * 16]))
    codes, sf = O.quantize_act_e8m0(x)
    assert sf[0, 0] == 0
    assert list(codes[0, :16]) == [0] * 16 and list(codes[0, 16:]) == [8] * 16


def test_e4m3_act_quant_worked_examples(golden_dir):
    for ex in _load(golden_dir, "act_quant_worked_examples.json")["e4m3_blocks"]:
        x = np.zeros((1, 32))
        x[0, 16] = ex["tensor_amax"]          # second block carries the tensor amax
        x[0, :len(ex["block"])] = ex["block"]
        codes, sf, s = O.quantize_act_e4m3(bf16_bits(x))
        assert s == np.float32(ex["tensor_amax"]) / np.float32(2688)
        assert int(sf[0, 0]) == ex["scale_byte"], ex
        assert list(codes[0, :len(ex["block"])]) == ex["codes"], ex


def test_e4m3_act_quant_fp32_recipe_and_exact_codes():
    """Scale steps against torch's FP32 arithmetic; code decisions against exact rationals."""
    w, _ = synth.config2(16)
    x = synth.config2(16)[1]
    codes, sf, s = O.quantize_act_e4m3(x)
    xt = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).float()
    amax_t = xt.abs().max()
    assert s == (amax_t / 2688.0).item()
    blocks = xt.reshape(16, -1, 16)
    t = (blocks.abs().amax(dim=2) / 6.0) / torch.tensor(s, dtype=torch.float32)
    sb_lib = t.clamp(max=448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(sf, sb_lib)
    denom = (torch.from_numpy(sf).view(torch.float8_e4m3fn).float() * torch.tensor(s, dtype=torch.float32)).numpy()
    rng = np.random.default_rng(3)
    xv = O.bf16_value(x)
    for _ in range(3000):
        m, kb, j = rng.integers(16), rng.integers(4096 // 16), rng.integers(16)
        val = Fraction(float(xv[m, kb * 16 + j]))
        d = Fraction(float(denom[m, kb]))
        mag = 0 if d == 0 else _rne_e2m1_fraction(val / d)
        assert int(codes[m, kb * 16 + j]) == (mag | (8 if np.signbit(xv[m, kb * 16 + j]) else 0))


def test_e4m3_zero_scale_block_gives_zero_codes():
    # tensor amax huge, one tiny block: amax_b/6/s underflows E4M3 -> scale byte 0 -> codes +-0
    x = np.zeros((1, 32))
    x[0, 16] = 3.0e38
    x[0, 0], x[0, 1] = 1e-3, -1e-3
    codes, sf, s = O.quantize_act_e4m3(bf16_bits(x))
    assert sf[0, 0] == 0
    assert codes[0, 0] == 0 and codes[0, 1] == 8


def test_fp4_packing_low_nibble_first():
    codes = np.array([[1, 2, 0xF, 0x8]], dtype=np.uint8)
    p = O.pack_fp4(codes)
    assert list(p[0]) == [0x21, 0x8F]
    assert np.array_equal(O.unpack_fp4(p), codes)


# ---------------------------------------------------------------------------
# Weight reconstruction: round trips through an encoder written here
# ---------------------------------------------------------------------------

def _encode_vq(target_codes, qn, qk):
    """Trivial exact VQ: per QBlock, the distinct 4-vectors become the codebook."""
    N, K = target_codes.shape
    idx = np.zeros((N, K // 4), dtype=np.uint8)
    cb = np.zeros((N // qn, K // qk, 256), dtype=np.uint16)
    for a in range(N // qn):
        for b in range(K // qk):
            blk = target_codes[a * qn:(a + 1) * qn, b * qk:(b + 1) * qk].reshape(qn, qk // 4, 4)
            keys = [tuple(int(c) for c in v) for v in blk.reshape(-1, 4)]
            table = sorted(set(keys))
            assert len(table) <= 256
            pos = {t: i for i, t in enumerate(table)}
            for i, t in enumerate(table):
                cb[a, b, i] = t[0] | (t[1] << 4) | (t[2] << 8) | (t[3] << 12)
            idx[a * qn:(a + 1) * qn, b * qk // 4:(b + 1) * qk // 4] = \
                np.array([pos[k] for k in keys], dtype=np.uint8).reshape(qn, qk // 4)
    return idx, cb


@pytest.mark.parametrize("qn,qk", [(8, 16), (16, 32), (32, 64)])
def test_weight_codes_round_trip(qn, qk):
    rng = np.random.default_rng(qn * 100 + qk)
    N, K = 64, 128
    target = np.zeros((N, K), dtype=np.uint8)
    for a in range(N // qn):
        for b in range(K // qk):
            palette = rng.integers(0, 16, size=(200, 4), dtype=np.uint8)
            pick = rng.integers(0, 200, size=(qn, qk // 4))
            target[a * qn:(a + 1) * qn, b * qk:(b + 1) * qk] = palette[pick].reshape(qn, qk)
    idx, cb = _encode_vq(target, qn, qk)
    w = synth.VQWeight("e8m0_b32", "prescale", N, K, qn, qk, idx, cb,
                       np.full((N, K // 32), 127, np.uint8), None, None, 1.0)
    assert np.array_equal(O.weight_codes(w), target)


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("ds", [8, 16, 32])
def test_scale_vq_round_trip(fmt, ds):
    """Scale VQ with groups of ds consecutive scales along K (Table 4 caption: ds = 8;
    Figure 3 b, c: higher scale-compression ratios): block scales drawn from a palette
    of ds-byte groups, encoded by an exact table written here, must come back."""
    rng = np.random.default_rng(11 + ds)
    B = O.BLOCK[fmt]
    N, K = 48, ds * B * 6
    palette = rng.integers(100, 140, size=(256, ds), dtype=np.uint8)
    groups = rng.integers(0, 256, size=(N, K // (ds * B)))
    target = palette[groups].reshape(N, K // B)
    table, inv = np.unique(target.reshape(-1, ds), axis=0, return_inverse=True)
    scb = np.zeros((256, ds), dtype=np.uint8)
    scb[:len(table)] = table
    sidx = inv.reshape(N, K // (ds * B)).astype(np.uint8)
    w = synth.VQWeight(fmt, "prescale_plus", N, K, N, K, np.zeros((N, K // 4), np.uint8),
                       np.zeros((1, 1, 256), np.uint16), None, sidx, scb, 1.0, ds)
    assert np.array_equal(O.weight_scale_bytes(w), target)
    # storage: one index byte per ds*B weights, plus the 256 x ds byte table
    assert O.bits_per_weight(fmt, "prescale_plus", N, K, N, K, scale_group=ds) == pytest.approx(
        8 / 4 + 4 * 4 * 256 / (N * K) + 8 / (ds * B) + 256 * ds * 8 / (N * K))
    assert O.storage_bytes(w) == N * K // 4 + 512 + N * K // (ds * B) + 256 * ds


# ---------------------------------------------------------------------------
# GEMM: exact integer special case and exact rationals
# ---------------------------------------------------------------------------

def test_linear_integer_special_case():
    """Block scales 2^-1 everywhere: 4*a and 4*w are integers (2 x E2M1 values),
    so 16*Y must equal an exact int64 matmul."""
    rng = np.random.default_rng(5)
    M, N, K = 24, 40, 256
    ca = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    cw = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    a_hat = O.dequant_act(ca, np.full((M, K // 32), 126, np.uint8), "e8m0_b32", 1.0)
    idx, cb = _encode_vq(cw, 8, 32)
    w = synth.VQWeight("e8m0_b32", "prescale", N, K, 8, 32, idx, cb,
                       np.full((N, K // 32), 126, np.uint8), None, None, 1.0)
    w_hat = O.dequant_weight(w)
    two = np.array([0, 1, 2, 3, 4, 6, 8, 12], dtype=np.int64)
    ia = np.where(ca & 8, -two[ca & 7], two[ca & 7])
    iw = np.where(cw & 8, -two[cw & 7], two[cw & 7])
    exact = ia @ iw.T
    assert np.array_equal((16 * O.linear(a_hat, w_hat)).astype(np.int64), exact)
    assert np.all(16 * O.linear(a_hat, w_hat) == exact)


def test_w4a4_linear_exact_rationals_tiny():
    """A 4 x 8 x 64 E4M3 case summed with exact fractions."""
    rng = np.random.default_rng(9)
    x = bf16_bits(rng.normal(size=(4, 64)))
    w = synth.make_weight(123, "e4m3_b16", "prescale", 8, 64, 0, 0)
    y, sabs = O.w4a4_linear(x, w)
    codes, sf, s = O.quantize_act_e4m3(x)
    a = O.dequant_act(codes, sf, "e4m3_b16", s)
    wh = O.dequant_weight(w)
    for m in range(4):
        for n in range(8):
            exact = sum(Fraction(float(a[m, k])) * Fraction(float(wh[n, k])) for k in range(64))
            assert abs(Fraction(float(y[m, n])) - exact) <= Fraction(2) ** -45 * max(1, abs(exact))


# ---------------------------------------------------------------------------
# The FP32 tensor scale of E4M3-B16 (Table 1: E4M3 block scales per 16 elements
# with an FP32 tensor scale): it multiplies every reconstructed activation and
# weight exactly once.  Each check below is computed without the oracle's
# dequant_* functions, from codes, scale bytes and tensor scales; a mutant of the
# oracle that drops, inverts or squares the factor must fail them.
# ---------------------------------------------------------------------------

_E4M3_ONE = 0x38                     # E4M3 byte of 1.0 (exponent 7 = bias, mantissa 0)
_TWICE_E2M1 = np.array([0, 1, 2, 3, 4, 6, 8, 12], dtype=np.int64)   # 2 x E2M1 magnitude


def _twice(codes):
    c = np.asarray(codes).astype(np.int64)
    return np.where(c & 8, -_TWICE_E2M1[c & 7], _TWICE_E2M1[c & 7])


def _e4m3_tscale_case(seed, M=12, N=24, K=256):
    """E4M3-B16 weight and activation codes, random positive block scales."""
    rng = np.random.default_rng(seed)
    ca = rng.integers(0, 16, size=(M, K), dtype=np.uint8)
    cw = rng.integers(0, 16, size=(N, K), dtype=np.uint8)
    sa = rng.integers(0x20, 0x50, size=(M, K // 16), dtype=np.uint8)
    sw = rng.integers(0x20, 0x50, size=(N, K // 16), dtype=np.uint8)
    idx, cb = _encode_vq(cw, 8, 64)
    return ca, cw, sa, sw, idx, cb


def _tensor_scale_pins_hold(O_mod) -> bool:
    """True when O_mod's reconstruction applies both FP32 tensor scales exactly once."""
    M, N, K = 12, 24, 256
    # (1) unit block scales, power-of-two tensor scales 2^-3 (weight), 2^-5 (activation):
    #     2a and 2w are integers, so 4 * 2^8 * Y equals an exact int64 matmul
    ca, cw, _, _, idx, cb = _e4m3_tscale_case(21, M, N, K)
    one_a = np.full((M, K // 16), _E4M3_ONE, np.uint8)
    one_w = np.full((N, K // 16), _E4M3_ONE, np.uint8)
    w = synth.VQWeight("e4m3_b16", "prescale", N, K, 8, 64, idx, cb, one_w, None, None, 2.0 ** -3)
    y = O_mod.linear(O_mod.dequant_act(ca, one_a, "e4m3_b16", 2.0 ** -5), O_mod.dequant_weight(w))
    exact = _twice(ca) @ _twice(cw).T
    if not np.array_equal(4.0 * 2.0 ** 8 * y, exact.astype(np.float64)):
        return False
    # (2) random E4M3 block scales and non-power-of-two FP32 tensor scales: Y equals the
    #     exact rational sum of code x block scale x tensor scale products (block scales
    #     decoded by torch's float8_e4m3fn cast, not by the oracle)
    ca, cw, sa, sw, idx, cb = _e4m3_tscale_case(22, M, N, K)
    ts_w = float(np.float32(1.0) / np.float32(2688.0))
    ts_a = float(np.float32(0.0123))
    w = synth.VQWeight("e4m3_b16", "prescale", N, K, 8, 64, idx, cb, sw, None, None, ts_w)
    y = O_mod.linear(O_mod.dequant_act(ca, sa, "e4m3_b16", ts_a), O_mod.dequant_weight(w))
    dec = lambda b: torch.from_numpy(np.ascontiguousarray(b)).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    va, vw = dec(sa), dec(sw)
    ia, iw = _twice(ca), _twice(cw)
    fa, fw = Fraction(ts_a), Fraction(ts_w)
    rng = np.random.default_rng(23)
    for _ in range(40):
        m, n = int(rng.integers(M)), int(rng.integers(N))
        ex = sum(Fraction(int(ia[m, k])) / 2 * Fraction(float(va[m, k // 16])) * fa *
                 Fraction(int(iw[n, k])) / 2 * Fraction(float(vw[n, k // 16])) * fw for k in range(K))
        if abs(Fraction(float(y[m, n])) - ex) > Fraction(2) ** -44 * max(abs(ex), Fraction(2) ** -200):
            return False
    return True


def test_tensor_scales_enter_exactly_once():
    assert _tensor_scale_pins_hold(O)


@pytest.mark.parametrize("mutant", ["drop", "invert", "square", "drop_weight"])
def test_tensor_scale_pins_catch_mutants(mutant):
    """The same pins on a copy of the oracle with a planted mistake in the tensor
    scale (on the CPU, in the oracle only): each mutant must fail them."""
    import types

    def dequant_act(codes, sf, fmt, tscale):
        B = O.BLOCK[fmt]
        S = np.repeat(O.scale_value(sf, fmt), B, axis=1)
        t = {"drop": 1.0, "invert": 1.0 / float(tscale), "square": float(tscale) ** 2,
             "drop_weight": float(tscale)}[mutant]
        return O.e2m1_value(codes) * S * t

    def dequant_weight(w):
        ts = 1.0 if mutant == "drop_weight" else w.w_tscale
        return dequant_act(O.weight_codes(w), O.weight_scale_bytes(w), w.fmt, ts)

    M_ = types.SimpleNamespace(linear=O.linear, dequant_act=dequant_act, dequant_weight=dequant_weight)
    assert not _tensor_scale_pins_hold(M_)


def test_w4a4_linear_scales_with_the_activation_tensor_scale():
    """E4M3-B16 end to end: multiplying the activation by 2^j multiplies its FP32
    tensor scale amax/2688 by 2^j and leaves every block scale byte and code alone,
    so the layer's output must scale by exactly 2^j (once, not squared or inverted)."""
    rng = np.random.default_rng(31)
    x = rng.normal(size=(6, 128))
    w = synth.make_weight(124, "e4m3_b16", "prescale", 16, 128, 0, 0)
    y0, _ = O.w4a4_linear(bf16_bits(x), w)
    for j in (-3, 5):
        yj, _ = O.w4a4_linear(bf16_bits(x * 2.0 ** j), w)
        assert np.array_equal(yj, y0 * 2.0 ** j)


def test_checksums_linearity():
    rng = np.random.default_rng(2)
    a = rng.normal(size=(33, 70))
    w = rng.normal(size=(21, 70))
    y = O.linear(a, w)
    row, col, abs_row, abs_col = O.checksums(a, w)
    assert np.allclose(row, y.sum(axis=1), rtol=0, atol=1e-10)
    assert np.allclose(col, y.sum(axis=0), rtol=0, atol=1e-10)
    assert np.allclose(abs_row, O.abs_linear(a, w).sum(axis=1))
    assert np.allclose(abs_col, O.abs_linear(a, w).sum(axis=0))


# ---------------------------------------------------------------------------
# Storage accounting vs the pages' BPE numbers (Table 1, Table 2, Table 4 caption)
# ---------------------------------------------------------------------------

def test_bpe_native_table1_table2(golden_dir):
    t1 = _load(golden_dir, "table1_formats.json")["formats"]
    t2 = _load(golden_dir, "table2_bpe.json")["values"]
    assert O.native_bits_per_weight("e8m0_b32") == t1["E8M0-B32-FP4"]["bpe"] == t2["E8M0-B32-FP4"]["native"]
    assert O.native_bits_per_weight("e4m3_b16") == t1["E4M3-B16-FP4"]["bpe"] == t2["E4M3-B16-FP4"]["native"]


def test_bpe_mxcode_table2(golden_dir):
    g = _load(golden_dir, "table2_bpe.json")
    N, K = g["readings"]["prescale_plus_tensor_shape"]
    for name, fmt in (("E4M3-B16-FP4", "e4m3_b16"), ("E8M0-B32-FP4", "e8m0_b32")):
        r = g["readings"][name]
        for strat in ("postscale", "prescale", "prescale_plus"):
            bpw = O.bits_per_weight(fmt, strat, N, K, r["qblock"], r["qblock"],
                                    postscale_block_scales=r["postscale_block_scales"])
            assert round(bpw, 2) == g["values"][name][strat], (name, strat, bpw)


def test_bpe_postscale_qb_table2(golden_dir):
    """PostScale-QB (one scale per QBlock) gives Table 2's PostScale column."""
    g = _load(golden_dir, "table2_bpe.json")
    for name, fmt in (("E4M3-B16-FP4", "e4m3_b16"), ("E8M0-B32-FP4", "e8m0_b32")):
        qb = g["readings"][name]["qblock"]
        bpw = O.bits_per_weight(fmt, "postscale_qb", 9216, 4096, qb, qb)
        assert round(bpw, 2) == g["values"][name]["postscale"], (name, bpw)


@pytest.mark.parametrize("fmt,qn,qk", [("e4m3_b16", 128, 256), ("e8m0_b32", 256, 128), ("e8m0_b32", 128, 512)])
def test_postscale_qb_dequant_expands_the_qblock_scale(fmt, qn, qk):
    """Dequantizing a PostScale-QB weight equals dequantizing the same weight with
    per-block scales copied, block by block, from the QBlock that holds the block
    (expanded here with explicit loops over rows and K ranges)."""
    w = synth.make_weight(9, fmt, "postscale_qb", 256, 1024, qn, qk)
    assert w.scales.shape == (256 // qn, 1024 // qk)
    B = O.BLOCK[fmt]
    per_block = np.zeros((256, 1024 // B), dtype=np.uint8)
    for n in range(256):
        for kb in range(1024 // B):
            k0 = kb * B                              # first input channel of the block
            per_block[n, kb] = w.scales[n // qn][k0 // qk]
    direct = type(w)(fmt, "postscale", 256, 1024, qn, qk, w.idx, w.cb, per_block, None, None, w.w_tscale)
    assert np.array_equal(O.weight_scale_bytes(w), per_block)
    assert np.array_equal(O.dequant_weight(w), O.dequant_weight(direct))
    assert O.storage_bytes(w) * 8 / (256 * 1024) == pytest.approx(
        O.bits_per_weight(fmt, "postscale_qb", 256, 1024, qn, qk))


def test_index_bits_table4_caption(golden_dir):
    g = _load(golden_dir, "table2_bpe.json")["index_bits_per_weight"]
    # a full-tensor codebook on a large tensor leaves only the index bits (+ direct scales)
    bpw = O.bits_per_weight("e8m0_b32", "postscale", 1 << 20, 1 << 20, 0, 0, postscale_block_scales=False)
    assert abs(bpw - g["value"]) < 1e-6


def test_storage_bytes_matches_bpe():
    w = synth.make_weight(1, "e4m3_b16", "prescale", 512, 1024, 256, 256)
    assert O.storage_bytes(w) * 8 / (512 * 1024) == pytest.approx(
        O.bits_per_weight("e4m3_b16", "prescale", 512, 1024, 256, 256))


# ---------------------------------------------------------------------------
# Generator sanity (closed forms of the sampling distributions)
# ---------------------------------------------------------------------------

def test_zipf_routing_first_choice_matches_closed_form():
    row_tok, off = synth.config4_routing()
    assert off[-1] == synth.MOE_TOKENS * synth.MOE_TOPK and np.all(np.diff(off) >= 0)
    # every token appears top_k times with distinct experts
    exp_of_row = np.repeat(np.arange(synth.MOE_EXPERTS), np.diff(off))
    pairs = set(zip(row_tok.tolist(), exp_of_row.tolist()))
    assert len(pairs) == synth.MOE_TOKENS * synth.MOE_TOPK
    # Gumbel-max: the arg-max choice follows p_i = i^-s / H exactly
    rng = synth.stream(99, "route")
    E, s, T = 128, 1.1, 200000
    logp = -s * np.log(np.arange(1, E + 1))
    first = np.argmax(logp[None, :] + rng.gumbel(size=(T, E)), axis=1)
    H = sum(i ** -s for i in range(1, E + 1))
    p1 = 1 / H
    assert abs(H - 4.431) < 5e-3
    assert abs(np.mean(first == 0) - p1) < 4 * math.sqrt(p1 * (1 - p1) / T)


# ---------------------------------------------------------------------------
# SwiGLU and the FP32-value quantization of the down projection's activation
# (MoE expert tensors, Table 4 caption): pinned to FP64 mathematics, to special
# values, and to the BF16 quantizers above on values both can take.
# ---------------------------------------------------------------------------

def test_exp_fp32_matches_the_exponential():
    x = np.linspace(-86.0, 88.0, 400001).astype(np.float32)
    x = np.concatenate([x, np.float32([0.0, -0.0, 1.0, -1.0, 0.5, 1e-30, -1e-30])])
    e = O.exp_fp32(x).astype(np.float64)
    ref = np.exp(x.astype(np.float64))
    assert np.all(np.abs(e - ref) <= 2 * 2.0 ** -24 * ref)          # within 2 ulp
    assert O.exp_fp32(np.float32(0.0)) == 1.0
    assert np.all(O.exp_fp32(np.float32([88.5, 100.0, 1e30])) == np.inf)
    assert np.all(O.exp_fp32(np.float32([-86.5, -100.0, -1e30])) == 0.0)
    # FP32 in, FP32 out, a fixed function of its input
    assert O.exp_fp32(x).dtype == np.float32
    assert np.array_equal(O.exp_fp32(x), O.exp_fp32(x.copy()))


def test_swiglu_fp32_matches_fp64_silu_times_up():
    rng = np.random.default_rng(41)
    g = np.concatenate([np.linspace(-40, 40, 200001), rng.normal(0, 4, 100000)]).astype(np.float32)
    u = rng.normal(0, 2, g.size).astype(np.float32)
    h = O.swiglu_fp32(g, u).astype(np.float64)
    gd, ud = g.astype(np.float64), u.astype(np.float64)
    ref = gd / (1.0 + np.exp(-gd)) * ud
    ok = np.abs(ref) > 1e-35
    assert np.all(np.abs(h - ref)[ok] <= 6 * 2.0 ** -24 * np.abs(ref[ok]))   # a few FP32 roundings
    # special values: SiLU(0) = 0, SiLU(g) = g for large g, -0 for very negative g
    sp = O.swiglu_fp32(np.float32([0.0, 100.0, -100.0, 3e38]), np.float32([5.0, 2.0, 7.0, 1.0]))
    assert sp[0] == 0.0 and sp[1] == 200.0 and sp[2] == 0.0 and np.signbit(sp[2]) and sp[3] == np.float32(3e38)


def test_fp32_value_quantizers_equal_the_bf16_ones_on_bf16_values():
    rng = np.random.default_rng(43)
    bits = bf16_bits(rng.normal(size=(6, 256)) * np.exp(rng.uniform(-10, 10, (6, 1))))
    vals = O.bf16_value(bits).astype(np.float32)
    c1, s1 = O.quantize_act_e8m0(bits)
    c2, s2 = O.quantize_values_e8m0(vals)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)
    ts = np.float32(0.0371)
    c1, s1, _ = O.quantize_act_e4m3(bits, ts)
    c2, s2 = O.quantize_values_e4m3(vals, ts)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_fp32_value_quantizers_exact_decisions():
    """Random FP32 values (24-bit mantissas, not BF16): the E8M0 exponent by the
    |v| / 2^e in [4, 8) characterisation, the E4M3 scale by torch's FP32 arithmetic
    and float8 cast, every code by exact rational rounding."""
    rng = np.random.default_rng(47)
    v = (rng.normal(size=(4, 64)) * np.exp(rng.uniform(-6, 6, (4, 1)))).astype(np.float32)
    codes, sf = O.quantize_values_e8m0(v)
    for r in range(4):
        for b in range(2):
            blk = [Fraction(float(t)) for t in v[r, 32 * b:32 * b + 32]]
            amax = max(abs(t) for t in blk)
            e = 0
            while amax / Fraction(2) ** e >= 8:
                e += 1
            while amax / Fraction(2) ** e < 4:
                e -= 1
            assert int(sf[r, b]) == e + 127
            for j, t in enumerate(blk):
                assert int(codes[r, 32 * b + j]) == _rne_e2m1_fraction(t / Fraction(2) ** e) | (8 if t < 0 else 0)
    s = np.float32(0.0123)
    codes, sb = O.quantize_values_e4m3(v, s)
    vt = torch.from_numpy(v).reshape(4, 4, 16)
    t = (vt.abs().amax(dim=2) / 6.0) / torch.tensor(s)
    assert np.array_equal(sb, t.clamp(max=448.0).to(torch.float8_e4m3fn).view(torch.uint8).numpy())
    denom = (torch.from_numpy(sb).view(torch.float8_e4m3fn).float() * torch.tensor(s)).numpy()
    for r in range(4):
        for k in range(64):
            d = Fraction(float(denom[r, k // 16]))
            val = Fraction(float(v[r, k]))
            mag = 0 if d == 0 else _rne_e2m1_fraction(val / d)
            assert int(codes[r, k]) == mag | (8 if val < 0 else 0)


def test_swiglu_quantize_splits_gate_and_up():
    rng = np.random.default_rng(53)
    y = rng.normal(0, 3, (5, 2 * 64)).astype(np.float32)
    c, s = O.swiglu_quantize(y, "e8m0_b32")
    c2, s2 = O.quantize_values_e8m0(O.swiglu_fp32(y[:, :64], y[:, 64:]))
    assert np.array_equal(c, c2) and np.array_equal(s, s2)
    c, s = O.swiglu_quantize(y, "e4m3_b16", 0.01)
    c2, s2 = O.quantize_values_e4m3(O.swiglu_fp32(y[:, :64], y[:, 64:]), 0.01)
    assert np.array_equal(c, c2) and np.array_equal(s, s2)
