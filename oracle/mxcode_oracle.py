"""CPU oracle for the MXCode W4A4 linear layer -- TEST INFRASTRUCTURE ONLY.

This is the plain, slow, exact reference that the CUDA path is checked
against.  Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline and
reference legs may import it; the library never does, and it shares no code
with the library (it has its own copies of every format rule).

What it computes, and where the method defines it
("MXCode: Vector Quantization for MX-Native Inference at Scale"):

* Formats (Table 1 and its caption): E2M1 elements; E8M0 block scales per 32
  elements (min 2^-127, max ~1.70e38); E4M3 block scales per 16 elements
  (min 2^-9, max 448) with an optional FP32 tensor scale.
* Weight reconstruction (abstract; Table 4 caption): a uint8 index per d=4
  consecutive weights along the input-channel axis selects one of K=256 FP4
  centroids of the weight's QBlock; the centroid's E2M1 codes are scaled by the
  MX block scale.  PostScale/PreScale store block scales directly; PreScale+
  VQ-codes groups of ds=8 scales with a Ks=256-entry scale codebook.
  PostScale-QB ("postscale_qb"): PostScale as Table 2's bits per weight imply
  (2.06 for E4M3-B16 at 256 x 256 QBlocks, 2.25 for E8M0-B32 at 128 x 128): the
  MXFP4-quantized codebook carries one scale, shared by every block of its
  QBlock, so no per-block weight scales are stored.
* W4A4 (abstract; Table 2 caption): activations are MX-quantized to FP4 too.
  The pages give no activation recipe; the oracle follows the OCP MX rule
  (shared scale from the block's amax, E2M1 round-to-nearest-even, saturate at
  +-6) and, for E4M3-B16, an FP32 tensor scale amax/(6*448).
* Storage accounting (Table 2 "Weight (BPE)" row; Figure 3 caption): indices +
  FP4 codebooks + scales (+ scale-VQ metadata), tensor scale excluded.
* The MoE FFN step between the gate/up and down projections (Table 4 caption:
  Qwen3's MoE expert tensors): h = SiLU(gate) * up in FP32 with a fixed FP32 exp,
  and the MX quantization of FP32 values (end of this file).

Where the pages leave a point open (the activation recipe, nibble order, scale-VQ
grouping, QBlock tiling, the PostScale storage), the function that decides it
states the reading it takes in its docstring.
Everything is FP64 except the FP32 steps of the E4M3 scale recipe and of SwiGLU,
which are done in FP32 on purpose because they are defined in FP32.

Parity pins: every function here is pinned by tests/test_oracle_pins.py to
something other than itself (closed forms, library routines, brute force,
round trips, the pages' own numbers).  None is "parity unpinned".
"""
from __future__ import annotations

import math
from typing import Optional

import numpy as np

E8M0_B32 = "e8m0_b32"
E4M3_B16 = "e4m3_b16"
BLOCK = {E8M0_B32: 32, E4M3_B16: 16}

# ---------------------------------------------------------------------------
# Element and scale formats (Table 1: "All use E2M1 elements and 8-bit block
# scales"; ranges of the block scales).
# ---------------------------------------------------------------------------

# E2M1: 1 sign bit (bit 3), 2 exponent bits, 1 mantissa bit.
E2M1_MAG = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


def e2m1_value(codes) -> np.ndarray:
    """Value of 4-bit E2M1 codes (bit 3 = sign)."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    mag = E2M1_MAG[c & 7]
    return np.where(c & 8, -mag, mag)


def e8m0_value(b) -> np.ndarray:
    """E8M0 scale byte b -> 2^(b-127).  0xFF is NaN and is rejected."""
    b = np.asarray(b).astype(np.int64)
    if np.any(b == 255):
        raise ValueError("E8M0 byte 0xFF is NaN")
    return np.ldexp(1.0, b - 127)


def e4m3_value(b) -> np.ndarray:
    """E4M3 (bias 7, no infinities, S.1111.111 = NaN) byte -> value."""
    b = np.asarray(b).astype(np.int64)
    s = (b >> 7) & 1
    e = (b >> 3) & 0xF
    m = b & 7
    if np.any((e == 15) & (m == 7)):
        raise ValueError("E4M3 NaN byte")
    mag = np.where(e == 0, m * 2.0 ** -9, np.ldexp(1.0 + m / 8.0, e - 7))
    return np.where(s == 1, -mag, mag)


_E4M3_POS_BYTES = np.arange(0, 127)             # 0x00 .. 0x7E: every non-negative finite value
_E4M3_POS_VALUES = e4m3_value(_E4M3_POS_BYTES)  # increasing


def e4m3_encode_rne_satfinite(v) -> np.ndarray:
    """Non-negative value -> nearest E4M3 byte (ties to even mantissa), saturating at 448.

    Nearest-value search over all 127 non-negative finite E4M3 values.  Values
    above 448 map to 448 (0x7E): the format's largest finite scale (Table 1).
    """
    v = np.asarray(v, dtype=np.float64)
    if np.any(v < 0) or np.any(np.isnan(v)):
        raise ValueError("E4M3 scale must be non-negative")
    flat = np.minimum(v.reshape(-1), 448.0)
    d = np.abs(flat[:, None] - _E4M3_POS_VALUES[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    # at most two candidates (adjacent bytes); prefer the even byte (= even mantissa)
    even = cand & ((_E4M3_POS_BYTES[None, :] & 1) == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    return _E4M3_POS_BYTES[pick].astype(np.uint8).reshape(v.shape)


def bf16_value(bits) -> np.ndarray:
    """BF16 bit patterns (uint16) -> FP64 (exact)."""
    b = np.asarray(bits).astype(np.uint32) << 16
    with np.errstate(invalid="ignore"):   # NaN patterns stay NaN
        return b.view(np.float32).astype(np.float64)


def e2m1_encode_rne(q) -> np.ndarray:
    """|q| -> E2M1 magnitude code 0..7: nearest value, ties to even code, saturating at 6.

    Ties sit between two adjacent codes, one even (mantissa bit 0) and one
    odd; round-half-to-even keeps the even one.  Anything above 6 is nearest
    to 6 (there is no larger E2M1 value), which is the saturation rule.
    """
    a = np.abs(np.asarray(q, dtype=np.float64)).reshape(-1)
    d = np.abs(a[:, None] - E2M1_MAG[None, :])
    dmin = d.min(axis=1, keepdims=True)
    cand = d == dmin
    even = cand & ((np.arange(8)[None, :] & 1) == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    return pick.astype(np.uint8).reshape(np.shape(q))


# ---------------------------------------------------------------------------
# Activation MX quantization (W4A4; OCP MX rule -- see module docstring)
# ---------------------------------------------------------------------------

def _signed_codes(x: np.ndarray, q: np.ndarray) -> np.ndarray:
    """E2M1 codes of x/scale = q, keeping the sign of x (so -0 -> 0x8)."""
    return e2m1_encode_rne(q) | (np.signbit(x).astype(np.uint8) << 3)


def quantize_act_e8m0(x_bits: np.ndarray):
    """E8M0-B32 activation quantization.

    Per block of 32 along K: amax = max|x|.  amax = 0 gives scale byte 0 and
    signed zero codes.  Otherwise e = floor(log2 amax) - 2 (2 = E2M1's largest
    exponent), clamped to [-127, 127], scale byte e+127, and every element
    becomes RNE_E2M1(x / 2^e), saturating at +-6.

    Returns (codes uint8 [M, K], sf uint8 [M, K/32]).
    """
    x = bf16_value(x_bits)
    M, K = x.shape
    xb = x.reshape(M, K // 32, 32)
    amax = np.abs(xb).max(axis=2)
    _, ex = np.frexp(amax)                    # amax = f * 2^ex, f in [0.5, 1)
    e = np.clip(ex.astype(np.int64) - 1 - 2, -127, 127)
    e = np.where(amax == 0, -127, e)
    q = xb / np.ldexp(1.0, e)[:, :, None]     # exact: division by a power of two
    codes = _signed_codes(xb, q)
    return codes.reshape(M, K), (e + 127).astype(np.uint8)


def tensor_scale_e4m3(x_bits: np.ndarray) -> np.float32:
    """FP32 activation tensor scale amax(|x|) / 2688 (2688 = 6 * 448); 1.0 if all zero."""
    amax = np.float32(np.abs(bf16_value(x_bits)).max()) if np.size(x_bits) else np.float32(0)
    if amax == 0:
        return np.float32(1.0)
    return np.float32(amax) / np.float32(2688.0)


def quantize_act_e4m3(x_bits: np.ndarray, tscale: Optional[float] = None):
    """E4M3-B16 activation quantization with an FP32 tensor scale s.

    s = amax_tensor/2688 in FP32 (or the caller's value).  Per block of 16:
    sb = E4M3_RNE_satfinite(fp32(fp32(amax_b / 6) / s)); sb = 0 gives signed
    zero codes; otherwise denom = fp32(value(sb) * s) and each element becomes
    RNE_E2M1(x / denom), decided exactly (FP64 division of a BF16 by an FP32
    cannot land on a rounding midpoint unless the exact quotient does).

    Returns (codes uint8 [M, K], sf uint8 [M, K/16], s as np.float32).
    """
    s = tensor_scale_e4m3(x_bits) if tscale is None else np.float32(tscale)
    x = bf16_value(x_bits)
    M, K = x.shape
    xb = x.reshape(M, K // 16, 16)
    amax = np.abs(xb).max(axis=2).astype(np.float32)
    t = (amax / np.float32(6.0)).astype(np.float32)
    t = (t / s).astype(np.float32)
    sb = e4m3_encode_rne_satfinite(np.where(np.isfinite(t), t, np.float64(448.0)))
    denom = (e4m3_value(sb).astype(np.float32) * s).astype(np.float32).astype(np.float64)
    safe = np.where(denom == 0, 1.0, denom)
    q = np.where((sb == 0)[:, :, None], 0.0, xb / safe[:, :, None])
    codes = _signed_codes(xb, q)
    return codes.reshape(M, K), sb.astype(np.uint8), np.float32(s)


def quantize_act(x_bits: np.ndarray, fmt: str, tscale: Optional[float] = None):
    """-> (codes [M,K], sf [M,K/B], tensor scale as float)."""
    if fmt == E8M0_B32:
        c, sf = quantize_act_e8m0(x_bits)
        return c, sf, 1.0
    c, sf, s = quantize_act_e4m3(x_bits, tscale)
    return c, sf, float(s)


def pack_fp4(codes: np.ndarray) -> np.ndarray:
    """[M, K] codes -> [M, K/2] bytes, element 2i in the low nibble of byte i."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] & 0xF) | ((c[:, 1::2] & 0xF) << 4)


def unpack_fp4(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.uint8)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def scale_value(sf, fmt: str) -> np.ndarray:
    return e8m0_value(sf) if fmt == E8M0_B32 else e4m3_value(sf)


def dequant_act(codes: np.ndarray, sf: np.ndarray, fmt: str, tscale: float) -> np.ndarray:
    """Exact value of quantized activations: code * block scale * tensor scale (FP64)."""
    B = BLOCK[fmt]
    S = np.repeat(scale_value(sf, fmt), B, axis=1)
    return e2m1_value(codes) * S * float(tscale)


# ---------------------------------------------------------------------------
# Weight reconstruction (abstract; Table 4 caption)
# ---------------------------------------------------------------------------

def weight_codes(w) -> np.ndarray:
    """FP4 codes [N, K] of a VQ weight: nibble (k mod 4) of cb[n//qn, k//qk, idx[n, k//4]]."""
    N, K, qn, qk = w.N, w.K, w.qn, w.qk
    n = np.arange(N)[:, None]
    k = np.arange(K)[None, :]
    entry = w.cb[n // qn, k // qk, w.idx[n, k // 4]]
    return ((entry >> (4 * (k % 4))) & 0xF).astype(np.uint8)


def weight_scale_bytes(w) -> np.ndarray:
    """Block-scale bytes [N, K/B]: stored directly, scb[sidx[n, kb//ds], kb % ds] (PreScale+,
    groups of ds consecutive scales along K; ds = 8 in Table 4's caption, larger ds are the
    higher scale-compression ratios of Figure 3 (b, c); the weight's `ds`, 8 if it has none),
    or the QBlock's scale scales[n//qn, (kb*B)//qk] (PostScale-QB)."""
    if w.strategy == "postscale_qb":
        B = BLOCK[w.fmt]
        n = np.arange(w.N)[:, None]
        kb = np.arange(w.K // B)[None, :]
        return np.asarray(w.scales, dtype=np.uint8)[n // w.qn, (kb * B) // w.qk]
    if w.strategy == "prescale_plus":
        KB = w.K // BLOCK[w.fmt]
        kb = np.arange(KB)[None, :]
        n = np.arange(w.N)[:, None]
        ds = getattr(w, "ds", 8)
        return w.scb[w.sidx[n, kb // ds], kb % ds].astype(np.uint8)
    return np.asarray(w.scales, dtype=np.uint8)


def dequant_weight(w) -> np.ndarray:
    """Exact W[N, K] (FP64) = E2M1(code) * block scale * tensor scale."""
    return dequant_act(weight_codes(w), weight_scale_bytes(w), w.fmt, w.w_tscale)


# ---------------------------------------------------------------------------
# The W4A4 linear layer
# ---------------------------------------------------------------------------

def linear(a_hat: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """Y[M, N] = sum_k a[m,k] w[n,k] in FP64."""
    return a_hat @ w_hat.T


def abs_linear(a_hat: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    """sum_k |a[m,k] w[n,k]|: the scale of the per-element tolerance."""
    return np.abs(a_hat) @ np.abs(w_hat).T


def w4a4_linear(x_bits: np.ndarray, w, y_rows=None, y_cols=None):
    """Quantize activations, reconstruct weights, multiply.

    Optional row/column subsets restrict the output to Y[y_rows][:, y_cols]
    (the activation quantization still sees the whole tensor, because the
    E4M3 tensor scale depends on all of it).  Returns (Y, sum|a w|).
    """
    codes, sf, s = quantize_act(x_bits, w.fmt)
    a_hat = dequant_act(codes, sf, w.fmt, s)
    w_hat = dequant_weight(w)
    if y_rows is not None:
        a_hat = a_hat[y_rows]
    if y_cols is not None:
        w_hat = w_hat[y_cols]
    return linear(a_hat, w_hat), abs_linear(a_hat, w_hat)


def checksums(a_hat: np.ndarray, w_hat: np.ndarray):
    """Row and column sums of Y = A W^T in O(MK + NK), by linearity.

    col[n] = sum_m Y[m,n] = sum_k (sum_m a[m,k]) w[n,k]
    row[m] = sum_n Y[m,n] = sum_k a[m,k] (sum_n w[n,k])
    Also returns the matching sums of |a w| for the tolerance.
    """
    col = w_hat @ a_hat.sum(axis=0)
    row = a_hat @ w_hat.sum(axis=0)
    abs_col = np.abs(w_hat) @ np.abs(a_hat).sum(axis=0)
    abs_row = np.abs(a_hat) @ np.abs(w_hat).sum(axis=0)
    return row, col, abs_row, abs_col


# ---------------------------------------------------------------------------
# Storage accounting (Table 1 BPE; Table 2 "Weight (BPE)"; Figure 3 caption)
# ---------------------------------------------------------------------------

def bits_per_weight(fmt: str, strategy: str, N: int, K: int, qn: int, qk: int,
                    n_centroids: int = 256, d: int = 4, scale_codebook: int = 256,
                    scale_group: int = 8, postscale_block_scales: bool = True) -> float:
    """Storage bits per weight: VQ indices + FP4 codebooks + scales (+ scale-VQ metadata).

    indices        log2(K)/d
    FP4 codebooks  K centroids x d elements x 4 bits, one codebook per qn x qk QBlock
    direct scales  8 bits per block of B
    PreScale+      log2(Ks) bits per group of ds scales, plus the Ks x ds byte scale
                   codebook of the tensor
    PostScale-QB   8 bits per QBlock
    The FP32 tensor scale is excluded (Table 1 caption).  postscale_block_scales=False
    is the PostScale reading in which no per-block weight scales are stored.
    """
    qn = N if qn in (0, None) else qn
    qk = K if qk in (0, None) else qk
    B = BLOCK[fmt]
    bits = math.log2(n_centroids) / d
    bits += 4.0 * d * n_centroids / (qn * qk)
    if strategy == "prescale_plus":
        bits += math.log2(scale_codebook) / (scale_group * B)
        bits += scale_codebook * scale_group * 8.0 / (N * K)
    elif strategy == "postscale_qb":
        bits += 8.0 / (qn * qk)
    elif strategy == "prescale" or postscale_block_scales:
        bits += 8.0 / B
    return bits


def native_bits_per_weight(fmt: str) -> float:
    """Native block-scaled FP4: 4 bits per element + one 8-bit scale per block (Table 1)."""
    return 4.0 + 8.0 / BLOCK[fmt]


def storage_bytes(w) -> int:
    """Bytes of the stored weight as this library keeps it (indices, codebooks, scales)."""
    n = w.idx.size + w.cb.size * 2
    if w.strategy == "prescale_plus":
        n += w.sidx.size + w.scb.size
    else:
        n += w.scales.size
    return int(n)


# ---------------------------------------------------------------------------
# SwiGLU between the MoE gate/up and down projections, and the MX quantization
# of its FP32 output (the down projection's W4A4 activation).  The pages name
# the MoE expert tensors (Table 4 caption: Qwen3's experts, whose FFN is
# h = SiLU(gate) * up); they give no arithmetic for it, so these are readings:
#
# * gate/up weight [2F, K]: rows [0, F) are the gate projection, rows [F, 2F)
#   the up projection; g and u are the layer's FP32 outputs (accumulator times
#   the FP32 tensor scales, as the linear layer returns them);
# * h = SiLU(g) * u with SiLU(g) = g / (1 + exp(-g)), every step one FP32
#   operation, so that the codes that h's quantization decides are decided in
#   the precision the kernel computes them in;
# * exp is a fixed FP32 function E, written out below (Cody and Waite's
#   two-constant reduction x = n ln2 + r, then the Taylor polynomial of e^r to
#   degree 7 by Horner's rule, then the exact scaling by 2^n); E(x) = +inf for
#   x > 88 and 0 for x < -86, where the FP32 result would be near overflow or
#   subnormal;
# * h is quantized by the activation rule above (blocks along h's channels),
#   applied to FP32 values instead of BF16 ones; for E4M3-B16 with a given FP32
#   tensor scale (a calibrated scale: h's global maximum is not known while the
#   gate/up tiles are still being produced).
# ---------------------------------------------------------------------------

_F32 = np.float32
_EXP_LOG2E = _F32(1.44269504088896341)
_EXP_C1 = _F32(0.693359375)                         # ln 2 rounded to 9 bits: n * C1 is exact
_EXP_C2 = _F32(0.6931471805599453 - 0.693359375)    # the rest of ln 2
_EXP_TAYLOR = [_F32(1.0 / math.factorial(i)) for i in range(7, -1, -1)]   # 1/7!, ..., 1/1!, 1/0!


def exp_fp32(x) -> np.ndarray:
    """E(x): e^x in FP32 by a fixed sequence of FP32 operations (no fused multiply-add).

    n = rint(x * log2 e); r = (x - n*C1) - n*C2 with C1 + C2 = ln 2; p = Taylor
    polynomial of e^r to degree 7 (Horner, one multiply and one add per step);
    E = p * 2^n.  +inf above 88, 0 below -86.
    """
    x = np.asarray(x, dtype=_F32)
    with np.errstate(over="ignore", invalid="ignore"):
        n = np.rint(x * _EXP_LOG2E).astype(_F32)
        r = (x - n * _EXP_C1) - n * _EXP_C2
        p = np.full_like(x, _EXP_TAYLOR[0])
        for c in _EXP_TAYLOR[1:]:
            p = p * r + c
        ni = np.clip(n, -126, 127).astype(np.int32)
        scale = ((ni + 127).astype(np.uint32) << 23).view(_F32)     # 2^n, exact
        e = p * scale
    e = np.where(x > _F32(88.0), _F32(np.inf), e)
    return np.where(x < _F32(-86.0), _F32(0.0), e).astype(_F32)


def swiglu_fp32(g, u) -> np.ndarray:
    """h = SiLU(g) * u = (g / (1 + E(-g))) * u, each operation in FP32."""
    g = np.asarray(g, dtype=_F32)
    u = np.asarray(u, dtype=_F32)
    with np.errstate(over="ignore", invalid="ignore", divide="ignore"):
        d = _F32(1.0) + exp_fp32(-g)
        return ((g / d) * u).astype(_F32)


def quantize_values_e8m0(x):
    """E8M0-B32 MX quantization of FP32 values [rows, F] (the rule of quantize_act_e8m0)."""
    x = np.asarray(x, dtype=_F32).astype(np.float64)
    M, F = x.shape
    xb = x.reshape(M, F // 32, 32)
    amax = np.abs(xb).max(axis=2)
    _, ex = np.frexp(amax)
    e = np.clip(ex.astype(np.int64) - 1 - 2, -127, 127)
    e = np.where(amax == 0, -127, e)
    codes = _signed_codes(xb, xb / np.ldexp(1.0, e)[:, :, None])
    return codes.reshape(M, F), (e + 127).astype(np.uint8)


def quantize_values_e4m3(x, tscale: float):
    """E4M3-B16 MX quantization of FP32 values [rows, F] with a given FP32 tensor
    scale s (the rule of quantize_act_e4m3)."""
    s = _F32(tscale)
    x = np.asarray(x, dtype=_F32).astype(np.float64)
    M, F = x.shape
    xb = x.reshape(M, F // 16, 16)
    amax = np.abs(xb).max(axis=2).astype(_F32)
    t = ((amax / _F32(6.0)).astype(_F32) / s).astype(_F32)
    sb = e4m3_encode_rne_satfinite(np.where(np.isfinite(t), t, np.float64(448.0)))
    denom = (e4m3_value(sb).astype(_F32) * s).astype(_F32).astype(np.float64)
    safe = np.where(denom == 0, 1.0, denom)
    q = np.where((sb == 0)[:, :, None], 0.0, xb / safe[:, :, None])
    return _signed_codes(xb, q).reshape(M, F), sb.astype(np.uint8)


def swiglu_quantize(y_gate_up, fmt: str, tscale: Optional[float] = None):
    """The down projection's activation from the FP32 gate/up output [rows, 2F]:
    h = swiglu_fp32(gate, up), then MX codes [rows, F] and block scales [rows, F/B]."""
    y = np.asarray(y_gate_up, dtype=_F32)
    F = y.shape[1] // 2
    h = swiglu_fp32(y[:, :F], y[:, F:])
    if fmt == E8M0_B32:
        return quantize_values_e8m0(h)
    return quantize_values_e4m3(h, tscale)
