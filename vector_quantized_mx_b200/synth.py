"""Seeded synthetic inputs for the MXCode W4A4 linear layer.

This module only *draws* data: random index bytes, random centroid codes,
random scale bytes and random BF16 activations, plus a Zipf expert routing.
It holds none of the layer's arithmetic (no decode, no quantizer, no GEMM), so
the CPU oracle and the CUDA path can both consume its output without sharing
any of the method's code.  Type conversions that a draw needs (float -> BF16,
float -> E4M3 byte) go through PyTorch's own casts.

Workload shapes follow the method's evaluation setting ("MXCode: Vector
Quantization for MX-Native Inference at Scale", Table 4 caption: VQ along the
input-channel axis with K=256 centroids of d=4 elements; PreScale+ with a
256-entry scale codebook over groups of 8 scales; Qwen3 (235B) expert tensors).

Every generator is a NumPy PCG64 stream keyed by (seed, role), so one tensor
role can be regenerated without drawing the others.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
import torch

FMT_E8M0_B32 = "e8m0_b32"
FMT_E4M3_B16 = "e4m3_b16"
FORMATS = (FMT_E8M0_B32, FMT_E4M3_B16)

POSTSCALE = "postscale"
PRESCALE = "prescale"
PRESCALE_PLUS = "prescale_plus"
POSTSCALE_QB = "postscale_qb"     # PostScale with one scale per QBlock (Table 2's 2.06 / 2.25 BPE)
STRATEGIES = (POSTSCALE, PRESCALE, PRESCALE_PLUS)

BLOCK = {FMT_E8M0_B32: 32, FMT_E4M3_B16: 16}

_ROLES = {"idx": 1, "cb": 2, "scale": 3, "sidx": 4, "scb": 5, "act": 6,
          "outlier": 7, "route": 8}


def stream(seed: int, role: str, sub: int = 0) -> np.random.Generator:
    """Independent PCG64 stream for one tensor role of one workload."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _ROLES[role], sub])))


# E2M1 magnitudes are 0, .5, 1, 1.5, 2, 3, 4, 6.  To draw "the E2M1 value
# nearest to a Gaussian sample" the sampler only needs the boundaries between
# neighbouring magnitudes; a continuous draw lands on a boundary with
# probability zero, so no tie rule is involved.
_E2M1_BOUNDARIES = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def draw_e2m1_codes(rng: np.random.Generator, shape, sigma: float = 1.5) -> np.ndarray:
    """4-bit E2M1 codes (bit 3 = sign) of Gaussian draws N(0, sigma^2)."""
    z = rng.normal(0.0, sigma, size=shape)
    mag = np.searchsorted(_E2M1_BOUNDARIES, np.abs(z)).astype(np.uint8)
    return mag | (np.signbit(z).astype(np.uint8) << 3)


def draw_codebooks(rng: np.random.Generator, n_qb: int, k_qb: int, n_centroids: int = 256,
                   d: int = 4, sigma: float = 1.5) -> np.ndarray:
    """FP4 codebooks [n_qb, k_qb, 256] as uint16: element t of a centroid in bits 4t..4t+3."""
    codes = draw_e2m1_codes(rng, (n_qb, k_qb, n_centroids, d), sigma).astype(np.uint16)
    packed = np.zeros((n_qb, k_qb, n_centroids), dtype=np.uint16)
    for t in range(d):
        packed |= codes[..., t] << np.uint16(4 * t)
    return packed


def draw_indices(rng: np.random.Generator, n: int, k: int, d: int = 4) -> np.ndarray:
    """uint8 VQ indices [n, k/d], uniform over 256 centroids."""
    return rng.integers(0, 256, size=(n, k // d), dtype=np.uint8)


def draw_e8m0_bytes(rng: np.random.Generator, shape, exp_lo: int, exp_hi: int) -> np.ndarray:
    """E8M0 scale bytes whose exponent is uniform over the integers [exp_lo, exp_hi]."""
    e = rng.integers(exp_lo, exp_hi + 1, size=shape)
    return (e + 127).astype(np.uint8)


def draw_e4m3_bytes(rng: np.random.Generator, shape, lo: float = 0.5, hi: float = 448.0) -> np.ndarray:
    """Positive E4M3 scale bytes: continuous U(lo, hi) rounded by torch's float8_e4m3fn cast."""
    u = np.clip(rng.uniform(lo, hi, size=shape), lo, hi).astype(np.float32)
    return torch.from_numpy(u).to(torch.float8_e4m3fn).view(torch.uint8).numpy().copy()


def draw_bf16_activations(rng: np.random.Generator, m: int, k: int,
                          outlier_cols: Optional[np.ndarray] = None,
                          outlier_factor: float = 20.0) -> np.ndarray:
    """BF16 bit patterns [m, k] of N(0,1) draws; listed columns are scaled before rounding."""
    z = rng.normal(0.0, 1.0, size=(m, k))
    if outlier_cols is not None and len(outlier_cols):
        z[:, outlier_cols] *= outlier_factor
    return torch.from_numpy(z).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def outlier_columns(rng: np.random.Generator, k: int, fraction: float = 0.01) -> np.ndarray:
    """round(fraction*k) input channels, chosen by a seeded permutation (same for every row)."""
    n = int(round(fraction * k))
    return np.sort(rng.permutation(k)[:n])


def zipf_topk_routing(rng: np.random.Generator, n_tokens: int, n_experts: int, top_k: int,
                      s: float = 1.1):
    """Top-k expert choice per token, weighted sampling without replacement from Zipf(s).

    Uses Gumbel-top-k on log p_i with p_i proportional to i^-s (expert id = rank - 1).
    Returns (row_token [n_tokens*top_k], offsets [n_experts+1]): rows sorted by expert,
    ties by token id.
    """
    logp = -s * np.log(np.arange(1, n_experts + 1, dtype=np.float64))
    keys = logp[None, :] + rng.gumbel(size=(n_tokens, n_experts))
    top = np.argpartition(-keys, top_k - 1, axis=1)[:, :top_k]
    tok = np.repeat(np.arange(n_tokens), top_k)
    exp = top.reshape(-1)
    order = np.lexsort((tok, exp))
    counts = np.bincount(exp, minlength=n_experts)
    offsets = np.zeros(n_experts + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    return tok[order], offsets


@dataclasses.dataclass
class VQWeight:
    """One VQ-coded weight W[N, K] in the logical (unpacked) layout.

    idx[n, j]      uint8, centroid of weights k = 4j..4j+3 of row n
    cb[a, b, c]    uint16, centroid c of QBlock (a, b) = (n // qn, k // qk)
    scales[n, kb]  uint8 block-scale byte (PostScale / PreScale), kb = k // B
    sidx[n, g]     uint8 scale-codebook index of scale group g = kb // 8 (PreScale+)
    scb[c, t]      uint8 scale codebook: 256 entries of ds scale bytes (PreScale+)
    w_tscale       FP32 tensor scale (1.0 for E8M0-B32)
    ds             PreScale+ scale group: ds consecutive block scales along K per index
    """
    fmt: str
    strategy: str
    N: int
    K: int
    qn: int
    qk: int
    idx: np.ndarray
    cb: np.ndarray
    scales: Optional[np.ndarray]
    sidx: Optional[np.ndarray]
    scb: Optional[np.ndarray]
    w_tscale: float
    ds: int = 8

    @property
    def block(self) -> int:
        return BLOCK[self.fmt]


def weight_rows(w: "VQWeight", r0: int, r1: int) -> "VQWeight":
    """Rows [r0, r1) of a logical VQ weight as a weight of their own (array slicing
    only).  Either r0 is a multiple of qn or the range lies inside one QBlock row,
    so QBlock row (r0 + i) // qn of the whole weight is row i // qn of the slice."""
    assert r0 % w.qn == 0 or r0 // w.qn == (r1 - 1) // w.qn
    q0, q1 = r0 // w.qn, (r1 - 1) // w.qn + 1
    scales = sidx = None
    if w.strategy == POSTSCALE_QB:
        scales = w.scales[q0:q1]
    elif w.strategy == PRESCALE_PLUS:
        sidx = w.sidx[r0:r1]
    else:
        scales = w.scales[r0:r1]
    return VQWeight(w.fmt, w.strategy, r1 - r0, w.K, w.qn, w.qk, w.idx[r0:r1], w.cb[q0:q1], scales, sidx, w.scb,
                    w.w_tscale, w.ds)


TSCALE_E4M3 = float(np.float32(1.0) / np.float32(2688.0))


def make_weight(seed: int, fmt: str, strategy: str, N: int, K: int, qn: int, qk: int,
                e8m0_exp=(-8, 1), sub: int = 0, ds: int = 8) -> VQWeight:
    """Draw one VQ weight; qn/qk = 0 means the QBlock spans the whole dimension; ds is the
    PreScale+ scale group (consecutive block scales per scale index)."""
    qn = N if qn in (0, None) else qn
    qk = K if qk in (0, None) else qk
    B = BLOCK[fmt]
    idx = draw_indices(stream(seed, "idx", sub), N, K)
    cb = draw_codebooks(stream(seed, "cb", sub), N // qn, K // qk)
    scales = sidx = scb = None
    if strategy == PRESCALE_PLUS:
        sidx = stream(seed, "sidx", sub).integers(0, 256, size=(N, K // (ds * B)), dtype=np.uint8)
        if fmt == FMT_E8M0_B32:
            scb = draw_e8m0_bytes(stream(seed, "scb", sub), (256, ds), *e8m0_exp)
        else:
            scb = draw_e4m3_bytes(stream(seed, "scb", sub), (256, ds))
    else:
        shape = (N // qn, K // qk) if strategy == POSTSCALE_QB else (N, K // B)   # per QBlock or per block
        if fmt == FMT_E8M0_B32:
            scales = draw_e8m0_bytes(stream(seed, "scale", sub), shape, *e8m0_exp)
        else:
            scales = draw_e4m3_bytes(stream(seed, "scale", sub), shape)
    w_tscale = 1.0 if fmt == FMT_E8M0_B32 else TSCALE_E4M3
    return VQWeight(fmt, strategy, N, K, qn, qk, idx, cb, scales, sidx, scb, w_tscale, ds)


def make_activations(seed: int, M: int, K: int, outliers: bool, sub: int = 0) -> np.ndarray:
    cols = outlier_columns(stream(seed, "outlier", sub), K) if outliers else None
    return draw_bf16_activations(stream(seed, "act", sub), M, K, cols)


# ---------------------------------------------------------------------------
# The five workloads.  Config 1 is the tiny all-at-once case; 2 is the decode
# GEMV shaped like a fused QKV projection; 3 the prefill GEMM; 4 the MoE expert
# layer; 5 the K=N=8192 sweep.
# ---------------------------------------------------------------------------

def config1():
    """Tiny single linear: PreScale, E8M0-B32, M=4, K=512, N=256, one codebook per tensor."""
    w = make_weight(1, FMT_E8M0_B32, PRESCALE, 256, 512, 0, 0, e8m0_exp=(-7, 0))
    x = make_activations(1, 4, 512, outliers=False)
    return w, x


def config2(M: int = 16):
    """Decode GEMV: PostScale, E4M3-B16, M in {1,4,16}, K=4096, N=9216, 256x256 QBlocks."""
    assert M in (1, 4, 16)
    w = make_weight(2, FMT_E4M3_B16, POSTSCALE, 9216, 4096, 256, 256)
    x = make_activations(2, 16, 4096, outliers=True)[:M].copy()
    return w, x


def config3():
    """Prefill GEMM: PreScale, E8M0-B32, M=8192, K=4096, N=9216, 256x256 QBlocks."""
    w = make_weight(3, FMT_E8M0_B32, PRESCALE, 9216, 4096, 256, 256, e8m0_exp=(-8, 1))
    x = make_activations(3, 8192, 4096, outliers=True)
    return w, x


MOE_EXPERTS = 128
MOE_TOKENS = 2048
MOE_TOPK = 8
MOE_HIDDEN = 4096
MOE_INTER = 1536


def config4_routing():
    """Zipf(1.1) top-8 routing of 2048 tokens over 128 experts -> (row_token, offsets)."""
    return zipf_topk_routing(stream(4, "route"), MOE_TOKENS, MOE_EXPERTS, MOE_TOPK)


def config4_expert(e: int, proj: str) -> VQWeight:
    """Expert e's gate/up [3072, 4096] or down [4096, 1536] weight: PreScale+, E4M3-B16."""
    if proj == "gate_up":
        return make_weight(4, FMT_E4M3_B16, PRESCALE_PLUS, 2 * MOE_INTER, MOE_HIDDEN, 256, 256, sub=2 * e)
    if proj == "down":
        return make_weight(4, FMT_E4M3_B16, PRESCALE_PLUS, MOE_HIDDEN, MOE_INTER, 256, 256, sub=2 * e + 1)
    raise ValueError(proj)


def config4_activations(proj: str, row_token: np.ndarray) -> np.ndarray:
    """Expert-sorted BF16 rows: each row is its token's activation (N(0,1))."""
    K = MOE_HIDDEN if proj == "gate_up" else MOE_INTER
    tokens = make_activations(4, MOE_TOKENS, K, outliers=False, sub=0 if proj == "gate_up" else 1)
    return tokens[row_token]


SWEEP_M = (1, 16, 128, 1024, 16384)
SWEEP_QB = (0, 1024, 256, 128)  # 0 = full tensor


def config5_weight(qb: int, strategy: str, fmt: str) -> VQWeight:
    return make_weight(5, fmt, strategy, 8192, 8192, qb, qb,
                       sub=SWEEP_QB.index(qb) * 16 + STRATEGIES.index(strategy) * 2 + FORMATS.index(fmt))


def config5_activations(M: int) -> np.ndarray:
    return make_activations(5, M, 8192, outliers=True, sub=SWEEP_M.index(M))
