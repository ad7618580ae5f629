"""Offline MXCode weight quantizer (host side, NumPy).

Turns a real-valued weight W[N, K] into the logical VQ layout that
mxc_pack_weight consumes (idx / cb / scales | sidx + scb, see mxc.h), for the
three strategies of "MXCode: Vector Quantization for MX-Native Inference at
Scale" (abstract): PostScale quantizes learned codebooks to MXFP4, PreScale
extracts the MX scales before codebook learning, PreScale+ additionally
VQ-codes those scales.  Vectors are d = 4 consecutive weights along the
input-channel axis with K = 256 centroids per QBlock, and PreScale+ codes
groups of ds = 8 scales with a Ks = 256-entry scale codebook (Table 4 caption).

The pages name the strategies but give no algorithm; this module takes the
plainest reading of each step:

* tensor scale (E4M3-B16): amax|W| / (6 * 448) in FP32, as for activations;
* MX block scales (PreScale): from the block amax by the OCP MX rule
  (E8M0: 2^(floor(log2 amax) - 2); E4M3: RNE of amax / 6 over the tensor scale);
* codebook learning: Lloyd k-means (seeded, a fixed number of iterations) on the
  4-vectors of each QBlock.  PreScale learns on the scale-normalized weights and
  rounds every centroid element to the nearest E2M1 value after each update, so
  the codebook is FP4 by construction; PostScale learns real-valued centroids
  on the weights and then MX-quantizes the codebook with one scale from the
  codebook's own amax (PostScale-QB stores that scale once per QBlock; PostScale
  with per-block storage repeats it for every block of the QBlock);
* PreScale+: k-means over groups of 8 consecutive block scales along K, in the
  log2 domain, centroids rounded to valid scale bytes; the FP4 indices are then
  re-assigned under the coded scales;
* indices: nearest (Euclidean) dequantized centroid, ties to the lower index.

quality() reports the weight SQNR, 10 log10(sum W^2 / sum (W - W_hat)^2), the
measure of Table 4 and Figures 2 and 3.  Nothing here runs on the GPU; the
result is a plain container that mxc.pack_weight uploads.
"""
from __future__ import annotations

import argparse
import math
from typing import Optional

import numpy as np

from .synth import VQWeight

BLOCK = {"e8m0_b32": 32, "e4m3_b16": 16}
E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
STRATEGIES = ("postscale", "prescale", "prescale_plus", "postscale_qb")


# ---------------------------------------------------------------------------
# Format rounding
# ---------------------------------------------------------------------------

def e2m1_codes(x: np.ndarray) -> np.ndarray:
    """Nearest E2M1 code of x (ties to the even code), saturating at +-6; bit 3 = sign."""
    a = np.abs(x)
    c = ((a > 0.25).astype(np.uint8) + (a >= 0.75) + (a > 1.25) + (a >= 1.75) + (a > 2.5) + (a >= 3.5)
         + (a > 5.0)).astype(np.uint8)
    return c | np.where(x < 0, 8, 0).astype(np.uint8)


def e2m1_values(codes: np.ndarray) -> np.ndarray:
    v = E2M1[codes & 7]
    return np.where(codes & 8, -v, v)


def e4m3_byte(v: np.ndarray) -> np.ndarray:
    """RNE E4M3 byte of v >= 0 (bias 7, max 448 = 0x7E, subnormals m * 2^-9), saturating."""
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros(v.shape, dtype=np.int64)
    sub = v < 2.0 ** -6
    out[sub] = np.rint(v[sub] * 512.0).astype(np.int64)          # 8 -> 0x08, the smallest normal
    nrm = ~sub
    e = np.floor(np.log2(np.where(nrm, v, 1.0))).astype(np.int64)
    m = np.rint((v / np.exp2(e) - 1.0) * 8.0).astype(np.int64)   # ties to even
    e = np.where(m == 8, e + 1, e)
    m = np.where(m == 8, 0, m)
    out[nrm] = ((e[nrm] + 7) << 3) | m[nrm]
    return np.clip(out, 0, 0x7E).astype(np.uint8)


def e4m3_value(b: np.ndarray) -> np.ndarray:
    b = np.asarray(b, dtype=np.int64)
    e, m = (b >> 3) & 0xF, b & 7
    return np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e - 7.0))


def scale_value(b: np.ndarray, fmt: str) -> np.ndarray:
    b = np.asarray(b)
    return np.exp2(b.astype(np.float64) - 127.0) if fmt == "e8m0_b32" else e4m3_value(b)


def scale_byte(amax: np.ndarray, fmt: str, tscale: float) -> np.ndarray:
    """MX scale byte of blocks (or codebooks) whose largest magnitude is amax."""
    amax = np.asarray(amax, dtype=np.float64)
    if fmt == "e8m0_b32":
        e = np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2
        return np.where(amax > 0, np.clip(e, -127, 127) + 127, 0).astype(np.uint8)
    t = (amax.astype(np.float32) / np.float32(6.0)).astype(np.float64) / tscale
    return e4m3_byte(t)


def tensor_scale(W: np.ndarray, fmt: str) -> float:
    if fmt == "e8m0_b32":
        return 1.0
    amax = float(np.max(np.abs(W))) if W.size else 0.0
    return float(np.float32(amax) / np.float32(2688.0)) if amax > 0 else 1.0


# ---------------------------------------------------------------------------
# k-means
# ---------------------------------------------------------------------------

def _assign(X: np.ndarray, C: np.ndarray) -> np.ndarray:
    d2 = (X * X).sum(1)[:, None] - 2.0 * X @ C.T + (C * C).sum(1)[None, :]
    return np.argmin(d2, axis=1)


def kmeans(X: np.ndarray, k: int, iters: int, rng: np.random.Generator, project=None):
    """Lloyd's algorithm on the rows of X; `project` maps centroids onto a grid after
    every update.  Empty clusters restart from a random row.  Returns (C, labels)."""
    V, d = X.shape
    C = X[rng.choice(V, size=k, replace=V < k)].copy()
    if project is not None:
        C = project(C)
    for _ in range(iters):
        lab = _assign(X, C)
        counts = np.bincount(lab, minlength=k)
        sums = np.stack([np.bincount(lab, weights=X[:, j], minlength=k) for j in range(d)], axis=1)
        empty = counts == 0
        C = np.where(empty[:, None], X[rng.integers(0, V, size=k)], sums / np.maximum(counts, 1)[:, None])
        if project is not None:
            C = project(C)
    return C, _assign(X, C)


def _fp4_grid(C: np.ndarray) -> np.ndarray:
    return e2m1_values(e2m1_codes(C))


def _pack_entries(codes: np.ndarray) -> np.ndarray:
    """[256, 4] E2M1 codes -> uint16 entries, element t in bits 4t..4t+3."""
    codes = codes.astype(np.uint16)
    return codes[:, 0] | (codes[:, 1] << 4) | (codes[:, 2] << 8) | (codes[:, 3] << 12)


# ---------------------------------------------------------------------------
# The strategies
# ---------------------------------------------------------------------------

def quantize_weight(W: np.ndarray, fmt: str, strategy: str, qn: int = 256, qk: int = 256, iters: int = 12,
                    seed: int = 0, n_centroids: int = 256, scale_codebook: int = 256,
                    scale_group: int = 8) -> VQWeight:
    """MXCode-quantizes W[N, K] (N % 128 == 0, K % 256 == 0; qn, qk as in mxc.h, 0 = whole
    dimension) and returns the logical VQ weight."""
    if fmt not in BLOCK or strategy not in STRATEGIES:
        raise ValueError(f"format {fmt!r} / strategy {strategy!r}")
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    qn = N if qn in (0, None) else qn
    qk = K if qk in (0, None) else qk
    if N % qn or K % qk or qk % 4:
        raise ValueError("QBlock must tile the tensor")
    B = BLOCK[fmt]
    rng = np.random.default_rng(seed)
    ts = tensor_scale(W, fmt)
    idx = np.zeros((N, K // 4), dtype=np.uint8)
    cb = np.zeros((N // qn, K // qk, n_centroids), dtype=np.uint16)
    scales = sidx = scb = None

    def vectors(A, a, b):       # QBlock (a, b) of A as rows of 4 consecutive weights along K
        return A[a * qn:(a + 1) * qn, b * qk:(b + 1) * qk].reshape(-1, 4)

    def put_idx(a, b, lab):
        idx[a * qn:(a + 1) * qn, b * qk // 4:(b + 1) * qk // 4] = lab.reshape(qn, qk // 4).astype(np.uint8)

    if strategy in ("prescale", "prescale_plus"):
        amax = np.abs(W).reshape(N, K // B, B).max(axis=2)
        sbytes = scale_byte(amax, fmt, ts)
        S = np.repeat(scale_value(sbytes, fmt) * ts, B, axis=1)               # [N, K]
        U = np.divide(W, S, out=np.zeros_like(W), where=S > 0)
        books = {}
        for a in range(N // qn):
            for b in range(K // qk):
                C, lab = kmeans(vectors(U, a, b), n_centroids, iters, rng, project=_fp4_grid)
                books[a, b] = C
                cb[a, b] = _pack_entries(e2m1_codes(C))
                put_idx(a, b, lab)
        if strategy == "prescale":
            scales = sbytes
        else:
            G = K // B // scale_group
            logs = np.log2(np.maximum(scale_value(sbytes, fmt), 2.0 ** -140)).reshape(N * G, scale_group)
            Cs, lab = kmeans(logs, scale_codebook, iters, rng)
            scb = e4m3_byte(np.exp2(Cs)) if fmt == "e4m3_b16" else \
                np.clip(np.rint(Cs) + 127, 0, 254).astype(np.uint8)
            # re-pick each group's entry among the rounded codebook, then re-assign indices
            lab = _assign(logs, np.log2(np.maximum(scale_value(scb, fmt), 2.0 ** -140)))
            sidx = lab.reshape(N, G).astype(np.uint8)
            coded = scb[sidx.reshape(-1)].reshape(N, K // B)
            S = np.repeat(scale_value(coded, fmt) * ts, B, axis=1)
            U = np.divide(W, S, out=np.zeros_like(W), where=S > 0)
            for (a, b), C in books.items():
                put_idx(a, b, _assign(vectors(U, a, b), C))
    else:
        Wt = W / ts
        qbytes = np.zeros((N // qn, K // qk), dtype=np.uint8)
        for a in range(N // qn):
            for b in range(K // qk):
                X = vectors(Wt, a, b)
                C, _ = kmeans(X, n_centroids, iters, rng)
                qbytes[a, b] = scale_byte(np.abs(C).max(), fmt, 1.0)
                q = scale_value(qbytes[a, b], fmt)
                codes = e2m1_codes(C / q) if q > 0 else np.zeros_like(C, dtype=np.uint8)
                cb[a, b] = _pack_entries(codes)
                put_idx(a, b, _assign(X, e2m1_values(codes) * q))
        if strategy == "postscale_qb":
            scales = qbytes
        else:                                          # the QBlock's scale in every block of it
            kb = np.arange(K // B)
            scales = qbytes[np.arange(N)[:, None] // qn, (kb[None, :] * B) // qk]
    return VQWeight(fmt, strategy, N, K, qn, qk, idx, cb, scales, sidx, scb, float(np.float32(ts)))


def dequantize(w: VQWeight) -> np.ndarray:
    """W_hat[N, K] = E2M1(centroid element) * block scale * tensor scale."""
    N, K, B = w.N, w.K, BLOCK[w.fmt]
    n = np.arange(N)[:, None]
    k = np.arange(K)[None, :]
    entry = w.cb[n // w.qn, k // w.qk, w.idx[n, k // 4]].astype(np.int64)
    vals = e2m1_values(((entry >> (4 * (k % 4))) & 0xF).astype(np.uint8))
    kb = np.arange(K // B)[None, :]
    if w.strategy == "prescale_plus":
        sb = w.scb[w.sidx[n, kb // 8], kb % 8]
    elif w.strategy == "postscale_qb":
        sb = w.scales[n // w.qn, (kb * B) // w.qk]
    else:
        sb = w.scales
    return vals * np.repeat(scale_value(sb, w.fmt), B, axis=1) * w.w_tscale


def sqnr_db(W: np.ndarray, W_hat: np.ndarray) -> float:
    err = float(np.sum((W - W_hat) ** 2))
    return math.inf if err == 0 else 10.0 * math.log10(float(np.sum(W * W)) / err)


def native_fp4(W: np.ndarray, fmt: str) -> np.ndarray:
    """W MX-quantized directly (the "Native FP4" rows of Tables 2 and 4), dequantized."""
    W = np.asarray(W, dtype=np.float64)
    N, K = W.shape
    B = BLOCK[fmt]
    ts = tensor_scale(W, fmt)
    sb = scale_byte(np.abs(W).reshape(N, K // B, B).max(axis=2), fmt, ts)
    S = np.repeat(scale_value(sb, fmt) * ts, B, axis=1)
    U = np.divide(W, S, out=np.zeros_like(W), where=S > 0)
    return e2m1_values(e2m1_codes(U)) * S


def quality(W: np.ndarray, w: VQWeight) -> dict:
    """SQNR of the MXCode weight and of native FP4 on the same tensor, and the storage
    bits per weight (indices + FP4 codebooks + scales (+ scale codebook))."""
    N, K = w.N, w.K
    bits = 8 * (w.idx.size + 2 * w.cb.size + (w.scales.size if w.scales is not None else 0)
                + (w.sidx.size + w.scb.size if w.sidx is not None else 0))
    return {"sqnr_db": sqnr_db(W, dequantize(w)), "native_fp4_sqnr_db": sqnr_db(W, native_fp4(W, w.fmt)),
            "bits_per_weight": bits / (N * K)}


def main(argv: Optional[list] = None) -> None:
    ap = argparse.ArgumentParser(description="MXCode-quantize a seeded Gaussian weight and report its SQNR")
    ap.add_argument("--n", type=int, default=512)
    ap.add_argument("--k", type=int, default=1024)
    ap.add_argument("--fmt", default="e4m3_b16", choices=sorted(BLOCK))
    ap.add_argument("--strategy", default="prescale", choices=STRATEGIES)
    ap.add_argument("--qb", type=int, default=256, help="square QBlock size (0 = whole tensor)")
    ap.add_argument("--iters", type=int, default=12)
    ap.add_argument("--seed", type=int, default=0)
    args = ap.parse_args(argv)
    W = np.random.default_rng(args.seed).normal(size=(args.n, args.k))
    w = quantize_weight(W, args.fmt, args.strategy, args.qb, args.qb, iters=args.iters, seed=args.seed)
    q = quality(W, w)
    print(f"{args.strategy} {args.fmt} QBlock {args.qb or 'tensor'}: SQNR {q['sqnr_db']:.2f} dB "
          f"({q['bits_per_weight']:.4f} bits/weight), native FP4 {q['native_fp4_sqnr_db']:.2f} dB")


if __name__ == "__main__":
    main()
