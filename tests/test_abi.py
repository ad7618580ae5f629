"""C-ABI checks that need no GPU: the library loads, exports every function that
include/mxc.h declares, reports layout sizes, packs weights on the host, and
rejects bad arguments synchronously (before touching any device)."""
import ctypes
import os
import re

import numpy as np
import pytest

from vector_quantized_mx_b200 import build, mxc, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build.build()
    return mxc.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "mxc.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(mxc_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported(L):
    names = declared_functions()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(mxc.EXPORTED)


def test_status_strings(L):
    for code in range(9):
        assert L.mxc_status_string(code)
    assert L.mxc_version() >= 100


def test_sf_bytes(L):
    assert L.mxc_sf_bytes(1, 512, 0) == 128 * 16
    assert L.mxc_sf_bytes(129, 4096, 1) == 256 * 256
    assert L.mxc_sf_bytes(0, 4096, 1) == 0
    assert L.mxc_sf_bytes(10, 4096, 2) == 0      # UE5M3: unsupported


def _pack(w):
    return mxc.pack_weight_host(w)


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("strategy", ["prescale", "prescale_plus", "postscale_qb"])
def test_pack_layouts(L, fmt, strategy):
    N, K = 256, 768
    w = synth.make_weight(7, fmt, strategy, N, K, 128, 256)
    h = _pack(w)
    # index tiles: [N/128][K/256][4 K-quarter slabs][128 rows][16 bytes]
    tiles = h["idx"].reshape(N // 128, K // 256, 4, 128, 16)
    for nt in range(N // 128):
        for ks in range(K // 256):
            for c in range(4):
                assert np.array_equal(tiles[nt, ks, c],
                                      w.idx[nt * 128:(nt + 1) * 128, ks * 64 + c * 16:ks * 64 + (c + 1) * 16])
    B = synth.BLOCK[fmt]
    if strategy == "prescale_plus":
        G = 256 // (8 * B)
        st = h["sidx"].reshape(N // 128, K // 256, 128, G)
        for nt in range(N // 128):
            for ks in range(K // 256):
                assert np.array_equal(st[nt, ks], w.sidx[nt * 128:(nt + 1) * 128, ks * G:(ks + 1) * G])
        assert h["scales"] is None
    elif strategy == "postscale_qb":                # one scale per QBlock, kept as [N/qn][K/qk]
        assert h["scales"].size == (N // 128) * (K // 256) and h["sidx"] is None
        assert np.array_equal(h["scales"].reshape(N // 128, K // 256), w.scales)
    else:
        assert h["scales"].size == L.mxc_sf_bytes(N, K, mxc.FMT[fmt])
        assert np.array_equal(mxc.sf_to_rows(h["scales"], N, K, fmt), w.scales)


@pytest.mark.parametrize("fmt", ["e8m0_b32", "e4m3_b16"])
@pytest.mark.parametrize("ds", [16, 32])
def test_pack_scale_index_units(L, fmt, ds):
    """PreScale+ with larger scale groups: the packed indices come in units of one
    256-channel stage (G = 256/(ds*B) groups per row) or of one group spanning
    ds*B/256 stages (G = 1); either way [N/128][U][128][G] with U*G = K/(ds*B)."""
    B = synth.BLOCK[fmt]
    N, K = 256, max(1024, 2 * ds * B)
    w = synth.make_weight(8, fmt, "prescale_plus", N, K, 128, 256, ds=ds)
    h = _pack(w)
    row = K // (ds * B)
    G = 256 // (ds * B) if ds * B <= 256 else 1
    U = row // G
    st = h["sidx"].reshape(N // 128, U, 128, G)
    for nt in range(N // 128):
        for u in range(U):
            assert np.array_equal(st[nt, u], w.sidx[nt * 128:(nt + 1) * 128, u * G:(u + 1) * G])
    assert h["scb"].size == 256 * ds
    keep = []
    hw = mxc._host_struct(w, keep)
    sizes = mxc._PackedSizes()
    assert L.mxc_packed_weight_sizes(ctypes.byref(hw), ctypes.byref(sizes)) == 0
    assert sizes.sidx == N * row and sizes.scb == 256 * ds
    for bad, status in ((12, 1), (64, 1)):              # only 8, 16 or 32
        hw.scale_group = bad
        assert L.mxc_packed_weight_sizes(ctypes.byref(hw), ctypes.byref(sizes)) == status


def test_sf_layout_word_holds_one_row(L):
    """Each 32-bit word of the SF layout holds four consecutive scales of one row."""
    N, K = 128, 512
    w = synth.make_weight(3, "e4m3_b16", "prescale", N, K, 0, 0)
    sf = _pack(w)["scales"].reshape(-1, 4)
    KB = K // 16
    for r in (0, 5, 31, 32, 77, 127):
        for kb4 in range(KB // 4):
            word = (kb4 * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4) // 4
            assert np.array_equal(sf[word], w.scales[r, 4 * kb4:4 * kb4 + 4])


def test_packed_sizes_rejects_bad_shapes(L):
    w = synth.make_weight(1, "e8m0_b32", "prescale", 256, 512, 0, 0)
    keep = []
    hw = mxc._host_struct(w, keep)
    sizes = mxc._PackedSizes()
    assert L.mxc_packed_weight_sizes(ctypes.byref(hw), ctypes.byref(sizes)) == 0
    assert sizes.idx == 256 * 128 and sizes.cb == 512
    hw.K = 500
    assert L.mxc_packed_weight_sizes(ctypes.byref(hw), ctypes.byref(sizes)) == 3   # alignment
    hw.K = 512
    for qn, qk, status in ((0, 32, 3), (0, 192, 3), (32, 0, 3), (192, 0, 3),   # QBlock sides the kernels refuse
                           (64, 64, 0), (64, 0, 0), (0, 64, 0), (0, 128, 0), (128, 256, 0)):
        hw.qn, hw.qk = qn, qk
        assert L.mxc_packed_weight_sizes(ctypes.byref(hw), ctypes.byref(sizes)) == status, (qn, qk)
    hw.qn = 0
    hw.qk = 0
    hw.fmt = 2
    assert L.mxc_packed_weight_sizes(ctypes.byref(hw), ctypes.byref(sizes)) == 2   # UE5M3 unsupported
    hw.fmt = 7
    assert L.mxc_packed_weight_sizes(ctypes.byref(hw), ctypes.byref(sizes)) == 1


def test_workspace_sizes(L):
    # every linear-layer workspace starts with a 4 KiB area of split-K arrival counters
    C = 4096
    # decode once: the counters, then the decoded weight (FP4 codes, then the SF-layout
    # scales), above 128 tokens when N is a multiple of 256 (the CTA-pair GEMM), else
    # from 1024 tokens
    assert L.mxc_linear_workspace_bytes(4096, 9216, 4096, 1) == C + 9216 * 4096 // 2 + 9216 * 4096 // 16
    assert L.mxc_linear_workspace_bytes(1024, 9216, 4096, 0) == C + 9216 * 4096 // 2 + 9216 * 4096 // 32
    assert L.mxc_linear_workspace_bytes(129, 9216, 4096, 1) == C + 9216 * 4096 // 2 + 9216 * 4096 // 16
    # 17..128 tokens (fused 128-token tiles): split-K partials [tile][rank][128][128] FP32
    assert L.mxc_linear_workspace_bytes(128, 9216, 4096, 1) == C + 72 * 2 * 128 * 128 * 4   # 72 tiles x 2 ranks
    assert L.mxc_linear_workspace_bytes(1023, 9344, 4096, 1) == 0          # N % 256 != 0: fused below 1024
    assert L.mxc_linear_workspace_bytes(1024, 9344, 4096, 1) == C + 9344 * 4096 // 2 + 9344 * 4096 // 16
    assert L.mxc_linear_workspace_bytes(16, 9216, 4096, 1) == 0            # decode: split-K in cluster SMEM
    # decode with more than two split-K ranks or slices past 2048 channels, all CTAs in
    # one wave of 148: the counters, then N/128 x ranks x 8 KiB of partial tiles
    assert L.mxc_linear_workspace_bytes(16, 4608, 8192, 1) == C + 36 * 4 * 8192       # 4 ranks of 2048
    assert L.mxc_linear_workspace_bytes(16, 4096, 4096, 1) == C + 32 * 4 * 4 * 2048   # 4 ranks of 1024
    assert L.mxc_linear_workspace_bytes(1, 256, 9216, 0) == C + 2 * 5 * 8192          # 5 ranks, last short
    assert L.mxc_linear_workspace_bytes(16, 128, 32768, 1) == C + 1 * 16 * 8192       # 16 ranks
    assert L.mxc_linear_workspace_bytes(16, 8192, 8192, 1) == 0            # 64 x 4 CTAs: two waves
    assert L.mxc_linear_workspace_bytes(16, 18432, 4096, 1) == 0           # 144 x 2 CTAs: two waves
    assert L.mxc_linear_workspace_bytes(17, 4608, 8192, 1) == C + 36 * 4 * 128 * 128 * 4   # 36 tiles x 4 ranks
    assert L.mxc_linear_workspace_bytes(16, 128, 65536, 1) == 0            # 32 ranks: past the limit
    assert L.mxc_moe_workspace_bytes(16384, 128, 3072, 4096, 1) >= 129 * 4
    assert L.mxc_grouped_sf_rows_bound(16384, 128) == 16384 + 128 * 128


def test_gpu_calls_reject_bad_arguments_synchronously(L):
    """Argument errors come back before any device work (safe without a GPU)."""
    a = mxc._MxTensor(16, 16, None, 4, 512, 256, 0)
    w = mxc._Weight(1, 0, 256, 512, 0, 0, 16, 16, 16, None, None, 1.0)
    y = 16
    # null tensor / weight
    assert L.mxc_linear(None, ctypes.byref(w), y, 256, 0, None, 0, None) == 1
    # format mismatch
    w.fmt = 1
    assert L.mxc_linear(ctypes.byref(a), ctypes.byref(w), y, 256, 0, None, 0, None) == 1
    w.fmt = 0
    # K not a multiple of 256
    a.K = 500
    assert L.mxc_linear(ctypes.byref(a), ctypes.byref(w), y, 256, 0, None, 0, None) == 3
    a.K = 512
    # ldq too small
    a.ldq = 128
    assert L.mxc_linear(ctypes.byref(a), ctypes.byref(w), y, 256, 0, None, 0, None) == 3
    a.ldq = 256
    # misaligned pointer
    w.idx = 17
    assert L.mxc_linear(ctypes.byref(a), ctypes.byref(w), y, 256, 0, None, 0, None) == 3
    w.idx = 16
    # UE5M3
    a.fmt = w.fmt = 2
    assert L.mxc_linear(ctypes.byref(a), ctypes.byref(w), y, 256, 0, None, 0, None) == 2
    a.fmt = w.fmt = 0
    # PreScale+ without its scale codebook
    w.strategy = 2
    assert L.mxc_linear(ctypes.byref(a), ctypes.byref(w), y, 256, 0, None, 0, None) == 1
    w.strategy = 1
    # ldy < N
    assert L.mxc_linear(ctypes.byref(a), ctypes.byref(w), y, 100, 0, None, 0, None) == 1
    # MoE: too many experts, zero experts
    table = (mxc._Weight * 1)(w)
    assert L.mxc_moe_linear(ctypes.byref(a), 16, table, 0, y, 256, 0, None, 0, None) == 1
    assert L.mxc_moe_linear(ctypes.byref(a), 16, table, 300, y, 256, 0, None, 0, None) == 2
    # quantize: bad K
    assert L.mxc_quantize_act(16, 4, 500, 512, 0, None, 16, 256, 16, None, 16, 256, None) == 3
    # quantize: E4M3 needs a tensor-scale output
    assert L.mxc_quantize_act(16, 4, 512, 512, 1, None, 16, 256, 16, None, 16, 256, None) == 1


def test_binding_fails_loudly_without_the_library(tmp_path, monkeypatch):
    """No CPU or library fallback: without libmxc.so every call raises."""
    monkeypatch.setattr(mxc, "_lib", None)
    monkeypatch.setattr(mxc, "_LIB_PATH", str(tmp_path / "libmxc.so"))
    with pytest.raises(RuntimeError, match="missing"):
        mxc.lib()
    w = synth.make_weight(1, "e8m0_b32", "prescale", 256, 512, 0, 0)
    with pytest.raises(RuntimeError, match="missing"):
        mxc.pack_weight_host(w)
