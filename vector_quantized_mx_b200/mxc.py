"""Python binding of the MXCode W4A4 C ABI (include/mxc.h).

Argument marshalling only: every step of the layer runs in libmxc.so.  PyTorch
provides device memory and the current CUDA stream.  The shared library is
loaded from this package directory; if it is missing, or the GPU is not an
sm_100 part, calls raise instead of falling back to anything else.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional, Sequence

import numpy as np
import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmxc.so")

FMT = {"e8m0_b32": 0, "e4m3_b16": 1, "ue5m3_b16": 2}
BLOCK = {"e8m0_b32": 32, "e4m3_b16": 16}
STRATEGY = {"postscale": 0, "prescale": 1, "prescale_plus": 2, "postscale_qb": 3}
OUT = {torch.float32: 0, torch.bfloat16: 1}

STATUS = {0: "MXC_OK", 1: "MXC_ERR_INVALID_ARG", 2: "MXC_ERR_UNSUPPORTED", 3: "MXC_ERR_ALIGNMENT",
          4: "MXC_ERR_WORKSPACE", 5: "MXC_ERR_CUDA", 6: "MXC_ERR_DEVICE_INVALID", 7: "MXC_ERR_TIMEOUT",
          8: "MXC_ERR_NO_DEVICE"}

EXPORTED = (
    "mxc_status_string", "mxc_version", "mxc_sf_bytes", "mxc_packed_weight_sizes", "mxc_pack_weight",
    "mxc_quantize_act_workspace_bytes", "mxc_linear_workspace_bytes", "mxc_moe_workspace_bytes",
    "mxc_grouped_sf_rows_bound", "mxc_quantize_act", "mxc_quantize_act_grouped", "mxc_linear",
    "mxc_native_linear", "mxc_moe_linear", "mxc_moe_linear_noalloc", "mxc_decode_weight", "mxc_get_device_error",
    "mxc_selftest_wait_timeout", "mxc_moe_gate_up_swiglu", "mxc_linear_workspace_bytes_for",
)


class MxcError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {STATUS.get(status, status)}")
        self.status = status


class _MxTensor(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("sf", ctypes.c_void_p), ("tscale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("K", ctypes.c_int64), ("ldq", ctypes.c_int64),
                ("fmt", ctypes.c_int)]


class _Weight(ctypes.Structure):
    _fields_ = [("strategy", ctypes.c_int), ("fmt", ctypes.c_int), ("N", ctypes.c_int64),
                ("K", ctypes.c_int64), ("qn", ctypes.c_int64), ("qk", ctypes.c_int64),
                ("idx", ctypes.c_void_p), ("cb", ctypes.c_void_p), ("scales", ctypes.c_void_p),
                ("sidx", ctypes.c_void_p), ("scb", ctypes.c_void_p), ("w_tscale", ctypes.c_float),
                ("scale_group", ctypes.c_int32)]


_WeightHost = _Weight  # identical field layout (mxc_weight_host)


class _PackedSizes(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_size_t), ("cb", ctypes.c_size_t), ("scales", ctypes.c_size_t),
                ("sidx", ctypes.c_size_t), ("scb", ctypes.c_size_t)]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded libmxc.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with python -m vector_quantized_mx_b200.build")
        L = ctypes.CDLL(_LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        sig = {
            "mxc_status_string": (ctypes.c_char_p, [ctypes.c_int]),
            "mxc_version": (ctypes.c_int, []),
            "mxc_sf_bytes": (sz, [i64, i64, ctypes.c_int]),
            "mxc_packed_weight_sizes": (ctypes.c_int, [ctypes.POINTER(_WeightHost), ctypes.POINTER(_PackedSizes)]),
            "mxc_pack_weight": (ctypes.c_int, [ctypes.POINTER(_WeightHost), vp, vp, vp]),
            "mxc_quantize_act_workspace_bytes": (sz, [i64, i64, ctypes.c_int]),
            "mxc_linear_workspace_bytes": (sz, [i64, i64, i64, ctypes.c_int]),
            "mxc_moe_workspace_bytes": (sz, [i64, i32, i64, i64, ctypes.c_int]),
            "mxc_linear_workspace_bytes_for": (sz, [ctypes.POINTER(_Weight), i64]),
            "mxc_grouped_sf_rows_bound": (i64, [i64, i32]),
            "mxc_quantize_act": (ctypes.c_int, [vp, i64, i64, i64, ctypes.c_int, vp, vp, i64, vp, vp, vp, sz, vp]),
            "mxc_quantize_act_grouped": (ctypes.c_int, [vp, i64, i64, i64, ctypes.c_int, vp, i32, vp, vp, i64, vp,
                                                        vp, vp, sz, vp]),
            "mxc_linear": (ctypes.c_int, [ctypes.POINTER(_MxTensor), ctypes.POINTER(_Weight), vp, i64, ctypes.c_int,
                                          vp, sz, vp]),
            "mxc_native_linear": (ctypes.c_int, [ctypes.POINTER(_MxTensor), ctypes.POINTER(_MxTensor), vp, i64,
                                                 ctypes.c_int, vp, sz, vp]),
            "mxc_moe_linear": (ctypes.c_int, [ctypes.POINTER(_MxTensor), vp, ctypes.POINTER(_Weight), i32, vp, i64,
                                              ctypes.c_int, vp, sz, vp]),
            "mxc_moe_linear_noalloc": (ctypes.c_int, [ctypes.POINTER(_MxTensor), vp, ctypes.POINTER(_Weight), i32,
                                                      vp, i64, ctypes.c_int, vp]),
            "mxc_decode_weight": (ctypes.c_int, [ctypes.POINTER(_Weight), vp, i64, vp, vp]),
            "mxc_get_device_error": (ctypes.c_int, [vp]),
            "mxc_selftest_wait_timeout": (ctypes.c_int, [i64, vp]),
            "mxc_moe_gate_up_swiglu": (ctypes.c_int, [ctypes.POINTER(_MxTensor), vp, ctypes.POINTER(_Weight), i32, vp,
                                                      vp, i64, vp, vp, sz, vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != 0:
        raise MxcError(status, what)


def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def sf_bytes(rows: int, K: int, fmt: str) -> int:
    return lib().mxc_sf_bytes(rows, K, FMT[fmt])


# ---------------------------------------------------------------------------
# Activations
# ---------------------------------------------------------------------------

@dataclass
class MXTensor:
    """An MX-quantized matrix on the device: FP4 codes, SF-layout scales, tensor scale."""
    q: torch.Tensor          # uint8 [rows, ldq]
    sf: torch.Tensor         # uint8, SF layout
    tscale: Optional[torch.Tensor]  # float32 [1] or None
    rows: int
    K: int
    fmt: str

    def _c(self) -> _MxTensor:
        # the C struct is rebuilt only when a field it holds has changed
        key = (self.q.data_ptr(), self.sf.data_ptr(), _ptr(self.tscale), self.rows, self.K, self.q.stride(0),
               self.fmt)
        c = self.__dict__.get("_cstruct")
        if c is None or c[0] != key:
            c = (key, _MxTensor(key[0], key[1], key[2], self.rows, self.K, key[5], FMT[self.fmt]))
            self.__dict__["_cstruct"] = c
        return c[1]


def empty_act(M: int, K: int, fmt: str, device) -> MXTensor:
    """Output buffers for quantize_act: FP4 codes, SF-layout scales, tensor scale."""
    q = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
    sf = torch.empty((max(1, sf_bytes(M, K, fmt)),), dtype=torch.uint8, device=device)
    ts = torch.empty((1,), dtype=torch.float32, device=device) if fmt == "e4m3_b16" else None
    return MXTensor(q, sf, ts, M, K, fmt)


def quantize_act(x: torch.Tensor, fmt: str, tscale_in: Optional[torch.Tensor] = None, out: Optional[MXTensor] = None,
                 ws: Optional[torch.Tensor] = None, stream=None) -> MXTensor:
    """mxc_quantize_act: BF16 [M, K] (device) -> MXTensor (written into `out` if given)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.is_cuda
    M, K = x.shape
    dev = x.device
    out = empty_act(M, K, fmt, dev) if out is None else out
    if ws is None:
        ws = torch.empty((lib().mxc_quantize_act_workspace_bytes(M, K, FMT[fmt]),), dtype=torch.uint8, device=dev)
    _check(lib().mxc_quantize_act(x.data_ptr(), M, K, x.stride(0), FMT[fmt], _ptr(tscale_in), out.q.data_ptr(),
                                  out.q.stride(0), out.sf.data_ptr(), _ptr(out.tscale), ws.data_ptr(), ws.numel(),
                                  _stream(stream)),
           "mxc_quantize_act")
    return out


def empty_act_grouped(M: int, K: int, E: int, fmt: str, device) -> MXTensor:
    """Output buffers for quantize_act_grouped (grouped SF layout, padding zeroed)."""
    rows_sf = lib().mxc_grouped_sf_rows_bound(M, E)
    q = torch.empty((M, K // 2), dtype=torch.uint8, device=device)
    sf = torch.zeros((max(1, sf_bytes(rows_sf, K, fmt)),), dtype=torch.uint8, device=device)
    ts = torch.empty((1,), dtype=torch.float32, device=device) if fmt == "e4m3_b16" else None
    return MXTensor(q, sf, ts, M, K, fmt)


def quantize_act_grouped(x: torch.Tensor, fmt: str, offsets: torch.Tensor, tscale_in=None,
                         out: Optional[MXTensor] = None, ws: Optional[torch.Tensor] = None,
                         stream=None) -> MXTensor:
    """mxc_quantize_act_grouped: rows sorted by group, offsets int32 [E+1] on the device."""
    assert x.dtype == torch.bfloat16 and offsets.dtype == torch.int32
    M, K = x.shape
    E = offsets.numel() - 1
    dev = x.device
    out = empty_act_grouped(M, K, E, fmt, dev) if out is None else out
    if ws is None:
        ws = torch.empty((lib().mxc_quantize_act_workspace_bytes(M, K, FMT[fmt]) + 4 * (E + 1),),
                         dtype=torch.uint8, device=dev)
    _check(lib().mxc_quantize_act_grouped(x.data_ptr(), M, K, x.stride(0), FMT[fmt], offsets.data_ptr(), E,
                                          _ptr(tscale_in), out.q.data_ptr(), out.q.stride(0), out.sf.data_ptr(),
                                          _ptr(out.tscale), ws.data_ptr(), ws.numel(), _stream(stream)),
           "mxc_quantize_act_grouped")
    return out


# ---------------------------------------------------------------------------
# Weights
# ---------------------------------------------------------------------------

@dataclass
class PackedWeight:
    """A VQ weight in the packed device layout (see mxc_weight in mxc.h)."""
    fmt: str
    strategy: str
    N: int
    K: int
    qn: int
    qk: int
    idx: torch.Tensor
    cb: torch.Tensor
    scales: Optional[torch.Tensor]
    sidx: Optional[torch.Tensor]
    scb: Optional[torch.Tensor]
    w_tscale: float
    ds: int = 8                 # PreScale+ scale group

    def _c(self) -> _Weight:
        key = (self.strategy, self.fmt, self.N, self.K, self.qn, self.qk, self.idx.data_ptr(), self.cb.data_ptr(),
               _ptr(self.scales), _ptr(self.sidx), _ptr(self.scb), self.w_tscale, self.ds)
        c = self.__dict__.get("_cstruct")
        if c is None or c[0] != key:
            c = (key, _Weight(STRATEGY[self.strategy], FMT[self.fmt], *key[2:]))
            self.__dict__["_cstruct"] = c
        return c[1]

    def storage_bytes(self) -> int:
        n = self.idx.numel() + self.cb.numel() * 2
        if self.strategy == "prescale_plus":
            return n + self.sidx.numel() + self.scb.numel()
        if self.strategy == "postscale_qb":
            return n + self.scales.numel()              # one scale per QBlock
        return n + self.N * self.K // BLOCK[self.fmt]


def _host_struct(w, keep: list) -> _WeightHost:
    def arr(a, dtype):
        if a is None:
            return None
        a = np.ascontiguousarray(a, dtype=dtype)
        keep.append(a)
        return a.ctypes.data
    return _WeightHost(STRATEGY[w.strategy], FMT[w.fmt], w.N, w.K, w.qn, w.qk, arr(w.idx, np.uint8),
                       arr(w.cb, np.uint16), arr(w.scales, np.uint8), arr(w.sidx, np.uint8), arr(w.scb, np.uint8),
                       float(w.w_tscale), int(getattr(w, "ds", 8)))


def pack_weight_host(w) -> dict:
    """mxc_pack_weight on host arrays -> dict of numpy arrays in the packed layout."""
    keep: list = []
    hw = _host_struct(w, keep)
    sizes = _PackedSizes()
    _check(lib().mxc_packed_weight_sizes(ctypes.byref(hw), ctypes.byref(sizes)), "mxc_packed_weight_sizes")
    idx = np.empty(sizes.idx, dtype=np.uint8)
    scales = np.empty(sizes.scales, dtype=np.uint8) if sizes.scales else None
    sidx = np.empty(sizes.sidx, dtype=np.uint8) if sizes.sidx else None
    _check(lib().mxc_pack_weight(ctypes.byref(hw), idx.ctypes.data,
                                 None if scales is None else scales.ctypes.data,
                                 None if sidx is None else sidx.ctypes.data), "mxc_pack_weight")
    return {"idx": idx, "scales": scales, "sidx": sidx,
            "cb": np.ascontiguousarray(w.cb, dtype=np.uint16).reshape(-1),
            "scb": None if w.scb is None else np.ascontiguousarray(w.scb, dtype=np.uint8).reshape(-1)}


def pack_weight(w, device="cuda") -> PackedWeight:
    """Packs a logical weight (any object with fmt/strategy/N/K/qn/qk/idx/cb/scales/sidx/scb/w_tscale)
    and uploads it."""
    h = pack_weight_host(w)

    def up(a):
        return None if a is None else torch.from_numpy(a).to(device)
    cb = torch.from_numpy(h["cb"].view(np.int16)).to(device)
    return PackedWeight(w.fmt, w.strategy, w.N, w.K, w.qn, w.qk, up(h["idx"]), cb, up(h["scales"]),
                        up(h["sidx"]), up(h["scb"]), float(w.w_tscale), int(getattr(w, "ds", 8)))


# ---------------------------------------------------------------------------
# Linear layers
# ---------------------------------------------------------------------------

def _out(M: int, N: int, dtype, dev) -> torch.Tensor:
    return torch.empty((M, N), dtype=dtype, device=dev)


def linear_workspace(M: int, N: int, K: int, fmt: str, device) -> torch.Tensor:
    """Workspace of mxc_linear / mxc_native_linear, zero-filled (its split-K arrival
    counters must be zero when a call starts; every call leaves them zero)."""
    n = lib().mxc_linear_workspace_bytes(M, N, K, FMT[fmt])
    return torch.zeros((max(n, 16),), dtype=torch.uint8, device=device)


def linear(a: MXTensor, w: PackedWeight, out_dtype=torch.float32, y: Optional[torch.Tensor] = None,
           ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """mxc_linear: y[M, N] = A . W^T with W decoded on the fly."""
    dev = a.q.device
    y = _out(a.rows, w.N, out_dtype, dev) if y is None else y
    at, wt = a._c(), w._c()
    if ws is None:
        n = lib().mxc_linear_workspace_bytes_for(ctypes.byref(wt), a.rows)
        ws = torch.zeros((max(n, 16),), dtype=torch.uint8, device=dev)
    _check(lib().mxc_linear(ctypes.byref(at), ctypes.byref(wt), y.data_ptr(), y.stride(0), OUT[y.dtype],
                            ws.data_ptr(), ws.numel(), _stream(stream)), "mxc_linear")
    return y


def native_linear(a: MXTensor, w: MXTensor, out_dtype=torch.float32, y: Optional[torch.Tensor] = None,
                  ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """mxc_native_linear: the same GEMM with a native block-scaled FP4 weight."""
    dev = a.q.device
    y = _out(a.rows, w.rows, out_dtype, dev) if y is None else y
    ws = linear_workspace(a.rows, w.rows, w.K, w.fmt, dev) if ws is None else ws
    at, wt = a._c(), w._c()
    _check(lib().mxc_native_linear(ctypes.byref(at), ctypes.byref(wt), y.data_ptr(), y.stride(0), OUT[y.dtype],
                                   ws.data_ptr(), ws.numel(), _stream(stream)), "mxc_native_linear")
    return y


def moe_linear(a: MXTensor, offsets: torch.Tensor, experts: Sequence[PackedWeight], out_dtype=torch.float32,
               y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """mxc_moe_linear: expert-grouped rows, expert e owning rows [offsets[e], offsets[e+1])."""
    E = len(experts)
    dev = a.q.device
    N = experts[0].N
    y = _out(a.rows, N, out_dtype, dev) if y is None else y
    if ws is None:
        ws = torch.empty((max(16, lib().mxc_moe_workspace_bytes(a.rows, E, N, a.K, FMT[a.fmt])),),
                         dtype=torch.uint8, device=dev)
    table = (_Weight * E)(*[w._c() for w in experts])
    at = a._c()
    _check(lib().mxc_moe_linear(ctypes.byref(at), offsets.data_ptr(), table, E, y.data_ptr(), y.stride(0),
                                OUT[y.dtype], ws.data_ptr(), ws.numel(), _stream(stream)), "mxc_moe_linear")
    return y


def moe_gate_up_swiglu(a: MXTensor, offsets: torch.Tensor, experts: Sequence[PackedWeight],
                       h_tscale: Optional[torch.Tensor] = None, out: Optional[MXTensor] = None,
                       ws: Optional[torch.Tensor] = None, stream=None) -> MXTensor:
    """mxc_moe_gate_up_swiglu: gate/up projection, SwiGLU and the down projection's MX
    quantization in one kernel.  Returns h as a grouped MXTensor (F = N/2 channels)
    that moe_linear takes over the same offsets.  h_tscale (float32 [1], device) is
    required for e4m3_b16."""
    E = len(experts)
    dev = a.q.device
    F = experts[0].N // 2
    if out is None:
        out = empty_act_grouped(a.rows, F, E, a.fmt, dev)
        if a.fmt == "e4m3_b16":
            out.tscale = h_tscale
    if ws is None:
        ws = torch.empty((max(16, lib().mxc_moe_workspace_bytes(a.rows, E, experts[0].N, a.K, FMT[a.fmt])),),
                         dtype=torch.uint8, device=dev)
    table = (_Weight * E)(*[w._c() for w in experts])
    at = a._c()
    _check(lib().mxc_moe_gate_up_swiglu(ctypes.byref(at), offsets.data_ptr(), table, E, _ptr(h_tscale),
                                        out.q.data_ptr(), out.q.stride(0), out.sf.data_ptr(), ws.data_ptr(),
                                        ws.numel(), _stream(stream)), "mxc_moe_gate_up_swiglu")
    return out


def moe_linear_noalloc(a: MXTensor, offsets: torch.Tensor, experts: Sequence[PackedWeight],
                       out_dtype=torch.float32, y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """mxc_moe_linear_noalloc: mxc_moe_linear without a caller workspace (for callers that
    cannot allocate device memory); the library uses a fixed device array instead."""
    E = len(experts)
    y = _out(a.rows, experts[0].N, out_dtype, a.q.device) if y is None else y
    table = (_Weight * E)(*[w._c() for w in experts])
    at = a._c()
    _check(lib().mxc_moe_linear_noalloc(ctypes.byref(at), offsets.data_ptr(), table, E, y.data_ptr(), y.stride(0),
                                        OUT[y.dtype], _stream(stream)), "mxc_moe_linear_noalloc")
    return y


def decode_weight(w: PackedWeight, stream=None) -> MXTensor:
    """mxc_decode_weight: the on-the-fly decode, written out as a native FP4 weight."""
    dev = w.idx.device
    q = torch.empty((w.N, w.K // 2), dtype=torch.uint8, device=dev)
    sf = torch.empty((sf_bytes(w.N, w.K, w.fmt),), dtype=torch.uint8, device=dev)
    wt = w._c()
    _check(lib().mxc_decode_weight(ctypes.byref(wt), q.data_ptr(), w.K // 2, sf.data_ptr(), _stream(stream)),
           "mxc_decode_weight")
    ts = torch.tensor([w.w_tscale], dtype=torch.float32, device=dev)
    return MXTensor(q, sf, ts, w.N, w.K, w.fmt)


def selftest_wait_timeout(limit_cycles: int, stream=None) -> None:
    """mxc_selftest_wait_timeout: a bounded device wait that is made to run out."""
    _check(lib().mxc_selftest_wait_timeout(limit_cycles, _stream(stream)), "mxc_selftest_wait_timeout")


def get_device_error(stream=None) -> int:
    """mxc_get_device_error: synchronizes the stream, returns and clears the device error word."""
    return lib().mxc_get_device_error(_stream(stream))


# ---------------------------------------------------------------------------
# Layout helper for callers that want the scales back in [rows, K/B] form
# ---------------------------------------------------------------------------

def sf_to_rows(sf: np.ndarray, rows: int, K: int, fmt: str) -> np.ndarray:
    """Reads an SF-layout buffer (mxc.h) back into a [rows, K/B] array of scale bytes."""
    KB = K // BLOCK[fmt]
    r = np.arange(rows)[:, None]
    kb = np.arange(KB)[None, :]
    off = ((r // 128) * (KB // 4) + kb // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + (kb % 4)
    return np.asarray(sf)[off]
