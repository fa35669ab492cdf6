"""Thin Python binding of the C ABI in include/qsa.h (ctypes).

Argument marshalling only: every step runs in the CUDA kernels of
libqsa_b200.so.  Tensors are torch CUDA tensors owned by the caller; the
functions pass their device pointers and the current CUDA stream, check the
returned status and raise ``QSAError`` with the library's message.  There is
no fallback: if the library is missing, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libqsa_b200.so")

HQ, D, HKV, GROUP, NG, HI, DI = 24, 256, 2, 32, 8, 4, 64
MAX_DECODE, MAX_SPLITS, MAX_TOPK, PART_STRIDE = 8, 64, 16384, 2 + 256
MODE_DECODE, MODE_PREFILL = 0, 1

_ERRORS = {1: "QSA_ERR_ARG", 2: "QSA_ERR_WORKSPACE", 3: "QSA_ERR_CUDA", 4: "QSA_ERR_TIMEOUT"}

# Every entry point the header declares, with its ctypes signature.
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float
SIGNATURES = {
    "qsa_workspace_bytes": (_SZ, [_I, _I, _I, _I, _I]),
    "qsa_cache_write": (_I, [_P, _I, _I, _P, _P, _P, _P]),
    "qsa_decode": (_I, [_P, _I, _I, _P, _P, _P, _P, _P, _I, _I, _F, _P, _SZ, _P, _P, _P]),
    "qsa_prefill_chunk": (_I, [_P, _I, _I, _P, _P, _P, _P, _P, _I, _F, _P, _SZ, _P, _P, _P]),
    "qsa_index_score": (_I, [_P, _I, _I, _P, _P, _P, _I64, _P]),
    "qsa_topk_workspace_bytes": (_SZ, [_I, _I, _I]),
    "qsa_topk": (_I, [_P, _I64, _I, _I, _I, _P, _SZ, _P, _P]),
    "qsa_attn": (_I, [_P, _I, _P, _P, _I, _I, _F, _P, _P, _P, _P]),
    "qsa_merge": (_I, [_P, _I, _I, _P, _P, _P]),
    "qsa_topk_static": (_I, [_P, _I64, _I, _I, _I, _P, _P]),
    "qsa_device_status": (_I, [_P, _P]),
    "qsa_selftest_wait_timeout": (_I, [_P]),
    "qsa_trace_begin": (_I, [_I, _P]),
    "qsa_trace_end": (_I, [_I, _P, _P, _P]),
    "qsa_last_error": (ctypes.c_char_p, []),
    "qsa_launch_count": (ctypes.c_uint64, []),
}


class QSAError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{_ERRORS.get(code, code)}: {msg}")
        self.code = code


class CacheStruct(ctypes.Structure):
    _fields_ = [("k", _P), ("v", _P), ("ks", _P), ("vs", _P), ("idx_key", _P),
                ("max_cells", ctypes.c_int32)]


class NewCellsStruct(ctypes.Structure):
    """qsa_new_cells: the step's own cells, appended by the step call itself."""
    _fields_ = [("k", _P), ("v", _P), ("idx_key", _P)]


def _new_cells(append, rows):
    """(struct, reference to keep alive) for append = (k, v, key) tensors, or (None, None)."""
    if append is None:
        return None, None
    k, v, key = append
    for t, name in ((k, "append k"), (v, "append v")):
        _dev(t, torch.float32, name)
        if t.shape[0] != rows:
            raise ValueError(f"{name} has {t.shape[0]} rows, the call has {rows}")
    _dev(key, torch.float16, "append idx_key")
    st = NewCellsStruct(k.data_ptr(), v.data_ptr(), key.data_ptr())
    return ctypes.byref(st), st


_lib = None


def load(path: str = LIB_PATH):
    """Load libqsa_b200.so (build it with top_sparse_attention_score_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library {path} is missing; run __graft_entry__.build()")
        lib = ctypes.CDLL(path)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _check(code: int) -> None:
    if code != 0:
        raise QSAError(code, load().qsa_last_error().decode())


def _ptr(t):
    # the signatures declare c_void_p: a plain int (or None for NULL) needs no wrapper
    return None if t is None else t.data_ptr()


# The raw handle of torch's current stream on the current device, without building
# a torch.cuda.Stream object per call (the public path below is the fallback).
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream):
    if stream is not None:
        return stream.cuda_stream
    if _raw_stream is not None:
        return _raw_stream(torch.cuda.current_device())
    return torch.cuda.current_stream().cuda_stream


def _dev(t: torch.Tensor, dtype, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


@dataclass
class DeviceCache:
    """The five cache arrays in device memory (layout of ``qsa_cache``)."""
    k: torch.Tensor        # int8    [cells][2][256]
    v: torch.Tensor        # int8    [cells][2][256]
    ks: torch.Tensor       # float16 [cells][2][8]
    vs: torch.Tensor       # float16 [cells][2][8]
    idx_key: torch.Tensor  # float16 [cells][64]

    @staticmethod
    def empty(cells: int, device="cuda") -> "DeviceCache":
        return DeviceCache(torch.zeros(cells, HKV, D, dtype=torch.int8, device=device),
                           torch.zeros(cells, HKV, D, dtype=torch.int8, device=device),
                           torch.zeros(cells, HKV, NG, dtype=torch.float16, device=device),
                           torch.zeros(cells, HKV, NG, dtype=torch.float16, device=device),
                           torch.zeros(cells, DI, dtype=torch.float16, device=device))

    @staticmethod
    def from_host(c, device="cuda") -> "DeviceCache":
        """Copy a synth.Cache (numpy arrays) to the device."""
        return DeviceCache(torch.from_numpy(c.k).to(device), torch.from_numpy(c.v).to(device),
                           torch.from_numpy(c.ks).to(device), torch.from_numpy(c.vs).to(device),
                           torch.from_numpy(c.idx_key).to(device))

    @property
    def cells(self) -> int:
        return self.k.shape[0]

    def struct(self) -> CacheStruct:
        _dev(self.k, torch.int8, "k")
        _dev(self.v, torch.int8, "v")
        _dev(self.ks, torch.float16, "ks")
        _dev(self.vs, torch.float16, "vs")
        _dev(self.idx_key, torch.float16, "idx_key")
        return CacheStruct(self.k.data_ptr(), self.v.data_ptr(), self.ks.data_ptr(),
                           self.vs.data_ptr(), self.idx_key.data_ptr(), self.cells)

    def ref(self) -> int:
        """Address of a qsa_cache for this cache, rebuilt (and checked again) whenever
        an array's storage or the cell count differs from the last call."""
        key = (self.k.data_ptr(), self.v.data_ptr(), self.ks.data_ptr(), self.vs.data_ptr(),
               self.idx_key.data_ptr(), self.k.shape[0])
        held = self.__dict__.get("_held")
        if held is None or held[0] != key:
            cs = self.struct()
            held = (key, cs, ctypes.addressof(cs))
            self.__dict__["_held"] = held
        return held[2]


def workspace_bytes(mode: int, rows: int, L: int, top_k: int, nsplit: int = 0) -> int:
    return int(load().qsa_workspace_bytes(mode, rows, L, top_k, nsplit))


def topk_workspace_bytes(rows: int, L: int, top_k: int) -> int:
    return int(load().qsa_topk_workspace_bytes(rows, L, top_k))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    return torch.empty(max(nbytes, 16), dtype=torch.uint8, device=device)


def cache_write(cache: DeviceCache, pos0: int, k, v, key, stream=None) -> None:
    _check(load().qsa_cache_write(cache.ref(), pos0, k.shape[0],
                                  _ptr(_dev(k, torch.float32, "k")), _ptr(_dev(v, torch.float32, "v")),
                                  _ptr(_dev(key, torch.float16, "key")), _stream(stream)))


def _opt(t, dtype, name):
    return None if t is None else _ptr(_dev(t, dtype, name))


def decode(cache: DeviceCache, L: int, q, iq, iw, top_k: int, nsplit: int = 0, scale: float = 1 / 16,
           ws=None, out=None, ids_out=None, stream=None, append=None, gate=None):
    """One decode step of n = q.shape[0] tokens.  append = (k, v, idx_key) writes the
    tokens' own cells at L - n .. L - 1 first (in the same call); gate multiplies the
    output by sigmoid(gate)."""
    n = q.shape[0]
    if ws is None:
        ws = workspace(workspace_bytes(MODE_DECODE, n, L, top_k, nsplit), q.device)
    if out is None:
        out = torch.empty(n, HQ, D, dtype=torch.float32, device=q.device)
    app, _keep = _new_cells(append, n)
    _check(load().qsa_decode(cache.ref(), L, n, app, _ptr(_dev(q, torch.float32, "q")),
                             _ptr(_dev(iq, torch.float16, "iq")), _ptr(_dev(iw, torch.float32, "iw")),
                             _opt(gate, torch.float32, "gate"), top_k, nsplit, scale, _ptr(ws), ws.numel(),
                             _ptr(out), _opt(ids_out, torch.int32, "ids_out"), _stream(stream)))
    return out


def prefill_chunk(cache: DeviceCache, pos0: int, q, iq, iw, top_k: int, scale: float = 1 / 16,
                  ws=None, out=None, ids_out=None, stream=None, append=None, gate=None):
    """One prompt chunk of T = q.shape[0] tokens at pos0.  append = (k, v, idx_key) writes
    the chunk's cells at pos0 .. pos0 + T - 1 first (in the same call)."""
    T = q.shape[0]
    if ws is None:
        ws = workspace(workspace_bytes(MODE_PREFILL, T, pos0 + T, top_k), q.device)
    if out is None:
        out = torch.empty(T, HQ, D, dtype=torch.float32, device=q.device)
    app, _keep = _new_cells(append, T)
    _check(load().qsa_prefill_chunk(cache.ref(), pos0, T, app, _ptr(_dev(q, torch.float32, "q")),
                                    _ptr(_dev(iq, torch.float16, "iq")),
                                    _ptr(_dev(iw, torch.float32, "iw")), _opt(gate, torch.float32, "gate"),
                                    top_k, scale, _ptr(ws), ws.numel(), _ptr(out),
                                    _opt(ids_out, torch.int32, "ids_out"), _stream(stream)))
    return out


def index_score(cache: DeviceCache, iq, iw, ncells: int, scores=None, stream=None):
    rows = iq.shape[0]
    if scores is None:
        ld = (ncells + 3) // 4 * 4
        scores = torch.empty(rows, ld, dtype=torch.float32, device=iq.device)
    _check(load().qsa_index_score(cache.ref(), rows, ncells, _ptr(_dev(iq, torch.float16, "iq")),
                                  _ptr(_dev(iw, torch.float32, "iw")),
                                  _ptr(_dev(scores, torch.float32, "scores")), scores.shape[1],
                                  _stream(stream)))
    return scores


def topk(scores, vis0: int, top_k: int, ws=None, ids=None, stream=None):
    rows, ld = scores.shape
    if ws is None:
        ws = workspace(topk_workspace_bytes(rows, vis0 + rows - 1, top_k), scores.device)
    if ids is None:
        ids = torch.empty(rows, top_k, dtype=torch.int32, device=scores.device)
    _check(load().qsa_topk(_ptr(_dev(scores, torch.float32, "scores")), ld, rows, vis0, top_k,
                           _ptr(ws), ws.numel(), _ptr(_dev(ids, torch.int32, "ids")), _stream(stream)))
    return ids


def attn(cache: DeviceCache, q, ids, nsplit: int = 1, scale: float = 1 / 16, part=None, out=None,
         stream=None, gate=None):
    rows, top_k = ids.shape
    if nsplit == 1 and out is None:
        out = torch.empty(rows, HQ, D, dtype=torch.float32, device=q.device)
    if nsplit > 1 and part is None:
        part = torch.empty(rows, HQ, nsplit, PART_STRIDE, dtype=torch.float32, device=q.device)
    _check(load().qsa_attn(cache.ref(), rows, _ptr(_dev(q, torch.float32, "q")),
                           _ptr(_dev(ids, torch.int32, "ids")), top_k, nsplit, scale,
                           _opt(gate, torch.float32, "gate"), _ptr(part), _ptr(out), _stream(stream)))
    return out if nsplit == 1 else part


def merge(part, out=None, stream=None, gate=None):
    rows, _, nsplit, _ = part.shape
    if out is None:
        out = torch.empty(rows, HQ, D, dtype=torch.float32, device=part.device)
    _check(load().qsa_merge(_ptr(_dev(part, torch.float32, "part")), rows, nsplit,
                            _opt(gate, torch.float32, "gate"), _ptr(_dev(out, torch.float32, "out")),
                            _stream(stream)))
    return out


class trace:
    """Per-kernel device times of the library calls made inside the block, on one stream:

        with qsa.trace() as t:
            qsa.decode(...)
        t.kernels  ->  [(name, ms), ...]

    Events between the kernels serialise them; the times are those of back-to-back kernels.
    """

    def __init__(self, capacity: int = 256, stream=None):
        self.capacity, self.stream, self.kernels = capacity, stream, []

    def __enter__(self):
        _check(load().qsa_trace_begin(self.capacity, _stream(self.stream)))
        return self

    def __exit__(self, *exc):
        n = ctypes.c_int(0)
        ms = (ctypes.c_float * self.capacity)()
        names = (ctypes.c_char_p * self.capacity)()
        _check(load().qsa_trace_end(self.capacity, ctypes.byref(n), ms, names))
        self.kernels = [(names[i].decode(), float(ms[i])) for i in range(min(n.value, self.capacity))]
        return False


def device_status(stream=None) -> int:
    """Read and clear the device's status word (0 or QSA_ERR_TIMEOUT); synchronises."""
    st = ctypes.c_int(0)
    _check(load().qsa_device_status(ctypes.byref(st), _stream(stream)))
    return st.value


def selftest_wait_timeout(stream=None) -> None:
    _check(load().qsa_selftest_wait_timeout(_stream(stream)))


def launch_count() -> int:
    return int(load().qsa_launch_count())


def last_error() -> str:
    return load().qsa_last_error().decode()
