"""Python binding of the hx C ABI (include/hx.h): argument marshalling only.

Every step of the coder runs in libhx.so: the codebook builder on the host, the histogram,
encode and decode kernels on the GPU. PyTorch supplies device memory and the current CUDA
stream; tensors are passed as raw pointers. There is no fallback: if the library is missing or
cannot load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import numpy as np

from . import build as _build

HX_OK, HX_ERR_ARG, HX_ERR_CUDA = 0, 1, 2
HX_ERR_UNCODABLE, HX_ERR_CORRUPT, HX_ERR_CODEBOOK, HX_ERR_TIMEOUT, HX_ERR_CAPACITY = 4, 8, 16, 32, 64
KIND_HUFFMAN, KIND_QLC, KIND_SHANNONIC, KIND_EXPGOLOMB = 0, 1, 2, 3
CHUNK, SUBSTREAMS, LMAX_MAX, QLC_LMAX = 4096, 8, 12, 11
CB_SEEN_ONLY = 1
TABLES_BYTES = 10240

HEADER = os.path.join(_build.INCLUDE, "hx.h")


class HxError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__(f"{what}: status {code} ({status_string(code)})")
        self.code = code


class _Codebook(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_uint8), ("lmax", ctypes.c_uint8),
                ("len", ctypes.c_uint8 * 256), ("code", ctypes.c_uint16 * 256),
                ("qlc_bits", ctypes.c_uint8 * 8), ("qlc_start", ctypes.c_uint16 * 9),
                ("rank2sym", ctypes.c_uint8 * 256), ("hash", ctypes.c_uint64),
                ("sh_nr", ctypes.c_uint8), ("sh_lo", ctypes.c_uint16 * 17),
                ("sh_f", ctypes.c_uint8 * 16)]


_lib = None


def declared_functions() -> list[str]:
    """Names of the functions include/hx.h declares."""
    with open(HEADER) as f:
        text = re.sub(r"/\*.*?\*/", "", f.read(), flags=re.S)
    return re.findall(r"^\s*(?:int|uint64_t|double|const char\*)\s+(hx_\w+)\s*\(", text,
                      flags=re.M)


def lib():
    """Load libhx.so (building it first when the sources are newer). Raises if it cannot."""
    global _lib
    if _lib is None:
        if not _build.up_to_date():
            _build.build()
        L = ctypes.CDLL(_build.LIB)
        P, u64, i32, u32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int, ctypes.c_uint32
        CB = ctypes.POINTER(_Codebook)
        sig = {
            "hx_build_codebook": (i32, [P, i32, u32, CB]),
            "hx_qlc_build": (i32, [P, i32, u32, CB]),
            "hx_codebook_tables": (i32, [CB, P]),
            "hx_codebook_upload": (i32, [CB, P, P]),
            "hx_histogram": (i32, [P, u64, P, P]),
            "hx_payload_offset": (u64, [u64]),
            "hx_sync_offset": (u64, [u64]),
            "hx_encode_bound": (u64, [u64]),
            "hx_scratch_bytes": (u64, [u64]),
            "hx_encode": (i32, [P, P, u64, P, u64, P, P, P, P]),
            "hx_decode": (i32, [P, P, u64, P, u64, P, P]),
            "hx_qlc_encode": (i32, [P, P, u64, P, u64, P, P, P, P]),
            "hx_qlc_decode": (i32, [P, P, u64, P, u64, P, P]),
            "hx_encode_noalloc": (i32, [P, P, u64, P, u64, P, P, P]),
            "hx_encode_bounded": (i32, [u32, P, P, u64, P, u64, P, P, P, u64, u64, u32, P]),
            "hx_shannonic_build": (i32, [P, i32, u32, CB]),
            "hx_expgolomb_build": (i32, [i32, i32, CB]),
            "hx_expgolomb_encode": (i32, [P, P, u64, P, u64, P, P, P, P]),
            "hx_expgolomb_decode": (i32, [P, P, u64, P, u64, P, P]),
            "hx_shannonic_encode_bound": (u64, [u64]),
            "hx_shannonic_encode": (i32, [P, P, u64, P, u64, P, P, P, P]),
            "hx_shannonic_decode": (i32, [P, P, u64, P, u64, P, P]),
            "hx_decode_set": (i32, [u32, P, u32, P, u64, P, u64, P, P]),
            "hx_planner_create": (i32, [ctypes.POINTER(_SessionConfig), P, P]),
            "hx_planner_codebook": (i32, [P, u64, CB]),
            "hx_planner_observe": (i32, [P, u64, P, P, P]),
            "hx_planner_destroy": (None, [P]),
            "hx_session_create": (i32, [ctypes.POINTER(_SessionConfig), P, P, u32, P]),
            "hx_session_encode": (i32, [P, P, u64, P, u64, P, P, P, P]),
            "hx_session_decode": (i32, [P, P, u64, P, u64, P, P]),
            "hx_session_drain": (i32, [P]),
            "hx_session_batch_info": (i32, [P, u64, ctypes.POINTER(_BatchInfo)]),
            "hx_session_destroy": (None, [P]),
            "hx_entropy": (ctypes.c_double, [P]),
            "hx_mean_length": (ctypes.c_double, [P, CB]),
            "hx_version": (i32, []),
            "hx_status_string": (ctypes.c_char_p, [i32]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().hx_status_string(int(code)).decode()


def _check(rc: int, what: str) -> None:
    if rc:
        raise HxError(rc, what)


class _SessionConfig(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_uint32), ("lmax", ctypes.c_uint32),
                ("max_distinct", ctypes.c_uint32), ("flags", ctypes.c_uint32),
                ("history", ctypes.c_uint32), ("lag", ctypes.c_uint32), ("drift", ctypes.c_double)]


class _BatchInfo(ctypes.Structure):
    _fields_ = [("hash", ctypes.c_uint64), ("slot", ctypes.c_uint32), ("observed", ctypes.c_int32),
                ("refreshed", ctypes.c_int32), ("pad", ctypes.c_uint32),
                ("symbols", ctypes.c_uint64), ("drift", ctypes.c_double)]


# ------------------------------------------------------------------------------ codebooks (host)
@dataclass
class Codebook:
    """A host codebook (hx_codebook)."""
    raw: _Codebook

    @property
    def kind(self) -> int:
        return self.raw.kind

    @property
    def lmax(self) -> int:
        return self.raw.lmax

    @property
    def len(self) -> np.ndarray:
        return np.frombuffer(bytes(self.raw.len), np.uint8).copy()

    @property
    def code(self) -> np.ndarray:
        return np.frombuffer(bytes(self.raw.code), np.uint16).copy()

    @property
    def qlc_bits(self) -> np.ndarray:
        return np.frombuffer(bytes(self.raw.qlc_bits), np.uint8).copy()

    @property
    def qlc_start(self) -> np.ndarray:
        return np.frombuffer(bytes(self.raw.qlc_start), np.uint16).copy()

    @property
    def rank2sym(self) -> np.ndarray:
        return np.frombuffer(bytes(self.raw.rank2sym), np.uint8).copy()

    @property
    def hash(self) -> int:
        return int(self.raw.hash)

    @property
    def sh_lo(self) -> np.ndarray:
        return np.frombuffer(bytes(self.raw.sh_lo), np.uint16)[: self.raw.sh_nr + 1].copy()

    @property
    def sh_f(self) -> np.ndarray:
        return np.frombuffer(bytes(self.raw.sh_f), np.uint8)[: self.raw.sh_nr].copy()

    def tables(self) -> bytes:
        buf = (ctypes.c_uint8 * TABLES_BYTES)()
        _check(lib().hx_codebook_tables(ctypes.byref(self.raw), buf), "hx_codebook_tables")
        return bytes(buf)

    def upload(self, device=None):
        """The table block as a device uint8 tensor (HX_TABLES_BYTES), copied on the current stream."""
        import torch
        t = torch.empty(TABLES_BYTES, dtype=torch.uint8, device=device or "cuda")
        _check(lib().hx_codebook_upload(ctypes.byref(self.raw), t.data_ptr(), _stream(t)),
               "hx_codebook_upload")
        return t


def _counts(counts) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.uint64).reshape(-1))
    if c.size != 256:
        raise ValueError("counts must have 256 entries")
    return c


def build_codebook(counts, lmax: int = 12, seen_only: bool = False) -> Codebook:
    c = _counts(counts)
    raw = _Codebook()
    _check(lib().hx_build_codebook(c.ctypes.data, int(lmax), CB_SEEN_ONLY if seen_only else 0,
                                   ctypes.byref(raw)), "hx_build_codebook")
    return Codebook(raw)


def qlc_build(counts, max_distinct: int = 4) -> Codebook:
    c = _counts(counts)
    raw = _Codebook()
    _check(lib().hx_qlc_build(c.ctypes.data, int(max_distinct), 0, ctypes.byref(raw)),
           "hx_qlc_build")
    return Codebook(raw)


def shannonic_build(counts, K: int = 16) -> Codebook:
    """hx_shannonic_build: range partition (at most K ranges) and 128-state tANS frequencies."""
    c = _counts(counts)
    raw = _Codebook()
    _check(lib().hx_shannonic_build(c.ctypes.data, int(K), 0, ctypes.byref(raw)),
           "hx_shannonic_build")
    return Codebook(raw)


def expgolomb_build(order: int = 5, map: int = 0) -> Codebook:
    """hx_expgolomb_build: Exp-Golomb of order 5..8 over a sign/magnitude (map 0) or zigzag
    (map 1) index of the byte."""
    raw = _Codebook()
    _check(lib().hx_expgolomb_build(int(order), int(map), ctypes.byref(raw)), "hx_expgolomb_build")
    return Codebook(raw)


def entropy(counts) -> float:
    """Shannon entropy of a 256-bin histogram, bits per symbol."""
    c = _counts(counts)
    return float(lib().hx_entropy(c.ctypes.data))


def mean_length(counts, cb: Codebook) -> float:
    """Mean code length (bits per symbol) of `cb` on data with this histogram."""
    c = _counts(counts)
    return float(lib().hx_mean_length(c.ctypes.data, ctypes.byref(cb.raw)))


# ------------------------------------------------------------------------------ layout helpers
def payload_offset(n: int) -> int:
    return int(lib().hx_payload_offset(n))


def sync_offset(n: int) -> int:
    return int(lib().hx_sync_offset(n))


def encode_bound(n: int, kind: int = KIND_HUFFMAN) -> int:
    if kind == KIND_SHANNONIC:
        return int(lib().hx_shannonic_encode_bound(n))
    return int(lib().hx_encode_bound(n))


def scratch_bytes(n: int) -> int:
    return int(lib().hx_scratch_bytes(n))


def stream_bytes(n: int, total_words: int) -> int:
    return payload_offset(n) + 4 * (int(total_words) + 2)


# ------------------------------------------------------------------------------ device calls
def _stream(t) -> int:
    import torch
    return torch.cuda.current_stream(t.device).cuda_stream


def _dev_u8(x, what):
    import torch
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.uint8 and x.is_contiguous()):
        raise TypeError(f"{what} must be a contiguous CUDA uint8 tensor")
    return x


def new_status(device=None):
    import torch
    return torch.zeros(1, dtype=torch.int32, device=device or "cuda")


def histogram(x, counts=None):
    """counts (int32[256] on the device) += histogram of x; returns counts."""
    import torch
    x = _dev_u8(x, "x")
    if counts is None:
        counts = torch.zeros(256, dtype=torch.int32, device=x.device)
    _check(lib().hx_histogram(x.data_ptr(), x.numel(), counts.data_ptr(), _stream(x)), "hx_histogram")
    return counts


def encode(tables, x, out=None, scratch=None, hist=None, status=None, kind: int = KIND_HUFFMAN):
    """Encode device bytes x with the device table block `tables`.

    Returns (out, status): out holds the stream (its first stream_size(out, n) bytes are
    meaningful), status is the device status word (0 when every check passed)."""
    import torch
    x = _dev_u8(x, "x")
    n = x.numel()
    if out is None:
        out = torch.empty(encode_bound(n, kind), dtype=torch.uint8, device=x.device)
    if scratch is None:
        scratch = torch.empty(scratch_bytes(n), dtype=torch.uint8, device=x.device)
    if status is None:
        status = new_status(x.device)
    fn = {KIND_HUFFMAN: lib().hx_encode, KIND_QLC: lib().hx_qlc_encode,
          KIND_SHANNONIC: lib().hx_shannonic_encode, KIND_EXPGOLOMB: lib().hx_expgolomb_encode}[kind]
    _check(fn(tables.data_ptr(), x.data_ptr(), n, out.data_ptr(), out.numel(), scratch.data_ptr(),
              hist.data_ptr() if hist is not None else None, status.data_ptr(), _stream(x)),
           "hx_encode")
    return out, status


def encode_bounded(tables, x, out, scratch, wait_ns: int, withhold: int = (1 << 64) - 1,
                   hist=None, status=None, kind: int = KIND_HUFFMAN, flush_rounds: int = 0):
    """hx_encode_bounded: encode() with the chunks' wait limit in nanoseconds and, for failure
    tests, one chunk (`withhold`) that never publishes its word count; `flush_rounds` is the
    chunks a warp codes between its flushes of the fused histogram (0: the default). Returns
    (out, status)."""
    x = _dev_u8(x, "x")
    out = _dev_u8(out, "out")
    if status is None:
        status = new_status(x.device)
    _check(lib().hx_encode_bounded(kind, tables.data_ptr(), x.data_ptr(), x.numel(),
                                   out.data_ptr(), out.numel(), scratch.data_ptr(),
                                   hist.data_ptr() if hist is not None else None,
                                   status.data_ptr(), int(wait_ns), int(withhold),
                                   int(flush_rounds), _stream(x)),
           "hx_encode_bounded")
    return out, status


NOALLOC_MAX_BYTES = 128 << 20


def encode_noalloc(tables, x, out, hist=None, status=None):
    """hx_encode_noalloc: Huffman encode whose scratch lives in the library (no allocation inside
    the call; `out` and `status` are the caller's). For callers that cannot allocate device
    memory at encode time. n <= NOALLOC_MAX_BYTES; calls overlapping on the GPU race."""
    x = _dev_u8(x, "x")
    out = _dev_u8(out, "out")
    if status is None:
        status = new_status(x.device)
    _check(lib().hx_encode_noalloc(tables.data_ptr(), x.data_ptr(), x.numel(), out.data_ptr(),
                                   out.numel(), hist.data_ptr() if hist is not None else None,
                                   status.data_ptr(), _stream(x)), "hx_encode_noalloc")
    return out, status


def decode(tables, stream, n: int, out=None, status=None, kind: int = KIND_HUFFMAN, nbytes=None):
    """Decode n bytes from the device stream. Returns (out, status)."""
    import torch
    stream = _dev_u8(stream, "stream")
    if out is None:
        out = torch.empty(max(n, 1), dtype=torch.uint8, device=stream.device)[:n]
    if status is None:
        status = new_status(stream.device)
    fn = {KIND_HUFFMAN: lib().hx_decode, KIND_QLC: lib().hx_qlc_decode,
          KIND_SHANNONIC: lib().hx_shannonic_decode, KIND_EXPGOLOMB: lib().hx_expgolomb_decode}[kind]
    _check(fn(tables.data_ptr(), stream.data_ptr(), int(nbytes or stream.numel()),
              out.data_ptr() if n else stream.data_ptr(), n, status.data_ptr(), _stream(stream)),
           "hx_decode")
    return out, status


def total_words(stream) -> int:
    """total_words from a stream header (reads 8 bytes back: synchronises with the stream)."""
    return int(np.frombuffer(stream[32:40].cpu().numpy().tobytes(), np.uint64)[0])


def stream_size(stream, n: int) -> int:
    return stream_bytes(n, total_words(stream))


MAX_TABLE_SET = 8


def decode_set(kind: int, tables, stream, n: int, out=None, status=None, nbytes=None):
    """hx_decode_set: decode with whichever of the device table blocks `tables` the stream's
    header hash names (picked on the device). Returns (out, status)."""
    import torch
    stream = _dev_u8(stream, "stream")
    if out is None:
        out = torch.empty(max(n, 1), dtype=torch.uint8, device=stream.device)[:n]
    if status is None:
        status = new_status(stream.device)
    ptrs = (ctypes.c_void_p * len(tables))(*[t.data_ptr() for t in tables])
    _check(lib().hx_decode_set(kind, ptrs, len(tables), stream.data_ptr(),
                               int(nbytes or stream.numel()),
                               out.data_ptr() if n else stream.data_ptr(), n, status.data_ptr(),
                               _stream(stream)), "hx_decode_set")
    return out, status


def _config(kind, history, lag, drift, lmax=12, max_distinct=4, seen_only=False):
    return _SessionConfig(kind=kind, lmax=lmax if kind == KIND_HUFFMAN else 0,
                          max_distinct=max_distinct if kind == KIND_QLC else 0,
                          flags=CB_SEEN_ONLY if seen_only else 0, history=history, lag=lag,
                          drift=float(drift))


class Planner:
    """hx_planner: the online loop's bookkeeping on the host (which codebook codes batch t)."""

    def __init__(self, kind=KIND_HUFFMAN, history=4, lag=2, drift=0.0, initial_counts=None,
                 **kw):
        self._cfg = _config(kind, history, lag, drift, **kw)
        init = None if initial_counts is None else _counts(initial_counts)
        h = ctypes.c_void_p()
        _check(lib().hx_planner_create(ctypes.byref(self._cfg),
                                       None if init is None else init.ctypes.data,
                                       ctypes.byref(h)), "hx_planner_create")
        self._h = h

    def codebook(self, batch: int) -> Codebook:
        raw = _Codebook()
        _check(lib().hx_planner_codebook(self._h, batch, ctypes.byref(raw)), "hx_planner_codebook")
        return Codebook(raw)

    def observe(self, batch: int, counts) -> tuple[bool, float]:
        c = _counts(counts)
        r, d = ctypes.c_int(), ctypes.c_double()
        _check(lib().hx_planner_observe(self._h, batch, c.ctypes.data, ctypes.byref(r),
                                        ctypes.byref(d)), "hx_planner_observe")
        return bool(r.value), float(d.value)

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h and _lib is not None:
            _lib.hx_planner_destroy(h)


class Session:
    """hx_session: encode a sequence of batches, each with the codebook of earlier batches'
    fused histograms; decode picks the table by the stream's codebook hash. The table slots,
    the histogram buffer and the status word are device tensors this object holds."""

    def __init__(self, device, kind=KIND_HUFFMAN, history=4, lag=2, drift=0.0,
                 initial_counts=None, slots=None, **kw):
        import torch
        self._cfg = _config(kind, history, lag, drift, **kw)
        self.kind = kind
        nslots = slots or min(MAX_TABLE_SET, lag + 2)
        self.slots = [torch.empty(TABLES_BYTES, dtype=torch.uint8, device=device)
                      for _ in range(nslots)]
        self.hist = torch.zeros(256, dtype=torch.int32, device=device)
        init = None if initial_counts is None else _counts(initial_counts)
        ptrs = (ctypes.c_void_p * nslots)(*[t.data_ptr() for t in self.slots])
        h = ctypes.c_void_p()
        _check(lib().hx_session_create(ctypes.byref(self._cfg),
                                       None if init is None else init.ctypes.data, ptrs, nslots,
                                       ctypes.byref(h)), "hx_session_create")
        self._h = h

    def encode(self, x, out, scratch, status):
        x = _dev_u8(x, "x")
        _check(lib().hx_session_encode(self._h, x.data_ptr(), x.numel(), out.data_ptr(),
                                       out.numel(), scratch.data_ptr(), self.hist.data_ptr(),
                                       status.data_ptr(), _stream(x)), "hx_session_encode")
        return out

    def decode(self, stream, n: int, out, status, nbytes=None):
        stream = _dev_u8(stream, "stream")
        _check(lib().hx_session_decode(self._h, stream.data_ptr(), int(nbytes or stream.numel()),
                                       out.data_ptr() if n else stream.data_ptr(), n,
                                       status.data_ptr(), _stream(stream)), "hx_session_decode")
        return out

    def drain(self):
        _check(lib().hx_session_drain(self._h), "hx_session_drain")

    def info(self, batch: int) -> dict:
        b = _BatchInfo()
        _check(lib().hx_session_batch_info(self._h, batch, ctypes.byref(b)),
               "hx_session_batch_info")
        return {"hash": int(b.hash), "slot": int(b.slot), "observed": bool(b.observed),
                "refreshed": bool(b.refreshed), "symbols": int(b.symbols),
                "drift": float(b.drift)}

    def __del__(self):
        h, self._h = getattr(self, "_h", None), None
        if h and _lib is not None:
            _lib.hx_session_destroy(h)
