"""CPU oracle of the fixed-codebook entropy coder (test infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import this
package. It wraps ``oracle.cpp`` (plain C++17, bit-serial) through ctypes and shares nothing with
the CUDA library. ``build()`` compiles it with g++ into ``oracle/liboracle.so``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "oracle.cpp")
LIB = os.path.join(HERE, "liboracle.so")

ERR_ARG, ERR_UNCODABLE, ERR_CORRUPT, ERR_CODEBOOK, ERR_CAPACITY = 1, 4, 8, 16, 64
KIND_HUFFMAN, KIND_QLC, KIND_SHANNONIC, KIND_EXPGOLOMB = 0, 1, 2, 3
SHN_K, SHN_L, SHN_R = 16, 128, 7
QLC_LMAX = 11

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.cpp with g++ (-O2, no GPU code) unless the library is newer than it."""
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run(["g++", "-std=c++17", "-O2", "-fPIC", "-shared", "-Wall", "-o", tmp, SRC],
                       check=True)
        os.replace(tmp, LIB)
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        P, u64, i32 = ctypes.c_void_p, ctypes.c_uint64, ctypes.c_int
        sig = {
            "orc_histogram": (None, [P, u64, P]),
            "orc_huffman_lengths": (i32, [P, i32, i32, P]),
            "orc_canonical_codes": (None, [P, P]),
            "orc_qlc_build": (i32, [P, i32, P, P, P, P, P]),
            "orc_hash_huffman": (u64, [i32, P]),
            "orc_hash_qlc": (u64, [P, P]),
            "orc_payload_offset": (u64, [u64]),
            "orc_sync_offset": (u64, [u64]),
            "orc_encode_bound": (u64, [u64]),
            "orc_encode_huffman": (i32, [i32, P, P, u64, P, u64, P]),
            "orc_decode_huffman": (i32, [i32, P, P, u64, P, u64]),
            "orc_encode_qlc": (i32, [P, P, P, P, u64, P, u64, P]),
            "orc_decode_qlc": (i32, [P, P, P, P, u64, P, u64]),
            "orc_entropy": (ctypes.c_double, [P]),
            "orc_fnv1a": (u64, [P, u64]),
            "orc_mean_length": (ctypes.c_double, [P, P]),
            "orc_shannonic_build": (i32, [P, i32, i32, P, P, P]),
            "orc_shannonic_partition": (i32, [P, i32, i32, P]),
            "orc_shannonic_normalise": (i32, [P, i32, P]),
            "orc_hash_shannonic": (u64, [i32, P, P]),
            "orc_shannonic_encode_bound": (u64, [u64]),
            "orc_encode_shannonic": (i32, [i32, P, P, P, u64, P, u64, P]),
            "orc_decode_shannonic": (i32, [i32, P, P, P, u64, P, u64]),
            "orc_expgolomb_codes": (i32, [i32, i32, P, P]),
            "orc_hash_expgolomb": (u64, [i32, i32]),
            "orc_encode_expgolomb": (i32, [i32, i32, P, u64, P, u64, P]),
            "orc_decode_expgolomb": (i32, [i32, i32, P, u64, P, u64]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def _u8(x) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(x, dtype=np.uint8).reshape(-1))


def histogram(x) -> np.ndarray:
    x = _u8(x)
    c = np.zeros(256, dtype=np.uint64)
    lib().orc_histogram(_p(x), x.size, _p(c))
    return c


def huffman_lengths(counts, lmax: int = 12, cover_all: bool = True) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.uint64))
    ln = np.zeros(256, dtype=np.uint8)
    rc = lib().orc_huffman_lengths(_p(c), int(lmax), int(bool(cover_all)), _p(ln))
    if rc:
        raise ValueError("lmax too small for the alphabet")
    return ln


def canonical_codes(lengths) -> np.ndarray:
    ln = _u8(lengths)
    code = np.zeros(256, dtype=np.uint32)
    lib().orc_canonical_codes(_p(ln), _p(code))
    return code


@dataclass
class Codebook:
    kind: int
    lmax: int
    len: np.ndarray        # u8[256]
    code: np.ndarray       # u32[256]
    bits: np.ndarray | None = None      # QLC u8[8]
    start: np.ndarray | None = None     # QLC u16[9]
    rank2sym: np.ndarray | None = None  # QLC u8[256]

    @property
    def hash(self) -> int:
        L = lib()
        if self.kind == KIND_HUFFMAN:
            return int(L.orc_hash_huffman(self.lmax, _p(self.len)))
        return int(L.orc_hash_qlc(_p(self.bits), _p(self.rank2sym)))


def huffman_codebook(counts, lmax: int = 12, cover_all: bool = True) -> Codebook:
    ln = huffman_lengths(counts, lmax, cover_all)
    return Codebook(KIND_HUFFMAN, lmax, ln, canonical_codes(ln))


def qlc_codebook(counts, max_distinct: int = 4) -> Codebook:
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.uint64))
    bits = np.zeros(8, np.uint8)
    start = np.zeros(9, np.uint16)
    r2s = np.zeros(256, np.uint8)
    ln = np.zeros(256, np.uint8)
    code = np.zeros(256, np.uint32)
    rc = lib().orc_qlc_build(_p(c), int(max_distinct), _p(bits), _p(start), _p(r2s), _p(ln), _p(code))
    if rc:
        raise ValueError("bad max_distinct")
    return Codebook(KIND_QLC, QLC_LMAX, ln, code, bits, start, r2s)


def payload_offset(n: int) -> int:
    return int(lib().orc_payload_offset(n))


def sync_offset(n: int) -> int:
    return int(lib().orc_sync_offset(n))


def encode_bound(n: int) -> int:
    return int(lib().orc_encode_bound(n))


@dataclass
class ShannonicBook:
    """[SHN] ranges lo[0..nr] over the byte values and their tANS frequencies f (sum 128)."""
    nr: int
    lo: np.ndarray  # i32[nr + 1]
    f: np.ndarray   # i32[nr]
    kind: int = KIND_SHANNONIC

    @property
    def hash(self) -> int:
        return int(lib().orc_hash_shannonic(self.nr, _p(self.lo), _p(self.f)))

    @property
    def offset_bits(self) -> np.ndarray:
        return np.array([int(np.ceil(np.log2(b - a))) if b - a > 1 else 0
                         for a, b in zip(self.lo[:-1], self.lo[1:])])


def shannonic_codebook(counts, K: int = SHN_K, cover_all: bool = True) -> ShannonicBook:
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.uint64))
    nr = ctypes.c_int()
    lo = np.zeros(SHN_K + 1, np.int32)
    f = np.zeros(SHN_K, np.int32)
    if lib().orc_shannonic_build(_p(c), int(K), int(cover_all), ctypes.byref(nr), _p(lo), _p(f)):
        raise ValueError("no Shannonic codebook for these counts")
    k = nr.value
    return ShannonicBook(k, lo[:k + 1].copy(), f[:k].copy())


def shannonic_partition(weights, K: int) -> np.ndarray:
    """The dynamic programme's partition of any alphabet (boundaries lo[0..nr])."""
    w = np.ascontiguousarray(np.asarray(weights, dtype=np.uint64))
    lo = np.zeros(K + 1, np.int32)
    k = lib().orc_shannonic_partition(_p(w), w.size, int(K), _p(lo))
    return lo[:k + 1].copy()


def shannonic_normalise(range_weights) -> np.ndarray:
    wr = np.ascontiguousarray(np.asarray(range_weights, dtype=np.uint64))
    f = np.zeros(wr.size, np.int32)
    lib().orc_shannonic_normalise(_p(wr), wr.size, _p(f))
    return f


@dataclass
class ExpGolombBook:
    """[EG] order and byte-to-index map (0 sign-magnitude, 1 two's complement zigzag)."""
    order: int
    map: int
    kind: int = KIND_EXPGOLOMB

    @property
    def hash(self) -> int:
        return int(lib().orc_hash_expgolomb(self.order, self.map))

    @property
    def codes(self) -> tuple[np.ndarray, np.ndarray]:
        ln = np.zeros(256, np.uint8)
        code = np.zeros(256, np.uint32)
        if lib().orc_expgolomb_codes(self.order, self.map, _p(ln), _p(code)):
            raise ValueError("bad Exp-Golomb order or map")
        return ln, code

    @property
    def len(self) -> np.ndarray:
        return self.codes[0]


def shannonic_encode_bound(n: int) -> int:
    return int(lib().orc_shannonic_encode_bound(n))


def encode(cb, x, cap: int | None = None) -> tuple[int, np.ndarray]:
    """Bit-serial encode into the chunked stream; returns (status, stream bytes)."""
    x = _u8(x)
    if cb.kind == KIND_EXPGOLOMB:
        cap = encode_bound(x.size) if cap is None else int(cap)
        out = np.zeros(max(cap, 1), dtype=np.uint8)
        written = ctypes.c_uint64(0)
        st = lib().orc_encode_expgolomb(cb.order, cb.map, _p(x), x.size, _p(out), cap,
                                        ctypes.byref(written))
        return int(st), out[: written.value] if written.value else out[: min(cap, 64)]
    if cb.kind == KIND_SHANNONIC:
        cap = shannonic_encode_bound(x.size) if cap is None else int(cap)
        out = np.zeros(max(cap, 1), dtype=np.uint8)
        written = ctypes.c_uint64(0)
        st = lib().orc_encode_shannonic(cb.nr, _p(cb.lo), _p(cb.f), _p(x), x.size, _p(out), cap,
                                        ctypes.byref(written))
        return int(st), out[: written.value] if written.value else out[: min(cap, 64)]
    cap = encode_bound(x.size) if cap is None else int(cap)
    out = np.zeros(max(cap, 1), dtype=np.uint8)
    written = ctypes.c_uint64(0)
    if cb.kind == KIND_HUFFMAN:
        st = lib().orc_encode_huffman(cb.lmax, _p(cb.len), _p(x), x.size, _p(out), cap,
                                      ctypes.byref(written))
    else:
        st = lib().orc_encode_qlc(_p(cb.bits), _p(cb.start), _p(cb.rank2sym), _p(x), x.size,
                                  _p(out), cap, ctypes.byref(written))
    return int(st), out[: written.value] if written.value else out[: min(cap, 64)]


def decode(cb, stream, n: int) -> tuple[int, np.ndarray]:
    """Bit-serial decode; returns (status, n bytes)."""
    s = _u8(stream)
    out = np.zeros(max(n, 1), dtype=np.uint8)
    if cb.kind == KIND_EXPGOLOMB:
        st = lib().orc_decode_expgolomb(cb.order, cb.map, _p(s), s.size, _p(out), n)
    elif cb.kind == KIND_SHANNONIC:
        st = lib().orc_decode_shannonic(cb.nr, _p(cb.lo), _p(cb.f), _p(s), s.size, _p(out), n)
    elif cb.kind == KIND_HUFFMAN:
        st = lib().orc_decode_huffman(cb.lmax, _p(cb.len), _p(s), s.size, _p(out), n)
    else:
        st = lib().orc_decode_qlc(_p(cb.bits), _p(cb.start), _p(cb.rank2sym), _p(s), s.size,
                                  _p(out), n)
    return int(st), out[:n]


def fnv1a(data: bytes) -> int:
    b = np.frombuffer(bytes(data), dtype=np.uint8).copy() if data else np.zeros(1, np.uint8)
    return int(lib().orc_fnv1a(_p(b), len(data)))


def entropy(counts) -> float:
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.uint64))
    return float(lib().orc_entropy(_p(c)))


def mean_length(counts, lengths) -> float:
    c = np.ascontiguousarray(np.asarray(counts, dtype=np.uint64))
    return float(lib().orc_mean_length(_p(c), _p(_u8(lengths))))


def session_schedule(hists, kind: int = KIND_HUFFMAN, history: int = 4, lag: int = 2,
                     drift: float = 0.0, initial_counts=None, lmax: int = 12,
                     max_distinct: int = 4, cover_all: bool = True):
    """The online single-stage loop, written out batch by batch.

    "Single-Stage Huffman Encoder for ML Compression", abstract: a batch is coded with the
    codebook of the average distribution of earlier batches. Batch t's codebook is built from the
    summed histograms of the batches observed once batch t - lag has been observed (at most the
    last `history` of them; `initial_counts`, or all ones, before any). Observing batch j computes
    its drift, mean code length under the codebook that coded it over its entropy, minus one;
    above `drift` (> 0) the history restarts from batch j (the drift refresh of the "Shannonic"
    review). Returns (codebook per batch, (refreshed, drift) per batch)."""
    init = np.ones(256, np.uint64) if initial_counts is None else np.asarray(initial_counts, np.uint64)

    def build(c):
        if kind == KIND_HUFFMAN:
            return huffman_codebook(c, lmax, cover_all)
        return qlc_codebook(c, max_distinct)

    window, books, seen = [], [], []

    def observe(j):
        h = np.asarray(hists[j], np.uint64)
        H = entropy(h)
        d, refresh = float("nan"), False
        if H > 0:
            d = mean_length(h, books[j].len) / H - 1.0
            refresh = drift > 0 and d > drift
        if refresh:
            window.clear()
        window.append(h)
        del window[:-history]
        seen.append((refresh, d))

    for t in range(len(hists)):
        if t >= lag:
            observe(t - lag)
        counts = np.sum(window, axis=0, dtype=np.uint64) if window else init
        books.append(build(counts))
    for j in range(max(0, len(hists) - lag), len(hists)):
        observe(j)
    return books, seen
