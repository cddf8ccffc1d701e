"""Host side of libhx.so (no GPU): the library loads, exports every symbol include/hx.h declares,
its codebook builder agrees with the oracle's, its layout helpers agree with the format, its
device table block is consistent, and host argument checks reject bad calls before any CUDA work.
"""
import ctypes
import subprocess

import numpy as np
import pytest

import datagen
from lossless_entropy_coding_fixed_b200 import hx
from lossless_entropy_coding_fixed_b200 import build as hxbuild


def test_library_builds_for_sm100a_and_exports_header():
    lib = hx.lib()
    names = hx.declared_functions()
    assert len(names) >= 15
    for name in names:
        assert hasattr(lib, name), name
    out = subprocess.run(["nm", "-D", "--defined-only", hxbuild.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    assert set(names) <= exported
    assert hx.lib().hx_version() == 1
    assert "-gencode" in hxbuild.ARCH and "arch=compute_100a,code=sm_100a" in hxbuild.ARCH


def _count_cases():
    cases = []
    for seed in range(25):
        zeros = [0.0, 0.3, 0.8][seed % 3]
        cases.append(datagen.random_counts(seed, zeros=zeros, skew=0.5 + 0.05 * seed))
    cases.append(np.zeros(256, np.uint64))
    one = np.zeros(256, np.uint64)
    one[200] = 9
    cases.append(one)
    cases.append(np.ones(256, np.uint64))
    return cases


@pytest.mark.parametrize("idx", range(28))
@pytest.mark.parametrize("lmax", [9, 12])
@pytest.mark.parametrize("seen_only", [False, True])
def test_builder_matches_oracle(orc, idx, lmax, seen_only):
    counts = _count_cases()[idx]
    try:
        ref = orc.huffman_codebook(counts, lmax=lmax, cover_all=not seen_only)
    except ValueError:
        with pytest.raises(hx.HxError):
            hx.build_codebook(counts, lmax=lmax, seen_only=seen_only)
        return
    cb = hx.build_codebook(counts, lmax=lmax, seen_only=seen_only)
    assert (cb.len == ref.len).all()
    assert (cb.code == ref.code).all()
    assert cb.hash == ref.hash and cb.kind == 0 and cb.lmax == lmax


@pytest.mark.parametrize("idx", range(28))
@pytest.mark.parametrize("maxd", [1, 3, 4, 8])
def test_qlc_builder_matches_oracle(orc, idx, maxd):
    counts = _count_cases()[idx]
    ref = orc.qlc_codebook(counts, max_distinct=maxd)
    q = hx.qlc_build(counts, max_distinct=maxd)
    assert (q.qlc_bits == ref.bits).all()
    assert (q.qlc_start == ref.start).all()
    assert (q.rank2sym == ref.rank2sym).all()
    assert (q.len == ref.len).all() and (q.code == ref.code).all()
    assert q.hash == ref.hash and q.kind == 1 and q.lmax == 11


def test_config_codebooks_match_oracle(orc):
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(1))
    assert (hx.build_codebook(counts).len == orc.huffman_codebook(counts).len).all()
    assert hx.qlc_build(counts).hash == orc.qlc_codebook(counts).hash


@pytest.mark.parametrize("n", [0, 1, 4095, 4096, 4097, 1 << 20, (1 << 30) + 7, (1 << 32) - 1])
def test_layout_helpers_match_oracle(orc, n):
    assert hx.payload_offset(n) == orc.payload_offset(n)
    assert hx.sync_offset(n) == orc.sync_offset(n)
    assert hx.encode_bound(n) == orc.encode_bound(n)
    assert hx.scratch_bytes(n) >= 8 * (-(-n // 4096))


def _tables(cb):
    t = np.frombuffer(cb.tables(), np.uint8)
    enc = t[:1024].view(np.uint32)
    dec = t[1024:1024 + 8192].view(np.uint16)
    r2s = t[9216:9472]
    area = t[9472:9504].view(np.uint32)
    return enc, dec, r2s, area


@pytest.mark.parametrize("kind", ["huffman", "qlc", "expgolomb"])
def test_table_block_consistent(orc, kind):
    counts = datagen.random_counts(5, zeros=0.4)
    cb = (hx.build_codebook(counts) if kind == "huffman" else hx.qlc_build(counts)
          if kind == "qlc" else hx.expgolomb_build(6, 0))
    enc, dec, r2s, area = _tables(cb)
    ln, code = cb.len.astype(np.int64), cb.code.astype(np.int64)
    assert (enc == (code << 4) | ln).all()
    # every 12-bit window decodes to the code word it starts with
    coded = np.nonzero(ln)[0]
    for w in range(4096):
        e = int(dec[w])
        s, flag, l = e >> 8, (e >> 4) & 15, e & 15
        if e == 0:  # no code word starts this window (only possible for an incomplete code)
            assert not any((w >> (12 - ln[t])) == code[t] for t in coded)
        else:  # (symbol << 8) | valid flag (bit 4) | length
            assert flag == 1 and l == ln[s] and (w >> (12 - l)) == code[s]
    if kind == "qlc":
        assert (r2s == cb.rank2sym).all()
        for a in range(8):
            st, fill, bits = int(area[a]) & 511, (int(area[a]) >> 9) & 511, int(area[a]) >> 18
            assert st == cb.qlc_start[a] and fill == cb.qlc_start[a + 1] - cb.qlc_start[a]
            assert bits == cb.qlc_bits[a]


def test_table_block_rejects_non_prefix_code():
    cb = hx.build_codebook(datagen.random_counts(2))
    cb.raw.len[0], cb.raw.code[0] = 1, 0
    cb.raw.len[1], cb.raw.code[1] = 2, 0  # "00" has "0" as a prefix
    with pytest.raises(hx.HxError):
        cb.tables()


def test_host_argument_checks_need_no_gpu():
    L = hx.lib()
    assert L.hx_build_codebook(None, 12, 0, None) == hx.HX_ERR_ARG
    c = np.ones(256, np.uint64)
    raw = hx._Codebook()
    assert L.hx_build_codebook(c.ctypes.data, 12, 0x80, ctypes.byref(raw)) == hx.HX_ERR_ARG
    assert L.hx_build_codebook(c.ctypes.data, 7, 0, ctypes.byref(raw)) == hx.HX_ERR_ARG
    assert L.hx_qlc_build(c.ctypes.data, 0, 0, ctypes.byref(raw)) == hx.HX_ERR_ARG
    assert L.hx_qlc_build(c.ctypes.data, 9, 0, ctypes.byref(raw)) == hx.HX_ERR_ARG
    # null buffers, oversize n and misaligned pointers are refused before any device work
    assert L.hx_encode(None, None, 16, None, 0, None, None, None, None) == hx.HX_ERR_ARG
    assert L.hx_encode(256, 256, 1 << 32, 256, 1 << 40, 256, None, 256, None) == hx.HX_ERR_ARG
    assert L.hx_encode(256, 257, 100, 256, 1 << 20, 256, None, 256, None) == hx.HX_ERR_ARG
    assert L.hx_encode(256, 256, 100, 256, 10, 256, None, 256, None) == hx.HX_ERR_ARG
    # the bounded-wait encode: same checks, plus the kind
    assert L.hx_encode_bounded(4, 256, 256, 100, 256, 1 << 20, 256, None, 256, 10, 0, 0,
                               None) == hx.HX_ERR_ARG  # no stream kind 4
    assert L.hx_encode_bounded(2, 256, 256, 100, 256, 1 << 20, 256, None, 256, 10, 0, 4097,
                               None) == hx.HX_ERR_ARG
    assert L.hx_encode_bounded(0, None, 256, 100, 256, 1 << 20, 256, None, 256, 10, 0, 0,
                               None) == hx.HX_ERR_ARG
    assert L.hx_encode_bounded(0, 256, 256, 100, 256, 1 << 20, 256, None, 256, 10, 0, 4097,
                               None) == hx.HX_ERR_ARG  # flush interval above the 24-bit bound
    assert L.hx_decode(None, 256, 100, 256, 4, 256, None) == hx.HX_ERR_ARG
    assert L.hx_decode(256, 264, 4096, 256, 4, 256, None) == hx.HX_ERR_ARG
    assert L.hx_decode(256, 256, 10, 256, 4, 256, None) == hx.HX_ERR_CORRUPT
    assert L.hx_histogram(None, 0, None, None) == hx.HX_ERR_ARG
    assert L.hx_histogram(257, 100, 256, None) == hx.HX_ERR_ARG
    assert hx.status_string(hx.HX_ERR_CORRUPT) == "corrupt stream"
