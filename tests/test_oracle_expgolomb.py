"""Pins of the oracle's Exp-Golomb code (the universal code the QLC page contrasts with).

Order 0 is the ue(v) code of ITU-T H.264 section 9.1, whose first code words are textbook
values; order k is order 0 of floor(v / 2^k) followed by the k low bits of v; the index map puts
a byte's sign in the low bit. The library's builder must give the same code words and hash.
"""
import numpy as np
import pytest

import datagen
from lossless_entropy_coding_fixed_b200 import hx

# ue(v) code words of v = 0..8 (H.264 Table 9-2)
UE = ["1", "010", "011", "00100", "00101", "00110", "00111", "0001000", "0001001"]


def _word(ln, code, b):
    return format(int(code[b]), "b").zfill(int(ln[b]))


def test_order0_is_the_textbook_code(orc):
    ln, code = orc.ExpGolombBook(0, 0).codes
    # map 0: byte b has index (b & 0x7f) << 1 | b >> 7, so indices 0..8 are these bytes
    bytes_of = [0, 128, 1, 129, 2, 130, 3, 131, 4]
    assert [_word(ln, code, b) for b in bytes_of] == UE


@pytest.mark.parametrize("k", [1, 3, 5, 8])
def test_order_k_is_order0_of_the_quotient_then_k_bits(orc, k):
    ln0, code0 = orc.ExpGolombBook(0, 1).codes
    lnk, codek = orc.ExpGolombBook(k, 1).codes
    zig = lambda b: (2 * (b - 256 * (b >= 128)) if b < 128 else -2 * (b - 256) - 1)
    by_index = {zig(b): b for b in range(256)}
    for v in range(256):
        q = v >> k
        if q not in by_index:
            continue
        expect = _word(ln0, code0, by_index[q]) + (format(v & ((1 << k) - 1), "b").zfill(k) if k else "")
        assert _word(lnk, codek, by_index[v]) == expect, (k, v)


def test_zigzag_map_for_twos_complement(orc):
    ln, code = orc.ExpGolombBook(0, 1).codes
    # 0 -> v0, -1 (0xff) -> v1, 1 -> v2, -2 (0xfe) -> v3, 2 -> v4
    assert [_word(ln, code, b) for b in (0, 255, 1, 254, 2)] == UE[:5]


@pytest.mark.parametrize("k,m", [(5, 0), (6, 1), (7, 0), (8, 1)])
def test_round_trip_and_library_codebook(orc, k, m):
    cb = orc.ExpGolombBook(k, m)
    lib = hx.expgolomb_build(k, m)
    ln, code = cb.codes
    assert (lib.len == ln).all() and (lib.code == code).all() and lib.hash == cb.hash
    assert ln.max() <= 12 and (ln >= k + 1).all()
    x = datagen.data(1, n=3 * 4096 + 77)
    st, s = orc.encode(cb, x)
    assert st == 0
    st, y = orc.decode(cb, s, x.size)
    assert st == 0 and (y == x).all()
    # a prefix code: the Kraft sum of the 256 code words is at most 1
    assert sum(2.0 ** -int(v) for v in ln) <= 1.0
