"""Pins of the oracle's Shannonic coder (range partition + 128-state tANS), on the CPU.

The "Shannonic" review page gives the method: a dynamic programme splits the 256 byte values into
at most K = 16 contiguous ranges minimising the range entropy plus fixed-width offset bits, the
range index is coded by tANS with 128 states, and the offset in ceil(log2 size) bits. Pinned here
by an exhaustive search on small alphabets (the partition), closed forms (the frequency
normalisation), a hand-built stream (one range: tANS then moves nothing), the coding efficiency
against the ideal code length, and the round trip with damage detection.
"""
import itertools
import math

import numpy as np
import pytest

import datagen


def _cost(w, lo):
    W = float(sum(w))
    c = 0.0
    for a, b in zip(lo[:-1], lo[1:]):
        wab = float(sum(w[a:b]))
        if wab:
            c += wab * math.log2(W / wab) + wab * math.ceil(math.log2(b - a)) if b - a > 1 else wab * math.log2(W / wab)
    return c


def _brute(w, K):
    n = len(w)
    best, arg = None, None
    for k in range(1, min(K, n) + 1):
        for cuts in itertools.combinations(range(1, n), k - 1):
            lo = [0, *cuts, n]
            c = _cost(w, lo)
            if best is None or c < best - 1e-9:
                best, arg = c, lo
    return best, arg


@pytest.mark.parametrize("seed", range(40))
def test_partition_is_the_exhaustive_optimum(orc, seed):
    rng = np.random.default_rng(seed)
    n, K = int(rng.integers(2, 11)), int(rng.integers(1, 5))
    w = rng.integers(1, 50, n) * rng.integers(1, 4, n) ** 3
    lo = orc.shannonic_partition(w, K)
    best, arg = _brute(list(map(int, w)), K)
    assert lo[0] == 0 and lo[-1] == n and len(lo) - 1 <= K
    assert _cost(list(map(int, w)), list(lo)) == pytest.approx(best, rel=1e-12, abs=1e-9)


def test_normalisation_closed_forms(orc):
    assert (orc.shannonic_normalise([5] * 16) == 8).all()
    f = orc.shannonic_normalise([1] * 15 + [10**9])
    assert (f[:15] == 1).all() and f[15] == 128 - 15
    f = orc.shannonic_normalise([3, 1])  # 96 and 32 exactly
    assert list(f) == [96, 32]
    f = orc.shannonic_normalise([1, 1, 1])  # 42 each, equal remainders: +1 to the two lowest
    assert list(f) == [43, 43, 42]
    rng = np.random.default_rng(2)
    for _ in range(200):
        wr = rng.integers(1, 10**6, int(rng.integers(1, 17)))
        f = orc.shannonic_normalise(wr)
        assert f.sum() == 128 and (f >= 1).all()
        ideal = wr * 128 / wr.sum()
        assert (np.abs(f - ideal) < 1 + (ideal < 1) * 1.0 + len(wr)).all()


def test_single_range_stream_by_hand(orc):
    """One range of all 256 values: f = 128, so every state step outputs no bits and keeps the
    state; a sub-stream is its bytes as 8-bit offsets from the last to the first, then 7 zero
    bits (the final state minus 128)."""
    cb = orc.ShannonicBook(1, np.array([0, 256], np.int32), np.array([128], np.int32))
    x = datagen.data(1, n=1000)
    st, s = orc.encode(cb, x)
    assert st == 0
    bits = []
    for k in range(2):
        sub = x[512 * k:min(1000, 512 * (k + 1))]
        for v in sub[::-1]:
            bits += [(int(v) >> (7 - i)) & 1 for i in range(8)]
        bits += [0] * 7
    nbits = len(bits)
    bits += [0] * (-nbits % 32)
    words = np.packbits(np.array(bits, np.uint8)).view(">u4").astype(np.uint32)
    P = orc.payload_offset(1000)
    assert (s[P:P + 4 * words.size].view(np.uint32) == words).all()
    S = orc.sync_offset(1000)
    sync = s[S:S + 16].view(np.uint16)
    assert sync[0] == nbits and sync[1] == 512 * 8 + 7 and (sync[2:] == nbits).all()


def test_coding_length_is_close_to_ideal(orc):
    """tANS codes range r in about log2(128 / f_r) bits: the payload must come within 1 % (plus
    7 bits per sub-stream) of sum over symbols of log2(128 / f_r) + offset bits."""
    x = datagen.data(1, n=1 << 20)
    h = orc.histogram(x)
    cb = orc.shannonic_codebook(h)
    ranges = np.searchsorted(cb.lo, np.arange(256), side="right") - 1
    ideal = sum(int(h[v]) * (math.log2(128 / cb.f[ranges[v]]) + cb.offset_bits[ranges[v]])
                for v in range(256))
    st, s = orc.encode(cb, x)
    S = orc.sync_offset(x.size)
    nc = (x.size + 4095) // 4096
    bits = int(s[S:S + 16 * nc].view(np.uint16)[::8].astype(np.int64).sum())
    assert st == 0
    assert abs(bits - 7 * 8 * nc - ideal) < 0.01 * ideal
    # and Shannon's bound holds for the whole code
    assert bits / x.size >= orc.entropy(h)


@pytest.mark.parametrize("cfg,n", [(1, 1), (1, 511), (1, 4097), (1, (1 << 20) - 3), (3, 4 * 8192)])
def test_round_trip_and_damage(orc, cfg, n):
    x = datagen.data(cfg, n=n) if cfg != 3 else datagen.data(3, n=1 << 26)[:n].copy()
    cb = orc.shannonic_codebook(orc.histogram(x))
    st, s = orc.encode(cb, x)
    assert st == 0 and s.size <= orc.shannonic_encode_bound(n)
    st, y = orc.decode(cb, s, n)
    assert st == 0 and (y == x).all()
    # A flipped offset bit changes one byte and nothing else (lengths come from the state and the
    # range, not from offsets); a flipped state bit derails the state chain, which must end in
    # state 128 exactly at the sub-stream's first bit -- caught, unless the chain happens to fall
    # back into step (tANS can resynchronise; the format carries no checksum).
    P = orc.payload_offset(n)
    rng = np.random.default_rng(n)
    flagged = 0
    for _ in range(40):
        t = s.copy()
        t[int(rng.integers(P, s.size - 8))] ^= np.uint8(1 << int(rng.integers(0, 8)))
        st, y = orc.decode(cb, t, n)
        flagged += st != 0
        assert st in (0, orc.ERR_CORRUPT)
    if n >= 4096:
        assert flagged >= 10
    other = orc.shannonic_codebook(datagen.random_counts(5))
    assert orc.decode(other, s, n)[0] == orc.ERR_CODEBOOK
