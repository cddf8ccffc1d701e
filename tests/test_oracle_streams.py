"""Oracle encode/decode pinned to hand-computed streams, prefix sums and round-trip identity.

"Lossless" means the decoder returns exactly the input bytes; the stream layout is the
chunked format written out in the oracle's header. No GPU.
"""
import numpy as np
import pytest

import datagen
from tests import _golden as G

HDR = 64


def parse(stream, n):
    st = np.asarray(stream, dtype=np.uint8)
    nc = -(-n // 4096)
    S = (64 + 4 * (nc + 1) + 15) // 16 * 16
    P = S + 16 * nc
    h = dict(magic=int(st[0:4].view(np.uint32)[0]), version=int(st[4]), kind=int(st[5]),
             lmax=int(st[6]), chunk=int(st[8:12].view(np.uint32)[0]),
             sub=int(st[12:16].view(np.uint32)[0]), n=int(st[16:24].view(np.uint64)[0]),
             n_chunks=int(st[24:32].view(np.uint64)[0]), total=int(st[32:40].view(np.uint64)[0]),
             hash=int(st[40:48].view(np.uint64)[0]))
    word_off = st[64:64 + 4 * (nc + 1)].view(np.uint32).copy()
    sync = st[S:S + 16 * nc].view(np.uint16).reshape(nc, 8).copy()
    payload = st[P:P + 4 * h["total"]].view(np.uint32).copy()
    guard = st[P + 4 * h["total"]:P + 4 * h["total"] + 8]
    return h, word_off, sync, payload, guard, P


def reference_bits(cb, x):
    """Independent construction of the payload with numpy bit arrays: per chunk, concatenate
    each symbol's code MSB-first, pad to 32 bits, pack to big-endian-bit u32 words."""
    words, word_off, sync = [], [0], []
    for c in range(0, len(x), 4096):
        seg = x[c:c + 4096]
        bits = []
        for s in seg:
            l = int(cb.len[s])
            bits.extend((int(cb.code[s]) >> (l - 1 - i)) & 1 for i in range(l))
        lens = cb.len[seg].astype(np.int64)
        starts = np.concatenate([[0], np.cumsum(lens)])
        nb = int(starts[-1])
        row = [nb] + [int(starts[512 * k]) if 512 * k < len(seg) else nb for k in range(1, 8)]
        sync.append(row)
        bits += [0] * (-len(bits) % 32)
        b = np.array(bits, dtype=np.uint8).reshape(-1, 32)
        w = (b.astype(np.uint64) << np.arange(31, -1, -1, dtype=np.uint64)).sum(axis=1)
        words += [int(v) for v in w]
        word_off.append(len(words))
    return np.array(words, np.uint32), np.array(word_off, np.uint32), np.array(sync, np.uint16)


def test_hand_streams(orc):
    cases = G.hand_streams()
    cb = orc.huffman_codebook(G.abc_counts(), cover_all=False)
    assert [int(cb.len[s]) for s in (0x41, 0x42, 0x43)] == [1, 2, 2]
    qlc = orc.qlc_codebook(np.ones(256, np.uint64))
    for name, c in cases.items():
        book = qlc if name.startswith("qlc") else cb
        st, s = orc.encode(book, c["x"])
        assert st == 0
        assert s.size == c["total"], name
        h, wo, sy, pay, guard, P = parse(s, c["x"].size)
        assert h["magic"] == 0x31305848 and bytes(s[:4]) == b"HX01"
        assert (h["version"], h["chunk"], h["sub"]) == (1, 4096, 8)
        assert h["kind"] == book.kind and h["lmax"] == (11 if book.kind else 12)
        assert h["n"] == c["x"].size and h["n_chunks"] == -(-c["x"].size // 4096)
        assert h["hash"] == book.hash
        assert list(wo) == c["word_off"], name
        assert list(sy.reshape(-1)) == c["sync"], name
        assert (pay == c["payload"]).all(), name
        assert (guard == 0).all()
        st, y = orc.decode(book, s, c["x"].size)
        assert st == 0 and (y == c["x"]).all()


@pytest.mark.parametrize("n", [0, 1, 2, 511, 512, 513, 1000, 4095, 4096, 4097, 8192, 3 * 4096 + 100])
@pytest.mark.parametrize("kind", ["huffman", "qlc"])
def test_round_trip_and_layout(orc, n, kind):
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(1))
    cb = orc.huffman_codebook(counts) if kind == "huffman" else orc.qlc_codebook(counts)
    x = datagen.data(1, n=max(n, 1))[:n] if n else np.zeros(0, np.uint8)
    st, s = orc.encode(cb, x)
    assert st == 0
    h, wo, sy, pay, guard, P = parse(s, n)
    assert s.size == P + 4 * (h["total"] + 2)
    assert h["total"] == wo[-1]
    words, ref_wo, ref_sync = reference_bits(cb, x)
    assert (wo == ref_wo).all()
    if n:
        assert (sy == ref_sync).all()
    assert (pay == words).all()
    st, y = orc.decode(cb, s, n)
    assert st == 0 and (y == x).all()


@pytest.mark.parametrize("kind", ["huffman", "qlc"])
def test_adversarial_symbol_mixes(orc, kind):
    counts = datagen.random_counts(11, skew=1.0)
    cb = orc.huffman_codebook(counts) if kind == "huffman" else orc.qlc_codebook(counts)
    longest = int(np.argmax(cb.len))
    shortest = int(np.argmin(np.where(cb.len > 0, cb.len, 99)))
    for x in (np.full(9000, longest, np.uint8), np.full(9000, shortest, np.uint8),
              datagen.uniform_bytes(9000, 5)):
        st, s = orc.encode(cb, x)
        assert st == 0
        st, y = orc.decode(cb, s, x.size)
        assert st == 0 and (y == x).all()
    st, s = orc.encode(cb, np.full(4096, longest, np.uint8))
    h, wo, sy, pay, guard, P = parse(s, 4096)
    assert int(sy[0, 0]) == 4096 * int(cb.len[longest])


def test_uncodable_symbol_flagged(orc):
    cb = orc.huffman_codebook(G.abc_counts(), cover_all=False)
    x = np.array([0x41, 0x44, 0x42], np.uint8)
    st, s = orc.encode(cb, x)
    assert st & orc.ERR_UNCODABLE
    # the uncodable byte emits no bits
    h, wo, sy, pay, guard, P = parse(s, 3)
    assert sy[0, 0] == 3


def test_capacity_flagged_with_size_in_header(orc):
    cb = orc.huffman_codebook(G.abc_counts(), cover_all=False)
    x = np.full(5000, 0x42, np.uint8)
    need = orc.encode(cb, x)[1].size
    st, s = orc.encode(cb, x, cap=need - 4)
    assert st & orc.ERR_CAPACITY
    h = parse(np.concatenate([s, np.zeros(1024, np.uint8)]), 5000)[0]
    assert orc.payload_offset(5000) + 4 * (h["total"] + 2) == need


@pytest.fixture(scope="module")
def setup(orc):
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(1))
    cb = orc.huffman_codebook(counts)
    x = datagen.data(1, n=3 * 4096 + 777)
    st, s = orc.encode(cb, x)
    assert st == 0
    return cb, x, s


class TestCorruption:
    def test_wrong_codebook(self, orc, setup):
        cb, x, s = setup
        other = orc.huffman_codebook(datagen.random_counts(1))
        assert orc.decode(other, s, x.size)[0] == orc.ERR_CODEBOOK
        q = orc.qlc_codebook(datagen.random_counts(1))
        assert orc.decode(q, s, x.size)[0] == orc.ERR_CODEBOOK

    def test_header_fields(self, orc, setup):
        cb, x, s = setup
        for off, val in [(0, 0x00), (4, 2), (9, 0), (12, 9)]:
            t = s.copy()
            t[off] = val
            assert orc.decode(cb, t, x.size)[0] == orc.ERR_CORRUPT
        assert orc.decode(cb, s, x.size + 1)[0] == orc.ERR_CORRUPT
        assert orc.decode(cb, s[:-20], x.size)[0] == orc.ERR_CORRUPT

    def test_index_tables(self, orc, setup):
        cb, x, s = setup
        t = s.copy()
        t[64 + 4:64 + 8] = np.array([10**6], np.uint32).view(np.uint8)  # word_off[1] past the end
        assert orc.decode(cb, t, x.size)[0] & orc.ERR_CORRUPT
        S = orc.sync_offset(x.size)
        t = s.copy()
        t[S + 2:S + 4] = np.array([60000], np.uint16).view(np.uint8)  # sync[0][1] beyond the chunk
        assert orc.decode(cb, t, x.size)[0] & orc.ERR_CORRUPT
        t = s.copy()
        t[S:S + 2] = np.array([int(t[S:S + 2].view(np.uint16)[0]) - 40], np.uint16).view(np.uint8)
        assert orc.decode(cb, t, x.size)[0] & orc.ERR_CORRUPT

    def test_payload_flips(self, orc, setup):
        cb, x, s = setup
        h, wo, sy, pay, guard, P = parse(s, x.size)
        rng = np.random.default_rng(0)
        for _ in range(60):
            c = int(rng.integers(0, len(sy)))
            bit = int(wo[c]) * 32 + int(rng.integers(0, int(sy[c, 0])))  # a valid (non-pad) bit
            t = s.copy()
            word = P + 4 * (bit // 32)
            b = 31 - bit % 32  # MSB-first inside a little-endian u32
            t[word + b // 8] ^= np.uint8(1 << (b % 8))
            st, y = orc.decode(cb, t, x.size)
            # a prefix code parses each bit string one way: a flip is caught or changes the bytes
            assert st & orc.ERR_CORRUPT or not (y == x).all()


def test_seen_only_codebook_rejects_unused_code_words(orc):
    # three symbols, Kraft sum 1: every prefix decodes. Two symbols with lmax 12 leaves no gap
    # either; a seen-only code over 3 symbols whose lengths are (1,2,2) is complete, so force a
    # gap with a QLC codebook whose last area is underfull.
    q = orc.qlc_codebook(np.ones(256, np.uint64), max_distinct=2)
    assert int(q.start[8]) == 256
    x = np.arange(256, dtype=np.uint8)
    st, s = orc.encode(q, x)
    assert st == 0
    P = orc.payload_offset(256)
    # an area index beyond the area's fill is corrupt: area 7 of this code is underfull iff
    # its capacity exceeds its fill
    cap = [1 << int(b) for b in q.bits]
    fill = [int(q.start[a + 1] - q.start[a]) for a in range(8)]
    assert sum(fill) == 256
    if cap[7] > fill[7]:
        t = s.copy()
        t[P:P + 4] = np.array([0xFFFFFFFF], np.uint32).view(np.uint8)
        assert orc.decode(q, t, 256)[0] & orc.ERR_CORRUPT
