"""GPU kernels against the CPU oracle, through the C ABI (libhx.so via the ctypes binding).

Integer/byte work, so the bar is bit-exact: the stream bytes the GPU writes equal the oracle's,
the bytes it decodes equal the input, its histogram equals the oracle's, and on damaged streams
it raises the same status bits the oracle returns. Sizes span several chunks and ragged tails.
"""
import numpy as np
import pytest

import datagen
from tests import _golden as G

torch = pytest.importorskip("torch")
from lossless_entropy_coding_fixed_b200 import hx  # noqa: E402

pytestmark = pytest.mark.gpu

SIZES = [1, 15, 16, 17, 511, 512, 513, 4095, 4096, 4097, 3 * 4096 + 100, 1 << 20, (1 << 20) + 13,
         (1 << 22) + 4097]


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.fixture(scope="module")
def books(orc, cuda):
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(1))
    hb, qb = hx.build_codebook(counts), hx.qlc_build(counts)
    return {
        "huffman": (hb, hb.upload(cuda), orc.huffman_codebook(counts), hx.KIND_HUFFMAN),
        "qlc": (qb, qb.upload(cuda), orc.qlc_codebook(counts), hx.KIND_QLC),
    }


def dev(x):
    return torch.from_numpy(np.ascontiguousarray(x)).cuda()


def gpu_encode(tables, x, kind, cap=None, hist=None):
    xd = dev(x)
    out = None if cap is None else torch.zeros(cap, dtype=torch.uint8, device="cuda")
    out, st = hx.encode(tables, xd, out=out, hist=hist, kind=kind)
    torch.cuda.synchronize()
    total = hx.total_words(out)
    size = min(out.numel(), hx.stream_bytes(x.size, total))
    return out[:size].cpu().numpy(), int(st.item()), total


def gpu_decode(tables, stream, n, kind):
    sd = dev(stream)
    out, st = hx.decode(tables, sd, n, kind=kind)
    torch.cuda.synchronize()
    return int(st.item()), out.cpu().numpy()


@pytest.mark.parametrize("n", [0, 1, 15, 17, 4096 * 3 + 5, 1 << 20, (1 << 22) + 3])
def test_histogram_parity(orc, cuda, n):
    x = datagen.data(1, n=max(n, 1))[:n] if n < (1 << 21) else datagen.uniform_bytes(n, 3)
    counts = hx.histogram(dev(x))
    torch.cuda.synchronize()
    assert (counts.cpu().numpy().astype(np.uint64) == orc.histogram(x)).all()
    hx.histogram(dev(x), counts)  # accumulates
    assert (counts.cpu().numpy().astype(np.uint64) == 2 * orc.histogram(x)).all()


@pytest.mark.parametrize("n", SIZES)
@pytest.mark.parametrize("kind", ["huffman", "qlc"])
def test_encode_decode_parity(orc, books, n, kind):
    cb, tables, ocb, k = books[kind]
    x = datagen.data(1, n=n) if n <= (1 << 20) else datagen.data(4, n=n)
    ost, ref = orc.encode(ocb, x)
    assert ost == 0
    got, st, _ = gpu_encode(tables, x, k)
    assert st == 0
    assert got.size == ref.size
    assert (got == ref).all(), np.nonzero(got != ref)[0][:10]
    st, y = gpu_decode(tables, ref, n, k)
    assert st == 0
    assert (y == x).all()


@pytest.mark.parametrize("kind", ["huffman", "qlc"])
def test_empty_input(orc, books, kind):
    cb, tables, ocb, k = books[kind]
    x = np.zeros(0, np.uint8)
    ost, ref = orc.encode(ocb, x)
    got, st, total = gpu_encode(tables, x, k)
    assert st == 0 and total == 0 and (got == ref).all()
    st, y = gpu_decode(tables, ref, 0, k)
    assert st == 0 and y.size == 0


def test_fused_histogram(orc, books):
    cb, tables, ocb, k = books["huffman"]
    x = datagen.data(4, n=(1 << 21) + 999)
    hist = torch.zeros(256, dtype=torch.int32, device="cuda")
    got, st, _ = gpu_encode(tables, x, k, hist=hist)
    assert st == 0
    assert (hist.cpu().numpy().astype(np.uint64) == orc.histogram(x)).all()
    assert (got == orc.encode(ocb, x)[1]).all()


@pytest.mark.parametrize("kind", ["huffman", "qlc"])
def test_adversarial_inputs(orc, kind, cuda):
    counts = datagen.random_counts(11, skew=1.0)
    cb = hx.build_codebook(counts) if kind == "huffman" else hx.qlc_build(counts)
    ocb = orc.huffman_codebook(counts) if kind == "huffman" else orc.qlc_codebook(counts)
    tables = cb.upload(cuda)
    k = cb.kind
    longest = int(np.argmax(ocb.len))
    shortest = int(np.argmin(np.where(ocb.len > 0, ocb.len, 99)))
    # chunks coded longer than 8 bits per symbol take the encoder's direct path; mixed runs
    # interleave direct and buffered chunks
    mixed = np.concatenate([np.full(4096, longest if i % 3 else shortest, np.uint8)
                            for i in range(7)] + [np.full(1000, longest, np.uint8)])
    for x in (np.full(5 * 4096 + 7, longest, np.uint8), np.full(5 * 4096 + 7, shortest, np.uint8),
              datagen.uniform_bytes(9 * 4096 + 77, 5), mixed):
        ref = orc.encode(ocb, x)[1]
        got, st, _ = gpu_encode(tables, x, k)
        assert st == 0 and (got == ref).all()
        st, y = gpu_decode(tables, ref, x.size, k)
        assert st == 0 and (y == x).all()
    # a full output buffer on the direct path: the header and index are written, no payload
    need = orc.encode(ocb, mixed)[1].size
    got, st, total = gpu_encode(tables, mixed, k, cap=need - 8)
    assert st == hx.HX_ERR_CAPACITY and hx.stream_bytes(mixed.size, total) == need


@pytest.mark.parametrize("lmax", [8, 9, 11])
def test_shorter_length_limits(orc, cuda, lmax):
    counts = datagen.random_counts(21, skew=1.2)
    cb, ocb = hx.build_codebook(counts, lmax=lmax), orc.huffman_codebook(counts, lmax=lmax)
    tables = cb.upload(cuda)
    x = datagen.uniform_bytes(3 * 4096 + 999, 8)
    ref = orc.encode(ocb, x)[1]
    got, st, _ = gpu_encode(tables, x, 0)
    assert st == 0 and (got == ref).all()
    st, y = gpu_decode(tables, ref, x.size, 0)
    assert st == 0 and (y == x).all()


def test_hand_streams_on_gpu(orc, cuda):
    cb = hx.build_codebook(G.abc_counts(), seen_only=True)
    qlc = hx.qlc_build(np.ones(256, np.uint64))
    for name, c in G.hand_streams().items():
        book = qlc if name.startswith("qlc") else cb
        tables = book.upload(cuda)
        got, st, _ = gpu_encode(tables, c["x"], book.kind)
        assert st == 0 and got.size == c["total"]
        P = hx.payload_offset(c["x"].size)
        assert (got[P:P + 4 * c["payload"].size].view(np.uint32) == c["payload"]).all(), name
        st, y = gpu_decode(tables, got, c["x"].size, book.kind)
        assert st == 0 and (y == c["x"]).all()


def test_uncodable_symbol(orc, cuda):
    counts = G.abc_counts()
    cb, ocb = hx.build_codebook(counts, seen_only=True), orc.huffman_codebook(counts, cover_all=False)
    tables = cb.upload(cuda)
    x = np.tile(np.array([0x41, 0x44, 0x42, 0x43], np.uint8), 3000)
    ost, ref = orc.encode(ocb, x)
    got, st, _ = gpu_encode(tables, x, 0)
    assert ost == st == hx.HX_ERR_UNCODABLE
    assert (got == ref).all()


def test_capacity(orc, books):
    cb, tables, ocb, k = books["huffman"]
    x = datagen.data(1, n=5 * 4096 + 3)
    ref = orc.encode(ocb, x)[1]
    need = ref.size
    P = hx.payload_offset(x.size)
    for cap in (need - 4, need // 2, P + 8):
        got, st, total = gpu_encode(tables, x, k, cap=cap)
        assert st == hx.HX_ERR_CAPACITY
        assert hx.stream_bytes(x.size, total) == need
        assert orc.encode(ocb, x, cap=cap)[0] & orc.ERR_CAPACITY
        # the header and the index are those of the whole stream; a payload word is either the
        # stream's own (a chunk that fitted) or untouched (zero), and none lies past the buffer
        assert got.size == cap and (got[:P] == ref[:P]).all()
        assert ((got[P:] == ref[P:cap]) | (got[P:] == 0)).all()
    got, st, _ = gpu_encode(tables, x, k, cap=need)
    assert st == 0 and (got == ref).all()


def test_wrong_kind_tables(books):
    cb, tables, ocb, k = books["huffman"]
    x = datagen.data(1, n=10000)
    _, st, _ = gpu_encode(tables, x, hx.KIND_QLC)
    assert st == hx.HX_ERR_ARG
    _, qt, _, _ = books["qlc"]
    ref, st0, _ = gpu_encode(tables, x, k)
    st, _ = gpu_decode(qt, ref, x.size, hx.KIND_HUFFMAN)
    assert st == hx.HX_ERR_ARG


def test_deterministic_repeat(books):
    cb, tables, ocb, k = books["huffman"]
    x = datagen.data(4, n=(1 << 23) + 12345)
    a, _, _ = gpu_encode(tables, x, k)
    b, _, _ = gpu_encode(tables, x, k)
    assert (a == b).all()


# --------------------------------------------------------------------------- damaged streams
@pytest.fixture(scope="module", params=["huffman", "qlc"])
def damaged_setup(orc, books, request):
    cb, tables, ocb, k = books[request.param]
    x = datagen.data(1, n=7 * 4096 + 777)
    st, s = orc.encode(ocb, x)
    assert st == 0
    return tables, ocb, x, s, k


def _damage_cases(s, n, orc):
    S = orc.sync_offset(n)
    cases = []
    for off, val in [(0, 0), (4, 2), (9, 0), (12, 9), (16, 1), (24, 3), (32, 0xff), (33, 0x7f)]:
        t = s.copy()
        t[off] = val
        cases.append(t)
    for c, v in [(1, 10**6), (3, 0), (8, 1)]:
        t = s.copy()
        t[64 + 4 * c:64 + 4 * c + 4] = np.array([v], np.uint32).view(np.uint8)
        cases.append(t)
    for c, k, v in [(0, 1, 60000), (2, 0, 5), (3, 4, 1), (7, 7, 0), (7, 5, 4000)]:
        t = s.copy()
        o = S + 16 * c + 2 * k
        t[o:o + 2] = np.array([v], np.uint16).view(np.uint8)
        cases.append(t)
    cases.append(s[:-12].copy())
    return cases


def test_damaged_index_and_header_statuses_match_oracle(orc, damaged_setup):
    tables, ocb, x, s, k = damaged_setup
    for i, t in enumerate(_damage_cases(s, x.size, orc)):
        ost, _ = orc.decode(ocb, t, x.size)
        st, _ = gpu_decode(tables, t, x.size, k)
        assert ost != 0, i
        assert st == ost, (i, st, ost)


def test_payload_bit_flips_match_oracle(orc, damaged_setup):
    tables, ocb, x, s, k = damaged_setup
    P = orc.payload_offset(x.size)
    rng = np.random.default_rng(1)
    for _ in range(40):
        t = s.copy()
        t[int(rng.integers(P, s.size - 8))] ^= np.uint8(1 << int(rng.integers(0, 8)))
        ost, oy = orc.decode(ocb, t, x.size)
        st, y = gpu_decode(tables, t, x.size, k)
        assert st == ost
        if st == 0:
            assert (y == oy).all()


def test_other_codebook_rejected(orc, damaged_setup, cuda):
    tables, ocb, x, s, k = damaged_setup
    if k != hx.KIND_HUFFMAN:
        pytest.skip("a Huffman table block against a Huffman stream")
    other = hx.build_codebook(datagen.random_counts(99)).upload(cuda)
    st, _ = gpu_decode(other, s, x.size, 0)
    assert st == hx.HX_ERR_CODEBOOK == orc.decode(orc.huffman_codebook(datagen.random_counts(99)), s, x.size)[0]


@pytest.mark.parametrize("kind", ["huffman", "qlc"])
@pytest.mark.parametrize("n", [4096, 5 * 4096 + 77, 1 << 20])
def test_flat_8bit_codes(orc, cuda, n, kind):
    """Every code 8 bits long (uniform counts: Huffman, or QLC with eight areas of 5 index bits):
    each 128-byte piece packs to exactly 32 words, so all 32 pieces of a chunk start in one
    shared-memory bank and the encoder takes its spread buffer layout for every chunk; every
    sub-stream is 128 words long, so the decoder's blocks take the voting loop and its 16-byte
    reader."""
    counts = np.ones(256, np.uint64)
    if kind == "huffman":
        cb, ocb = hx.build_codebook(counts), orc.huffman_codebook(counts)
    else:
        cb, ocb = hx.qlc_build(counts), orc.qlc_codebook(counts)
    assert (ocb.len == 8).all()
    tables = cb.upload(cuda)
    x = datagen.uniform_bytes(n, 9)
    ref = orc.encode(ocb, x)[1]
    got, st, _ = gpu_encode(tables, x, cb.kind)
    assert st == 0 and (got == ref).all()
    st, y = gpu_decode(tables, ref, n, cb.kind)
    assert st == 0 and (y == x).all()


def test_mixed_buffer_layouts(orc, books):
    """Chunks of bytes whose codes are all 8 bits long (spread layout) between chunks of the
    workload's law (plain layout), in one stream."""
    cb, tables, ocb, k = books["huffman"]
    eight = np.flatnonzero(ocb.len == 8).astype(np.uint8)
    assert eight.size > 0
    rng = np.random.default_rng(31)
    law = datagen.data(1, n=6 * 4096)
    parts = [rng.choice(eight, 4096) if i % 2 else law[i * 4096:(i + 1) * 4096] for i in range(6)]
    x = np.concatenate(parts + [rng.choice(eight, 1500)]).astype(np.uint8)
    ref = orc.encode(ocb, x)[1]
    got, st, _ = gpu_encode(tables, x, k)
    assert st == 0 and (got == ref).all()
