"""The Shannonic coder on the GPU (k_sh_encode, k_sh_decode) against the oracle.

Byte work, so the bar is bit-exact: the stream the GPU writes equals the oracle's byte for byte,
decoding returns the input, the fused histogram equals the oracle's, and on damaged streams the
GPU raises the status bits the oracle returns.
"""
import numpy as np
import pytest

import datagen

torch = pytest.importorskip("torch")
from lossless_entropy_coding_fixed_b200 import hx  # noqa: E402

pytestmark = pytest.mark.gpu
K = hx.KIND_SHANNONIC


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _book(orc, counts, cuda):
    cb = hx.shannonic_build(counts)
    ocb = orc.shannonic_codebook(counts)
    assert cb.hash == ocb.hash
    return cb.upload(cuda), ocb


def _enc(tables, x, cap=None, hist=None):
    xd = torch.from_numpy(np.ascontiguousarray(x)).cuda()
    out = torch.zeros(cap if cap else hx.encode_bound(x.size, K), dtype=torch.uint8, device="cuda")
    out, st = hx.encode(tables, xd, out=out, hist=hist, kind=K)
    torch.cuda.synchronize()
    total = hx.total_words(out)
    size = min(out.numel(), hx.stream_bytes(x.size, total))
    return out[:size].cpu().numpy(), int(st.item()), total


def _dec(tables, s, n):
    y, st = hx.decode(tables, torch.from_numpy(s).cuda(), n, kind=K)
    torch.cuda.synchronize()
    return int(st.item()), y.cpu().numpy()


@pytest.mark.parametrize("n", [1, 15, 511, 512, 513, 4095, 4096, 4097, 3 * 4096 + 100,
                               (1 << 20) - 3, (1 << 22) + 4097])
def test_encode_decode_parity(orc, cuda, n):
    x = datagen.data(1, n=n) if n <= 1 << 20 else datagen.data(4, n=n)
    tables, ocb = _book(orc, sum(orc.histogram(b) for b in datagen.prior_batches(1)), cuda)
    ost, ref = orc.encode(ocb, x)
    got, st, _ = _enc(tables, x)
    assert ost == st == 0
    assert got.size == ref.size and (got == ref).all()
    st, y = _dec(tables, ref, n)
    assert st == 0 and (y == x).all()


@pytest.mark.parametrize("cfg", [2, 3, 5])
def test_other_laws(orc, cuda, cfg):
    x = (datagen.data(cfg, n=1 << 22) if cfg == 2 else
         datagen.data(3, n=1 << 26)[: 1 << 22].copy() if cfg == 3 else datagen.data(5, shard=3)[: 1 << 22].copy())
    tables, ocb = _book(orc, orc.histogram(x), cuda)
    hist = torch.zeros(256, dtype=torch.int32, device=cuda)
    got, st, _ = _enc(tables, x, hist=hist)
    ref = orc.encode(ocb, x)[1]
    assert st == 0 and (got == ref).all()
    assert (hist.cpu().numpy().astype(np.uint64) == orc.histogram(x)).all()
    st, y = _dec(tables, ref, x.size)
    assert st == 0 and (y == x).all()


def test_adversarial_inputs(orc, cuda):
    """A skewed table and data made of its rarest bytes: up to 15 bits per byte."""
    counts = datagen.random_counts(11, skew=1.0)
    tables, ocb = _book(orc, counts, cuda)
    rare = int(np.argmin(counts))
    for x in (np.full(5 * 4096 + 7, rare, np.uint8), datagen.uniform_bytes(9 * 4096 + 77, 5)):
        ref = orc.encode(ocb, x)[1]
        got, st, _ = _enc(tables, x)
        assert st == 0 and (got == ref).all()
        st, y = _dec(tables, ref, x.size)
        assert st == 0 and (y == x).all()


def test_parked_and_recoded_groups(orc, cuda):
    """The encoder parks each sub-stream's bits in shared memory (113 words, 7.06 bits per
    symbol) and codes a group of 4 chunks again, straight into the payload, when one of its
    sub-streams is longer. Runs of the codebook's rarest byte make some groups long: a whole
    chunk, a single sub-stream, and a run across a chunk boundary, among groups that fit."""
    x = datagen.data(4, n=64 * 4096 + 123)
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(1))
    tables, ocb = _book(orc, counts, cuda)
    rare = np.uint8(np.argmin(counts))
    x[20 * 4096:21 * 4096] = rare
    x[41 * 4096 + 3 * 512:41 * 4096 + 4 * 512] = rare
    x[51 * 4096 - 700:51 * 4096 + 300] = rare
    x[-50:] = rare
    hist = torch.zeros(256, dtype=torch.int32, device=cuda)
    ref = orc.encode(ocb, x)[1]
    got, st, _ = _enc(tables, x, hist=hist)
    assert st == 0 and got.size == ref.size and (got == ref).all()
    assert (hist.cpu().numpy().astype(np.uint64) == orc.histogram(x)).all()
    st, y = _dec(tables, ref, x.size)
    assert st == 0 and (y == x).all()
    # a buffer that ends inside the stream: the header and the index are whole, a payload word is
    # the stream's own or untouched (zero), in recoded groups as in the others
    P = hx.payload_offset(x.size)
    for cap in (ref.size // 2, ref.size - 4):
        got, st, total = _enc(tables, x, cap=cap)
        assert st == hx.HX_ERR_CAPACITY and hx.stream_bytes(x.size, total) == ref.size
        assert got.size == cap and (got[:P] == ref[:P]).all()
        assert ((got[P:] == ref[P:cap]) | (got[P:] == 0)).all()


def test_capacity_and_wrong_tables(orc, cuda):
    x = datagen.data(1, n=5 * 4096 + 3)
    tables, ocb = _book(orc, orc.histogram(x), cuda)
    full = orc.encode(ocb, x)[1]
    need = full.size
    P = hx.payload_offset(x.size)
    for cap in (need - 4, need // 2, P + 8):
        got, st, total = _enc(tables, x, cap=cap)
        assert st == hx.HX_ERR_CAPACITY and hx.stream_bytes(x.size, total) == need
        # the header and the index are those of the whole stream; a payload word is either the
        # stream's own (a chunk that fitted) or untouched (zero), and none lies past the buffer
        assert got.size == cap and (got[:P] == full[:P]).all()
        assert ((got[P:] == full[P:cap]) | (got[P:] == 0)).all()
    got, st, _ = _enc(tables, x, cap=need)
    assert st == 0 and (got == full).all()
    huff = hx.build_codebook(orc.histogram(x)).upload(cuda)
    _, st, _ = _enc(huff, x)
    assert st == hx.HX_ERR_ARG
    ref = orc.encode(ocb, x)[1]
    y, st = hx.decode(huff, torch.from_numpy(ref).cuda(), x.size, kind=K)
    torch.cuda.synchronize()
    assert int(st.item()) == hx.HX_ERR_ARG


def test_damaged_streams_match_oracle(orc, cuda):
    x = datagen.data(1, n=7 * 4096 + 777)
    tables, ocb = _book(orc, orc.histogram(x), cuda)
    st, s = orc.encode(ocb, x)
    S, P = orc.sync_offset(x.size), orc.payload_offset(x.size)
    cases = []
    for off, val in [(0, 0), (5, 1), (9, 0), (33, 0x7f)]:
        t = s.copy()
        t[off] = val
        cases.append(t)
    for c, k, v in [(0, 1, 60000), (2, 0, 5), (3, 4, 1), (7, 7, 0), (7, 5, 4000)]:
        t = s.copy()
        t[S + 16 * c + 2 * k:S + 16 * c + 2 * k + 2] = np.array([v], np.uint16).view(np.uint8)
        cases.append(t)
    rng = np.random.default_rng(3)
    for _ in range(30):
        t = s.copy()
        t[int(rng.integers(P, s.size - 8))] ^= np.uint8(1 << int(rng.integers(0, 8)))
        cases.append(t)
    cases.append(s[:-12].copy())
    for i, t in enumerate(cases):
        ost, oy = orc.decode(ocb, t, x.size)
        st, y = _dec(tables, t, x.size)
        assert st == ost, (i, st, ost)
        if st == 0:
            assert (y == oy).all(), i
