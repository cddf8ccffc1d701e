"""Randomised GPU parity of the single-pass encoder and the decoder against the oracle.

Each case draws a codebook (Huffman with a random length limit, cover-all or seen-only, or a QLC
code with a random number of distinct widths) from a random histogram, and a random input of a
random size whose bytes follow another random law, so that chunks differ in length and the
encoder's chunk order and look-back see uneven work. The GPU stream must equal the oracle's byte
for byte (statuses included), the fused histogram must equal the oracle's, and decoding must give
the input back. Two encodes running at the same time on two streams, each with its own scratch,
must both be exact too.
"""
import numpy as np
import pytest

import datagen

torch = pytest.importorskip("torch")
from lossless_entropy_coding_fixed_b200 import hx  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


def _case(orc, seed):
    rng = np.random.default_rng(9000 + seed)
    counts = datagen.random_counts(seed, alphabet=int(rng.integers(2, 257)),
                                   zeros=float(rng.choice([0.0, 0.3])),
                                   skew=float(rng.uniform(0.3, 1.5)))
    if counts.sum() == 0:
        counts[0] = 1
    kind = int(rng.integers(0, 3))
    if kind == 2:  # QLC
        md = int(rng.integers(1, 9))
        return counts, hx.qlc_build(counts, max_distinct=md), orc.qlc_codebook(counts, md), rng
    seen = kind == 1
    m = int((counts > 0).sum()) if seen else 256
    lmax = int(rng.integers(max(8, int(np.ceil(np.log2(max(m, 2))))), 13))
    return (counts, hx.build_codebook(counts, lmax=lmax, seen_only=seen),
            orc.huffman_codebook(counts, lmax=lmax, cover_all=not seen), rng)


@pytest.mark.parametrize("seed", range(24))
def test_random_codebooks_and_sizes(orc, cuda, seed):
    counts, cb, ocb, rng = _case(orc, seed)
    assert cb.hash == ocb.hash
    n = int(rng.choice([int(rng.integers(0, 5000)), int(rng.integers(4096, 300000)),
                        int(rng.integers(1 << 20, 3 << 20))]))
    # bytes from a law close to the codebook's (or uniform), so some chunks are longer
    if rng.random() < 0.7:
        p = counts.astype(np.float64) + (0.0 if getattr(cb, "kind", 0) == 1 else 0.05)
        p /= p.sum()
        x = rng.choice(256, size=n, p=p).astype(np.uint8)
    else:
        x = rng.integers(0, 256, n, dtype=np.uint8)
    if cb.kind == hx.KIND_HUFFMAN and not (cb.len > 0).all():
        coded = np.flatnonzero(cb.len > 0)
        if rng.random() < 0.8:  # mostly codable inputs; sometimes an uncodable byte
            x = coded[rng.integers(0, coded.size, n)].astype(np.uint8)
    tables = cb.upload(cuda)
    xd = torch.from_numpy(x).to(cuda)
    hist = torch.zeros(256, dtype=torch.int32, device=cuda)
    out, st = hx.encode(tables, xd, hist=hist, kind=cb.kind)
    torch.cuda.synchronize()
    ost, ref = orc.encode(ocb, x)
    assert int(st.item()) == ost
    size = hx.stream_size(out, n)
    assert size == ref.size and (out[:size].cpu().numpy() == ref).all()
    assert (hist.cpu().numpy().astype(np.uint64) == orc.histogram(x)).all()
    if ost == 0:
        y, st2 = hx.decode(tables, out[:size], n, kind=cb.kind)
        torch.cuda.synchronize()
        assert int(st2.item()) == 0 and torch.equal(y, xd)


def test_two_encodes_on_two_streams(orc, cuda):
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(1))
    hb, qb = hx.build_codebook(counts), hx.qlc_build(counts)
    xs = [datagen.data(4, n=(8 << 20) + 123), datagen.data(2, n=(6 << 20) + 4097)]
    refs = [orc.encode(orc.huffman_codebook(counts), xs[0])[1],
            orc.encode(orc.qlc_codebook(counts), xs[1])[1]]
    streams = [torch.cuda.Stream(cuda), torch.cuda.Stream(cuda)]
    outs = []
    for x, cb, s in zip(xs, (hb, qb), streams):
        with torch.cuda.stream(s):
            xd = torch.from_numpy(x).to(cuda)
            outs.append(hx.encode(cb.upload(cuda), xd, kind=cb.kind))
    torch.cuda.synchronize()
    for (out, st), ref, x in zip(outs, refs, xs):
        assert int(st.item()) == 0
        assert hx.stream_size(out, x.size) == ref.size
        assert (out[:ref.size].cpu().numpy() == ref).all()


@pytest.mark.parametrize("kind", ["qlc", "expgolomb"])
def test_bounded_wait_other_kinds(orc, cuda, kind):
    """A withheld chunk times out the chunks after it for the QLC and Exp-Golomb encoders too;
    with no chunk withheld the stream equals the oracle's."""
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(1))
    if kind == "qlc":
        cb, ocb = hx.qlc_build(counts), orc.qlc_codebook(counts)
    else:
        cb, ocb = hx.expgolomb_build(6, 0), orc.ExpGolombBook(6, 0)
    n = 50 * 4096 + 9
    x = datagen.data(1, n=n)
    xd = torch.from_numpy(x).to(cuda)
    tables = cb.upload(cuda)
    out = torch.zeros(hx.encode_bound(n), dtype=torch.uint8, device=cuda)
    scratch = torch.empty(hx.scratch_bytes(n), dtype=torch.uint8, device=cuda)
    _, st = hx.encode_bounded(tables, xd, out, scratch, wait_ns=2_000_000, withhold=7,
                              kind=cb.kind)
    torch.cuda.synchronize()
    assert int(st.item()) & hx.HX_ERR_TIMEOUT
    _, st = hx.encode_bounded(tables, xd, out, scratch, wait_ns=10 ** 9, kind=cb.kind)
    torch.cuda.synchronize()
    ref = orc.encode(ocb, x)[1]
    assert int(st.item()) == 0 and (out[:ref.size].cpu().numpy() == ref).all()
