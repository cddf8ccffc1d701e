"""The online single-stage loop on the GPU (hx_session) and table-set decode (hx_decode_set).

Every batch's stream must equal the oracle's encode of that batch with the codebook the oracle's
schedule assigns it (bit-exact), the session must report the same codebook hashes and drift
refreshes, and the streams must decode back through the hash-picked table slots.
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


def _batches():
    """Five e4m3 N(0, 0.5) batches, then five of a wide normal on bytes; ragged sizes."""
    rng = np.random.default_rng(11)
    sizes = [3 * 4096 + 100, 1 << 16, 5 * 4096, 70001, 4096, (1 << 16) + 3, 12345, 4 * 4096 + 1,
             1 << 15, 9999]
    xs = []
    for i, n in enumerate(sizes):
        if i < 5:
            xs.append(datagen.data(1, n=1 << 20)[i * 100000:i * 100000 + n].copy())
        else:
            xs.append(np.clip(rng.normal(0, 1, n) * 60 + 128, 0, 255).astype(np.uint8))
    return xs


@pytest.mark.parametrize("kind", [hx.KIND_HUFFMAN, hx.KIND_QLC])
def test_session_matches_oracle_schedule(orc, cuda, kind):
    xs = _batches()
    init = orc.histogram(datagen.data(1, n=1 << 14))
    m, lag, drift = 3, 2, 0.1
    books, seen = orc.session_schedule([orc.histogram(x) for x in xs], kind, m, lag, drift,
                                       initial_counts=init)
    sess = hx.Session(cuda, kind, history=m, lag=lag, drift=drift, initial_counts=init)
    outs, stats = [], []
    for x in xs:
        n = x.size
        out = torch.empty(hx.encode_bound(n), dtype=torch.uint8, device=cuda)
        scratch = torch.empty(hx.scratch_bytes(n), dtype=torch.uint8, device=cuda)
        st = torch.zeros(1, dtype=torch.int32, device=cuda)
        sess.encode(torch.from_numpy(x).to(cuda), out, scratch, st)
        outs.append(out)
        stats.append(st)
    torch.cuda.synchronize()
    sess.drain()
    for t, x in enumerate(xs):
        ost, ref = orc.encode(books[t], x)
        assert ost == 0 and int(stats[t].item()) == 0
        assert (outs[t][:ref.size].cpu().numpy() == ref).all(), t
        info = sess.info(t)
        assert info["hash"] == books[t].hash and info["observed"] and info["symbols"] == x.size
        assert info["refreshed"] == seen[t][0]
        assert info["drift"] == pytest.approx(seen[t][1], rel=1e-12, abs=1e-12)
    assert any(r for r, _ in seen)  # the switch refreshed
    # a slot holds the codebook of the last batch that used it; a stream decodes through the
    # slots exactly when its codebook is still in one of them
    infos = [sess.info(t) for t in range(len(xs))]
    live = {}
    for i in infos:
        live[i["slot"]] = i["hash"]
    assert books[-1].hash in live.values()
    for t, x in enumerate(xs):
        y = torch.empty(x.size, dtype=torch.uint8, device=cuda)
        st = torch.zeros(1, dtype=torch.int32, device=cuda)
        sess.decode(outs[t], x.size, y, st)
        torch.cuda.synchronize()
        if infos[t]["hash"] in live.values():
            assert int(st.item()) == 0 and (y.cpu().numpy() == x).all(), t
        else:
            assert int(st.item()) == hx.HX_ERR_CODEBOOK, t


def test_old_stream_after_slot_reuse_is_refused(orc, cuda):
    """Two slots and a new codebook every batch: an early stream's table is gone."""
    rng = np.random.default_rng(5)
    sess = hx.Session(cuda, hx.KIND_HUFFMAN, history=1, lag=1, drift=0.0, slots=2)
    outs, xs = [], []
    for t in range(6):
        x = np.clip(rng.normal(0, 1, 20000) * (10 + 15 * t) + 128, 0, 255).astype(np.uint8)
        out = torch.empty(hx.encode_bound(x.size), dtype=torch.uint8, device=cuda)
        scratch = torch.empty(hx.scratch_bytes(x.size), dtype=torch.uint8, device=cuda)
        st = torch.zeros(1, dtype=torch.int32, device=cuda)
        sess.encode(torch.from_numpy(x).to(cuda), out, scratch, st)
        outs.append(out)
        xs.append(x)
    torch.cuda.synchronize()
    hashes = [sess.info(t)["hash"] for t in range(6)]
    assert len(set(hashes[1:])) == 5  # every batch after the first brought a new codebook
    y = torch.empty(xs[0].size, dtype=torch.uint8, device=cuda)
    st = torch.zeros(1, dtype=torch.int32, device=cuda)
    sess.decode(outs[1], xs[1].size, y, st)
    torch.cuda.synchronize()
    assert int(st.item()) == hx.HX_ERR_CODEBOOK
    st.zero_()
    y = torch.empty(xs[5].size, dtype=torch.uint8, device=cuda)
    sess.decode(outs[5], xs[5].size, y, st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and (y.cpu().numpy() == xs[5]).all()


@pytest.mark.parametrize("kind", [hx.KIND_HUFFMAN, hx.KIND_QLC])
def test_decode_set_picks_by_hash(orc, cuda, kind):
    books, streams, xs = [], [], []
    for seed in range(3):
        counts = datagen.random_counts(40 + seed)
        cb = hx.build_codebook(counts) if kind == hx.KIND_HUFFMAN else hx.qlc_build(counts)
        x = datagen.data(1, n=3 * 4096 + 77 * (seed + 1))
        out, st = hx.encode(cb.upload(cuda), torch.from_numpy(x).to(cuda), kind=kind)
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        books.append(cb.upload(cuda))
        streams.append(out)
        xs.append(x)
    empty = torch.zeros(hx.TABLES_BYTES, dtype=torch.uint8, device=cuda)
    for i, (s, x) in enumerate(zip(streams, xs)):
        for order in ([empty, books[2], books[0], books[1]], books[::-1]):
            y, st = hx.decode_set(kind, order, s, x.size)
            torch.cuda.synchronize()
            assert int(st.item()) == 0 and (y.cpu().numpy() == x).all(), (i, len(order))
        others = [b for j, b in enumerate(books) if j != i]
        _, st = hx.decode_set(kind, others, s, x.size)
        torch.cuda.synchronize()
        assert int(st.item()) == hx.HX_ERR_CODEBOOK
