"""The largest input one call takes (n = 2^32 - 1 bytes, 2^20 chunks, the last one ragged), on the
GPU, with the checks that hold at any size and the oracle on sampled chunks.

Every chunk's bits start on a word boundary and depend on its own bytes only, so the oracle's
stream for one chunk's bytes alone holds that chunk's sync row and payload words. The input is a
seeded 64 MiB cfg-4 batch repeated 64 times, less the final byte, so its histogram is 64 times the
batch's minus that byte.
"""
import numpy as np
import pytest

import datagen

torch = pytest.importorskip("torch")
from lossless_entropy_coding_fixed_b200 import hx  # noqa: E402

pytestmark = pytest.mark.gpu

N = (1 << 32) - 1
TILE = 1 << 26
CHUNK = 4096


@pytest.fixture(scope="module")
def setup(orc):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    tile = datagen.data(4, n=TILE)
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(4))
    x = torch.from_numpy(tile).cuda().repeat(N // TILE + 1)[:N]
    hist = orc.histogram(tile).astype(np.uint64) * np.uint64(N // TILE + 1)
    hist[tile[-1]] -= np.uint64(1)
    yield tile, counts, x, hist
    del x
    torch.cuda.empty_cache()


def chunk_bytes(tile, c):
    lo, hi = c * CHUNK, min(N, (c + 1) * CHUNK)
    return np.concatenate([tile, tile])[lo % TILE:lo % TILE + (hi - lo)]


@pytest.mark.parametrize("kind", ["huffman", "qlc", "shannonic"])
def test_max_size_stream(orc, setup, kind):
    tile, counts, x, hist_expected = setup
    if kind == "huffman":
        cb, ocb = hx.build_codebook(counts), orc.huffman_codebook(counts)
    elif kind == "qlc":
        cb, ocb = hx.qlc_build(counts), orc.qlc_codebook(counts)
    else:  # 2^18 groups of 4 chunks in the Shannonic encoder's look-back
        cb, ocb = hx.shannonic_build(counts), orc.shannonic_codebook(counts)
    tables = cb.upload()
    hist = torch.zeros(256, dtype=torch.int32, device="cuda")
    out, st = hx.encode(tables, x, hist=hist, kind=cb.kind)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert (hist.cpu().numpy().view(np.uint32).astype(np.uint64) == hist_expected).all()

    nc = N // CHUNK + 1
    assert nc == 1 << 20
    size = hx.stream_size(out, N)
    S, P = hx.sync_offset(N), hx.payload_offset(N)
    head = out[:P].cpu().numpy()
    woff = head[64:64 + 4 * (nc + 1)].view(np.uint32).astype(np.int64)
    sync = head[S:S + 16 * nc].view(np.uint16).reshape(nc, 8).astype(np.int64)
    total = hx.total_words(out)
    # the index at any size: word offsets are the prefix sums of the chunks' padded bit counts
    assert woff[0] == 0 and woff[-1] == total and size == P + 4 * (total + 2)
    assert (np.diff(woff) == (sync[:, 0] + 31) // 32).all()
    assert (np.diff(sync[:, 1:], axis=1) >= 0).all() and (sync[:, 7] <= sync[:, 0]).all()

    # sampled chunks against the oracle, byte for byte: both ends, the 2^31 byte boundary, the
    # ragged last chunk (4095 bytes), and seeded random ones
    rng = np.random.default_rng(97)
    picks = sorted({0, 1, (1 << 19) - 1, 1 << 19, nc - 2, nc - 1,
                    *rng.integers(0, nc, 10).tolist()})
    for c in picks:
        xc = chunk_bytes(tile, c)
        assert xc.size == (CHUNK if c < nc - 1 else N - c * CHUNK)
        ost, ref = orc.encode(ocb, xc)
        assert ost == 0
        Sc, Pc = hx.sync_offset(xc.size), hx.payload_offset(xc.size)
        ref_sync = ref[Sc:Sc + 16].view(np.uint16).astype(np.int64)
        ref_words = ref[Pc:ref.size - 8].view(np.uint32)
        assert (sync[c] == ref_sync).all(), c
        assert woff[c + 1] - woff[c] == ref_words.size, c
        got = out[P + 4 * woff[c]:P + 4 * woff[c + 1]].cpu().numpy().view(np.uint32)
        assert (got == ref_words).all(), c

    y, st = hx.decode(tables, out[:size], N, kind=cb.kind)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(y, x)
    del out, y
    torch.cuda.empty_cache()
