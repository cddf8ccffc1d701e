"""Many encode/decode round trips of random sizes and offsets, through the C ABI.

The single-pass encoder takes each chunk's word offset from the chunks before it while they are
still being coded (a decoupled look-back over a window of 64 chunks), and the fused histogram's
counts are flushed by warps while other warps keep counting. Both are races that a few fixed cases
could miss, so this runs 400 random cases: sizes from 1 byte to 32 MiB at random offsets into one
batch, each of the three prefix-code kinds and the Shannonic coder (whose encoder parks each
sub-stream in shared memory and learns a group's offset the same way), half of the Huffman and
Shannonic cases with the fused histogram.
Every stream must decode back to its input with status 0, every fused histogram must equal the
bytes' counts, and every 10th stream up to 4 MiB must equal the oracle's byte for byte.
"""
import numpy as np
import pytest

import datagen

torch = pytest.importorskip("torch")
from lossless_entropy_coding_fixed_b200 import hx  # noqa: E402

pytestmark = pytest.mark.gpu


def test_random_round_trips():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    dev = torch.device("cuda:0")
    rng = np.random.default_rng(20261203)
    pool = datagen.data(4, n=1 << 25)
    pool_d = torch.from_numpy(pool).to(dev)
    prior = sum(oracle.histogram(b) for b in datagen.prior_batches(1))
    books = [(hx.build_codebook(prior), oracle.huffman_codebook(prior)),
             (hx.qlc_build(prior), oracle.qlc_codebook(prior)),
             (hx.expgolomb_build(7, 0), None),
             (hx.shannonic_build(prior), oracle.shannonic_codebook(prior))]
    books = [(cb, cb.upload(dev), ocb) for cb, ocb in books]
    compared = 0
    for it in range(400):
        n = int(rng.integers(1, 1 << 25)) if rng.random() < 0.7 else int(rng.integers(1, 1 << 16))
        off = int(rng.integers(0, (1 << 25) - n + 1)) & ~15  # inputs are 16-byte aligned
        n = min(n, (1 << 25) - off)
        cb, tables, ocb = books[int(rng.integers(0, len(books)))]
        x = pool_d[off:off + n]
        hist = None
        if cb.kind in (hx.KIND_HUFFMAN, hx.KIND_SHANNONIC) and rng.random() < 0.5:
            hist = torch.zeros(256, dtype=torch.int32, device=dev)
        out, st = hx.encode(tables, x, hist=hist, kind=cb.kind)
        y, st2 = hx.decode(tables, out, n, kind=cb.kind)
        torch.cuda.synchronize()
        case = (it, n, off, cb.kind)
        assert int(st.item()) == 0 and int(st2.item()) == 0, case
        assert torch.equal(x, y), case
        if hist is not None:
            counts = np.bincount(pool[off:off + n], minlength=256).astype(np.uint64)
            assert (hist.cpu().numpy().astype(np.uint64) == counts).all(), case
        if ocb is not None and it % 10 == 0 and n <= 1 << 22:
            ref = oracle.encode(ocb, pool[off:off + n])[1]
            size = hx.stream_size(out, n)
            assert size == ref.size and (out[:size].cpu().numpy() == ref).all(), case
            compared += 1
    assert compared >= 10
