"""The single-pass encoder's bounded wait (failure detection without a GPU fault), and the other
knob hx_encode_bounded exposes, the fused histogram's flush interval.

Each chunk learns its word offset from the chunks before it. A chunk that never publishes its
word count (the `withhold` argument of hx_encode_bounded) makes every later chunk's wait run out:
they raise HX_ERR_TIMEOUT and write no payload, the kernel still completes, and the context stays
usable (a normal encode right after it equals the oracle's stream).
"""
import numpy as np
import pytest

import datagen

torch = pytest.importorskip("torch")
from lossless_entropy_coding_fixed_b200 import hx  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    counts = sum(oracle.histogram(b) for b in datagen.prior_batches(1))
    cb = hx.build_codebook(counts)
    return oracle, cb.upload(torch.device("cuda:0")), oracle.huffman_codebook(counts)


def _buffers(n):
    out = torch.zeros(hx.encode_bound(n), dtype=torch.uint8, device="cuda")
    scratch = torch.empty(hx.scratch_bytes(n), dtype=torch.uint8, device="cuda")
    return out, scratch


@pytest.mark.parametrize("withhold", [0, 3, 39])
def test_withheld_chunk_times_out_and_context_survives(setup, withhold):
    orc, tables, ocb = setup
    n = 40 * 4096 - 100
    x = datagen.data(1, n=n)
    xd = torch.from_numpy(x).cuda()
    out, scratch = _buffers(n)
    _, st = hx.encode_bounded(tables, xd, out, scratch, wait_ns=2_000_000, withhold=withhold)
    torch.cuda.synchronize()
    status = int(st.item())
    if withhold == 39:  # the last chunk: nothing waits for it, the stream is whole
        assert status == 0
    else:
        assert status & hx.HX_ERR_TIMEOUT
    # the context still works: a normal encode equals the oracle's stream
    out2, scratch2 = _buffers(n)
    _, st2 = hx.encode(tables, xd, out=out2, scratch=scratch2)
    torch.cuda.synchronize()
    ref = orc.encode(ocb, x)[1]
    assert int(st2.item()) == 0 and (out2[:ref.size].cpu().numpy() == ref).all()


def test_generous_limit_and_no_withheld_chunk_equals_oracle(setup):
    orc, tables, ocb = setup
    n = (1 << 20) + 777
    x = datagen.data(4, n=n)
    out, scratch = _buffers(n)
    _, st = hx.encode_bounded(tables, torch.from_numpy(x).cuda(), out, scratch,
                              wait_ns=10 ** 9, withhold=n)  # a chunk index past the end
    torch.cuda.synchronize()
    ref = orc.encode(ocb, x)[1]
    assert int(st.item()) == 0 and (out[:ref.size].cpu().numpy() == ref).all()


@pytest.mark.parametrize("flush_rounds", [1, 2])
def test_fused_histogram_flushed_every_chunk(setup, flush_rounds):
    """Each warp clears the shared counts into the histogram after every (or every second) chunk
    it codes, while the other warps keep counting: the histogram and the stream still equal the
    oracle's."""
    orc, tables, ocb = setup
    n = (1 << 24) + 777
    x = datagen.data(4, n=n)
    out, scratch = _buffers(n)
    hist = torch.zeros(256, dtype=torch.int32, device="cuda")
    _, st = hx.encode_bounded(tables, torch.from_numpy(x).cuda(), out, scratch, wait_ns=10 ** 9,
                              hist=hist, flush_rounds=flush_rounds)
    torch.cuda.synchronize()
    ref = orc.encode(ocb, x)[1]
    assert int(st.item()) == 0 and (out[:ref.size].cpu().numpy() == ref).all()
    assert (hist.cpu().numpy().astype(np.uint64) == orc.histogram(x)).all()


@pytest.mark.parametrize("withhold", [0, 4, 9])
def test_shannonic_withheld_group_times_out_and_context_survives(setup, withhold):
    """The Shannonic encoder's look-back runs over groups of 4 chunks: a group that never
    publishes its word count makes the groups after it time out (group 9 is the last of 40
    chunks: nothing waits for it)."""
    orc = setup[0]
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(1))
    tables = hx.shannonic_build(counts).upload(torch.device("cuda:0"))
    ocb = orc.shannonic_codebook(counts)
    n = 40 * 4096 - 100
    x = datagen.data(1, n=n)
    xd = torch.from_numpy(x).cuda()
    k = hx.KIND_SHANNONIC
    out = torch.zeros(hx.encode_bound(n, k), dtype=torch.uint8, device="cuda")
    scratch = torch.empty(hx.scratch_bytes(n), dtype=torch.uint8, device="cuda")
    _, st = hx.encode_bounded(tables, xd, out, scratch, wait_ns=2_000_000, withhold=withhold,
                              kind=k)
    torch.cuda.synchronize()
    status = int(st.item())
    ref = orc.encode(ocb, x)[1]
    if withhold == 9:
        assert status == 0 and (out[:ref.size].cpu().numpy() == ref).all()
    else:
        assert status & hx.HX_ERR_TIMEOUT
    out2 = torch.zeros_like(out)
    _, st2 = hx.encode(tables, xd, out=out2, scratch=scratch, kind=k)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0 and (out2[:ref.size].cpu().numpy() == ref).all()
