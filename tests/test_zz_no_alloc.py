"""The allocation-free encode entry point (hx_encode_noalloc), called through the C ABI.

Some callers cannot allocate device memory when they encode: code running under a framework
whose caching allocator has reserved the device's memory, or a latency-critical path that cannot
take cudaMalloc's implicit synchronisation. hx_encode_noalloc keeps its scratch in a fixed array
inside the library instead. It must write exactly the stream hx_encode writes (bit-exact, as for
every byte-valued result here), on two calls in a row that reuse that array.

This file is collected last, so a run that stops at its first failure has run every other test.
"""
import ctypes

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
    dev = torch.device("cuda:0")
    counts = np.zeros(256, np.uint64)
    for b in datagen.prior_batches(1):
        counts += np.bincount(b, minlength=256).astype(np.uint64)
    tables = hx.build_codebook(counts).upload(dev)
    return dev, tables


def _raw_noalloc(tables, x, out, hist, status):
    L = hx.lib()
    return L.hx_encode_noalloc(ctypes.c_void_p(tables.data_ptr()), ctypes.c_void_p(x.data_ptr()),
                               x.numel(), ctypes.c_void_p(out.data_ptr()), out.numel(),
                               ctypes.c_void_p(hist.data_ptr()), ctypes.c_void_p(status.data_ptr()),
                               ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("n", [(1 << 24) + 777, 4096 * 3 + 5])
def test_noalloc_equals_encode_twice(setup, n):
    dev, tables = setup
    x = torch.from_numpy(datagen.data(4, n=n)).to(dev)
    ref, st = hx.encode(tables, x)
    hist_ref = torch.zeros(256, dtype=torch.int32, device=dev)
    hx.histogram(x, hist_ref)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    size = hx.stream_size(ref, n)
    for _ in range(2):  # the second call reuses (and must re-clear) the library's scratch
        out = torch.full((hx.encode_bound(n),), 0xA5, dtype=torch.uint8, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        hist = torch.zeros(256, dtype=torch.int32, device=dev)
        assert _raw_noalloc(tables, x, out, hist, status) == 0
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert hx.stream_size(out, n) == size
        assert torch.equal(out[:size], ref[:size])
        assert torch.equal(hist, hist_ref)


@pytest.mark.parametrize("n", [128 << 20, (100 << 20) + 4095])
def test_noalloc_equals_oracle_at_the_limit(setup, n):
    """The largest input the library's array is sized for (HX_NOALLOC_MAX_BYTES exactly), and a
    ragged size: the stream equals the oracle's byte for byte."""
    import oracle
    dev, tables = setup
    assert n <= hx.NOALLOC_MAX_BYTES
    counts = sum(oracle.histogram(b) for b in datagen.prior_batches(1))
    xh = datagen.data(4, n=n)
    x = torch.from_numpy(xh).to(dev)
    out = torch.full((hx.encode_bound(n),), 0xA5, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    hist = torch.zeros(256, dtype=torch.int32, device=dev)
    assert _raw_noalloc(tables, x, out, hist, status) == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = oracle.encode(oracle.huffman_codebook(counts), xh)[1]
    assert hx.stream_size(out, n) == ref.size
    assert (out[:ref.size].cpu().numpy() == ref).all()
    assert (hist.cpu().numpy().astype(np.uint64) == oracle.histogram(xh)).all()


def test_noalloc_refuses_oversize(setup):
    dev, tables = setup
    n = (128 << 20) + 1
    x = torch.empty(n, dtype=torch.uint8, device=dev)
    out = torch.empty(hx.payload_offset(n) + 16, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    hist = torch.zeros(256, dtype=torch.int32, device=dev)
    assert _raw_noalloc(tables, x, out, hist, status) == hx.HX_ERR_ARG
    torch.cuda.synchronize()
    assert int(status.item()) == 0
