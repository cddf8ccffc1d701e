"""Full-size workloads on the GPU against the oracle: the streams the benchmark times.

For each workload the codebook comes from its prior batches (cfg 3: its own histogram), the GPU
stream must equal the oracle's byte for byte, the GPU must decode it back to the input, the
fused histogram must equal the oracle's, and the payload bits per symbol must equal the oracle's
mean code length on the data.
"""
import numpy as np
import pytest

import datagen

torch = pytest.importorskip("torch")
from lossless_entropy_coding_fixed_b200 import hx  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")


def prior_counts(orc, cfg, layer=0):
    return sum(orc.histogram(b) for b in datagen.prior_batches(cfg, layer))


def check_workload(orc, x, counts, kind):
    if kind == "huffman":
        cb, ocb = hx.build_codebook(counts), orc.huffman_codebook(counts)
    else:
        cb, ocb = hx.qlc_build(counts), orc.qlc_codebook(counts)
    assert cb.hash == ocb.hash
    tables = cb.upload()
    xd = torch.from_numpy(x).cuda()
    hist = torch.zeros(256, dtype=torch.int32, device="cuda")
    out, st = hx.encode(tables, xd, hist=hist, kind=cb.kind)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    size = hx.stream_size(out, x.size)
    ost, ref = orc.encode(ocb, x)
    assert ost == 0 and size == ref.size
    got = out[:size].cpu().numpy()
    assert (got == ref).all()
    h = orc.histogram(x)
    assert (hist.cpu().numpy().astype(np.uint64) == h).all()
    y, st = hx.decode(tables, out[:size], x.size, kind=cb.kind)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert torch.equal(y, xd)
    # payload bits per symbol = the oracle's mean code length on this data
    nc = -(-x.size // 4096)
    S = hx.sync_offset(x.size)
    bits = got[S:S + 16 * nc].view(np.uint16).reshape(nc, 8)[:, 0].astype(np.int64).sum()
    assert bits / x.size == pytest.approx(orc.mean_length(h, ocb.len), rel=1e-12)
    del out, y, xd
    torch.cuda.empty_cache()
    return bits / x.size


@pytest.mark.parametrize("kind", ["huffman", "qlc"])
def test_cfg2_ffn_mix_256mib(orc, kind):
    x = datagen.data(2)
    check_workload(orc, x, prior_counts(orc, 2), kind)


@pytest.mark.parametrize("kind", ["huffman", "qlc"])
def test_cfg3_int8_per_tensor_64mib(orc, kind):
    x = datagen.data(3)
    counts = orc.histogram(x)
    check_workload(orc, x, counts, kind)


@pytest.mark.parametrize("kind", ["huffman", "qlc"])
def test_cfg4_e4m3_1gib(orc, kind):
    x = datagen.data(4)
    bps = check_workload(orc, x, prior_counts(orc, 4), kind)
    h = orc.histogram(x)
    per_shard = orc.mean_length(h, orc.huffman_lengths(h, cover_all=False))
    if kind == "huffman":
        assert bps <= per_shard * 1.01  # fixed codebook within 1% of the per-shard code
    assert bps >= orc.entropy(h)


@pytest.mark.parametrize("layer", range(16))
def test_cfg5_layer_shards(orc, layer):
    """Every layer (so every dtype and law of the batch): one shard with its layer's Huffman
    codebook, another with its layer's QLC (32 of the 64 shards)."""
    counts = prior_counts(orc, 5, layer)
    x = datagen.data(5, shard=4 * layer + layer % 4)
    bps = check_workload(orc, x, counts, "huffman")
    h = orc.histogram(x)
    assert bps >= orc.mean_length(h, orc.huffman_lengths(h, cover_all=False)) >= orc.entropy(h)
    x = datagen.data(5, shard=4 * layer + (layer + 2) % 4)
    check_workload(orc, x, counts, "qlc")
