"""The compressed all-gather's exchange on CPU ranks (gloo, world size 2), with a stand-in coder:
the real one needs a GPU. Checks the size exchange, the padding to the longest stream, the
reassembly in rank order and the refusal of unequal shards."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from lossless_entropy_coding_fixed_b200 import collective, hx


class StandInCodec(collective.Codec):
    """A 'stream' in the library's layout with the shard's bytes as payload: header with
    total_words, then the bytes at the payload offset (the length depends on the shard)."""

    def bound(self, n):
        return hx.payload_offset(n) + n + 64

    def encode(self, tables, x, out):
        n = x.numel()
        keep = n - int(x[0]) % 7  # streams of different lengths on different ranks
        words = (keep + 3) // 4
        out.zero_()
        out[32:40] = torch.tensor([words], dtype=torch.int64).view(torch.uint8)
        P = hx.payload_offset(n)
        out[P:P + n] = x

    def decode(self, tables, stream, n, out):
        P = hx.payload_offset(n)
        assert stream.numel() == hx.stream_bytes(n, int(stream[32:40].view(torch.int64)[0]))
        out.copy_(stream[P:P + n]) if stream.numel() >= P + n else out.copy_(torch.cat(
            [stream[P:], torch.zeros(P + n - stream.numel(), dtype=torch.uint8)]))


def _run(rank, world, port, n, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = torch.from_numpy(np.random.default_rng(rank).integers(0, 256, n, dtype=np.uint8))
        out, sizes = collective.compressed_all_gather(x, None, codec=StandInCodec())
        results[rank] = (out.numpy().copy(), sizes)
    finally:
        dist.destroy_process_group()


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_two_ranks_gather_in_rank_order():
    n, world = 10000, 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        port = _port()
        procs = [ctx.Process(target=_run, args=(r, world, port, n, results)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
            assert p.exitcode == 0
        expect = np.concatenate([np.random.default_rng(r).integers(0, 256, n, dtype=np.uint8)
                                 for r in range(world)])
        keep = [n - int(expect[r * n]) % 7 for r in range(world)]
        for r in range(world):
            out, sizes = results[r]
            assert sizes == [hx.stream_bytes(n, (k + 3) // 4) for k in keep]
            for q in range(world):
                got = out[q * n:(q + 1) * n]
                # the stand-in keeps the whole shard whenever the stream holds it
                assert (got[:keep[q] - 3] == expect[q * n:q * n + keep[q] - 3]).all()


class LosslessStandIn(collective.Codec):
    """A lossless stand-in: the header's total_words covers the bytes plus 0..2 spare words that
    depend on the first byte, so streams differ in length across ranks and parts."""

    def bound(self, n):
        return hx.stream_bytes(n, (n + 3) // 4 + 2)

    def words(self, x):
        return (x.numel() + 3) // 4 + (int(x[0]) % 3 if x.numel() else 0)

    def encode(self, tables, x, out):
        n = x.numel()
        out.zero_()
        out[32:40] = torch.tensor([self.words(x)], dtype=torch.int64).view(torch.uint8)
        P = hx.payload_offset(n)
        out[P:P + n] = x

    def decode(self, tables, stream, n, out):
        assert stream.numel() == hx.stream_bytes(n, int(stream[32:40].view(torch.int64)[0]))
        P = hx.payload_offset(n)
        out.copy_(stream[P:P + n])


class OracleCodec(collective.Codec):
    """The CPU oracle as the coder: real streams in the library's format, so a merged stream can
    be checked against the oracle's stream of all ranks' bytes (not against merge_streams)."""

    def __init__(self):
        import datagen
        import oracle
        self.oracle = oracle
        self.cb = oracle.huffman_codebook(sum(oracle.histogram(b)
                                              for b in datagen.prior_batches(1)))

    def bound(self, n):
        return self.oracle.encode_bound(n)

    def encode(self, tables, x, out):
        st = self.oracle.encode(self.cb, x.numpy())[1]
        out[:st.size] = torch.from_numpy(st)

    def decode(self, tables, stream, n, out):
        status, y = self.oracle.decode(self.cb, stream.numpy(), n)
        assert status == 0
        out.copy_(torch.from_numpy(y))


CASES = [(10000, 1), (10000, 3), (10000, 6), (3 * 4096, 2), (0, 3), (1, 4)]
MERGED = [(3 * 4096, 1), (3 * 4096, 2)]


def _shard(rank, n):
    return torch.from_numpy(np.random.default_rng(100 + rank).integers(0, 256, n, dtype=np.uint8))


def _run_parts(rank, world, port, results):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = []
        for n, parts in CASES:
            out, sent = collective.compressed_all_gather(_shard(rank, n), None,
                                                         codec=LosslessStandIn(), parts=parts)
            res.append((out.numpy().copy(), sent))
        for n, parts in MERGED:  # one global stream instead of the decoded bytes
            st, sent = collective.compressed_all_gather(_shard(rank, n), None,
                                                        codec=OracleCodec(), parts=parts,
                                                        decode=False)
            res.append((st.numpy().copy(), sent))
        try:  # a merged stream of shards that are not whole chunks: every rank refuses
            collective.compressed_all_gather(_shard(rank, 5000), None, codec=LosslessStandIn(),
                                             decode=False)
            res.append("accepted")
        except ValueError:
            res.append("refused")
        try:  # a merged stream of 2^32 bytes or more: refused before any coding (the shard is
            # never touched, so its pages are never committed)
            collective.compressed_all_gather(torch.empty(1 << 31, dtype=torch.uint8), None,
                                             codec=LosslessStandIn(), decode=False)
            res.append("accepted")
        except ValueError:
            res.append("refused")
        try:  # unequal shards: every rank must refuse, none may hang
            collective.compressed_all_gather(_shard(rank, 4096 + rank), None,
                                             codec=LosslessStandIn(), parts=2)
            res.append("accepted")
        except ValueError:
            res.append("refused")
        results[rank] = res
    finally:
        dist.destroy_process_group()


def test_parts_pipeline_two_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    with ctx.Manager() as m:
        results = m.dict()
        port = _port()
        procs = [ctx.Process(target=_run_parts, args=(r, world, port, results))
                 for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(180)
            assert p.exitcode == 0
        codec = LosslessStandIn()
        for r in range(world):
            res = results[r]
            assert res[-3:] == ["refused", "refused", "refused"]
            merged = res[len(CASES):len(CASES) + len(MERGED)]
            oc = OracleCodec()
            for (n, parts), (st, sent) in zip(MERGED, merged):
                # the oracle's stream of every rank's bytes in rank order
                whole = np.concatenate([_shard(q, n).numpy() for q in range(world)])
                expect = oc.oracle.encode(oc.cb, whole)[1]
                assert st.size == expect.size and (st == expect).all(), (n, parts)
            for (n, parts), (out, sent) in zip(CASES, res[:len(CASES)]):
                shards = [_shard(q, n) for q in range(world)]
                assert (out == np.concatenate([s.numpy() for s in shards])).all(), (n, parts)
                bounds = collective.part_bounds(n, parts)
                assert len(bounds) == max(1, min(parts, -(-n // 4096)))
                assert sent == [sum(hx.stream_bytes(hi - lo, codec.words(s[lo:hi]))
                                    for lo, hi in bounds) for s in shards], (n, parts)


# ------------------------------------------------------------------ one global stream
@pytest.fixture(scope="module")
def orc_books():
    import datagen
    import oracle
    counts = sum(oracle.histogram(b) for b in datagen.prior_batches(1))
    return oracle, datagen, [oracle.huffman_codebook(counts), oracle.qlc_codebook(counts),
                             oracle.shannonic_codebook(counts), oracle.ExpGolombBook(6, 0)]


@pytest.mark.parametrize("cuts", [[0, 5 * 4096 + 777], [0, 8192, 16384, 5 * 4096 + 777],
                                  [0, 4096, 4096, 12288, 5 * 4096 + 777], [0, 4096, 8192]])
def test_merge_streams_equals_stream_of_whole(orc_books, cuts):
    """Streams of consecutive chunk-aligned pieces, merged, are byte for byte the oracle's
    stream of the whole input (every chunk codes the same bytes from a word boundary)."""
    oracle, datagen, books = orc_books
    x = datagen.data(1, n=cuts[-1])
    for cb in books:
        pieces = [torch.from_numpy(oracle.encode(cb, x[a:b])[1]) for a, b in zip(cuts, cuts[1:])]
        merged = collective.merge_streams(pieces, [b - a for a, b in zip(cuts, cuts[1:])])
        assert (merged.numpy() == oracle.encode(cb, x)[1]).all()


def test_merge_streams_refusals(orc_books):
    oracle, datagen, books = orc_books
    x = datagen.data(1, n=3 * 4096)
    a = torch.from_numpy(oracle.encode(books[0], x[:4096])[1])
    b = torch.from_numpy(oracle.encode(books[1], x[4096:])[1])
    with pytest.raises(ValueError):  # another codebook
        collective.merge_streams([a, b], [4096, 8192])
    c = torch.from_numpy(oracle.encode(books[0], x[:4000])[1])
    d = torch.from_numpy(oracle.encode(books[0], x[4000:])[1])
    with pytest.raises(ValueError):  # a piece that is not whole chunks
        collective.merge_streams([c, d], [4000, 8288])
    e = torch.from_numpy(oracle.encode(books[0], x[4096:])[1])
    with pytest.raises(ValueError):  # a size that its stream's header does not code
        collective.merge_streams([a, e], [4096, 4096])
    with pytest.raises(ValueError):  # 2^32 bytes or more cannot be one stream
        collective.merge_streams([a, e], [1 << 31, 1 << 31])
