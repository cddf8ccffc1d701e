"""The compressed all-gather on a GPU with NCCL and the real coder (each of the four stream
kinds), as one rank (the exchange between two ranks is covered on CPU ranks), in a child process
so the process group does not outlive the test."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


def _port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(port, q):
    import datetime

    import torch.distributed as dist

    import datagen
    from lossless_entropy_coding_fixed_b200 import collective, hx
    import oracle

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1,
                            timeout=datetime.timedelta(seconds=60), device_id=torch.device("cuda:0"))
    try:
        res = {}
        prior = sum(oracle.histogram(b) for b in datagen.prior_batches(1))
        books = {hx.KIND_HUFFMAN: (hx.build_codebook(prior), oracle.huffman_codebook(prior)),
                 hx.KIND_QLC: (hx.qlc_build(prior), oracle.qlc_codebook(prior)),
                 hx.KIND_SHANNONIC: (hx.shannonic_build(prior), oracle.shannonic_codebook(prior)),
                 hx.KIND_EXPGOLOMB: (hx.expgolomb_build(6, 0), oracle.ExpGolombBook(6, 0))}
        for kind, (cb, ocb) in books.items():
            for parts in (1, 3):
                x = datagen.data(1, n=(1 << 20) - 77)
                out, sizes = collective.compressed_all_gather(
                    torch.from_numpy(x).cuda(), cb.upload("cuda"), codec=collective.Codec(kind),
                    parts=parts)
                torch.cuda.synchronize()
                ref = sum(int(oracle.encode(ocb, x[lo:hi])[1].size)
                          for lo, hi in collective.part_bounds(x.size, parts))
                # the stream bytes themselves: kept coded, the parts merge into the oracle's
                # stream of the whole shard
                xs = x[:(x.size // 4096) * 4096]
                st, _ = collective.compressed_all_gather(
                    torch.from_numpy(xs).cuda(), cb.upload("cuda"), codec=collective.Codec(kind),
                    parts=parts, decode=False)
                torch.cuda.synchronize()
                same = bool(np.array_equal(st.cpu().numpy(), oracle.encode(ocb, xs)[1]))
                res[(kind, parts)] = (bool((out.cpu().numpy() == x).all()), sizes, ref, same)
        q.put(res)
    finally:
        dist.destroy_process_group()


def test_one_rank_round_trip():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_rank, args=(_port(), q))
    p.start()
    res = q.get(timeout=300)
    p.join(120)
    assert p.exitcode == 0
    assert len(res) == 8
    for case, (ok, sizes, ref_size, same_stream) in res.items():
        assert ok and sizes == [ref_size] and same_stream, case
