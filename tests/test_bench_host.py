"""bench.py's host logic on CPU: the max-over-ranks timing across 2 gloo ranks (the N > 1 path
has no data-path collective, only this reduction), the whole-job throughput, and the reference
(oracle) arm on a bounded sample, including its silent exit on ranks other than 0."""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout
from types import SimpleNamespace

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, dist, torch.device("cpu"))
        out[rank] = ms
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(2, port, out), nprocs=2, join=True)
        assert dict(out) == {0: 15.0, 1: 15.0}


def test_job_throughput_is_whole_job():
    assert bench.job_gbs(1, 4 << 30, 1.0) == pytest.approx(4 * 1.073741824e9 / 1e-3 / 1e9)
    assert bench.job_gbs(8, 1 << 30, 2.0) == pytest.approx(8 * bench.job_gbs(1, 1 << 30, 2.0))
    assert bench.max_over_ranks(3.5, None, None) == 3.5


def test_reference_arm_runs_oracle_on_rank0_only():
    args = SimpleNamespace(steps=2, warmup=1)
    buf = io.StringIO()
    with redirect_stdout(buf):
        assert bench.cpu_reference(args, rank=1, ws=2) == 0
    assert buf.getvalue() == ""
    with redirect_stdout(buf):
        assert bench.cpu_reference(args, rank=0, ws=1) == 0
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] > 0
    assert line["cpu_baseline"]["kind"] == "oracle"
    assert line["cpu_baseline"]["cores"] == (os.cpu_count() or 1)
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["higher_is_better"] is True


def test_oracle_slices_are_chunk_aligned_and_cover_the_input():
    import numpy as np
    x = np.arange(5 * 4096 + 77, dtype=np.uint64).astype(np.uint8)
    for threads in (1, 2, 3, 8, 64):
        sl = bench._oracle_slices(x, threads)
        assert len(sl) <= threads and all(s.size % 4096 == 0 for s in sl[:-1])
        assert (np.concatenate(sl) == x).all()


def test_roofline_entry_arithmetic():
    r = bench.roofline_entry("k", [(2e9, 1.0), (1e9, 0.5)], 6000.0, "measured")
    assert r["algorithmic_bytes_per_launch"] == 1.5e9 and r["ms_per_launch"] == 0.75
    assert r["achieved"] == pytest.approx(1.5e9 / 0.75e-3 / 1e9)
    assert r["frac"] == pytest.approx(r["achieved"] / 6000.0)
    assert r["frac_spec"] == pytest.approx(r["achieved"] / bench.SPEC_HBM_GBS)
    assert r["launches_per_step"] == 2


def test_code_only_ignores_comments_and_layout():
    src = 'int f(int a) {  // the sum\n  /* two\n lines */ return a + 1;\n}\nconst char* s = "a // b";\n'
    same = 'int f(int a) { return a + 1; }\n// another note\nconst char* s = "a // b";'
    changed = 'int f(int a) { return a + 2; }\nconst char* s = "a // b";'
    assert bench.code_only(src) == bench.code_only(same)
    assert bench.code_only(src) != bench.code_only(changed)
    assert '"a // b"' in bench.code_only(src)
