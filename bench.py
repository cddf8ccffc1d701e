#!/usr/bin/env python3
"""Benchmark of the fixed-codebook entropy coder on B200: one JSON line on rank 0.

Workload (one step): a 1 GiB batch of e4m3 bytes (fp32 N(0,1)*0.5, RNE-saturating cast), the
fixed Huffman codebook (package-merge, Lmax 12) and the Quad Length Code built from the summed
histogram of 4 earlier 1 MiB batches of the same law. A step runs the whole hot path on the batch:
Huffman encode with the histogram fused in, Huffman decode, QLC encode, QLC decode. The metric is
uncompressed bytes through the codec per second (4 x 1 GiB per step) and bits per symbol.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hx|reference]

Timing: W untimed steps, then exactly K steps between a barrier + synchronize on both sides,
CUDA events on the stream the kernels run on, max over ranks. The inputs (1 GiB) are larger than
the 126 MB L2, so no flush is needed between steps. `--impl reference` times the CPU oracle (the
reference implementation of this build) on a bounded sample of the same workload, rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

N_BYTES = 1 << 30
WORKLOAD = ("cfg4: 1 GiB e4m3 bytes of N(0,1)*0.5; fixed Huffman (Lmax 12) and QLC (8 areas) "
            "from 4 prior 1 MiB batches; step = Huffman encode(+fused histogram) + decode + "
            "QLC encode + decode")
METRIC = "encode & decode GB/s (uncompressed) at 1 B200, % of HBM roofline; bits/symbol"
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ["lossless_entropy_coding_fixed_b200/csrc/hx_kernels.cu",
                  "lossless_entropy_coding_fixed_b200/csrc/hx_tables.h"]


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=100)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="hx", choices=["hx", "reference"])
    p.add_argument("--n", type=int, default=N_BYTES, help="bytes per batch (default 1 GiB)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-online", action="store_true")
    p.add_argument("--no-shannonic", action="store_true")
    p.add_argument("--no-expgolomb", action="store_true")
    return p.parse_args()


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), ws


def max_over_ranks(ms: float, pg, device) -> float:
    """The slowest rank's time: every rank calls this at the same point (a MAX all-reduce)."""
    if pg is None:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def job_gbs(world: int, bytes_per_rank_step: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank moves its own batch each step (weak scaling)."""
    return world * bytes_per_rank_step / (ms_per_step * 1e-3) / 1e9


def code_only(text: str) -> str:
    """C/C++/CUDA source with its comments removed and every run of whitespace made one space,
    so that an edit of comments or layout leaves the kernels' hash unchanged."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if c in "\"'":  # a string or character literal, copied whole
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        elif text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        else:
            out.append(c)
            i += 1
    return " ".join("".join(out).split())


def kernel_source_hash() -> str:
    """Hash of the kernel sources' code (comments and layout excluded): the DRAM traffic record
    is used only while it matches."""
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), encoding="utf-8") as fh:
            h.update(code_only(fh.read()).encode())
    return h.hexdigest()[:16]


def hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on this source."""
    try:
        with open(os.path.join(ROOT, "profiles", "dram_traffic.json")) as f:
            rec = json.load(f)
    except Exception:
        return None
    if rec.get("kernel_source_sha") != kernel_source_hash():
        return None
    k = rec.get("kernels", {}).get(kernel)
    if not k or rec.get("n") is None:
        return None
    return k["dram_bytes_per_launch"] * (N_BYTES / rec["n"])


class ClockSampler:
    """nvidia-smi samples during the timed region (SM clock, throttle reasons)."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index, self.proc, self.out = index, None, None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                self.out = None

    def summary(self):
        if not self.out:
            return None
        rows = [r.split(", ") for r in self.out.strip().splitlines() if r.count(",") >= 8]
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        if not sm:
            return None
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip() == "Active"})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": float(rows[0][2]),
                "reasons": reasons, "samples": len(sm)}


# ---------------------------------------------------------------------------------------------
def cpu_reference(args, rank, ws):
    """The oracle on a bounded sample of the workload (rank 0 only)."""
    if rank != 0:
        return 0
    import oracle
    import datagen
    sample = 1 << 20
    counts = sum(oracle.histogram(b) for b in datagen.prior_batches(4))
    hb, qb = oracle.huffman_codebook(counts), oracle.qlc_codebook(counts)
    x = datagen.data(4, n=sample)

    def step():
        _, sh = oracle.encode(hb, x)
        oracle.decode(hb, sh, x.size)
        _, sq = oracle.encode(qb, x)
        oracle.decode(qb, sq, x.size)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    value = 4 * sample * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_bytes_per_step": sample},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": f"first {sample} bytes of the 1 GiB batch per step, "
                                   "single-thread bit-serial C++"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline_leg(counts):
    """Time the oracle as it stands on a 64 MiB slice of the workload (~10-30 s, one core)."""
    import oracle
    import datagen
    sample = 64 << 20
    x = datagen.data(4, n=sample)
    hb, qb = oracle.huffman_codebook(counts), oracle.qlc_codebook(counts)
    t0 = time.perf_counter()
    _, sh = oracle.encode(hb, x)
    oracle.decode(hb, sh, x.size)
    _, sq = oracle.encode(qb, x)
    oracle.decode(qb, sq, x.size)
    dt = time.perf_counter() - t0
    return {"value": 4 * sample / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {sample >> 20} MiB of the batch through the same 4 codec calls "
                      f"({dt:.1f} s, single-thread bit-serial C++)"}


def shannonic_leg(dev, hx, torch, x, prior, h, scratch, y, status, steps):
    """The Shannonic coder (range partition + 128-state tANS) on the same batch and prior:
    encode and decode device time per call (CUDA events, inputs resident), bits per symbol."""
    n = x.numel()
    cb = hx.shannonic_build(prior)
    t = cb.upload(dev)
    out = torch.empty(hx.encode_bound(n, hx.KIND_SHANNONIC), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    res = {}
    for name, fn in (("encode", lambda: hx.encode(t, x, out=out, scratch=scratch, status=status,
                                                  kind=hx.KIND_SHANNONIC)),
                     ("decode", lambda: hx.decode(t, out, n, out=y, status=status,
                                                  kind=hx.KIND_SHANNONIC))):
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = a.elapsed_time(b) / steps
    assert int(status.item()) == 0 and torch.equal(x, y)
    size = hx.stream_size(out, n)
    return {"encode_ms": res["encode"], "decode_ms": res["decode"],
            "encode_GB_per_s_uncompressed": n / (res["encode"] * 1e-3) / 1e9,
            "decode_GB_per_s_uncompressed": n / (res["decode"] * 1e-3) / 1e9,
            "ranges": int(cb.raw.sh_nr),
            "bits_per_symbol": {"framed": size * 8 / n, "tans_ideal": hx.mean_length(h, cb)}}


def expgolomb_leg(dev, hx, torch, x, h, scratch, y, status, steps):
    """Exp-Golomb (the QLC page's universal-code contrast) on the same batch: the order 5..8 with
    the shortest mean length on the batch's own histogram (sign-magnitude index, e4m3), encode and
    decode device time per call, bits per symbol."""
    n = x.numel()
    books = {k: hx.expgolomb_build(k, 0) for k in (5, 6, 7, 8)}
    order = min(books, key=lambda k: hx.mean_length(h, books[k]))
    t = books[order].upload(dev)
    out = torch.empty(hx.encode_bound(n), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    res = {}
    for name, fn in (("encode", lambda: hx.encode(t, x, out=out, scratch=scratch, status=status,
                                                  kind=hx.KIND_EXPGOLOMB)),
                     ("decode", lambda: hx.decode(t, out, n, out=y, status=status,
                                                  kind=hx.KIND_EXPGOLOMB))):
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            fn()
        b.record(stream)
        torch.cuda.synchronize(dev)
        res[name] = a.elapsed_time(b) / steps
    assert int(status.item()) == 0 and torch.equal(x, y)
    return {"order": order, "encode_ms": res["encode"], "decode_ms": res["decode"],
            "bits_per_symbol": {"framed": hx.stream_size(out, n) * 8 / n,
                                "payload": hx.mean_length(h, books[order])}}


def online_leg(dev, hx, datagen, torch):
    """The online single-stage loop (hx_session) over 16 batches of 64 MiB: e4m3 activations
    whose scale drifts 3 % per batch, switching law at batch 10 (datagen.online_batch). Every
    batch is encoded with the codebook of the earlier batches' fused histograms (history 4, lag 2,
    drift refresh above 5 % over entropy) and decoded through the hash-picked table slots.
    Inputs resident in HBM; device time over the whole sequence."""
    xs_host = [datagen.online_batch(t, 1 << 26) for t in range(16)]
    xs = [torch.from_numpy(x).to(dev) for x in xs_host]
    n = xs[0].numel()
    prior = np.bincount(datagen.online_batch(0, 1 << 20), minlength=256).astype(np.uint64)
    bound = hx.encode_bound(n)
    outs = [torch.empty(bound, dtype=torch.uint8, device=dev) for _ in range(4)]
    scratch = torch.empty(hx.scratch_bytes(n), dtype=torch.uint8, device=dev)
    y = torch.empty(n, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def run():
        sess = hx.Session(dev, hx.KIND_HUFFMAN, history=4, lag=2, drift=0.05,
                          initial_counts=prior)
        sizes = []
        t0 = time.perf_counter()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for t, x in enumerate(xs):
            out = outs[t % 4]
            sess.encode(x, out, scratch, status)
            sess.decode(out, n, y, status)
        b.record(stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - t0
        sess.drain()
        for t in range(len(xs)):
            sizes.append(sess.info(t))
        return a.elapsed_time(b), wall, sess, sizes

    run()  # warm-up (a fresh session each run: the schedule restarts)
    ms, wall, sess, infos = run()
    assert int(status.item()) == 0, f"status {int(status.item())}"
    # bits: each tensor under the codebook the session used, against its own optimal code
    fixed = own = ent = 0.0
    planner = hx.Planner(hx.KIND_HUFFMAN, 4, 2, 0.05, initial_counts=prior)
    for t, x in enumerate(xs_host):
        h = np.bincount(x, minlength=256).astype(np.uint64)
        if t >= 2:
            planner.observe(t - 2, np.bincount(xs_host[t - 2], minlength=256))
        cb = planner.codebook(t)
        assert cb.hash == infos[t]["hash"]
        fixed += hx.mean_length(h, cb)
        own += hx.mean_length(h, hx.build_codebook(h, seen_only=True))
        ent += hx.entropy(h)
    k = len(xs)
    return {"workload": "16 x 64 MiB e4m3 batches, N(0, 0.5*1.03^t) drifting, FFN-mixture law "
                        "from batch 10; Huffman, history 4, lag 2, drift refresh 5 %; initial "
                        "codebook from 1 MiB of batch 0's law",
            "GB_per_s_uncompressed": 2 * k * n / (ms * 1e-3) / 1e9, "ms": ms,
            "host_wall_ms": wall * 1e3, "refreshes": sum(i["refreshed"] for i in infos),
            "codebooks": len({i["hash"] for i in infos}),
            "bits_per_symbol": {"online": fixed / k, "per_tensor_huffman": own / k,
                                "entropy": ent / k}}


# ---------------------------------------------------------------------------------------------
def main():
    args = parse()
    rank, local_rank, ws = dist_env()
    if args.impl == "reference":
        return cpu_reference(args, rank, ws)

    import torch
    import datagen
    from lossless_entropy_coding_fixed_b200 import hx

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    pg = None
    if ws > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
        pg = dist

    n = args.n
    # codebooks from the prior batches (host, off the data path)
    pc = torch.zeros(256, dtype=torch.int32, device=dev)
    for b in datagen.prior_batches(4):
        hx.histogram(torch.from_numpy(b).to(dev), pc)
    prior = pc.cpu().numpy().astype(np.uint64)
    t0 = time.perf_counter()
    hcb = hx.build_codebook(prior)
    t1 = time.perf_counter()
    qcb = hx.qlc_build(prior)
    t2 = time.perf_counter()
    x_host = datagen.data(4, n=n)
    x = torch.from_numpy(x_host).to(dev)
    ht, qt = hcb.upload(dev), qcb.upload(dev)
    bound = hx.encode_bound(n)
    sh = torch.empty(bound, dtype=torch.uint8, device=dev)
    sq = torch.empty(bound, dtype=torch.uint8, device=dev)
    scratch = torch.empty(hx.scratch_bytes(n), dtype=torch.uint8, device=dev)
    y = torch.empty(n, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    # one fused-histogram row per timed step, so no counter is reset inside the timed region
    hist = torch.zeros(args.steps + 1, 256, dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    ops = ["huffman_encode", "huffman_decode", "qlc_encode", "qlc_decode"]
    # one event pair per kernel launch: an encode is two launches (measure, then pack)
    kern = ["huffman_measure", "huffman_pack", "huffman_decode",
            "qlc_measure", "qlc_pack", "qlc_decode"]
    ev = {k: [] for k in kern}

    def step(record: bool, row: int = 0):
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(7)] if record else None
        mark = (lambda i: marks[i].record(stream)) if record else (lambda i: None)
        mark(0)
        hx.encode_passes(ht, x, sh, scratch, hist=hist[row], status=status,
                         kind=hx.KIND_HUFFMAN, between=lambda: mark(1))
        mark(2)
        hx.decode(ht, sh, n, out=y, status=status, kind=hx.KIND_HUFFMAN)
        mark(3)
        hx.encode_passes(qt, x, sq, scratch, status=status, kind=hx.KIND_QLC,
                         between=lambda: mark(4))
        mark(5)
        hx.decode(qt, sq, n, out=y, status=status, kind=hx.KIND_QLC)
        mark(6)
        if record:
            for i, k in enumerate(kern):
                ev[k].append((marks[i], marks[i + 1]))

    for _ in range(max(3, args.warmup)):
        step(False, args.steps)
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, f"status {int(status.item())}"
    # correctness of the timed configuration: both codecs round-trip the batch
    hx.decode(ht, sh, n, out=y, status=status)
    assert torch.equal(y, x)
    hx.decode(qt, sq, n, out=y, status=status, kind=hx.KIND_QLC)
    assert torch.equal(y, x)
    torch.cuda.synchronize(dev)

    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index) as clocks:
        start.record(stream)
        for i in range(args.steps):
            step(True, i)
        end.record(stream)
        torch.cuda.synchronize(dev)
    if pg:
        pg.barrier()
    elapsed_ms = max_over_ranks(start.elapsed_time(end), pg, dev)
    assert int(status.item()) == 0, f"status {int(status.item())}"
    per_kernel_ms = {k: sum(a.elapsed_time(b) for a, b in ev[k]) / args.steps for k in kern}
    per_op_ms = {"huffman_encode": per_kernel_ms["huffman_measure"] + per_kernel_ms["huffman_pack"],
                 "huffman_decode": per_kernel_ms["huffman_decode"],
                 "qlc_encode": per_kernel_ms["qlc_measure"] + per_kernel_ms["qlc_pack"],
                 "qlc_decode": per_kernel_ms["qlc_decode"]}

    # sizes and bits per symbol
    rows = hist[: args.steps].cpu().numpy().astype(np.uint64)
    h = rows[0]
    assert int(h.sum()) == n and (rows == h).all()
    size_h, size_q = hx.stream_size(sh, n), hx.stream_size(sq, n)
    payload_bits_h = hx.mean_length(h, hcb)
    payload_bits_q = hx.mean_length(h, qcb)
    per_shard = hx.mean_length(h, hx.build_codebook(h, seen_only=True))
    H = hx.entropy(h)
    alg_bytes = {"huffman_encode": n + size_h, "huffman_decode": size_h + n,
                 "qlc_encode": n + size_q, "qlc_decode": size_q + n}
    ms_per_step = elapsed_ms / args.steps
    value = job_gbs(ws, 4 * n, ms_per_step)
    peak, peak_kind = hbm_peak()
    # Algorithmic bytes of each kernel launch: measure reads the batch and writes the sync rows;
    # pack reads the batch and writes the stream; decode reads the stream and writes the batch.
    index = 16 * ((n + 4095) // 4096)
    kernels = {  # kernel name -> [(algorithmic bytes, ms) per launch in a step]
        "k_measure": [(n + index, per_kernel_ms["huffman_measure"]),
                      (n + index, per_kernel_ms["qlc_measure"])],
        "k_pack": [(n + size_h, per_kernel_ms["huffman_pack"]),
                   (n + size_q, per_kernel_ms["qlc_pack"])],
        "k_decode<0>": [(size_h + n, per_kernel_ms["huffman_decode"])],
        "k_decode<1>": [(size_q + n, per_kernel_ms["qlc_decode"])],
    }
    # the dominant kernel: the largest share of the step
    kernel_name = max(kernels, key=lambda k: sum(ms for _, ms in kernels[k]))
    launches = kernels[kernel_name]
    bytes_per_launch = sum(b for b, _ in launches) / len(launches)
    ms_per_launch = sum(ms for _, ms in launches) / len(launches)
    achieved = bytes_per_launch / (ms_per_launch * 1e-3) / 1e9

    # end to end through the public API with host buffers: every step uploads its batch from
    # pinned memory, runs the four codec calls and downloads both streams (their sizes read from
    # the headers). Steps are pipelined over two buffer slots and three streams (upload, codec,
    # download), so one step's upload and the previous step's download overlap each other and
    # the codec calls, as a caller streaming batches through the library would run them.
    e2e = None
    if not args.no_e2e:
        x_pin = torch.from_numpy(x_host).pin_memory()
        out_h = torch.empty(bound, dtype=torch.uint8).pin_memory()
        out_q = torch.empty(bound, dtype=torch.uint8).pin_memory()
        st_host = torch.empty(1, dtype=torch.int32).pin_memory()
        hdr = torch.empty(2, 64, dtype=torch.uint8).pin_memory()
        s_in, s_out, s_hdr = (torch.cuda.Stream(dev) for _ in range(3))
        slots = [{"x": x, "sh": sh, "sq": sq},
                 {"x": torch.empty_like(x), "sh": torch.empty_like(sh),
                  "sq": torch.empty_like(sq)}]
        for sl in slots:
            sl["used"] = torch.cuda.Event()  # the codec calls are done with the slot's input
            sl["free"] = torch.cuda.Event()  # the slot's streams have been downloaded
            sl["used"].record(stream)
            sl["free"].record(s_out)

        def upload_and_code(sl):
            s_in.wait_event(sl["used"])
            with torch.cuda.stream(s_in):
                sl["x"].copy_(x_pin, non_blocking=True)
            up = torch.cuda.Event()
            up.record(s_in)
            stream.wait_event(up)
            stream.wait_event(sl["free"])
            done = []
            for t, kind, key in ((ht, hx.KIND_HUFFMAN, "sh"), (qt, hx.KIND_QLC, "sq")):
                hx.encode(t, sl["x"], out=sl[key], scratch=scratch, status=status, kind=kind)
                e = torch.cuda.Event()
                e.record(stream)
                done.append(e)
                hx.decode(t, sl[key], n, out=y, status=status, kind=kind)
            sl["used"].record(stream)
            return sl, done

        def download(sl, done):
            for j, (e, key) in enumerate(zip(done, ("sh", "sq"))):
                s_hdr.wait_event(e)
                with torch.cuda.stream(s_hdr):
                    hdr[j].copy_(sl[key][:64], non_blocking=True)
            got = torch.cuda.Event()
            got.record(s_hdr)
            got.synchronize()  # the host needs both stream sizes to copy them
            d2h = 0
            for j, (key, host) in enumerate((("sh", out_h), ("sq", out_q))):
                size = hx.stream_bytes(n, int(hdr[j][32:40].numpy().view(np.uint64)[0]))
                s_out.wait_event(done[j])
                with torch.cuda.stream(s_out):
                    host[:size].copy_(sl[key][:size], non_blocking=True)
                d2h += size + 64
            s_out.wait_event(sl["used"])
            with torch.cuda.stream(s_out):
                st_host.copy_(status, non_blocking=True)  # the step's status word
            sl["free"].record(s_out)
            return d2h + 4

        def run(k, start=None):
            if start is not None:
                s_in.wait_event(start)
            pending, d2h = None, 0
            for t in range(k):
                nxt = upload_and_code(slots[t % 2])
                if pending:
                    d2h = download(*pending)
                pending = nxt
            d2h = download(*pending)
            end = torch.cuda.Event()
            end.record(s_out)
            stream.wait_event(end)
            return d2h

        run(2)  # untimed: both slots once
        torch.cuda.synchronize(dev)
        k_e2e = max(3, min(args.steps, 10))
        if pg:
            pg.barrier()
        torch.cuda.synchronize(dev)
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        d2h = run(k_e2e, start=s0)
        s1.record(stream)
        torch.cuda.synchronize(dev)
        assert int(st_host.item()) == 0
        e2e_ms = max_over_ranks(s0.elapsed_time(s1) / k_e2e, pg, dev)
        e2e = {"value": job_gbs(ws, 4 * n, e2e_ms), "unit": "GB/s",
               "h2d_bytes_per_step": n, "d2h_bytes_per_step": d2h, "steps": k_e2e,
               "path": "pinned host batch -> H2D -> 4 codec calls -> D2H of both streams; steps "
                       "pipelined over 2 buffer slots on upload / codec / download streams"}

    shannonic = None
    if not args.no_shannonic:
        shannonic = shannonic_leg(dev, hx, torch, x, prior, h, scratch, y, status,
                                  max(3, min(args.steps, 10)))

    expgolomb = None
    if not args.no_expgolomb:
        expgolomb = expgolomb_leg(dev, hx, torch, x, h, scratch, y, status,
                                  max(3, min(args.steps, 10)))

    online = None
    if not args.no_online:
        online = online_leg(dev, hx, datagen, torch)

    cpu = None
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_leg(prior)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "u8", "data": "synthetic",
            "config": {"workload": WORKLOAD, "n_bytes_per_gpu": n, "chunk": 4096,
                       "substreams": 8, "lmax": 12,
                       "l2": "inputs larger than L2 (1 GiB per tensor vs 126 MB), no flush",
                       "parallelism": f"replicas x{ws} (independent batches, no collective)"},
            "ops": {o: {"ms": per_op_ms[o], "GB_per_s_uncompressed": n / (per_op_ms[o] * 1e-3) / 1e9,
                        "hbm_GB_per_s_algorithmic": alg_bytes[o] / (per_op_ms[o] * 1e-3) / 1e9,
                        "hbm_frac_algorithmic": alg_bytes[o] / (per_op_ms[o] * 1e-3) / 1e9 / peak}
                    for o in ops},
            "kernels_ms": per_kernel_ms,
            "bits_per_symbol": {"huffman_payload": payload_bits_h,
                                "huffman_framed": size_h * 8 / n,
                                "qlc_payload": payload_bits_q, "qlc_framed": size_q * 8 / n,
                                "per_shard_huffman": per_shard, "entropy": H,
                                "fixed_vs_per_shard": payload_bits_h / per_shard - 1,
                                "fixed_vs_entropy": payload_bits_h / H - 1},
            "host_codebook_build_us": {"huffman": (t1 - t0) * 1e6, "qlc": (t2 - t1) * 1e6},
            "roofline": {"bound": "hbm", "kernel": kernel_name,
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": achieved / peak,
                         "traffic": recorded_traffic(kernel_name),
                         "algorithmic_bytes_per_launch": bytes_per_launch,
                         "launches_per_step": len(launches), "ms_per_launch": ms_per_launch},
            "cpu_baseline": cpu,
            "e2e": e2e,
            "online": online,
            "shannonic": shannonic,
            "expgolomb": expgolomb,
            "gpu_launches": 6 * args.steps,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
