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
SPEC_HBM_GBS = 8000.0  # the B200's HBM3e specification (DGX figure)
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
    p.add_argument("--no-configs", action="store_true")
    p.add_argument("--no-cfg5", action="store_true")
    p.add_argument("--no-collective", action="store_true")
    p.add_argument("--quick", action="store_true",
                   help="the headline step only (no e2e, legs, configs or CPU baseline)")
    a = p.parse_args()
    if a.quick:
        for k in ("no_e2e", "no_cpu_baseline", "no_online", "no_shannonic", "no_expgolomb",
                  "no_configs", "no_cfg5", "no_collective"):
            setattr(a, k, True)
    return a


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
def _oracle_slices(x, threads):
    """Chunk-aligned slices of x, one per thread."""
    per = -(-x.size // threads)
    per = -(-per // 4096) * 4096
    return [x[i:i + per] for i in range(0, x.size, per)]


def oracle_codec_pass(books, x, threads: int) -> float:
    """The oracle as it stands, encoding and decoding x with each codebook: x is cut into
    chunk-aligned slices, each coded as its own stream on its own thread (ctypes releases the
    interpreter lock). Returns the seconds taken."""
    import oracle
    from concurrent.futures import ThreadPoolExecutor
    slices = _oracle_slices(x, threads)

    def one(sl):
        for cb in books:
            st, s = oracle.encode(cb, sl)
            assert st == 0
            st, y = oracle.decode(cb, s, sl.size)
            assert st == 0 and (y == sl).all()

    t0 = time.perf_counter()
    if threads == 1:
        for sl in slices:
            one(sl)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(one, slices))
    return time.perf_counter() - t0


def cpu_reference(args, rank, ws):
    """The oracle on a bounded sample of the workload, on all host cores (rank 0 only)."""
    if rank != 0:
        return 0
    import oracle
    import datagen
    cores = os.cpu_count() or 1
    sample = 4 << 20
    counts = sum(oracle.histogram(b) for b in datagen.prior_batches(4))
    books = (oracle.huffman_codebook(counts), oracle.qlc_codebook(counts))
    x = datagen.data(4, n=sample)
    for _ in range(args.warmup):
        oracle_codec_pass(books, x, cores)
    dt = sum(oracle_codec_pass(books, x, cores) for _ in range(args.steps))
    value = 4 * sample * args.steps / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u8",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "sample_bytes_per_step": sample},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": f"first {sample >> 20} MiB of the 1 GiB batch per step, in "
                                   f"{cores} chunk-aligned slices on {cores} threads: Huffman and "
                                   "QLC encode + decode, bit-serial C++"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def cpu_baseline_leg(counts):
    """Time the oracle as it stands on a slice of the workload: one thread on 16 MiB, and all host
    cores on 64 MiB in chunk-aligned slices (~10-30 s in all)."""
    import oracle
    import datagen
    cores = os.cpu_count() or 1
    books = (oracle.huffman_codebook(counts), oracle.qlc_codebook(counts))
    x1 = datagen.data(4, n=16 << 20)
    dt1 = oracle_codec_pass(books, x1, 1)
    xa = datagen.data(4, n=64 << 20)
    dta = oracle_codec_pass(books, xa, cores)
    return {"value": 4 * xa.size / dta / 1e9, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"first 64 MiB of the batch through the same 4 codec calls, cut into {cores} "
                      f"chunk-aligned slices on {cores} threads ({dta:.1f} s, bit-serial C++)",
            "single_thread": {"value": 4 * x1.size / dt1 / 1e9, "unit": "GB/s", "cores": 1,
                              "sample": f"first 16 MiB, one thread ({dt1:.1f} s)"}}


def roofline_entry(kernel, launches, peak, peak_kind):
    """HBM roofline of one kernel from its launches in a step: [(algorithmic bytes, ms)]."""
    b = sum(x for x, _ in launches) / len(launches)
    ms = sum(t for _, t in launches) / len(launches)
    achieved = b / (ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": achieved, "peak": peak,
            "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
            "frac_spec": achieved / SPEC_HBM_GBS, "peak_spec": SPEC_HBM_GBS,
            "algorithmic_bytes_per_launch": b, "launches_per_step": len(launches),
            "ms_per_launch": ms}


def graph_ms(torch, fn, reps: int) -> float:
    """Device time of one fn() call: reps calls captured in a CUDA graph, replayed (no launch
    gaps; for inputs too small to hide the host's launch time)."""
    fn()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(reps):
            fn()
    g.replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    g.replay()
    b.record()
    torch.cuda.synchronize()
    del g
    return a.elapsed_time(b) / reps


def config_numbers(dev, hx, torch, x, prior, peak, kinds=("huffman", "qlc"), reps=20, graph=False):
    """Encode and decode of one input with the fixed codebooks from `prior`: time per call
    (inputs resident), GB/s, roofline fraction, bits per symbol against per-shard Huffman and
    the entropy. Checks the round trip."""
    n = x.numel()
    h = np.bincount(x.cpu().numpy(), minlength=256).astype(np.uint64)
    per_shard = hx.mean_length(h, hx.build_codebook(h, seen_only=True))
    H = hx.entropy(h)
    out = torch.empty(hx.encode_bound(n), dtype=torch.uint8, device=dev)
    scratch = torch.empty(hx.scratch_bytes(n), dtype=torch.uint8, device=dev)
    y = torch.empty(n, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    res = {"n": n, "entropy": H, "per_shard_huffman": per_shard}
    for name in kinds:
        cb = hx.build_codebook(prior) if name == "huffman" else hx.qlc_build(prior)
        t = cb.upload(dev)
        enc = lambda: hx.encode(t, x, out=out, scratch=scratch, status=status, kind=cb.kind)
        dec = lambda: hx.decode(t, out, n, out=y, status=status, kind=cb.kind)
        enc()
        dec()
        torch.cuda.synchronize()
        assert int(status.item()) == 0 and torch.equal(x, y)
        size = hx.stream_size(out, n)
        r = {}
        for op, fn in (("encode", enc), ("decode", dec)):
            if graph:
                ms = graph_ms(torch, fn, reps)
            else:
                for _ in range(3):
                    fn()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                for _ in range(reps):
                    fn()
                b.record()
                torch.cuda.synchronize()
                ms = a.elapsed_time(b) / reps
            alg = (n + size) / (ms * 1e-3) / 1e9
            r[op] = {"ms": ms, "GB_per_s_uncompressed": n / (ms * 1e-3) / 1e9,
                     "hbm_frac_algorithmic": alg / peak, "hbm_frac_spec": alg / SPEC_HBM_GBS}
        assert int(status.item()) == 0
        bits = hx.mean_length(h, cb)
        r["bits_per_symbol"] = {"payload": bits, "framed": size * 8 / n,
                                "vs_per_shard": bits / per_shard - 1, "vs_entropy": bits / H - 1}
        res[name] = r
    return res


def configs_leg(dev, hx, datagen, torch, peak):
    """cfg 1 (1 MiB, timed through CUDA graphs of 200 calls), cfg 2 (256 MiB FFN mixture, codebook
    from 8 prior 256 MiB batches) and cfg 3 (64 MiB INT8 weights, per-tensor codebook)."""
    out = {}
    for cfg in (1, 2, 3):
        prior = sum(np.bincount(b, minlength=256) for b in datagen.prior_batches(cfg))
        x = torch.from_numpy(datagen.data(cfg)).to(dev)
        out[f"cfg{cfg}"] = config_numbers(dev, hx, torch, x, prior.astype(np.uint64), peak,
                                          reps=200 if cfg == 1 else 20, graph=cfg == 1)
        del x
    return out


def cfg5_leg(dev, hx, datagen, torch):
    """cfg 5: 64 tensors of 64 MiB (16 layers x 4 shards, e4m3 and INT8, laws and scales per
    layer); each shard coded with its layer's fixed Huffman codebook (4 prior batches). Per
    shard: fixed-codebook bits per symbol against a per-shard Huffman code and the entropy (the
    drift); the whole batch's encode and decode time on the device (inputs resident)."""
    rows = []
    enc_ms = dec_ms = 0.0
    total = 0
    out = torch.empty(hx.encode_bound(datagen.CFG5_TENSOR), dtype=torch.uint8, device=dev)
    scratch = torch.empty(hx.scratch_bytes(datagen.CFG5_TENSOR), dtype=torch.uint8, device=dev)
    y = torch.empty(datagen.CFG5_TENSOR, dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    for layer in range(16):
        prior = sum(np.bincount(b, minlength=256) for b in datagen.prior_batches(5, layer))
        cb = hx.build_codebook(prior.astype(np.uint64))
        t = cb.upload(dev)
        law = datagen.cfg5_layer(layer)
        for j in range(datagen.CFG5_SHARDS):
            shard = layer * datagen.CFG5_SHARDS + j
            xh = datagen.data(5, shard=shard)
            x = torch.from_numpy(xh).to(dev)
            n = x.numel()
            h = np.bincount(xh, minlength=256).astype(np.uint64)
            ms = {}
            for op, fn in (("enc", lambda: hx.encode(t, x, out=out, scratch=scratch,
                                                      status=status)),
                           ("dec", lambda: hx.decode(t, out, n, out=y, status=status))):
                fn()
                a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record()
                fn()
                b.record()
                torch.cuda.synchronize()
                ms[op] = a.elapsed_time(b)
            assert int(status.item()) == 0 and torch.equal(x, y)
            enc_ms += ms["enc"]
            dec_ms += ms["dec"]
            total += n
            fixed = hx.mean_length(h, cb)
            own = hx.mean_length(h, hx.build_codebook(h, seen_only=True))
            rows.append({"shard": shard, "layer": layer, "dtype": law["dtype"],
                         "family": law["family"], "scale": round(law["scale"], 4),
                         "fixed_bits": round(fixed, 4), "per_shard_bits": round(own, 4),
                         "entropy": round(hx.entropy(h), 4),
                         "drift": round(fixed / own - 1, 5),
                         "framed_bits": round(hx.stream_size(out, n) * 8 / n, 4)})
    drifts = [r["drift"] for r in rows]
    return {"shards": len(rows), "bytes": total,
            "encode_GB_per_s": total / (enc_ms * 1e-3) / 1e9,
            "decode_GB_per_s": total / (dec_ms * 1e-3) / 1e9,
            "drift_mean": float(np.mean(drifts)), "drift_max": float(np.max(drifts)),
            "drift_min": float(np.min(drifts)),
            "fixed_bits_mean": float(np.mean([r["fixed_bits"] for r in rows])),
            "per_shard_bits_mean": float(np.mean([r["per_shard_bits"] for r in rows])),
            "rows": rows}


def collective_leg(dev, hx, datagen, torch, tables, prior):
    """The compressed all-gather on one rank (NCCL, a process group of one): ms per GiB through
    compressed_all_gather with 1 and 4 parts, against Huffman encode + decode alone. No figure
    exists for 2 or more GPUs (every run here has one)."""
    import datetime
    import torch.distributed as dist
    from lossless_entropy_coding_fixed_b200 import collective
    n = 1 << 28
    x = torch.from_numpy(datagen.data(4, n=n)).to(dev)
    own = not dist.is_initialized()
    if own:
        store = dist.TCPStore("127.0.0.1", 0, 1, True, timeout=datetime.timedelta(seconds=60))
        dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=dev,
                                timeout=datetime.timedelta(seconds=60))
    try:
        res = {"n": n}
        for parts in (1, 4):
            out, sent = collective.compressed_all_gather(x, tables, parts=parts)
            torch.cuda.synchronize()
            assert torch.equal(out, x)
            t0 = time.perf_counter()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(5):
                collective.compressed_all_gather(x, tables, parts=parts)
            b.record()
            torch.cuda.synchronize()
            res[f"parts{parts}_ms_per_GiB"] = a.elapsed_time(b) / 5 * (1 << 30) / n
            res[f"parts{parts}_wall_ms_per_GiB"] = (time.perf_counter() - t0) / 5 * 1e3 * (1 << 30) / n
        st = hx.new_status(dev)
        out = torch.empty(hx.encode_bound(n), dtype=torch.uint8, device=dev)
        y = torch.empty_like(x)
        scratch = torch.empty(hx.scratch_bytes(n), dtype=torch.uint8, device=dev)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(5):
            hx.encode(tables, x, out=out, scratch=scratch, status=st)
            hx.decode(tables, out, n, out=y, status=st)
        b.record()
        torch.cuda.synchronize()
        res["codec_alone_ms_per_GiB"] = a.elapsed_time(b) / 5 * (1 << 30) / n
        res["note"] = "one rank: the exchange is a local NCCL all-gather; no NVLink figure"
        return res
    finally:
        if own:
            dist.destroy_process_group()


E2E_SLOTS = 3  # buffer slots of the end-to-end pipeline (2: 50.6 GB/s, 3: 55.6, 4: 55.5)


def e2e_leg(args, dev, hx, torch, pg, ws, x_host, ht, qt, n, bound, scratch, status):
    """End to end through the public API with host buffers, both directions of a link: every step
    uploads its batch from pinned memory, encodes it with both codebooks and downloads the two
    streams (sender), then uploads the two streams, decodes them and downloads both decoded
    batches (receiver). Steps are pipelined over E2E_SLOTS buffer slots. Each kind of transfer
    has its own copy stream (batch up, streams down, streams up, decoded batches down) and encode
    and decode their own compute streams, so one step's transfers overlap the next step's;
    events order every reuse of a buffer. Every step's copies are inside the timed region."""
    x_pin = torch.from_numpy(x_host).pin_memory()
    host_y = [torch.empty(n, dtype=torch.uint8).pin_memory() for _ in range(2)]
    st_host = torch.empty(1, dtype=torch.int32).pin_memory()
    stream = torch.cuda.current_stream(dev)
    up_x, down_st, up_st, down_y, s_hdr, s_enc, s_dec = (torch.cuda.Stream(dev) for _ in range(7))
    books = ((ht, hx.KIND_HUFFMAN), (qt, hx.KIND_QLC))
    slots = []
    for _ in range(E2E_SLOTS):
        sl = {"x": torch.empty(n, dtype=torch.uint8, device=dev),
              "st": [torch.empty(bound, dtype=torch.uint8, device=dev) for _ in range(2)],
              "rx": [torch.empty(bound, dtype=torch.uint8, device=dev) for _ in range(2)],
              "y": [torch.empty(n, dtype=torch.uint8, device=dev) for _ in range(2)],
              "host_st": [torch.empty(bound, dtype=torch.uint8).pin_memory() for _ in range(2)],
              "hdr": torch.empty(2, 64, dtype=torch.uint8).pin_memory()}
        # the slot's last encode, header read, stream download, stream upload, decode and
        # decoded download
        for name, s_ in (("enc", s_enc), ("hdr_ev", s_hdr), ("stdown", down_st),
                         ("stup", up_st), ("dec", s_dec), ("ydown", down_y)):
            sl[name] = torch.cuda.Event()
            sl[name].record(s_)
        slots.append(sl)
    counted = {"h2d": 0, "d2h": 0}

    def sender(sl):
        up_x.wait_event(sl["enc"])  # the slot's last encode has read its batch
        with torch.cuda.stream(up_x):
            sl["x"].copy_(x_pin, non_blocking=True)
        up = torch.cuda.Event()
        up.record(up_x)
        s_enc.wait_event(up)
        s_enc.wait_event(sl["stdown"])  # the slot's last streams are downloaded
        with torch.cuda.stream(s_enc):
            for j, (t, kind) in enumerate(books):
                hx.encode(t, sl["x"], out=sl["st"][j], scratch=scratch, status=status, kind=kind)
        sl["enc"].record(s_enc)
        s_hdr.wait_event(sl["enc"])
        with torch.cuda.stream(s_hdr):
            for j in range(2):
                sl["hdr"][j].copy_(sl["st"][j][:64], non_blocking=True)
        sl["hdr_ev"].record(s_hdr)
        return n

    def link(sl):
        # the streams' sizes (their headers), then stream bytes down and back up
        sl["hdr_ev"].synchronize()
        sizes = [hx.stream_bytes(n, int(sl["hdr"][j][32:40].numpy().view(np.uint64)[0]))
                 for j in range(2)]
        down_st.wait_event(sl["enc"])
        down_st.wait_event(sl["stup"])  # the slot's host stream buffers were read
        with torch.cuda.stream(down_st):
            for j in range(2):
                sl["host_st"][j][:sizes[j]].copy_(sl["st"][j][:sizes[j]], non_blocking=True)
        sl["stdown"].record(down_st)
        up_st.wait_event(sl["stdown"])
        up_st.wait_event(sl["dec"])  # the slot's last decode has read its received streams
        with torch.cuda.stream(up_st):
            for j in range(2):
                sl["rx"][j][:sizes[j]].copy_(sl["host_st"][j][:sizes[j]], non_blocking=True)
        sl["stup"].record(up_st)
        s_dec.wait_event(sl["stup"])
        s_dec.wait_event(sl["ydown"])  # the slot's last decoded batches are downloaded
        with torch.cuda.stream(s_dec):
            for j, (t, kind) in enumerate(books):
                hx.decode(t, sl["rx"][j], n, out=sl["y"][j], status=status, kind=kind,
                          nbytes=sizes[j])
        sl["dec"].record(s_dec)
        down_y.wait_event(sl["dec"])
        with torch.cuda.stream(down_y):
            for j in range(2):
                host_y[j].copy_(sl["y"][j], non_blocking=True)
            st_host.copy_(status, non_blocking=True)
        sl["ydown"].record(down_y)
        # (bytes up, bytes down): the streams up; headers, streams, decoded batches, status down
        return sum(sizes), 64 * 2 + sum(sizes) + 2 * n + 4

    def run(k):
        counted["h2d"] = counted["d2h"] = 0
        for s_ in (up_x, down_st, up_st, down_y, s_hdr, s_enc, s_dec):
            s_.wait_stream(stream)
        pending = None
        for t in range(k):
            sl = slots[t % E2E_SLOTS]
            counted["h2d"] += sender(sl)
            if pending is not None:
                up, down = link(pending)
                counted["h2d"] += up
                counted["d2h"] += down
            pending = sl
        up, down = link(pending)
        counted["h2d"] += up
        counted["d2h"] += down
        for s_ in (up_x, down_st, up_st, down_y, s_hdr, s_enc, s_dec):
            stream.wait_stream(s_)

    run(E2E_SLOTS)  # untimed: every slot once
    torch.cuda.synchronize(dev)
    k = max(3, min(args.steps, 10))
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s0.record(stream)
    run(k)
    s1.record(stream)
    torch.cuda.synchronize(dev)
    assert int(st_host.item()) == 0
    assert torch.equal(host_y[0], x_pin) and torch.equal(host_y[1], x_pin)
    e2e_ms = max_over_ranks(s0.elapsed_time(s1) / k, pg, dev)
    return {"value": job_gbs(ws, 4 * n, e2e_ms), "unit": "GB/s",
            "h2d_bytes_per_step": counted["h2d"] // k, "d2h_bytes_per_step": counted["d2h"] // k,
            "steps": k,
            "path": "pinned host batch -> H2D -> Huffman and QLC encode -> D2H of both streams "
                    "-> H2D of both streams -> decode -> D2H of both decoded batches; steps "
                    f"pipelined over {E2E_SLOTS} buffer slots, each transfer kind on its own "
                    "copy stream, encode and decode on their own streams"}


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
    ev = {o: [] for o in ops}

    def step(record: bool, row: int = 0):
        marks = [torch.cuda.Event(enable_timing=True) for _ in range(5)] if record else None
        mark = (lambda i: marks[i].record(stream)) if record else (lambda i: None)
        mark(0)
        hx.encode(ht, x, out=sh, scratch=scratch, hist=hist[row], status=status,
                  kind=hx.KIND_HUFFMAN)
        mark(1)
        hx.decode(ht, sh, n, out=y, status=status, kind=hx.KIND_HUFFMAN)
        mark(2)
        hx.encode(qt, x, out=sq, scratch=scratch, status=status, kind=hx.KIND_QLC)
        mark(3)
        hx.decode(qt, sq, n, out=y, status=status, kind=hx.KIND_QLC)
        mark(4)
        if record:
            for i, o in enumerate(ops):
                ev[o].append((marks[i], marks[i + 1]))

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
    per_op_ms = {o: sum(a.elapsed_time(b) for a, b in ev[o]) / args.steps for o in ops}

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
    # Each op is one launch of the library's kernel (an encode also clears its look-back words
    # first, inside the op's time): k_encode reads the batch and writes the stream, k_decode reads
    # the stream and writes the batch.
    kernels = {"k_encode": ["huffman_encode", "qlc_encode"],
               "k_decode": ["huffman_decode", "qlc_decode"]}
    roof = {k: roofline_entry(k, [(alg_bytes[o], per_op_ms[o]) for o in v], peak, peak_kind)
            for k, v in kernels.items()}
    # the dominant kernel: the largest share of the step
    kernel_name = max(roof, key=lambda k: roof[k]["ms_per_launch"] * roof[k]["launches_per_step"])

    # the histogram on its own (the frequency analysis that defines the next codebook), over the
    # same batch: device time per call, inputs resident
    hc = torch.zeros(256, dtype=torch.int32, device=dev)
    for _ in range(3):
        hx.histogram(x, hc)
    a_, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a_.record(stream)
    for _ in range(10):
        hx.histogram(x, hc)
    b_.record(stream)
    torch.cuda.synchronize(dev)
    hist_ms = a_.elapsed_time(b_) / 10
    assert (hc.cpu().numpy().astype(np.uint64) == h * 13).all()
    histogram = {"ms": hist_ms, "GB_per_s": n / (hist_ms * 1e-3) / 1e9,
                 "hbm_frac": n / (hist_ms * 1e-3) / 1e9 / peak}

    e2e = None
    if not args.no_e2e:
        e2e = e2e_leg(args, dev, hx, torch, pg, ws, x_host, ht, qt, n, bound, scratch, status)

    # the side legs run on one GPU only: their figures are per-GPU and rank 0 alone reports them,
    # and cfg5 alone builds 8 GiB of input on the host
    side = ws == 1
    shannonic = None
    if side and not args.no_shannonic:
        shannonic = shannonic_leg(dev, hx, torch, x, prior, h, scratch, y, status,
                                  max(3, min(args.steps, 10)))

    expgolomb = None
    if side and not args.no_expgolomb:
        expgolomb = expgolomb_leg(dev, hx, torch, x, h, scratch, y, status,
                                  max(3, min(args.steps, 10)))
    del x, y, sh, sq, scratch
    torch.cuda.empty_cache()

    online = None
    if side and not args.no_online:
        online = online_leg(dev, hx, datagen, torch)

    configs = None
    if side and not args.no_configs:
        configs = configs_leg(dev, hx, datagen, torch, peak)

    cfg5 = None
    if side and not args.no_cfg5:
        cfg5 = cfg5_leg(dev, hx, datagen, torch)

    collective = None
    if side and not args.no_collective:
        collective = collective_leg(dev, hx, datagen, torch, ht, prior)

    cpu = None
    if rank == 0 and side and not args.no_cpu_baseline:
        cpu = cpu_baseline_leg(prior)

    if rank == 0:
        main_roof = dict(roof[kernel_name])
        main_roof["traffic"] = recorded_traffic(kernel_name)
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
                        "hbm_frac_algorithmic": alg_bytes[o] / (per_op_ms[o] * 1e-3) / 1e9 / peak,
                        "hbm_frac_spec": alg_bytes[o] / (per_op_ms[o] * 1e-3) / 1e9 / SPEC_HBM_GBS}
                    for o in ops},
            "bits_per_symbol": {"huffman_payload": payload_bits_h,
                                "huffman_framed": size_h * 8 / n,
                                "qlc_payload": payload_bits_q, "qlc_framed": size_q * 8 / n,
                                "per_shard_huffman": per_shard, "entropy": H,
                                "fixed_vs_per_shard": payload_bits_h / per_shard - 1,
                                "fixed_vs_entropy": payload_bits_h / H - 1},
            "host_codebook_build_us": {"huffman": (t1 - t0) * 1e6, "qlc": (t2 - t1) * 1e6},
            "roofline": main_roof,
            "roofline_kernels": {k: dict(v, traffic=recorded_traffic(k)) for k, v in roof.items()},
            "histogram": histogram,
            "cpu_baseline": cpu,
            "e2e": e2e,
            "configs": configs,
            "cfg5_drift": cfg5,
            "collective": collective,
            "online": online,
            "shannonic": shannonic,
            "expgolomb": expgolomb,
            # the library's kernels in the timed region: per step two k_encode, two k_decode
            "gpu_launches": 4 * args.steps,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if pg:
        pg.barrier()
        pg.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
