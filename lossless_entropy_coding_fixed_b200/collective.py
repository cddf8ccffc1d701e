"""Compressed all-gather: the pages' use of the coder ("Quad Length Codes ...", abstract:
collective operations in LLM training and serving are bound by network bandwidth, and lossless
compression relieves them; "Single-Stage Huffman Encoder ...", abstract: sender and receiver
share a fixed codebook, so only coded data travels).

Every rank encodes its shard with the shared table block, the ranks exchange stream sizes and
then the streams themselves (one NCCL all-gather of buffers padded to the largest stream), and
every rank decodes every stream. With several parts per shard the three stages overlap: one
part's exchange runs while the next part is encoded and the previous one decoded. The coding
runs in libhx.so; the exchange is torch.distributed (NCCL on GPUs).
"""
from __future__ import annotations

from dataclasses import dataclass

from . import hx

HEADER_TOTAL_WORDS = slice(32, 40)  # u64 total_words in the stream header


@dataclass
class Codec:
    """The four calls the exchange needs; the default is the library. (Tests on CPU ranks pass a
    stand-in, since the coder itself needs a GPU.)"""
    kind: int = hx.KIND_HUFFMAN

    def bound(self, n: int) -> int:
        return hx.encode_bound(n, self.kind)

    def encode(self, tables, x, out):
        hx.encode(tables, x, out=out, kind=self.kind)

    def decode(self, tables, stream, n: int, out):
        hx.decode(tables, stream, n, out=out, kind=self.kind)

    def stream_bytes(self, n: int, total_words: int) -> int:
        return hx.stream_bytes(n, total_words)


def _round16(v: int) -> int:
    return (v + 15) // 16 * 16


def part_bounds(n: int, parts: int) -> list[tuple[int, int]]:
    """[lo, hi) byte ranges of at most `parts` contiguous parts of n bytes, each a whole number of
    chunks (HX_CHUNK symbols) but the last."""
    chunks = -(-n // hx.CHUNK)
    if chunks == 0:
        return [(0, 0)]
    parts = max(1, min(parts, chunks))
    per = -(-chunks // parts) * hx.CHUNK
    return [(lo, min(n, lo + per)) for lo in range(0, n, per)]


def _host_ints(tensors, work, side):
    """The values of one-element int64 tensors that an async collective fills, on the host. On a
    GPU a side stream waits for the collective and copies them, so the host does not wait for
    the codec work queued on the current stream after it."""
    import torch
    if side is None:
        work.wait()
        return [int(t.item()) for t in tensors]
    host = torch.empty(len(tensors), dtype=torch.int64, pin_memory=True)
    with torch.cuda.stream(side):
        work.wait()
        for i, t in enumerate(tensors):
            t.record_stream(side)
            host[i:i + 1].copy_(t, non_blocking=True)
        done = torch.cuda.Event()
        done.record(side)
    done.synchronize()
    return host.tolist()


def merge_streams(streams, ns):
    """One stream of sum(ns) bytes from the streams of consecutive pieces of it, each piece but the
    last a whole number of chunks. The headers must agree on version, kind, lmax and codebook
    hash; the word offsets are rebased by the payload words before each piece, and the sync rows
    and payload words are concatenated. The result is the stream the encoder writes for the whole
    input (its chunks code the same bytes from the same word boundaries)."""
    import torch

    if not streams or len(streams) != len(ns):
        raise ValueError("merge_streams needs one size per stream")
    if any(n % hx.CHUNK for n in ns[:-1]):
        raise ValueError("every piece but the last must be a whole number of chunks")
    if sum(ns) >= 1 << 32:
        raise ValueError("a stream codes fewer than 2^32 bytes; the merged input is larger")
    head = streams[0][:64]
    for st in streams[1:]:
        if not (torch.equal(st[:8], head[:8]) and torch.equal(st[40:48], head[40:48])):
            raise ValueError("the streams were not coded with the same codebook")
    for st, n in zip(streams, ns):
        hn, hc = (int(v) for v in st[16:32].view(torch.int64).tolist())
        if hn != n or hc != -(-n // hx.CHUNK):
            raise ValueError(f"a stream's header codes {hn} bytes, not the {n} given for it")
    totals = [int(st[32:40].view(torch.int64)[0]) for st in streams]
    chunks = [-(-n // hx.CHUNK) for n in ns]
    n_all, words = sum(ns), sum(totals)
    if words >= 1 << 32:
        raise ValueError("the merged payload exceeds 2^32 words")
    out = torch.zeros(hx.stream_bytes(n_all, words), dtype=torch.uint8, device=head.device)
    out[:64] = head
    out[16:40] = torch.tensor([n_all, sum(chunks), words], dtype=torch.int64).view(torch.uint8)
    woff = out[64:64 + 4 * (sum(chunks) + 1)].view(torch.int32)
    S, P = hx.sync_offset(n_all), hx.payload_offset(n_all)
    c0 = w0 = 0
    for st, n, nc, tw in zip(streams, ns, chunks, totals):
        own = st[64:64 + 4 * nc].view(torch.int32).to(torch.int64) & 0xFFFFFFFF
        woff[c0:c0 + nc] = (own + w0).to(torch.int32)  # u32 bits, below 2^32
        s_i, p_i = hx.sync_offset(n), hx.payload_offset(n)
        out[S + 16 * c0:S + 16 * (c0 + nc)] = st[s_i:s_i + 16 * nc]
        out[P + 4 * w0:P + 4 * (w0 + tw)] = st[p_i:p_i + 4 * tw]
        c0, w0 = c0 + nc, w0 + tw
    woff[c0:c0 + 1] = torch.tensor([words], dtype=torch.int64).to(torch.int32)
    return out


def compressed_all_gather(x, tables, group=None, codec: Codec | None = None, parts: int = 1,
                          decode: bool = True):
    """All-gather of equal-size uint8 shards through the coder.

    x: this rank's shard (contiguous uint8 tensor, the same size on every rank); tables: the
    shared table block (device uint8 tensor). Returns (gathered, sizes): gathered holds
    world_size * n bytes in rank order, sizes the stream bytes each rank sent. With
    decode=False, gathered is instead the one stream of all ranks' bytes in rank order
    (merge_streams of the received streams; with 2 or more ranks n must be a whole number of
    chunks), for a receiver that keeps the data coded.

    With parts > 1 the shard is coded as that many chunk-aligned parts, each its own stream, in a
    three-stage pipeline: part p is encoded while part p - 1 is exchanged and part p - 2 decoded.
    A part's exchange is sized by the ranks' stream sizes (one small all-gather, read on the host)
    and moves every stream padded to the longest. Every rank takes the same collective steps."""
    import torch
    import torch.distributed as dist

    codec = codec or Codec()
    world = dist.get_world_size(group)
    n = x.numel()
    dev = x.device
    # the shard sizes first: every rank sees them all, so unequal shards stop every rank here
    ns = [torch.empty(1, dtype=torch.int64, device=dev) for _ in range(world)]
    dist.all_gather(ns, torch.tensor([n], dtype=torch.int64, device=dev), group=group)
    if any(int(v.item()) != n for v in ns):
        raise ValueError("compressed_all_gather needs the same shard size on every rank")
    if not decode and world > 1 and n % hx.CHUNK:
        raise ValueError("a merged stream needs shards of whole chunks")
    if not decode and world * n >= 1 << 32:
        raise ValueError("a merged stream codes fewer than 2^32 bytes; world * n is larger")
    bounds = part_bounds(n, parts)
    # decoded shards go to rows of a multiple of 16 bytes (the decoder's output alignment)
    row = _round16(n)
    rows = torch.empty(world * row if decode else 0, dtype=torch.uint8, device=dev)
    sent = [0] * world
    side = torch.cuda.Stream(dev) if x.is_cuda else None
    live = {}

    def code(p):  # encode part p, then start the exchange of its stream sizes
        lo, hi = bounds[p]
        stream = torch.empty(_round16(codec.bound(hi - lo)), dtype=torch.uint8, device=dev)
        codec.encode(tables, x[lo:hi], stream)
        total = stream[HEADER_TOTAL_WORDS].view(torch.int64).clone()
        sizes = [torch.empty(1, dtype=torch.int64, device=dev) for _ in range(world)]
        live[p] = {"stream": stream, "sizes": sizes,
                   "work": dist.all_gather(sizes, total, group=group, async_op=True)}

    def send(p):  # start the exchange of part p's streams, padded to the longest
        st, (lo, hi) = live[p], bounds[p]
        totals = _host_ints(st["sizes"], st["work"], side)
        st["bytes"] = [codec.stream_bytes(hi - lo, t) for t in totals]
        span = _round16(max(st["bytes"]))
        st["recv"] = [torch.empty(span, dtype=torch.uint8, device=dev) for _ in range(world)]
        st["work"] = dist.all_gather(st["recv"], st["stream"][:span], group=group,
                                     async_op=True)

    kept = {}

    def unpack(p):  # decode every rank's stream of part p into its place (or keep it)
        st, (lo, hi) = live.pop(p), bounds[p]
        st["work"].wait()
        for r in range(world):
            if decode:
                codec.decode(tables, st["recv"][r][:st["bytes"][r]], hi - lo,
                             rows[r * row + lo:r * row + hi])
            else:
                kept[(r, p)] = st["recv"][r][:st["bytes"][r]]
            sent[r] += st["bytes"][r]

    for p in range(len(bounds) + 2):
        if p < len(bounds):
            code(p)
        if 0 <= p - 1 < len(bounds):
            send(p - 1)
        if 0 <= p - 2 < len(bounds):
            unpack(p - 2)
    if not decode:
        order = [(r, p) for r in range(world) for p in range(len(bounds))]
        return merge_streams([kept[k] for k in order],
                             [bounds[p][1] - bounds[p][0] for _, p in order]), sent
    out = rows if row == n else rows.view(world, row)[:, :n].reshape(-1)
    return out, sent
