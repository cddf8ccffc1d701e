"""Compressed all-gather: the pages' use of the coder ("Quad Length Codes ...", abstract:
collective operations in LLM training and serving are bound by network bandwidth, and lossless
compression relieves them; "Single-Stage Huffman Encoder ...", abstract: sender and receiver
share a fixed codebook, so only coded data travels).

Every rank encodes its shard with the shared table block, the ranks exchange stream sizes and
then the streams themselves (one NCCL all-gather of buffers padded to the largest stream), and
every rank decodes every stream. The coding runs in libhx.so; the exchange is torch.distributed
(NCCL on GPUs).
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


def compressed_all_gather(x, tables, group=None, codec: Codec | None = None):
    """All-gather of equal-size uint8 shards through the coder.

    x: this rank's shard (contiguous uint8 tensor, the same size on every rank); tables: the
    shared table block (device uint8 tensor). Returns (gathered, sizes): gathered holds
    world_size * n bytes in rank order, sizes the stream bytes each rank sent. One host sync
    reads the stream sizes, to size the exchange."""
    import torch
    import torch.distributed as dist

    codec = codec or Codec()
    world = dist.get_world_size(group)
    n = x.numel()
    stream = torch.empty(_round16(codec.bound(n)), dtype=torch.uint8, device=x.device)
    codec.encode(tables, x, stream)
    # the stream size, from its header's total_words (on the device)
    total = stream[HEADER_TOTAL_WORDS].view(torch.int64)
    mine = torch.stack([torch.tensor(n, device=x.device, dtype=torch.int64), total[0]])
    sizes = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(sizes, mine, group=group)
    host = [tuple(int(v) for v in s.tolist()) for s in sizes]
    if any(hn != n for hn, _ in host):
        raise ValueError("compressed_all_gather needs the same shard size on every rank")
    nbytes = [codec.stream_bytes(n, tw) for _, tw in host]
    span = _round16(max(nbytes))  # every rank sends the same length: the longest stream
    recv = [torch.empty(span, dtype=torch.uint8, device=x.device) for _ in range(world)]
    dist.all_gather(recv, stream[:span], group=group)
    out = torch.empty(world * n, dtype=torch.uint8, device=x.device)
    for r in range(world):
        codec.decode(tables, recv[r][:nbytes[r]], n, out[r * n:(r + 1) * n])
    return out, nbytes
