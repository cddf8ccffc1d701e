"""Fixed-codebook lossless entropy coding of 8-bit tensor symbols (e4m3 / INT8 bytes) on B200.

Single-stage Huffman ("Single-Stage Huffman Encoder for ML Compression"): a length-limited
canonical codebook fixed from the summed histograms of earlier batches; the stream carries only
the codebook's hash. Quad Length Codes ("Quad Length Codes for Lossless Compression of e4m3"):
3-bit area prefix + fixed-width in-area index. The work runs in libhx.so (include/hx.h); the
module ``hx`` is its Python binding.
"""
from . import hx  # noqa: F401
from .hx import (  # noqa: F401
    Codebook, HxError, build_codebook, qlc_build, histogram, encode, decode, encode_bound,
    payload_offset, scratch_bytes, stream_size, KIND_HUFFMAN, KIND_QLC,
)

__all__ = ["hx", "Codebook", "HxError", "build_codebook", "qlc_build", "histogram", "encode",
           "decode", "encode_bound", "payload_offset", "scratch_bytes", "stream_size",
           "KIND_HUFFMAN", "KIND_QLC"]
