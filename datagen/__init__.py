"""Seeded synthetic 8-bit tensor symbols (e4m3 and INT8 bytes) for the fixed-codebook coder.

This module only makes inputs. It holds none of the coder's arithmetic: no histogram, no code
lengths, no bit packing. Both the CUDA library's tests/benchmark and the CPU oracle take their
inputs from here, so neither side depends on the other for data.

The pages the coder follows ("Single-Stage Huffman Encoder for ML Compression", abstract; "Quad
Length Codes for Lossless Compression of e4m3", abstract and Figures 1, 4) measure real model
tensors (Gemma 2B shards, FFN1/FFN2 e4m3 activations) that are not available here. The five
workloads below stand in for them:

  cfg 1: 2^20 e4m3 bytes of N(0,1)*0.5; codebook from 4 prior 2^20 batches of the same law.
  cfg 2: 2^28 e4m3 bytes of a per-element mixture, 0.9 Laplace(0, b=0.3) + 0.1 N(0, sd=3);
         codebook from the summed histogram of 8 prior 2^28 batches.
  cfg 3: 2^26 INT8 bytes: an 8192x8192 Student-t(nu=4)*0.02 matrix quantised per row
         (scale = absmax/127, round half to even, clamp +-127); per-tensor codebook.
  cfg 4: 2^30 e4m3 bytes of the cfg-1 law; codebook from the cfg-1 prior batches.
  cfg 5: 64 tensors of 2^26 bytes, 16 layers x 4 shards. Layer l is e4m3 when l is even and
         INT8 otherwise, of family [Laplace, normal, Student-t4][l mod 3], at a scale drawn
         log-uniformly from [0.01, 3] with seed 5000+l. Each layer's codebook sums 4 prior
         2^26 batches of that layer.

Seeds: data of cfg k uses 1000+k (cfg-5 tensor t = 4*l + s uses 1500+t); prior batch j of cfg k
uses 2000+100k+j (cfg-5 layer l, batch j uses 2500+10l+j). Every array is built from blocks of
2^22 values, block b drawn from ``np.random.default_rng([seed, b])``, so the bytes do not depend
on how many threads draw them.

The e4m3 cast is OCP E4M3FN (bias 7, largest finite 448, no infinities): clamp to +-448, then
round to nearest even via torch's float8_e4m3fn conversion. INT8 bytes are two's complement.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

E4M3_MAX = 448.0
BLOCK = 1 << 22          # values per independently seeded block
INT8_COLS = 8192         # row length of the INT8 matrices (cfg 3 and cfg 5)
CFG5_LAYERS = 16
CFG5_SHARDS = 4
CFG5_TENSOR = 1 << 26

SIZES = {1: 1 << 20, 2: 1 << 28, 3: 1 << 26, 4: 1 << 30, 5: CFG5_LAYERS * CFG5_SHARDS * CFG5_TENSOR}
N_PRIOR = {1: 4, 2: 8, 3: 0, 4: 4, 5: 4}


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


# ----------------------------------------------------------------------------------------------
# Casts
# ----------------------------------------------------------------------------------------------
def e4m3_bytes(x: np.ndarray) -> np.ndarray:
    """fp32 values -> OCP E4M3FN bit patterns (uint8): clamp to +-448, round to nearest even."""
    x = np.clip(np.asarray(x, dtype=np.float32), -E4M3_MAX, E4M3_MAX)
    t = torch.from_numpy(np.ascontiguousarray(x)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy().copy()


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    """E4M3FN bit patterns -> float64 values, written from the format definition (NaN for 0x7F/0xFF)."""
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    normal = sign * (1.0 + m / 8.0) * np.power(2.0, e - 7)
    sub = sign * (m / 8.0) * 2.0 ** -6
    v = np.where(e == 0, sub, normal)
    return np.where((b & 0x7F) == 0x7F, np.nan, v)


def int8_rowwise_bytes(mat: np.ndarray) -> np.ndarray:
    """Symmetric per-row INT8: scale = absmax/127, q = round-half-even(x/scale) clamped to +-127.

    Arithmetic is fp32 as numpy evaluates it on fp32 arrays; an all-zero row uses scale 1.
    Returns the two's-complement bytes, row-major.
    """
    mat = np.asarray(mat, dtype=np.float32)
    absmax = np.max(np.abs(mat), axis=1, keepdims=True)
    scale = np.where(absmax > 0, absmax / np.float32(127.0), np.float32(1.0)).astype(np.float32)
    q = np.clip(np.rint(mat / scale), -127, 127).astype(np.int8)
    return q.reshape(-1).view(np.uint8)


# ----------------------------------------------------------------------------------------------
# Laws
# ----------------------------------------------------------------------------------------------
def _draw(family: str, rng: np.random.Generator, count: int, scale: float) -> np.ndarray:
    if family == "normal":
        return rng.standard_normal(count, dtype=np.float32) * np.float32(scale)
    if family == "laplace":
        return rng.laplace(0.0, scale, count).astype(np.float32)
    if family == "student_t4":
        return (rng.standard_t(4.0, count) * scale).astype(np.float32)
    if family == "ffn_mix":  # per-element Bernoulli(0.1) choice between N(0, sd=3) and Laplace(0, 0.3)
        pick = rng.random(count) < 0.1
        lap = rng.laplace(0.0, 0.3, count)
        nor = rng.standard_normal(count) * 3.0
        return np.where(pick, nor, lap).astype(np.float32)
    raise ValueError(f"unknown family {family!r}")


def tensor_bytes(family: str, dtype: str, n: int, seed: int, scale: float = 1.0) -> np.ndarray:
    """n bytes of `family` at `scale`, cast to `dtype` ("e4m3" or "int8"), block-seeded by `seed`."""
    out = np.empty(n, dtype=np.uint8)
    if dtype == "int8":
        if n % INT8_COLS:
            raise ValueError("INT8 tensors are whole rows of 8192")
    elif dtype != "e4m3":
        raise ValueError(f"unknown dtype {dtype!r}")
    nblk = (n + BLOCK - 1) // BLOCK

    def one(b: int) -> None:
        lo, hi = b * BLOCK, min(n, (b + 1) * BLOCK)
        rng = np.random.default_rng([seed, b])
        x = _draw(family, rng, hi - lo, scale)
        if dtype == "e4m3":
            out[lo:hi] = e4m3_bytes(x)
        else:  # BLOCK is a multiple of INT8_COLS, so a block holds whole rows
            out[lo:hi] = int8_rowwise_bytes(x.reshape(-1, INT8_COLS))

    if nblk == 1:
        one(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(one, range(nblk)))
    return out


# ----------------------------------------------------------------------------------------------
# Workloads
# ----------------------------------------------------------------------------------------------
def cfg5_layer(layer: int) -> dict:
    """dtype, family and scale of cfg-5 layer `layer` (scale log-uniform on [0.01, 3], seed 5000+l)."""
    rng = np.random.default_rng(5000 + layer)
    scale = float(math.exp(rng.uniform(math.log(0.01), math.log(3.0))))
    return {"dtype": "e4m3" if layer % 2 == 0 else "int8",
            "family": ["laplace", "normal", "student_t4"][layer % 3],
            "scale": scale}


def _law(cfg: int, layer: int | None = None) -> tuple[str, str, float]:
    if cfg in (1, 4):
        return "normal", "e4m3", 0.5
    if cfg == 2:
        return "ffn_mix", "e4m3", 1.0
    if cfg == 3:
        return "student_t4", "int8", 0.02
    if cfg == 5:
        p = cfg5_layer(layer)
        return p["family"], p["dtype"], p["scale"]
    raise ValueError(f"unknown config {cfg}")


def data(cfg: int, shard: int = 0, n: int | None = None) -> np.ndarray:
    """The input bytes of config `cfg` (cfg 5: tensor `shard` in 0..63). `n` truncates the draw
    to its first n bytes (same bytes as the full draw's prefix, whole blocks)."""
    if cfg == 5:
        layer = shard // CFG5_SHARDS
        family, dtype, scale = _law(5, layer)
        full, seed = CFG5_TENSOR, 1500 + shard
    else:
        family, dtype, scale = _law(cfg)
        full, seed = SIZES[cfg], 1000 + cfg
    n = full if n is None else int(n)
    if n > full:
        raise ValueError("n beyond the configuration's size")
    if dtype == "int8" and n % INT8_COLS:
        # draw whole rows, then cut: the prefix of the full matrix
        rows = -(-n // INT8_COLS)
        return tensor_bytes(family, dtype, rows * INT8_COLS, seed, scale)[:n]
    return tensor_bytes(family, dtype, n, seed, scale)


def prior_batches(cfg: int, layer: int = 0):
    """Yield the prior batches whose summed histogram defines the fixed codebook of `cfg`
    (cfg 4 shares cfg 1's; cfg 3 is per-tensor, so its only batch is the tensor itself)."""
    if cfg == 3:
        yield data(3)
        return
    if cfg == 4:
        cfg = 1
    if cfg == 5:
        family, dtype, scale = _law(5, layer)
        for j in range(N_PRIOR[5]):
            yield tensor_bytes(family, dtype, CFG5_TENSOR, 2500 + 10 * layer + j, scale)
        return
    family, dtype, scale = _law(cfg)
    for j in range(N_PRIOR[cfg]):
        yield tensor_bytes(family, dtype, SIZES[cfg], 2000 + 100 * cfg + j, scale)


def online_batch(t: int, n: int, switch: int = 10) -> np.ndarray:
    """Batch t of the online-loop workload: e4m3 activations whose scale drifts 3 % per batch
    (N(0, 0.5 * 1.03^t)) up to batch `switch`, then the cfg-2 FFN mixture law (an abrupt change).
    Seed 7000 + t."""
    if t < switch:
        return tensor_bytes("normal", "e4m3", n, 7000 + t, 0.5 * 1.03 ** t)
    return tensor_bytes("ffn_mix", "e4m3", n, 7000 + t, 1.0)


def uniform_bytes(n: int, seed: int) -> np.ndarray:
    """n independent uniform bytes (edge-case and adversarial tests)."""
    return np.random.default_rng(seed).integers(0, 256, n, dtype=np.uint8)


def random_counts(seed: int, alphabet: int = 256, zeros: float = 0.0, skew: float = 1.0) -> np.ndarray:
    """A random 256-bin count vector: `alphabet` leading bins drawn geometric-like, a fraction
    `zeros` of them forced to 0, the rest of the 256 bins 0."""
    rng = np.random.default_rng(seed)
    c = np.zeros(256, dtype=np.uint64)
    w = np.floor(np.exp(rng.uniform(0, 12 * skew, alphabet))).astype(np.uint64)
    if zeros:
        w[rng.random(alphabet) < zeros] = 0
    c[:alphabet] = w
    return c
