"""Pins of the CPU oracle to facts outside itself (no GPU).

Each test ties one oracle function to something the pages, a published standard or plain
mathematics fixes: brute-force optimal prefix codes, textbook Huffman, the RFC 1951 worked
example, the QLC tables printed on the page, closed forms of the entropy, FNV-1a test vectors
and hand-computed streams.
"""
import heapq
import itertools
import math

import numpy as np
import pytest

import datagen
from tests import _golden as G


def cost(w, ln):
    return int(sum(int(a) * int(b) for a, b in zip(w, ln)))


def kraft_units(ln, lmax=12):
    """Kraft sum times 2^lmax, exact integer."""
    return sum(1 << (lmax - int(l)) for l in ln if l)


def brute_force_cost(weights, lmax):
    """Minimum sum(w*len) over all prefix codes with lengths <= lmax (Kraft <= 1), by
    enumerating length multisets; the rearrangement inequality gives the best assignment."""
    w = sorted(weights, reverse=True)
    m = len(w)
    if m == 1:
        return w[0]
    top = min(lmax, m - 1)
    best = None
    for ls in itertools.combinations_with_replacement(range(1, top + 1), m):
        if sum(2.0 ** -l for l in ls) <= 1.0 + 1e-12:
            c = sum(a * b for a, b in zip(w, ls))
            best = c if best is None else min(best, c)
    return best


def textbook_huffman_cost(weights):
    """Classic Huffman by repeatedly merging the two lightest nodes; cost = sum of merges.
    Also returns the maximum depth."""
    if len(weights) == 1:
        return weights[0], 1
    h = [(w, i, 0) for i, w in enumerate(weights)]
    heapq.heapify(h)
    total, k = 0, len(weights)
    while len(h) > 1:
        a, _, da = heapq.heappop(h)
        b, _, db = heapq.heappop(h)
        total += a + b
        heapq.heappush(h, (a + b, k, max(da, db) + 1))
        k += 1
    return total, h[0][2]


# --------------------------------------------------------------------------- package-merge
@pytest.mark.parametrize("seed", range(60))
def test_package_merge_equals_brute_force_small_alphabets(orc, seed):
    rng = np.random.default_rng(seed)
    m = int(rng.integers(1, 9))
    lmax = int(rng.integers(max(1, math.ceil(math.log2(max(m, 2)))), 9))
    weights = (rng.integers(1, 1000, m) if seed % 3 else 2 ** rng.integers(0, 20, m)).astype(np.uint64)
    syms = rng.choice(256, m, replace=False)
    counts = np.zeros(256, np.uint64)
    counts[syms] = weights
    ln = orc.huffman_lengths(counts, lmax=lmax, cover_all=False)
    assert (ln[counts == 0] == 0).all()
    assert ln.max() <= lmax
    assert cost(counts, ln) == brute_force_cost([int(v) for v in weights], lmax)
    if m >= 2:
        assert kraft_units(ln, 12) == 1 << 12  # the optimum is a complete code


@pytest.mark.parametrize("seed", range(20))
def test_package_merge_equals_textbook_huffman_when_limit_does_not_bind(orc, seed):
    counts = datagen.random_counts(seed, alphabet=int(np.random.default_rng(seed).integers(2, 257)),
                                   skew=0.6)
    counts[counts == 0] = 1
    w = [int(v) for v in counts if v]
    ref, depth = textbook_huffman_cost(w)
    ln = orc.huffman_lengths(counts, lmax=12, cover_all=False)
    if depth <= 12:
        assert cost(counts, ln) == ref
    else:  # the limit binds: the limited code can only cost more
        assert cost(counts, ln) >= ref


@pytest.mark.parametrize("seed", range(20))
def test_full_codes_kraft_exact_and_mean_in_entropy_bounds(orc, seed):
    counts = datagen.random_counts(100 + seed, skew=0.7, zeros=0.3)
    ln = orc.huffman_lengths(counts, lmax=12, cover_all=True)
    assert (ln >= 1).all() and ln.max() <= 12
    assert kraft_units(ln) == 1 << 12
    w = np.maximum(counts, 1)
    H = orc.entropy(w)
    mean = orc.mean_length(w, ln)
    assert H - 1e-12 <= mean < H + 1


def test_lmax_binds_exactly(orc):
    counts = np.zeros(256, np.uint64)
    counts[:8] = [1, 2, 4, 8, 16, 32, 64, 128]  # unconstrained depth 7
    ln = orc.huffman_lengths(counts, lmax=3, cover_all=False)
    assert list(ln[:8]) == [3] * 8
    ln = orc.huffman_lengths(counts, lmax=12, cover_all=False)
    assert list(ln[:8]) == [7, 7, 6, 5, 4, 3, 2, 1]
    with pytest.raises(ValueError):
        orc.huffman_lengths(counts, lmax=2, cover_all=False)


def test_dyadic_distribution_mean_equals_entropy(orc):
    counts = np.zeros(256, np.uint64)
    counts[[10, 20, 30, 40, 50]] = [8, 4, 2, 1, 1]
    ln = orc.huffman_lengths(counts, cover_all=False)
    assert [int(ln[s]) for s in (10, 20, 30, 40, 50)] == [1, 2, 3, 4, 4]
    assert orc.mean_length(counts, ln) == pytest.approx(orc.entropy(counts), abs=1e-15)


def test_degenerate_alphabets(orc):
    counts = np.zeros(256, np.uint64)
    assert orc.huffman_lengths(counts, cover_all=False).max() == 0
    counts[7] = 5
    ln = orc.huffman_lengths(counts, cover_all=False)
    assert ln[7] == 1 and ln.sum() == 1
    ln = orc.huffman_lengths(np.zeros(256, np.uint64), cover_all=True)
    assert (ln == 8).all()  # all weights equal: the balanced code


def test_tie_break_rule_on_equal_weights(orc):
    # five equal weights: optimal codes have two lengths-2 and three lengths-3 (or 3x2 + 2x3);
    # leaves sort by symbol, so the first packages take the smallest symbols -> longer codes.
    counts = np.zeros(256, np.uint64)
    counts[[3, 1, 4, 0, 2]] = 1
    ln = orc.huffman_lengths(counts, cover_all=False)
    assert list(ln[:5]) == [3, 3, 2, 2, 2]


# --------------------------------------------------------------------------- canonical codes
def test_canonical_codes_rfc1951_example(orc):
    ex = G.rfc1951()
    ln = np.zeros(256, np.uint8)
    for s, l, _ in ex:
        ln[ord(s)] = l
    code = orc.canonical_codes(ln)
    for s, l, c in ex:
        assert format(int(code[ord(s)]), f"0{l}b") == c


@pytest.mark.parametrize("seed", range(10))
def test_canonical_codes_prefix_free(orc, seed):
    counts = datagen.random_counts(200 + seed, zeros=0.5)
    ln = orc.huffman_lengths(counts, cover_all=False)
    code = orc.canonical_codes(ln)
    words = sorted(format(int(code[s]), f"0{int(ln[s])}b") for s in range(256) if ln[s])
    for a, b in zip(words, words[1:]):
        assert not b.startswith(a)


# --------------------------------------------------------------------------- QLC
def qlc_dp_cost(weights, max_distinct):
    """Optimal QLC cost by dynamic programming over areas (a different algorithm from the
    oracle's enumeration): state = (areas used, ranks covered, last width, distinct widths)."""
    order = sorted(range(256), key=lambda s: (-int(weights[s]), s))
    pre = [0]
    for s in order:
        pre.append(pre[-1] + int(weights[s]))
    INF = float("inf")
    best = {(0, -1, 0): 0}  # (ranks covered, last width, distinct) -> cost
    for _ in range(8):
        nxt = {}
        for (r, lb, d), c in best.items():
            for b in range(max(lb, 0), 9):
                nd = d + (1 if b != lb else 0)
                if nd > max_distinct:
                    continue
                take = min(1 << b, 256 - r)
                key = (r + take, b, nd)
                v = c + (pre[r + take] - pre[r]) * (3 + b)
                if v < nxt.get(key, INF):
                    nxt[key] = v
        best = nxt
    return min(c for (r, _, _), c in best.items() if r == 256)


@pytest.mark.parametrize("seed,maxd", [(s, d) for s in range(6) for d in (1, 2, 4, 8)])
def test_qlc_search_optimal_by_dp(orc, seed, maxd):
    counts = datagen.random_counts(300 + seed, skew=0.8, zeros=0.2 * (seed % 2))
    q = orc.qlc_codebook(counts, max_distinct=maxd)
    assert len(set(int(b) for b in q.bits)) <= maxd
    assert list(q.bits) == sorted(q.bits)
    assert cost(counts, q.len) == qlc_dp_cost(counts, maxd)


def test_qlc_code_structure(orc):
    counts = datagen.random_counts(7, skew=0.9)
    q = orc.qlc_codebook(counts)
    assert q.start[0] == 0 and q.start[8] == 256
    assert sum(2.0 ** -int(l) for l in q.len) <= 1.0
    for a in range(8):
        for r in range(int(q.start[a]), int(q.start[a + 1])):
            s = int(q.rank2sym[r])
            assert q.len[s] == 3 + q.bits[a]
            assert int(q.code[s]) >> int(q.bits[a]) == a
            assert int(q.code[s]) & ((1 << int(q.bits[a])) - 1) == r - q.start[a]
    # ranking: weight descending, ties to the smaller symbol
    ranked = [int(s) for s in q.rank2sym]
    assert ranked == sorted(range(256), key=lambda s: (-int(counts[s]), s))


def test_qlc_uniform_is_identity_code(orc):
    q = orc.qlc_codebook(np.full(256, 7, np.uint64))
    assert list(q.bits) == [5] * 8
    assert (q.code == np.arange(256)).all() and (q.len == 8).all()
    assert orc.mean_length(np.ones(256, np.uint64), q.len) == 8.0 == orc.entropy(np.ones(256, np.uint64))
    q1 = orc.qlc_codebook(datagen.random_counts(1), max_distinct=1)
    assert list(q1.bits) == [5] * 8


def test_qlc_reproduces_table1_on_gaussian_e4m3(orc):
    """Table 1's six printed areas come out of the area search on an e4m3 N(0, 0.5) histogram."""
    counts = sum(orc.histogram(b) for b in datagen.prior_batches(1))
    q = orc.qlc_codebook(counts)
    for row in G.qlc_tables()[1]:
        a = row["area"] - 1
        assert format(a, "03b") == row["code"]
        assert int(q.bits[a]) == row["bits"]
        assert 3 + int(q.bits[a]) == row["len"]
        assert int(q.start[a]) == row["first"]
        assert int(q.start[a + 1]) - 1 == row["last"]
        assert int(q.start[a + 1] - q.start[a]) == row["nsym"]
    assert len(set(int(b) for b in q.bits)) == 4


def test_qlc_table2_prefix_is_feasible(orc):
    """Table 2's printed areas come out of the area search on a PMF with two dominant symbols
    over a geometric tail (the shape of a sorted post-activation PMF): weights 3200, 3200, then
    1000*0.97^r for the remaining ranks r, placed on a random permutation of the byte values."""
    w = np.zeros(256, np.uint64)
    order = np.random.default_rng(3).permutation(256)
    prof = [3200, 3200] + [max(1, int(1000 * 0.97 ** r)) for r in range(254)]
    w[order] = prof
    q = orc.qlc_codebook(w)
    assert len(set(int(b) for b in q.bits)) == 4
    rows = G.qlc_tables()[2]
    assert [int(b) for b in q.bits[:6]] == [r["bits"] for r in rows]
    assert [int(q.start[a]) for a in range(6)] == [r["first"] for r in rows]


# --------------------------------------------------------------------------- entropy, hash
def test_entropy_closed_forms(orc):
    assert orc.entropy(np.ones(256, np.uint64)) == pytest.approx(8.0, abs=1e-12)
    c = np.zeros(256, np.uint64)
    c[[0, 1]] = 5
    assert orc.entropy(c) == pytest.approx(1.0, abs=1e-15)
    c[[0, 1, 2]] = [2, 1, 1]
    assert orc.entropy(c) == pytest.approx(1.5, abs=1e-15)
    assert orc.entropy(np.zeros(256, np.uint64)) == 0.0


def test_fnv1a_published_vectors(orc):
    for data, h in G.fnv_vectors():
        assert orc.fnv1a(data) == h


def test_codebook_hash_serialisation(orc):
    cb = orc.huffman_codebook(G.abc_counts(), cover_all=False)
    assert cb.hash == orc.fnv1a(bytes([0, 12]) + cb.len.tobytes())
    q = orc.qlc_codebook(np.ones(256, np.uint64))
    assert q.hash == orc.fnv1a(bytes([1, 11]) + q.bits.tobytes() + q.rank2sym.tobytes())


# --------------------------------------------------------------------------- histogram
def test_histogram_hand_counted(orc):
    """Small inputs counted by hand, the empty input and a last byte that differs included."""
    for raw, bins in G.histograms():
        want = np.zeros(256, np.uint64)
        for v, c in bins.items():
            want[v] = c
        got = orc.histogram(np.frombuffer(raw, dtype=np.uint8))
        assert got.dtype == np.uint64 and (got == want).all(), raw.hex()


@pytest.mark.parametrize("n", [0, 1, 15, 16, 17, 4095, 4096, 4097, 3 * 4096 + 100])
def test_histogram_closed_form_ramp(orc, n):
    """x[i] = i mod 256: every bin holds floor(n/256), and the first n mod 256 bins one more,
    so a dropped or doubled byte at any ragged length changes a bin."""
    x = (np.arange(n) % 256).astype(np.uint8)
    want = np.full(256, n // 256, np.uint64)
    want[: n % 256] += 1
    assert (orc.histogram(x) == want).all()
    assert int(orc.histogram(x).sum()) == n


@pytest.mark.parametrize("seed", range(4))
def test_histogram_equals_bincount(orc, seed):
    """Against numpy's bincount on random and skewed inputs of ragged sizes."""
    rng = np.random.default_rng(seed)
    for n in (0, 1, 17, 4097, 65537):
        x = rng.integers(0, 256, n, dtype=np.uint8) if seed % 2 else \
            np.minimum(rng.geometric(0.1, n), 255).astype(np.uint8)
        assert (orc.histogram(x) == np.bincount(x, minlength=256).astype(np.uint64)).all()
