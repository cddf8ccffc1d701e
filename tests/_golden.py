"""Readers for the text fixtures under tests/golden/ (each fixture cites its source)."""
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _lines(name):
    with open(os.path.join(GOLDEN, name)) as f:
        for ln in f:
            ln = ln.strip()
            if ln and not ln.startswith("#"):
                yield ln


def rfc1951():
    return [(s, int(l), c) for s, l, c in (ln.split() for ln in _lines("rfc1951_canonical.txt"))]


def qlc_tables():
    rows = {}
    for ln in _lines("qlc_tables.txt"):
        t, area, acode, nsym, sbits, clen, r0, r1 = ln.split()
        rows.setdefault(int(t), []).append(dict(area=int(area), code=acode, nsym=int(nsym),
                                                bits=int(sbits), len=int(clen),
                                                first=int(r0), last=int(r1)))
    return rows


def fnv_vectors():
    out = []
    for ln in _lines("fnv1a64_vectors.txt"):
        q, h = ln.rsplit(" ", 1)
        out.append((q.strip('"').encode(), int(h, 16)))
    return out


def _runs(items, width):
    vals = []
    for it in items.split():
        k, v = it.split("*") if "*" in it else ("1", it)
        vals += [int(v, 16)] * int(k)
    return vals


def hand_streams():
    cases = {}
    for ln in _lines("streams_hand.txt"):
        name, inp, wo, sy, pw, total = [p.strip() for p in ln.split("|")]
        x = np.array(_runs(inp, 2), dtype=np.uint8)
        words = []
        for it in pw.split():
            k, v = it.split("*") if "*" in it else ("1", it)
            words += [int(v, 16)] * int(k)
        cases[name] = dict(x=x, word_off=[int(v) for v in wo.split()],
                           sync=[int(v) for v in sy.split()],
                           payload=np.array(words, dtype=np.uint32), total=int(total))
    return cases


def abc_counts():
    c = np.zeros(256, dtype=np.uint64)
    c[0x41], c[0x42], c[0x43] = 2, 1, 1
    return c


def histograms():
    """(bytes, {value: count}) from histogram_hand.txt."""
    out = []
    for ln in _lines("histogram_hand.txt"):
        data, bins = (t.strip() for t in ln.split("|"))
        raw = b"" if data == "-" else bytes.fromhex(data)
        out.append((raw, {int(v): int(c) for v, c in (b.split(":") for b in bins.split())}))
    return out
