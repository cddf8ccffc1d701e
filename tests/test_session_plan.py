"""The online single-stage loop's schedule (which codebook codes batch t), on the host.

The oracle writes the loop out batch by batch (``oracle.session_schedule``); it is pinned here by
properties that do not restate its rule -- scale invariance of the code under summed identical
histograms, a single refresh at a distribution switch, the restart of the history there -- and
the library's planner (``hx_planner``, the bookkeeping ``hx_session`` runs) must hand out the
same codebook hash for every batch and flag the same refreshes.
"""
import numpy as np
import pytest

import datagen
from lossless_entropy_coding_fixed_b200 import hx


def _switch_hists(orc, before=5, after=5, n=1 << 16):
    """Histograms of e4m3 N(0, 0.5) batches, then of a different law (a wide normal on bytes)."""
    rng = np.random.default_rng(3)
    hs = [orc.histogram(datagen.data(1, n=n)) for _ in range(before)]
    for _ in range(after):
        x = np.clip(rng.normal(0, 1, n) * 60 + 128, 0, 255).astype(np.uint8)
        hs.append(orc.histogram(x))
    return hs


def test_stationary_batches_give_the_batch_code(orc):
    """Summing k copies of one histogram scales the weights, which leaves the optimal
    length-limited code unchanged: from batch lag on, the code is the batch's own."""
    h = orc.histogram(datagen.data(1, n=1 << 16))
    for lag, m in ((1, 1), (2, 4), (3, 2)):
        books, seen = orc.session_schedule([h] * 8, orc.KIND_HUFFMAN, m, lag)
        own = orc.huffman_codebook(h)
        first = orc.huffman_codebook(np.ones(256, np.uint64))
        for t, b in enumerate(books):
            assert b.hash == (own.hash if t >= lag else first.hash), (lag, m, t)
        assert not any(r for r, _ in seen)


def test_switch_refreshes_once_and_restarts_history(orc):
    hs = _switch_hists(orc)
    books, seen = orc.session_schedule(hs, orc.KIND_HUFFMAN, history=4, lag=1, drift=0.1)
    drifts = np.array([d for _, d in seen])
    # batch 0 is coded with the all-ones code (far off); the others up to the switch are close
    assert drifts[0] > 0.1 and (drifts[1:5] < 0.05).all() and drifts[5] > 0.1
    assert [r for r, _ in seen] == [True, False, False, False, False, True, False, False, False, False]
    # after the refresh at batch 5 the history holds batch 5 alone, then grows again
    assert books[6].hash == orc.huffman_codebook(hs[5]).hash
    assert books[7].hash == orc.huffman_codebook(hs[5] + hs[6]).hash
    # without a threshold the old batches stay in the window
    books0, seen0 = orc.session_schedule(hs, orc.KIND_HUFFMAN, history=4, lag=1, drift=0.0)
    assert not any(r for r, _ in seen0)
    assert books0[6].hash == orc.huffman_codebook(hs[2] + hs[3] + hs[4] + hs[5]).hash


@pytest.mark.parametrize("kind", [hx.KIND_HUFFMAN, hx.KIND_QLC])
@pytest.mark.parametrize("m,lag,drift", [(4, 2, 0.0), (2, 1, 0.1), (3, 2, 0.1), (1, 3, 0.02)])
def test_planner_matches_oracle_schedule(orc, kind, m, lag, drift):
    hs = _switch_hists(orc)
    init = orc.histogram(datagen.data(1, n=1 << 14))
    books, seen = orc.session_schedule(hs, kind, m, lag, drift, initial_counts=init)
    p = hx.Planner(kind, m, lag, drift, initial_counts=init)
    for t in range(len(hs)):
        if t >= lag:
            r, d = p.observe(t - lag, hs[t - lag])
            assert r == seen[t - lag][0]
            assert d == pytest.approx(seen[t - lag][1], rel=1e-12, abs=1e-12)
        assert p.codebook(t).hash == books[t].hash, t


def test_planner_rejects_out_of_order_use():
    p = hx.Planner(hx.KIND_HUFFMAN, 2, 2, 0.0)
    p.codebook(0)
    p.codebook(1)
    with pytest.raises(hx.HxError):
        p.codebook(2)  # batch 0 not observed yet
    with pytest.raises(hx.HxError):
        p.observe(1, np.ones(256))  # batch 0 comes first
    p.observe(0, np.ones(256))
    p.codebook(2)
    for bad in (dict(history=0), dict(history=65), dict(lag=0), dict(lag=9),
                dict(kind=2), dict(drift=float("nan"))):
        kw = dict(kind=hx.KIND_HUFFMAN, history=2, lag=1, drift=0.0) | bad
        with pytest.raises(hx.HxError):
            hx.Planner(**kw)
