"""The synthetic-input generators: the e4m3 cast against the OCP E4M3FN definition, the INT8
per-row quantiser against its definition, and determinism of the seeded draws. No GPU."""
import numpy as np

import datagen


def e4m3_reference(v: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even onto the finite E4M3FN values (written from the format: bias 7,
    3 mantissa bits, subnormals at exponent 0, 0x7F/0xFF NaN), after clamping to +-448."""
    codes = np.arange(256, dtype=np.uint8)
    vals = datagen.e4m3_decode(codes)
    keep = ~np.isnan(vals) & (codes < 0x80)  # non-negative finite codes (0x00..0x7E)
    pos_codes, pos_vals = codes[keep], vals[keep]
    order = np.argsort(pos_vals)
    pos_codes, pos_vals = pos_codes[order], pos_vals[order]
    out = np.empty(v.shape, np.uint8)
    for i, x in enumerate(np.asarray(v, np.float64)):
        a = min(abs(x), 448.0)
        j = np.searchsorted(pos_vals, a)
        if j < len(pos_vals) and pos_vals[j] == a:
            c = pos_codes[j]
        else:
            lo, hi = j - 1, j
            dl, dh = a - pos_vals[lo], pos_vals[hi] - a
            if dl < dh:
                c = pos_codes[lo]
            elif dh < dl:
                c = pos_codes[hi]
            else:  # tie: the even mantissa (even code)
                c = pos_codes[lo] if pos_codes[lo] % 2 == 0 else pos_codes[hi]
        out[i] = c | (0x80 if np.signbit(x) else 0)
    return out


def test_e4m3_cast_matches_definition():
    vals = datagen.e4m3_decode(np.arange(256, dtype=np.uint8))
    finite = np.unique(vals[~np.isnan(vals)])
    pos = np.sort(finite[finite >= 0])
    mids = (pos[:-1] + pos[1:]) / 2
    f32 = lambda a: np.asarray(a, np.float32)
    probes = np.concatenate([
        finite, mids, -mids,
        np.nextafter(f32(mids), f32(np.inf)), np.nextafter(f32(mids), f32(-np.inf)),
        -np.nextafter(f32(mids), f32(np.inf)),
        [448.0, 449.0, 464.0, 480.0, 1e6, -1e6, 1e-9, -1e-9, 2.0 ** -10, -0.0],
    ]).astype(np.float32)
    got = datagen.e4m3_bytes(probes)
    ref = e4m3_reference(probes)
    assert (got == ref).all(), np.nonzero(got != ref)
    # every finite value maps to its own code
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    assert (datagen.e4m3_bytes(datagen.e4m3_decode(codes).astype(np.float32)) == codes).all()


def test_int8_rowwise_definition():
    rng = np.random.default_rng(0)
    m = (rng.standard_t(4, (16, 8192)) * 0.02).astype(np.float32)
    m[3, 17] = 0.0
    q = datagen.int8_rowwise_bytes(m).view(np.int8).reshape(16, 8192).astype(np.int64)
    scale = np.abs(m).max(axis=1, keepdims=True) / np.float32(127)
    assert (np.abs(q).max(axis=1) == 127).all()
    assert (q >= -127).all()
    err = np.abs(q * scale.astype(np.float64) - m)
    assert (err <= scale / 2 * (1 + 1e-5)).all()
    # round half to even on exact ties
    t = np.array([[127.0, 0.5, 1.5, 2.5, -0.5, -2.5]], np.float32)
    assert list(datagen.int8_rowwise_bytes(t).view(np.int8)) == [127, 0, 2, 2, 0, -2]


def test_seeded_and_blockwise_deterministic():
    a = datagen.data(1)
    b = datagen.data(1)
    assert (a == b).all() and a.size == 1 << 20
    assert (datagen.data(1, n=5000) == a[:5000]).all()
    p = list(datagen.prior_batches(1))
    assert len(p) == 4 and not (p[0] == p[1]).all()
    x3 = datagen.data(3, n=8192 * 3 + 5)
    assert x3.size == 8192 * 3 + 5
    assert int(x3.view(np.int8).min()) >= -127


def test_cfg5_layers():
    layers = [datagen.cfg5_layer(l) for l in range(16)]
    assert all(0.01 <= p["scale"] <= 3 for p in layers)
    assert [p["dtype"] for p in layers[:4]] == ["e4m3", "int8", "e4m3", "int8"]
    assert [p["family"] for p in layers[:3]] == ["laplace", "normal", "student_t4"]
    x = datagen.data(5, shard=5, n=1 << 16)
    assert x.size == 1 << 16
