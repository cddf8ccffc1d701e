"""Exp-Golomb streams on the GPU (the prefix-code kernels with a kind-3 table) against the oracle:
bit-exact streams, exact decode, and the oracle's status on damaged streams."""
import numpy as np
import pytest

import datagen

torch = pytest.importorskip("torch")
from lossless_entropy_coding_fixed_b200 import hx  # noqa: E402

pytestmark = pytest.mark.gpu
K = hx.KIND_EXPGOLOMB


@pytest.fixture(scope="module")
def cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return torch.device("cuda:0")


@pytest.mark.parametrize("order,map_,cfg,n", [(5, 0, 1, 1), (5, 0, 1, 4097), (7, 0, 1, (1 << 20) - 3),
                                              (6, 1, 3, 4 * 8192), (8, 1, 3, 3 * 4096 + 5)])
def test_parity(orc, cuda, order, map_, cfg, n):
    x = datagen.data(cfg, n=n) if cfg == 1 else datagen.data(3, n=1 << 26)[:n].copy()
    cb, ocb = hx.expgolomb_build(order, map_), orc.ExpGolombBook(order, map_)
    tables = cb.upload(cuda)
    ost, ref = orc.encode(ocb, x)
    out, st = hx.encode(tables, torch.from_numpy(x).cuda(), kind=K)
    torch.cuda.synchronize()
    got = out[:ref.size].cpu().numpy()
    assert ost == int(st.item()) == 0 and (got == ref).all()
    y, st = hx.decode(tables, torch.from_numpy(ref).cuda(), n, kind=K)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and (y.cpu().numpy() == x).all()


def test_damage_matches_oracle(orc, cuda):
    x = datagen.data(1, n=5 * 4096 + 333)
    cb, ocb = hx.expgolomb_build(6, 0), orc.ExpGolombBook(6, 0)
    tables = cb.upload(cuda)
    _, s = orc.encode(ocb, x)
    P = orc.payload_offset(x.size)
    rng = np.random.default_rng(8)
    for _ in range(30):
        t = s.copy()
        t[int(rng.integers(P, s.size - 8))] ^= np.uint8(1 << int(rng.integers(0, 8)))
        ost, oy = orc.decode(ocb, t, x.size)
        y, st = hx.decode(tables, torch.from_numpy(t).cuda(), x.size, kind=K)
        torch.cuda.synchronize()
        assert int(st.item()) == ost
        if ost == 0:
            assert (y.cpu().numpy() == oy).all()


def test_crowded_reader_damage_matches_oracle(orc, cuda):
    """Order 7 on e4m3 bytes: almost every code is 8 bits, so sub-streams start on one bank of
    their lines and the decoder's blocks take the voting loop with its 16-byte reader. Flipped
    payload bits and damaged sync entries must raise the oracle's statuses there too."""
    x = datagen.data(1, n=40 * 4096 + 333)
    cb, ocb = hx.expgolomb_build(7, 0), orc.ExpGolombBook(7, 0)
    tables = cb.upload(cuda)
    _, s = orc.encode(ocb, x)
    S, P = orc.sync_offset(x.size), orc.payload_offset(x.size)
    first = [0] + [int(v) for v in s[S + 2:S + 16].view(np.uint16)]
    banks = [(b >> 5) & 31 for b in first]
    assert max(banks.count(b) for b in banks) >= 4  # the first chunk looks crowded
    rng = np.random.default_rng(12)
    cases = []
    for _ in range(30):
        t = s.copy()
        t[int(rng.integers(P, s.size - 8))] ^= np.uint8(1 << int(rng.integers(0, 8)))
        cases.append(t)
    for c, k, v in [(0, 3, 4100), (5, 1, 0), (9, 7, 30000), (33, 4, 16385)]:
        t = s.copy()
        o = S + 16 * c + 2 * k
        t[o:o + 2] = np.array([v], np.uint16).view(np.uint8)
        cases.append(t)
    flagged = 0
    for t in cases:
        ost, oy = orc.decode(ocb, t, x.size)
        y, st = hx.decode(tables, torch.from_numpy(t).cuda(), x.size, kind=K)
        torch.cuda.synchronize()
        assert int(st.item()) == ost
        flagged += ost != 0
        if ost == 0:
            assert (y.cpu().numpy() == oy).all()
    assert flagged >= 4  # at least the sync damages
