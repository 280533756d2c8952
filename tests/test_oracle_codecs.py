"""Pins of the oracle's element codecs (E2M1 codes, UE4M3 block scales).

Independent references: the hand-derived fixtures in tests/golden/ and the ml_dtypes
library's float4_e2m1fn / float8_e4m3fn conversions (round-to-nearest-even).
"""
import ml_dtypes
import numpy as np

from _golden import rows


def test_e2m1_decode_matches_grid(orc):
    grid = {int(a): float(b) for a, b in (r.split() for r in rows("e2m1_grid.txt"))}
    for c in range(8):
        assert orc.e2m1_decode(np.array([c]))[0] == grid[c]
        assert orc.e2m1_decode(np.array([c | 8]))[0] == -grid[c]
        assert np.signbit(orc.e2m1_decode(np.array([c | 8]))[0])


def test_e2m1_hand_ties(orc):
    for r in rows("e2m1_round.txt"):
        v, c = r.split()
        assert orc.e2m1_encode(np.array([float(v)], np.float32))[0] == int(c), r


def _e2m1_probe_set():
    grid = np.array([0, .5, 1, 1.5, 2, 3, 4, 6], np.float32)
    mids = (grid[1:] + grid[:-1]) / 2
    pts = np.concatenate([grid, mids, [6.5, 7, 8, 100, 1e30, 1e-30, 1e-45]]).astype(np.float32)
    near = np.concatenate([np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))])
    rnd = np.random.default_rng(7).uniform(-8, 8, 200000).astype(np.float32)
    allv = np.concatenate([pts, near, rnd])
    return np.concatenate([allv, -allv]).astype(np.float32)


def test_e2m1_encode_vs_ml_dtypes(orc):
    v = _e2m1_probe_set()
    ours = orc.e2m1_encode(v)
    ref = v.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(v[i]), int(ours[i]), int(ref[i])) for i in bad[:10]]


def test_e4m3_decode_vs_ml_dtypes(orc):
    c = np.arange(256, dtype=np.uint8)
    ours = orc.e4m3_decode(c)
    ref = c.view(ml_dtypes.float8_e4m3fn).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert set(np.nonzero(nan)[0]) == {0x7F, 0xFF}
    assert np.array_equal(ours[~nan], ref[~nan])
    assert orc.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert orc.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9


def test_e4m3_hand_ties(orc):
    for r in rows("e4m3_round.txt"):
        v, c = r.split()
        assert orc.e4m3_encode(np.array([float(v)], np.float32))[0] == int(c, 16), r


def test_e4m3_encode_vs_ml_dtypes(orc):
    vals = orc.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    mids = (vals[1:] + vals[:-1]) / 2
    pts = np.concatenate([vals, mids]).astype(np.float32)
    near = np.concatenate([np.nextafter(pts, np.float32(np.inf)), np.nextafter(pts, np.float32(0))])
    rng = np.random.default_rng(11)
    rnd = np.exp(rng.uniform(np.log(2.0 ** -14), np.log(448.0), 300000)).astype(np.float32)
    v = np.concatenate([pts, near, rnd, [0.0, 1e-40, 2.0 ** -11]]).astype(np.float32)
    v = v[v <= 448.0]
    ours = orc.e4m3_encode(v)
    ref = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(v[i]), int(ours[i]), int(ref[i])) for i in bad[:10]]


def test_e4m3_satfinite(orc):
    v = np.array([448.0, 448.5, 463.9, 464.0, 480.0, 1e4, 3e38], np.float32)
    assert np.all(orc.e4m3_encode(v) == 0x7E)
