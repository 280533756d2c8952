"""Pins of the oracle's block quantizer, scale-factor layout and weight quantizer:
hand-derived worked examples, closed forms and invariants."""
import numpy as np

from _golden import rows
from vla_action_head_b200 import synth


def test_block_worked_examples(orc):
    for r in rows("block16_examples.txt"):
        g, ys, s, cs = (p.strip() for p in r.split("|"))
        y = np.array([float(t) for t in ys.split()], np.float32)
        codes, sbyte = orc.quantize_block16(y, float(g))
        assert sbyte == int(s, 16), r
        assert [int(c) for c in codes] == [int(t, 16) for t in cs.split()], (r, codes)


def _blocks(seed, n, scale_lo=-3, scale_hi=3):
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((n, 16)).astype(np.float32)
    y *= np.exp(rng.uniform(scale_lo, scale_hi, (n, 1))).astype(np.float32)
    return y


def _unpack(codes8):
    c = np.asarray(codes8, np.uint8)
    out = np.empty(c.size * 2, np.uint8)
    out[0::2] = c & 15
    out[1::2] = c >> 4
    return out


def test_amax_maps_to_six(orc):
    """For a normal, unsaturated scale the largest |y| lands on magnitude 6: t = a/(6g) is
    rounded to s within half an E4M3 step (2^-4 relative), so a/S lies in
    [6/1.0625, 6/0.9375], which E2M1 rounds to 6."""
    y = _blocks(1, 4000)
    for g in (1.0, 0.25, 3.0):
        for blk in y:
            codes, s = orc.quantize_block16(blk, g)
            t = np.float32(np.abs(blk).max()) / np.float32(6 * g)
            if not (2.0 ** -6 <= t <= 448):
                continue
            u = _unpack(codes)
            i = int(np.argmax(np.abs(blk)))
            assert (u[i] & 7) == 7, (g, blk, s)


def test_zero_block(orc):
    codes, s = orc.quantize_block16(np.zeros(16, np.float32), 1.0)
    assert s == 0 and not codes.any()


def test_constant_block(orc):
    """A constant block c: every code is magnitude 6 with c's sign and 6*S is within
    half an E4M3 step (2^-4 relative) of |c| (normal scale range)."""
    for c in (1.0, -0.37, 12.5, -300.0, 2.0 ** -3):
        for g in (1.0, 0.5):
            codes, s = orc.quantize_block16(np.full(16, c, np.float32), g)
            u = _unpack(codes)
            assert np.all(u == (7 | (8 if c < 0 else 0)))
            S = float(orc.e4m3_decode(np.array([s]))[0]) * g
            assert abs(6 * S - abs(c)) <= 2.0 ** -4 * abs(c) * (1 + 1e-6)


def test_dequant_error_bound(orc):
    """|y - yhat| <= half the local E2M1 grid gap times S (gap 0.5 below 2, 1 below 4,
    2 up to 6; the top element can exceed 6 by at most 6*2^-4/(1-2^-4) < 1 = gap/2)."""
    y = _blocks(3, 3000, -2, 2)
    for blk in y:
        codes, s = orc.quantize_block16(blk, 1.0)
        S = float(orc.e4m3_decode(np.array([s]))[0])
        yh = orc.e2m1_decode(_unpack(codes)).astype(np.float64) * S
        v = np.abs(blk.astype(np.float64)) / S
        half_gap = np.where(v < 2, 0.25, np.where(v < 4, 0.5, 1.0))
        assert np.all(np.abs(blk - yh) <= half_gap * S * (1 + 1e-5) + 1e-30)


def test_quantize_rows_matches_blocks(orc):
    y = _blocks(5, 3 * 12).reshape(3, 192)
    codes, sf = orc.quantize_rows(y, 0.75)
    for r in range(3):
        for b in range(12):
            c, s = orc.quantize_block16(y[r, b * 16:(b + 1) * 16], 0.75)
            assert np.array_equal(codes[r, b * 8:(b + 1) * 8], c)
            assert sf[orc.sf_offset(r, b, 192)] == s


def test_sf_offsets_golden(orc):
    for r in rows("sf_offsets.txt"):
        row, kb, K, off = (int(t) for t in r.split())
        assert orc.sf_offset(row, kb, K) == off, r


def test_sf_layout_is_a_bijection(orc):
    for rws, K in ((1, 64), (41, 1536), (130, 320), (256, 4320)):
        rp = (rws + 127) // 128 * 128
        nb = (K + 63) // 64 * 4
        offs = np.array([orc.sf_offset(r, b, K) for r in range(rp) for b in range(nb)])
        assert offs.size == orc.sf_bytes(rws, K)
        assert np.array_equal(np.sort(offs), np.arange(offs.size))


def test_sf_padding_stays_zero(orc):
    y = _blocks(9, 41 * 6).reshape(41, 96)  # K = 96: 6 real blocks of 8 (padded to 64-atoms)
    codes, sf = orc.quantize_rows(y, 1.0)
    real = {orc.sf_offset(r, b, 96) for r in range(41) for b in range(6)}
    pad = [i for i in range(sf.size) if i not in real]
    assert len(pad) == sf.size - 41 * 6 and not sf[pad].any()


def test_weight_quantizer_global_scale(orc):
    w = synth.bf16_normal(77, (64, 128), 0.0, 0.02)
    codes, sf, g = orc.quantize_weight(w)
    wf = synth.bf16_bits_to_f32(w)
    amax = np.float32(np.abs(wf).max())
    assert g == np.float32(amax / np.float32(2688.0))
    r, k = np.unravel_index(int(np.argmax(np.abs(wf))), wf.shape)
    assert sf[orc.sf_offset(int(r), int(k) // 16, 128)] == 0x7E
    u = _unpack(codes[r])
    assert (u[k] & 7) == 7
    # every block equals the activation quantizer at the same global scale
    c2, sf2 = orc.quantize_rows(wf, g)
    assert np.array_equal(c2, codes) and np.array_equal(sf2, sf)


def test_weight_quantizer_zero_and_interleave(orc):
    z = np.zeros((32, 64), np.uint16)
    codes, sf, g = orc.quantize_weight(z)
    assert g == 1.0 and not codes.any() and not sf.any()
    w = synth.bf16_normal(78, (64, 64), 0.0, 0.02)
    c0, s0, g0 = orc.quantize_weight(w)
    ci, si, gi = orc.quantize_weight(w, interleave_gate_up=True)
    assert g0 == gi
    for j in range(32):
        assert np.array_equal(ci[2 * j], c0[j])
        assert np.array_equal(ci[2 * j + 1], c0[32 + j])
        for b in range(4):
            assert si[orc.sf_offset(2 * j, b, 64)] == s0[orc.sf_offset(j, b, 64)]
            assert si[orc.sf_offset(2 * j + 1, b, 64)] == s0[orc.sf_offset(32 + j, b, 64)]
