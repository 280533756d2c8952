"""CPU checks of the FP4-output acceptance rule (parity.check_fp4_output) that every
bias+GELU / GeGLU -> FP4 GPU parity test goes through.  The "GPU" outputs here are made by
the oracle's own block quantizer and then altered on the host: a legitimate one-step scale
difference at an E4M3 rounding boundary must pass; a planted mistake must fail."""
import numpy as np
import pytest

from parity import check_fp4_output

ROWS, K, G = 64, 1024, 1.0


def _quantize(orc, h):
    """Oracle FP4 of fp64 h [ROWS, K] (quantized as fp32, as the epilogue's oracle does)."""
    return orc.quantize_rows(h.astype(np.float32), G)


def _put_block(orc, codes, sf, r, b, y32):
    """Quantizes one 16-value block with the oracle and writes it at (row r, block b)."""
    c8, s = orc.quantize_block16(y32, G)
    codes[r, 8 * b:8 * b + 8] = c8
    sf[orc.sf_offset(r, b, K)] = s
    return s


def _e4m3_mid(orc, s):
    """Midpoint between UE4M3 byte s and s + 1."""
    v = orc.e4m3_decode(np.array([s, s + 1], np.uint8)).astype(np.float64)
    return 0.5 * (v[0] + v[1])


@pytest.fixture()
def case(orc):
    rng = np.random.default_rng(7)
    h = rng.standard_normal((ROWS, K)).astype(np.float32).astype(np.float64)
    # block (3, 5): amax set so that t = a / (6 g) sits 2^-13 below the midpoint between
    # bytes 0x30 and 0x31 -- the oracle rounds down, an fp32 h a hair larger rounds up
    blk = h[3, 80:96]
    blk *= 0.9 / np.abs(blk).max()
    t_mid = _e4m3_mid(orc, 0x30)
    a = float(np.float32(6.0 * G * t_mid * (1 - 2.0 ** -13)))
    j = int(np.argmax(np.abs(blk)))
    blk[j] = np.copysign(a, blk[j])
    h[3, 80:96] = blk
    ref_codes, ref_sf = _quantize(orc, h)
    return h, ref_codes, ref_sf


def _gpu_like(orc, h, ref_codes, ref_sf):
    """A legitimate kernel result: block (3, 5) quantized from h (1 + 2^-11), which crosses
    the E4M3 boundary (one scale step up, codes re-rounded at that scale)."""
    codes, sf = ref_codes.copy(), ref_sf.copy()
    y = (h[3, 80:96] * (1 + 2.0 ** -11)).astype(np.float32)
    s = _put_block(orc, codes, sf, 3, 5, y)
    assert s == orc.sf_gather(ref_sf, ROWS, K)[3, 5] + 1
    return codes, sf


def test_boundary_scale_step_passes(orc, case):
    h, rc, rs = case
    gc, gs = _gpu_like(orc, h, rc, rs)
    check_fp4_output(orc, gc, gs, rc, rs, h, G, ROWS, K)


def test_identical_output_passes(orc, case):
    h, rc, rs = case
    assert check_fp4_output(orc, rc.copy(), rs.copy(), rc, rs, h, G, ROWS, K) == 0.0


def test_garbage_codes_in_a_stepped_block_fail(orc, case):
    """The hole of the old rule: codes were never looked at where the scales differ."""
    h, rc, rs = case
    gc, gs = _gpu_like(orc, h, rc, rs)
    gc[3, 40:48] = 0x77  # block 5 of row 3: every code +6
    with pytest.raises(AssertionError, match="E2M1 rounding"):
        check_fp4_output(orc, gc, gs, rc, rs, h, G, ROWS, K)


def test_sign_flip_in_a_stepped_block_fails(orc, case):
    h, rc, rs = case
    gc, gs = _gpu_like(orc, h, rc, rs)
    gc[3, 40:48] ^= 0x88  # every code's sign bit
    with pytest.raises(AssertionError):
        check_fp4_output(orc, gc, gs, rc, rs, h, G, ROWS, K)


def test_scale_step_away_from_a_boundary_fails(orc, case):
    """A one-step scale difference (codes consistent with it) where t is nowhere near an
    E4M3 rounding boundary is a bug, not fp32 rounding."""
    h, rc, rs = case
    gc, gs = rc.copy(), rs.copy()
    r, b = 10, 7
    s_ref = int(orc.sf_gather(rs, ROWS, K)[r, b])
    S_up = float(orc.e4m3_decode(np.array([s_ref + 1], np.uint8))[0]) * G
    gs[orc.sf_offset(r, b, K)] = s_ref + 1
    y = h[r, 16 * b:16 * b + 16].astype(np.float32)
    v = orc.e2m1_encode((y.astype(np.float64) / S_up).astype(np.float32))
    gc[r, 8 * b:8 * b + 8] = (v[0::2] | (v[1::2] << 4)).astype(np.uint8)
    with pytest.raises(AssertionError, match="away from an E4M3 rounding boundary"):
        check_fp4_output(orc, gc, gs, rc, rs, h, G, ROWS, K)


def test_far_code_in_an_equal_scale_block_fails(orc, case):
    h, rc, rs = case
    gc, gs = rc.copy(), rs.copy()
    c = gc[20, 100]
    lo = c & 15
    gc[20, 100] = (c & 0xF0) | ((lo & 8) | ((lo & 7) + 3 if (lo & 7) < 4 else (lo & 7) - 3))
    with pytest.raises(AssertionError, match="E2M1 rounding"):
        check_fp4_output(orc, gc, gs, rc, rs, h, G, ROWS, K)


def test_two_step_scale_fails(orc, case):
    h, rc, rs = case
    gc, gs = rc.copy(), rs.copy()
    off = orc.sf_offset(30, 2, K)
    gs[off] = gs[off] + 2
    with pytest.raises(AssertionError, match="more than one step"):
        check_fp4_output(orc, gc, gs, rc, rs, h, G, ROWS, K)


def test_row_selection(orc, case):
    """sel: the rows compared are a subset (h_ref holds just them)."""
    h, rc, rs = case
    gc, gs = _gpu_like(orc, h, rc, rs)
    sel = np.array([0, 3, 17, 63] + list(range(30, 42)))  # 1024 blocks: one stepped
    check_fp4_output(orc, gc, gs, rc, rs, h[sel], G, ROWS, K, sel=sel)
    gc[3, 40:48] = 0x77
    with pytest.raises(AssertionError):
        check_fp4_output(orc, gc, gs, rc, rs, h[sel], G, ROWS, K, sel=sel)
