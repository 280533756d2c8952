"""Pins of the oracle's 16-point Hadamard block rotation and its uniform INT4 (E0M3)
element grid ("Pi0.5 Thor NVFP4 End-to-End Results", §Full-INT4 Decoder Activations +
Hadamard Rotation and §E0M3 Uniform-INT4 Decoder Weights): hand-derived worked examples,
the Sylvester matrix from scipy, orthogonality, closed forms and invariants."""
import numpy as np
import pytest
import scipy.linalg

from _golden import rows
from vla_action_head_b200 import synth


def _hexes(txt):
    return np.array([float.fromhex(t) for t in txt.split()], np.float64)


# ---- rotation ----------------------------------------------------------------------------
def test_hadamard_hand_cases(orc):
    """Rounding order, signs and the 1/4 scale of the butterfly, bit for bit."""
    for r in rows("hadamard16.txt"):
        a, b = r.split("|")
        y, want = _hexes(a), _hexes(b)
        got = orc.hadamard16(y.astype(np.float32)).astype(np.float64)
        assert np.array_equal(got, want), (r, got)
        assert np.array_equal(np.signbit(got), np.signbit(want)), r


def _matrix(orc):
    """The rotation applied to the 16 unit vectors (exact: every partial sum is +-1 or 0)."""
    return orc.hadamard16(np.eye(16, dtype=np.float32)).astype(np.float64).T  # column j = R e_j


def test_rotation_is_sylvester_hadamard_over_four(orc):
    R = _matrix(orc)
    assert np.array_equal(4.0 * R, scipy.linalg.hadamard(16).astype(np.float64))


def test_rotation_orthonormal_and_involutive(orc):
    H = 4.0 * _matrix(orc)
    assert np.array_equal(H @ H.T, 16.0 * np.eye(16))
    R = H / 4.0
    assert np.array_equal(R @ R, np.eye(16))
    # rotating twice returns the block exactly where every partial sum is exact in fp32
    rng = np.random.default_rng(1)
    y = rng.integers(-64, 65, (500, 16)).astype(np.float32)
    assert np.array_equal(orc.hadamard16(orc.hadamard16(y)), y)


def test_rotation_close_to_fp64_product(orc):
    """fp32 butterfly vs the fp64 product H y / 4: four rounded stages, each within half an
    ulp of a partial sum bounded by sum |y|."""
    rng = np.random.default_rng(2)
    y = (rng.standard_normal((2000, 16)) * np.exp(rng.uniform(-4, 4, (2000, 1)))).astype(np.float32)
    H = scipy.linalg.hadamard(16).astype(np.float64)
    want = y.astype(np.float64) @ H.T / 4.0
    got = orc.hadamard16(y).astype(np.float64)
    bound = 4 * 2.0 ** -24 * np.abs(y).astype(np.float64).sum(axis=1, keepdims=True) / 4.0
    assert np.all(np.abs(got - want) <= bound)


def test_rotation_preserves_dot_products(orc):
    """The GEMM is unchanged by rotating both operands' blocks (fp64, no quantization)."""
    rng = np.random.default_rng(3)
    a = rng.standard_normal((64, 16))
    w = rng.standard_normal((64, 16))
    R = scipy.linalg.hadamard(16).astype(np.float64) / 4.0
    assert np.allclose(((a @ R.T) * (w @ R.T)).sum(1), (a * w).sum(1), rtol=0, atol=1e-12)


# ---- E0M3 ----------------------------------------------------------------------------------
def test_e0m3_decode_closed_form(orc):
    c = np.arange(16, dtype=np.uint8)
    want = np.where(c & 8, -1.0, 1.0) * (c & 7)
    assert np.array_equal(orc.e0m3_decode(c).astype(np.float64), want)


def test_e0m3_hand_rounding(orc):
    for r in rows("e0m3_round.txt"):
        v, c = (t.strip() for t in r.split("|"))
        assert orc.e0m3_encode(np.array([float(v)], np.float32))[0] == int(c, 16), r


def test_e0m3_encode_against_rint(orc):
    """Against numpy's round-half-to-even on 200k values spanning the grid and beyond."""
    rng = np.random.default_rng(4)
    v = (rng.uniform(-9, 9, 200000)).astype(np.float32)
    v[:64] = np.arange(-16, 16, 0.5, dtype=np.float32)  # every tie
    mag = np.minimum(np.rint(np.abs(v.astype(np.float64))), 7).astype(np.uint8)
    want = mag | (np.signbit(v).astype(np.uint8) << 3)
    assert np.array_equal(orc.e0m3_encode(v), want)


def test_e0m3_block_worked_examples(orc):
    for r in rows("e0m3_blocks.txt"):
        g, ys, s, cs = (p.strip() for p in r.split("|"))
        y = np.array([float(t) for t in ys.split()], np.float32)
        codes, sbyte = orc.quantize_block16_ex(y, float(g), orc.E0M3)
        assert sbyte == int(s, 16), r
        assert [int(c) for c in codes] == [int(t, 16) for t in cs.split()], (r, codes)


def _unpack(c8):
    c8 = np.asarray(c8, np.uint8)
    out = np.empty(c8.shape[:-1] + (c8.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c8 & 15
    out[..., 1::2] = c8 >> 4
    return out


def test_e0m3_amax_maps_to_seven_and_error_bound(orc):
    """Normal, unsaturated scale: a / S lies in [7 / 1.0625, 7 / 0.9375] = [6.59, 7.47], which
    rounds to 7; every element is within half a step (S / 2) of its dequantized value."""
    rng = np.random.default_rng(5)
    for g in (1.0, 0.125, 3.0):
        y = (rng.standard_normal((3000, 16)) * np.exp(rng.uniform(-3, 3, (3000, 1)))).astype(np.float32)
        codes, sf = orc.quantize_rows(y, g, flags=orc.E0M3)
        deq = orc.dequantize(codes, sf, g, y.shape[0], 16, flags=orc.E0M3)
        s = orc.sf_gather(sf, y.shape[0], 16)[:, 0]
        S = orc.e4m3_decode(s).astype(np.float64) * np.float32(g)
        normal = (s >= 0x08) & (s < 0x7E)
        q = _unpack(codes)
        i_max = np.argmax(np.abs(y), axis=1)
        assert np.all((q[np.arange(len(y)), i_max] & 7)[normal] == 7)
        err = np.abs(y.astype(np.float64) - deq)
        assert np.all(err[normal] <= (0.5 * S[normal, None]) * (1 + 2.0 ** -20))


def test_e0m3_zero_block(orc):
    codes, s = orc.quantize_block16_ex(np.zeros(16, np.float32), 1.0, orc.E0M3)
    assert s == 0 and not codes.any()


# ---- quantizers under the options ----------------------------------------------------------
def test_rotated_rows_quantize_the_rotated_block(orc):
    """ROTATE = the plain block quantizer applied to the rotated block (structure)."""
    rng = np.random.default_rng(6)
    y = rng.standard_normal((8, 64)).astype(np.float32)
    for fmt in (0, orc.E0M3):
        c1, s1 = orc.quantize_rows(y, 1.0, flags=orc.ROTATE | fmt)
        yr = orc.hadamard16(y.reshape(-1, 16)).reshape(8, 64)
        c2, s2 = orc.quantize_rows(yr, 1.0, flags=fmt)
        assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_rotated_norm_quantize_is_norm_then_rotated_quantize(orc):
    x = synth.bf16_normal(synth.seed_of(60, synth.X), (5, 256))
    ga = synth.bf16_normal(synth.seed_of(60, synth.GAMMA), (256,), 1.0, 0.1)
    for flags in (orc.ROTATE, orc.E0M3, orc.ROTATE | orc.E0M3):
        c1, s1 = orc.quantize_norm(x, "rmsnorm", gamma=ga, eps=1e-6, flags=flags)
        y = orc.norm_rows(x, "rmsnorm", gamma=ga, eps=1e-6)
        c2, s2 = orc.quantize_rows(y, 1.0, flags=flags)
        assert np.array_equal(c1, c2) and np.array_equal(s1, s2)


@pytest.mark.parametrize("flags,qmax", [(0, 6), (1, 6), (2, 7), (3, 7)])
def test_weight_global_scale_and_top_block(orc, flags, qmax):
    """g = amax of the quantized (rotated) values / (qmax * 448); the block holding that
    amax takes the largest scale byte (0x7E = 448) and its element the top magnitude."""
    w = synth.bf16_normal(synth.seed_of(61, synth.W0), (64, 128), 0.0, 0.02)
    codes, sf, g = orc.quantize_weight_ex(w, flags=flags)
    wf = synth.bf16_bits_to_f32(w).reshape(-1, 16)
    vals = orc.hadamard16(wf) if flags & orc.ROTATE else wf
    amax = np.float32(np.abs(vals).max())
    assert np.float32(g) == np.float32(amax / np.float32(qmax * 448))
    flat = np.argmax(np.abs(vals))
    r, b = divmod(flat // 16, 128 // 16)
    assert orc.sf_gather(sf, 64, 128)[r, b] == 0x7E
    q = _unpack(codes).reshape(-1, 16)
    assert q[flat // 16, flat % 16] & 7 == 7


def test_weight_ex_without_options_equals_the_plain_quantizers(orc):
    w = synth.bf16_normal(synth.seed_of(62, synth.W0), (32, 96), 0.0, 0.02)
    for inter in (False, True):
        assert all(np.array_equal(a, b) or a == b
                   for a, b in zip(orc.quantize_weight_ex(w, inter), orc.quantize_weight(w, inter)))
        assert all(np.array_equal(a, b) or a == b
                   for a, b in zip(orc.quantize_weight_ex(w, inter, mse=True), orc.quantize_weight_mse(w, inter)))


def test_rotated_gemm_approximates_the_unrotated_product(orc):
    """Rotating both operands leaves the product alone up to quantization error: the GEMM
    of rotated NVFP4 operands tracks x w^T (fp64, unquantized) as closely as the unrotated
    GEMM does."""
    M, N, K = 16, 64, 512
    x = synth.bf16_normal(synth.seed_of(63, synth.X), (M, K))
    w = synth.bf16_normal(synth.seed_of(63, synth.W0), (N, K), 0.0, 0.02)
    exact = synth.bf16_bits_to_f32(x).astype(np.float64) @ synth.bf16_bits_to_f32(w).astype(np.float64).T
    cos = {}
    for flags in (0, orc.ROTATE):
        ac, asf = orc.quantize_norm(x, "none", flags=flags)
        wc, wsf, gw = orc.quantize_weight_ex(w, flags=flags)
        v = orc.gemm(ac, asf, 1.0, M, wc, wsf, gw, N, K)["v"]
        cos[flags] = (v * exact).sum() / np.sqrt((v * v).sum() * (exact * exact).sum())
    assert cos[orc.ROTATE] > 0.99 and cos[0] > 0.99


@pytest.mark.parametrize("epi", ["bias_gelu_rht", "geglu_rht"])
def test_rotated_fp4_epilogue_structure(orc, epi):
    """The rotated FP4 epilogues: codes = the rotated quantizer on (float)h, and h_out = the
    fp64 rotation of the unrotated epilogue's h."""
    M, N, K = 4, 128, 256
    x = synth.bf16_normal(synth.seed_of(64, synth.X), (M, K))
    w = synth.bf16_normal(synth.seed_of(64, synth.W0), (N, K), 0.0, 0.02)
    bias = synth.bf16_normal(synth.seed_of(64, synth.BIAS0), (N,), 0.0, 0.01)
    ac, asf = orc.quantize_norm(x, "none")
    wc, wsf, gw = orc.quantize_weight(w)
    plain = orc.gemm(ac, asf, 1.0, M, wc, wsf, gw, N, K, epi=epi[:-4], bias=bias)
    rot = orc.gemm(ac, asf, 1.0, M, wc, wsf, gw, N, K, epi=epi, bias=bias)
    n_out = plain["h"].shape[1]
    c2, s2 = orc.quantize_rows(plain["h"].astype(np.float32), 1.0, flags=orc.ROTATE)
    assert np.array_equal(rot["codes"], c2) and np.array_equal(rot["sf"], s2)
    R = scipy.linalg.hadamard(16).astype(np.float64) / 4.0
    want = (plain["h"].reshape(M, n_out // 16, 16) @ R.T).reshape(M, n_out)
    assert np.allclose(rot["h"], want, rtol=0, atol=1e-12 * np.abs(plain["h"]).max())
