"""Pins of the oracle's MSE-searched weight block scales ("Pi0.5 Thor NVFP4 End-to-End
Results", §E0M3 Uniform-INT4 Decoder Weights and §Fused GeGLU FFN in the Decoder: the
decoder's NVFP4 weights are MSE-quantized).  The pins do not re-run the oracle's formula:
hand-derived blocks, an exhaustive search written with ml_dtypes' E2M1 / E4M3 codecs, the
exact scaling law of a power-of-two factor, sign symmetry, and the guarantee that the
search never does worse than the amax scale (measured through the dequantizer)."""
import ml_dtypes
import numpy as np
import pytest

from _golden import rows
from vla_action_head_b200 import synth


def _golden():
    out = []
    for line in rows("mse_block_scales.txt"):
        name, g, ys, s_amax, e_amax, s_mse, e_mse, codes = [c.strip() for c in line.split("|")]
        out.append(dict(name=name, g=float(g), y=np.array([float(v) for v in ys.split()], np.float32),
                        s_amax=int(s_amax, 16), e_amax=float(e_amax), s_mse=int(s_mse, 16), e_mse=float(e_mse),
                        codes=np.array([int(c, 16) for c in codes.split()], np.uint8)))
    return out


@pytest.mark.parametrize("case", _golden(), ids=lambda c: c["name"])
def test_hand_derived_blocks(orc, case):
    s, codes = orc.quantize_block16_mse(case["y"], case["g"])
    assert s == case["s_mse"]
    assert np.array_equal(codes, case["codes"])
    assert orc.block_sse(case["y"], case["g"], s)[0] == case["e_mse"]
    # the amax quantizer's byte and its error, as derived by hand
    codes_a = np.zeros(8, np.uint8)
    y = np.ascontiguousarray(case["y"])
    s_a = orc.lib().orc_quantize_block16(y.ctypes.data, case["g"], codes_a.ctypes.data)
    assert s_a == case["s_amax"]
    assert orc.block_sse(case["y"], case["g"], s_a)[0] == case["e_amax"]


# ---- an exhaustive search written independently, with ml_dtypes' codecs -----------------
_E4M3 = np.arange(127, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float32)


def _search(y, g):
    """(best byte, codes) by trying every byte 0x00..0x7E; E in fp64, index order."""
    best, best_e, best_q = None, None, None
    for s in range(127):
        ds = _E4M3[s]
        if ds == 0.0:
            q = np.zeros(16, np.float32)
        else:
            r = np.float32(1.0) / (ds * np.float32(g))
            v = np.clip(y * r, -6.0, 6.0).astype(np.float32)  # satfinite, then round to nearest even
            q = v.astype(ml_dtypes.float4_e2m1fn).astype(np.float32)
        e = 0.0
        for i in range(16):
            d = float(y[i]) - float(q[i]) * float(ds) * float(g)
            e = e + d * d
        if best is None or e < best_e:
            best, best_e, best_q = s, e, q
    nib = best_q.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    codes = (nib[0::2] | (nib[1::2] << 4)).astype(np.uint8)
    return best, codes


def test_exhaustive_search_matches(orc):
    rng = np.random.default_rng(9)
    for trial in range(60):
        # bf16-valued weights of a few shapes of distribution, at assorted global scales
        kind = trial % 3
        if kind == 0:
            y = rng.normal(0.0, 0.02, 16)
        elif kind == 1:
            y = rng.standard_t(3, 16) * 0.05
        else:
            y = rng.normal(0.0, 0.02, 16)
            y[rng.integers(16)] *= 12.0  # one outlier
        y = y.astype(ml_dtypes.bfloat16).astype(np.float32)
        g = float(np.float32(np.abs(y).max() / 2688.0 * rng.choice([0.5, 1.0, 3.0])))
        s, codes = orc.quantize_block16_mse(y, g)
        s_ref, codes_ref = _search(y.astype(np.float32), g)
        assert s == s_ref, (trial, s, s_ref)
        assert np.array_equal(codes, codes_ref), trial


def test_power_of_two_law(orc):
    """Doubling the block moves the best normal scale up one binade (+8 in the byte) and
    multiplies E by 4 exactly."""
    rng = np.random.default_rng(11)
    for _ in range(40):
        y = rng.normal(0.0, 0.3, 16).astype(ml_dtypes.bfloat16).astype(np.float32)
        s1, c1 = orc.quantize_block16_mse(y, 1.0)
        s2, c2 = orc.quantize_block16_mse(2.0 * y, 1.0)
        assert 16 <= s1 and s1 + 8 <= 0x7E
        assert s2 == s1 + 8 and np.array_equal(c1, c2)
        assert orc.block_sse(2.0 * y, 1.0, s2)[0] == 4.0 * orc.block_sse(y, 1.0, s1)[0]


def test_sign_symmetry(orc):
    rng = np.random.default_rng(12)
    for _ in range(40):
        y = rng.normal(0.0, 0.3, 16).astype(np.float32)
        y[np.abs(y) < 1e-3] = 0.5  # no zeros: -0.0 keeps its sign bit
        s1, c1 = orc.quantize_block16_mse(y, 1.0)
        s2, c2 = orc.quantize_block16_mse(-y, 1.0)
        assert s1 == s2 and np.array_equal(c2, c1 ^ 0x88)


def test_never_worse_than_amax_and_same_global_scale(orc):
    """Per block, the MSE choice's squared error (through the fp64 dequantizer) is at most
    the amax choice's; the global scale is the same amax / 2688."""
    N, K = 48, 256
    w = synth.bf16_normal(synth.seed_of(80, synth.W0), (N, K), 0.0, 0.02)
    wf = w.view(ml_dtypes.bfloat16).astype(np.float64)
    ca, sa, ga = orc.quantize_weight(w)
    cm, sm, gm = orc.quantize_weight_mse(w)
    assert ga == gm
    da = orc.dequantize(ca, sa, ga, N, K)
    dm = orc.dequantize(cm, sm, gm, N, K)
    ea = ((wf - da) ** 2).reshape(N, K // 16, 16).sum(-1)
    em = ((wf - dm) ** 2).reshape(N, K // 16, 16).sum(-1)
    assert np.all(em <= ea * (1 + 1e-12) + 1e-300)
    assert em.sum() < 0.95 * ea.sum()  # the search buys a real reduction on Gaussian weights
    assert not np.array_equal(sa, sm)


def test_interleave_permutes_rows(orc):
    N, K = 16, 64
    w = synth.bf16_normal(synth.seed_of(81, synth.W0), (N, K), 0.0, 0.02)
    c0, s0, g0 = orc.quantize_weight_mse(w)
    c1, s1, g1 = orc.quantize_weight_mse(w, interleave_gate_up=True)
    assert g0 == g1
    perm = [(r // 2) if r % 2 == 0 else N // 2 + r // 2 for r in range(N)]
    assert np.array_equal(c1, c0[perm])
    for r in range(N):
        for b in range(K // 16):
            assert s1[orc.sf_offset(r, b, K)] == s0[orc.sf_offset(perm[r], b, K)]
