"""Pins of the oracle's gated residual update and its bf16 rounding ("Pi0.5 Thor NVFP4
End-to-End Results", §Implemented Path: gated residual update + Pi0.5 AdaRMSNorm + gate
output + NVFP4/SFA in one launch before Gate+Up and the next layer's QKV)."""
import ml_dtypes
import numpy as np
import pytest

from _golden import rows
from vla_action_head_b200 import synth


def _bf16(vals):
    return np.asarray(vals, np.float32).astype(ml_dtypes.bfloat16).view(np.uint16)


def test_f32_to_bf16_matches_ml_dtypes(orc):
    rng = np.random.default_rng(7)
    v = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 200000),
        # every tie between adjacent bf16 values over a range of exponents, and +-1 fp32 ulp
        ((np.arange(-300, 300, dtype=np.int64)[:, None] * 2 + 1) * 2 ** 15 +
         (np.arange(40, 200)[None, :] << 23)).astype(np.uint32).view(np.float32).ravel(),
        np.array([0.0, -0.0, np.inf, -np.inf, 3.4e38, -3.4e38, 1e-40, -1e-40, 1.17549435e-38], np.float32),
    ]).astype(np.float32)
    ties = v[(v.view(np.uint32) & 0xFFFF) == 0x8000]
    assert ties.size > 1000
    v = np.concatenate([v, np.nextafter(ties, np.float32(np.inf)), np.nextafter(ties, np.float32(-np.inf))])
    assert np.array_equal(orc.f32_to_bf16(v), v.astype(ml_dtypes.bfloat16).view(np.uint16))
    nan = orc.f32_to_bf16(np.array([np.nan, -np.nan], np.float32))
    assert np.all(np.isnan(nan.view(ml_dtypes.bfloat16).astype(np.float32)))


def test_gated_residual_golden(orc):
    for line in rows("gated_residual.txt"):
        xs, gs, ds, hs = line.split()
        x, g, d = _bf16([float(xs)]), _bf16([float(gs)]), _bf16([float(ds)])
        # the fixture's inputs are exact bf16 values
        for s, b in ((xs, x), (gs, g), (ds, d)):
            assert float(b.view(ml_dtypes.bfloat16)[0]) == float(s), s
        h = orc.gated_residual(x.reshape(1, 1), d.reshape(1, 1), g)
        assert int(h[0, 0]) == int(hs, 16), line


def test_gated_residual_special_cases(orc):
    x = synth.bf16_normal(1, (5, 48))
    d = synth.bf16_normal(2, (5, 48))
    zero = np.zeros((5, 48), np.uint16)
    assert np.array_equal(orc.gated_residual(x, zero, _bf16(np.full(48, 3.0))), x)
    assert np.array_equal(orc.gated_residual(x, d, np.zeros(48, np.uint16)), x)
    assert np.array_equal(orc.gated_residual(x, d, None), orc.gated_residual(x, d, _bf16(np.ones(48))))
    neg = (x ^ 0x8000).astype(np.uint16)
    assert np.all(orc.gated_residual(x, neg, None) == 0)  # x + (-x) = +0


def test_gated_residual_against_numpy(orc):
    """Independent arithmetic: numpy fp32 product and sum, ml_dtypes rounding."""
    x = synth.bf16_normal(3, (17, 1024))
    d = synth.bf16_normal(4, (17, 1024))
    g = synth.bf16_normal(5, (1024,), 0.0, 0.5)
    f = lambda b: b.view(ml_dtypes.bfloat16).astype(np.float32)  # noqa: E731
    want = (f(x) + f(g)[None, :] * f(d)).astype(ml_dtypes.bfloat16).view(np.uint16)
    assert np.array_equal(orc.gated_residual(x, d, g), want)


@pytest.mark.parametrize("kind", ["adarms", "rmsnorm", "layernorm", "adaln"])
def test_residual_front_end_reductions(orc, kind):
    """With gate 0 the fused front-end is the plain norm of x; with d = 0 too."""
    x = synth.bf16_normal(6, (9, 256))
    d = synth.bf16_normal(7, (9, 256))
    sc = synth.bf16_normal(8, (256,), 0.0, 0.1)
    sh = synth.bf16_normal(9, (256,), 0.0, 0.1)
    ga = synth.bf16_normal(10, (256,), 1.0, 0.1)
    kw = dict(gamma=ga, beta=sh, scale=sc, shift=sh, eps=1e-6)
    h, c, s = orc.residual_quantize_norm(x, d, np.zeros(256, np.uint16), kind, **kw)
    rc, rs = orc.quantize_norm(x, kind, **kw)
    assert np.array_equal(h, x) and np.array_equal(c, rc) and np.array_equal(s, rs)
    h, c, s = orc.residual_quantize_norm(x, np.zeros_like(x), sc, kind, **kw)
    assert np.array_equal(h, x) and np.array_equal(c, rc) and np.array_equal(s, rs)
