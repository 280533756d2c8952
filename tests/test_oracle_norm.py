"""Pins of the oracle's norm front-ends against torch's fp64 library routines
(layer_norm, rms_norm), closed forms of the modulation, and the fused == two-step
structure."""
import numpy as np
import torch
import torch.nn.functional as F

from vla_action_head_b200 import synth

F32_EPS = 2.0 ** -24


def _x(seed, rows, K, std=1.0, mean=0.0):
    return synth.bf16_normal(seed, (rows, K), mean, std)


def _f(b):
    return torch.from_numpy(synth.bf16_bits_to_f32(b).astype(np.float64))


def _close(y, ref, scale):
    """fp32 result vs fp64 reference: a few roundings of terms of size `scale`."""
    err = np.abs(y.astype(np.float64) - ref)
    assert np.all(err <= 8 * F32_EPS * scale + 1e-30), float(np.max(err / (scale + 1e-30)))


def test_layernorm_vs_torch(orc):
    x = _x(1, 7, 1536)
    ga = synth.bf16_normal(2, (1536,), 1.0, 0.1)
    be = synth.bf16_normal(3, (1536,), 0.0, 0.1)
    y = orc.norm_rows(x, "layernorm", gamma=ga, beta=be, eps=1e-5)
    ref = F.layer_norm(_f(x), (1536,), _f(ga), _f(be), eps=1e-5).numpy()
    n = F.layer_norm(_f(x), (1536,), eps=1e-5).numpy()
    _close(y, ref, np.abs(n * _f(ga).numpy()) + np.abs(_f(be).numpy()))


def test_rmsnorm_vs_torch(orc):
    x = _x(4, 5, 2048, 2.0, 0.3)
    ga = synth.bf16_normal(5, (2048,), 1.0, 0.1)
    y = orc.norm_rows(x, "rmsnorm", gamma=ga, eps=1e-6)
    ref = F.rms_norm(_f(x), (2048,), _f(ga), eps=1e-6).numpy()
    _close(y, ref, np.abs(ref))


def test_adaln_reduces_to_layernorm(orc):
    x = _x(6, 4, 512)
    z = np.zeros(512, np.uint16)  # bf16 +0
    y = orc.norm_rows(x, "adaln", scale=z, shift=z, eps=1e-6)
    ref = F.layer_norm(_f(x), (512,), eps=1e-6).numpy()
    _close(y, ref, np.abs(ref))


def test_adaln_scale_minus_one_gives_shift(orc):
    """(1 + scale) with scale = -1 zeroes the normalized term: y == shift exactly."""
    x = _x(7, 3, 256)
    minus1 = synth.f32_to_bf16_bits(np.full(256, -1.0, np.float32))
    sh = synth.bf16_normal(8, (256,), 0.0, 0.1)
    y = orc.norm_rows(x, "adaln", scale=minus1, shift=sh)
    assert np.array_equal(y, np.broadcast_to(synth.bf16_bits_to_f32(sh), y.shape))


def test_adaln_moments(orc):
    """Constant scale s and shift c: each row has mean c and std (1+s) (population)."""
    x = _x(9, 6, 1536)
    s, c = 0.25, -0.5
    sc = synth.f32_to_bf16_bits(np.full(1536, s, np.float32))
    sh = synth.f32_to_bf16_bits(np.full(1536, c, np.float32))
    y = orc.norm_rows(x, "adaln", scale=sc, shift=sh, eps=1e-6).astype(np.float64)
    assert np.allclose(y.mean(1), c, atol=1e-5)
    assert np.allclose(y.std(1), 1 + s, rtol=1e-4)


def test_adarms_reduces_to_rmsnorm_and_shift(orc):
    x = _x(10, 4, 1024)
    z = np.zeros(1024, np.uint16)
    y = orc.norm_rows(x, "adarms", scale=z, eps=1e-6)
    ref = F.rms_norm(_f(x), (1024,), eps=1e-6).numpy()
    _close(y, ref, np.abs(ref))
    sc = synth.bf16_normal(11, (1024,), 0.0, 0.1)
    y1 = orc.norm_rows(x, "adarms", scale=sc, eps=1e-6).astype(np.float64)
    opl = 1.0 + synth.bf16_bits_to_f32(sc).astype(np.float64)
    _close(y1, ref * opl, np.abs(ref * opl))
    minus1 = synth.f32_to_bf16_bits(np.full(1024, -1.0, np.float32))
    sh = synth.bf16_normal(12, (1024,), 0.0, 0.1)
    y2 = orc.norm_rows(x, "adarms", scale=minus1, shift=sh)
    assert np.array_equal(y2, np.broadcast_to(synth.bf16_bits_to_f32(sh), y2.shape))


def test_layernorm_constant_row_is_zero_block(orc):
    x = synth.f32_to_bf16_bits(np.full((2, 64), 3.25, np.float32))
    y = orc.norm_rows(x, "layernorm", eps=1e-5)
    assert not np.any(y)
    codes, sf = orc.quantize_norm(x, "layernorm", eps=1e-5)
    assert not codes.any() and not sf.any()


def test_none_is_identity(orc):
    x = np.random.default_rng(0).standard_normal((3, 80)).astype(np.float32)
    assert np.array_equal(orc.norm_rows(x, "none"), x)
    xb = _x(13, 3, 80)
    assert np.array_equal(orc.norm_rows(xb, "none"), synth.bf16_bits_to_f32(xb))


def test_fused_equals_two_step(orc):
    """Fused norm -> FP4 equals norm followed by the plain quantizer on the same fp32 y."""
    K = 1536
    x = _x(14, 9, K)
    ga = synth.bf16_normal(15, (K,), 1.0, 0.1)
    be = synth.bf16_normal(16, (K,), 0.0, 0.1)
    sc = synth.bf16_normal(17, (K,), 0.0, 0.1)
    sh = synth.bf16_normal(18, (K,), 0.0, 0.1)
    for kind, kw in (("layernorm", dict(gamma=ga, beta=be)), ("rmsnorm", dict(gamma=ga)),
                     ("adaln", dict(scale=sc, shift=sh)), ("adarms", dict(scale=sc)),
                     ("none", {})):
        for g in (1.0, 0.3):
            c1, s1 = orc.quantize_norm(x, kind, eps=1e-6, g=g, **kw)
            y = orc.norm_rows(x, kind, eps=1e-6, **kw)
            c2, s2 = orc.quantize_rows(y, g)
            assert np.array_equal(c1, c2) and np.array_equal(s1, s2), kind
