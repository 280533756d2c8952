"""Pins of the oracle's block-scaled GEMM and epilogues: brute force against torch fp64
matmul on operands dequantized independently (ml_dtypes decoders, scales chosen
densely by the test), closed forms, one-hot selection, and torch's tanh-GELU."""
import ml_dtypes
import numpy as np
import torch
import torch.nn.functional as F

from vla_action_head_b200 import synth


def _pack(codes):
    """codes [rows, K] (4-bit) -> bytes [rows, K/2], element 2j in the low nibble."""
    c = np.asarray(codes, np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def _place_sf(orc, scales, K):
    rows = scales.shape[0]
    sf = np.zeros(orc.sf_bytes(rows, K), np.uint8)
    for r in range(rows):
        for b in range(scales.shape[1]):
            sf[orc.sf_offset(r, b, K)] = scales[r, b]
    return sf


def _deq(codes, scales, g):
    e = np.asarray(codes, np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    s = np.asarray(scales, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return e * np.repeat(s, 16, axis=1) * g


def _rand_operand(rng, rows, K):
    codes = rng.integers(0, 16, (rows, K), dtype=np.uint8)
    scales = rng.integers(0x20, 0x48, (rows, K // 16), dtype=np.uint8)  # 2^-3 .. 2^2
    return codes, scales


def test_brute_force_tiny(orc):
    rng = np.random.default_rng(3)
    for M, N, K in ((1, 8, 64), (3, 64, 128), (2, 40, 64)):
        ca, sa = _rand_operand(rng, M, K)
        cw, sw = _rand_operand(rng, N, K)
        gA, gW = 0.75, 1.5
        bias = synth.bf16_normal(5, (N,), 0, 0.5)
        res = synth.bf16_normal(6, (M, N), 0, 0.5)
        ref = torch.from_numpy(_deq(ca, sa, gA)) @ torch.from_numpy(_deq(cw, sw, gW)).T
        ref = ref.numpy()
        b = synth.bf16_bits_to_f32(bias).astype(np.float64)
        r = synth.bf16_bits_to_f32(res).astype(np.float64)
        args = (_pack(ca), _place_sf(orc, sa, K), gA, M, _pack(cw), _place_sf(orc, sw, K), gW, N, K)
        for epi, exp in (("none", ref), ("bias", ref + b), ("residual", ref + r),
                         ("bias_residual", ref + b + r)):
            out = orc.gemm(*args, epi=epi, bias=bias, residual=res)["v"]
            assert np.allclose(out, exp, rtol=1e-13, atol=1e-12), epi


def test_all_six_closed_form(orc):
    """Every element code 6 (0x7), one scale per operand: v = 36 K dec(sA) dec(sW) gA gW."""
    M, N, K = 2, 16, 256
    ca = np.full((M, K), 7, np.uint8)
    cw = np.full((N, K), 7, np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)  # 1.0
    sw = np.full((N, K // 16), 0x41, np.uint8)  # 2.25
    out = orc.gemm(_pack(ca), _place_sf(orc, sa, K), 0.5, M, _pack(cw), _place_sf(orc, sw, K),
                   0.25, N, K)["v"]
    assert np.all(out == 36 * K * 1.0 * 2.25 * 0.5 * 0.25)


def test_one_hot_selects_weight_column(orc):
    rng = np.random.default_rng(4)
    M, N, K = 4, 32, 128
    cw, sw = _rand_operand(rng, N, K)
    wd = _deq(cw, sw, 1.25)
    ca = np.zeros((M, K), np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    ks = [0, 17, 64, 127]
    for m, k in enumerate(ks):
        ca[m, k] = 2  # value 1.0
    out = orc.gemm(_pack(ca), _place_sf(orc, sa, K), 1.0, M, _pack(cw), _place_sf(orc, sw, K),
                   1.25, N, K)["v"]
    for m, k in enumerate(ks):
        assert np.array_equal(out[m], wd[:, k])


def test_row_subset_equals_full(orc):
    rng = np.random.default_rng(5)
    M, N, K = 9, 48, 192
    ca, sa = _rand_operand(rng, M, K)
    cw, sw = _rand_operand(rng, N, K)
    args = (_pack(ca), _place_sf(orc, sa, K), 1.0, M, _pack(cw), _place_sf(orc, sw, K), 1.0, N, K)
    full = orc.gemm(*args)["v"]
    sub = orc.gemm(*args, rows=[7, 2, 3])["v"]
    assert np.array_equal(sub, full[[7, 2, 3]])


def test_gelu_tanh_vs_torch(orc):
    z = np.concatenate([np.linspace(-12, 12, 4001), [0.0, 1e-8, -1e-8, 30.0, -30.0]])
    ref = F.gelu(torch.from_numpy(z), approximate="tanh").numpy()
    ours = np.array([orc.gelu_tanh(v) for v in z])
    # 0.5 z (1 + tanh u) cancels for negative z: compare on the scale of |z|
    assert np.all(np.abs(ours - ref) <= 1e-15 * np.abs(z))


def test_fp4_epilogues(orc):
    rng = np.random.default_rng(6)
    M, N, K = 5, 64, 128
    ca, sa = _rand_operand(rng, M, K)
    cw, sw = _rand_operand(rng, N, K)
    bias = synth.bf16_normal(7, (N,), 0, 0.5)
    args = (_pack(ca), _place_sf(orc, sa, K), 0.01, M, _pack(cw), _place_sf(orc, sw, K), 0.02, N, K)
    v0 = orc.gemm(*args, epi="bias", bias=bias)["v"]
    gl = orc.gemm(*args, epi="bias_gelu", bias=bias, g_out=0.5)
    assert np.array_equal(gl["v"], v0)
    zt = torch.from_numpy(v0)
    assert np.all(np.abs(gl["h"] - F.gelu(zt, approximate="tanh").numpy()) <= 1e-15 * np.abs(v0))
    c2, s2 = orc.quantize_rows(gl["h"].astype(np.float32), 0.5)
    assert np.array_equal(gl["codes"], c2) and np.array_equal(gl["sf"], s2)
    gg = orc.gemm(*args, epi="geglu", bias=None, g_out=0.5)
    v1 = orc.gemm(*args, epi="none")["v"]
    h = F.gelu(torch.from_numpy(v1[:, 0::2]), approximate="tanh").numpy() * v1[:, 1::2]
    assert np.all(np.abs(gg["h"] - h) <= 1e-15 * np.abs(v1[:, 0::2] * v1[:, 1::2]))
    c3, s3 = orc.quantize_rows(gg["h"].astype(np.float32), 0.5)
    assert np.array_equal(gg["codes"], c3) and np.array_equal(gg["sf"], s3)


def test_gemm_on_quantized_layer_tracks_bf16_matmul(orc):
    """End to end on the oracle: quantize x and W, GEMM, compare with the bf16 values'
    fp64 matmul.  NVFP4 error is a few percent per element; cosine stays above 0.99."""
    M, N, K = 8, 96, 512
    x = synth.bf16_normal(8, (M, K))
    w = synth.bf16_normal(9, (N, K), 0, 0.02)
    ca, sa = orc.quantize_norm(x, "none", g=1.0)
    cw, sw, gW = orc.quantize_weight(w)
    out = orc.gemm(ca, sa, 1.0, M, cw, sw, gW, N, K)["v"]
    ref = synth.bf16_bits_to_f32(x).astype(np.float64) @ synth.bf16_bits_to_f32(w).astype(np.float64).T
    cos = (out * ref).sum() / np.sqrt((out * out).sum() * (ref * ref).sum())
    assert cos > 0.99
