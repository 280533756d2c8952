"""GPU parity of the quantizer options against the oracle: the 16-point Hadamard block
rotation ("Pi0.5 Thor NVFP4 End-to-End Results", §Full-INT4 Decoder Activations + Hadamard
Rotation) and uniform INT4 elements (same page, §E0M3 Uniform-INT4 Decoder Weights) in the
norm front-end, the gated residual front-end and the weight quantizers (bit for bit), the
rotated FP4-output epilogues, and GEMMs on rotated operands (the GEMM bar)."""
import ctypes as C

import numpy as np
import pytest

from _golden import rows
from parity import check_fp4_output, check_gemm_bf16, dev_bf16, dev_f32, host, to_gpu_fp4
from vla_action_head_b200 import nvfp4, synth

pytestmark = pytest.mark.gpu

FLAGS = {"rot": (True, "e2m1"), "e0m3": (False, "e0m3"), "rot_e0m3": (True, "e0m3")}


@pytest.fixture(scope="module", autouse=True)
def _probe():
    nvfp4.probe()


def _oflags(orc, rotate, fmt):
    return (orc.ROTATE if rotate else 0) | (orc.E0M3 if fmt == "e0m3" else 0)


def _crafted():
    """fp32 blocks: the hand-derived rotation cases, the E0M3 worked examples, every E0M3
    tie at scale 1 (amax 7), signed zeros, subnormal and saturated scales, random blocks
    over 21 binades."""
    out = []
    for r in rows("hadamard16.txt"):
        out.append(np.array([float.fromhex(t) for t in r.split("|")[0].split()], np.float32))
    for r in rows("e0m3_blocks.txt"):
        out.append(np.array([float(t) for t in r.split("|")[1].split()], np.float32))
    ties = np.arange(0.5, 7.0, 1.0, dtype=np.float32)
    for t in ties:
        for v in (t, np.nextafter(t, np.float32(9)), np.nextafter(t, np.float32(0))):
            b = np.zeros(16, np.float32)
            b[0] = 7.0
            b[1:8] = v
            b[8:15] = -v
            b[15] = -1e-9
            out.append(b)
    out.append(np.full(16, -0.0, np.float32))
    for a in (1e-4, 0.02, 7.5 * 448 * 2):
        out.append(np.linspace(-a, a, 16).astype(np.float32))
    rng = np.random.default_rng(3)
    r = rng.standard_normal((252, 16)).astype(np.float32)
    r *= np.exp(rng.uniform(-12, 9, (252, 1))).astype(np.float32)
    blocks = np.concatenate([np.stack(out), r])
    pad = (-len(blocks)) % 4
    return np.concatenate([blocks, np.zeros((pad, 16), np.float32)]).reshape(-1, 64)


@pytest.mark.parametrize("opt", list(FLAGS))
@pytest.mark.parametrize("g", [1.0, 0.37])
def test_plain_quantizer_options_bit_exact(orc, opt, g):
    rotate, fmt = FLAGS[opt]
    x = _crafted()
    q = nvfp4.quantize_norm(dev_f32(x), "none", global_scale=g, rotate=rotate, fmt=fmt)
    rc, rs = orc.quantize_rows(x, g, flags=_oflags(orc, rotate, fmt))
    assert np.array_equal(host(q.codes), rc), np.argwhere(host(q.codes) != rc)[:8]
    assert np.array_equal(host(q.sf), rs)


def _params(wl, K, kind):
    p = {}
    if kind in ("layernorm", "rmsnorm"):
        p["gamma"] = synth.bf16_normal(synth.seed_of(wl, synth.GAMMA), (K,), 1.0, 0.1)
    if kind == "layernorm":
        p["beta"] = synth.bf16_normal(synth.seed_of(wl, synth.BETA), (K,), 0.0, 0.1)
    if kind in ("adaln", "adarms"):
        p["scale"] = synth.bf16_normal(synth.seed_of(wl, synth.MOD_SCALE), (K,), 0.0, 0.1)
    if kind == "adaln":
        p["shift"] = synth.bf16_normal(synth.seed_of(wl, synth.MOD_SHIFT), (K,), 0.0, 0.1)
    return p


@pytest.mark.parametrize("opt", list(FLAGS))
@pytest.mark.parametrize("kind,M,K", [("adaln", 41, 1536), ("layernorm", 41, 1536), ("adarms", 50, 1024),
                                      ("rmsnorm", 968, 2048), ("none", 33, 4096), ("rmsnorm", 3, 16384)])
def test_norm_quantize_options_bit_exact(orc, opt, kind, M, K):
    rotate, fmt = FLAGS[opt]
    wl = 70
    x = synth.bf16_normal(synth.seed_of(wl, synth.X), (M, K))
    p = _params(wl, K, kind)
    eps = 1e-5 if kind == "layernorm" else 1e-6
    q = nvfp4.quantize_norm(dev_bf16(x), kind, eps=eps, rotate=rotate, fmt=fmt,
                            **{k: dev_bf16(v) for k, v in p.items()})
    rc, rs = orc.quantize_norm(x, kind, eps=eps, flags=_oflags(orc, rotate, fmt), **p)
    assert np.array_equal(host(q.codes), rc)
    assert np.array_equal(host(q.sf), rs)


@pytest.mark.parametrize("opt", ["rot", "rot_e0m3"])
def test_residual_front_end_options_bit_exact(orc, opt):
    import torch
    rotate, fmt = FLAGS[opt]
    M, K, wl = 50, 1024, 71
    x = synth.bf16_normal(synth.seed_of(wl, synth.X), (M, K))
    d = synth.bf16_normal(synth.seed_of(wl, synth.RESIDUAL), (M, K))
    gate = synth.bf16_normal(synth.seed_of(wl, synth.GAMMA), (K,), 0.0, 0.5)
    sc = synth.bf16_normal(synth.seed_of(wl, synth.MOD_SCALE), (K,), 0.0, 0.1)
    h_out = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    h, q = nvfp4.residual_quantize_norm(dev_bf16(x), dev_bf16(d), dev_bf16(gate), "adarms", scale=dev_bf16(sc),
                                        eps=1e-6, h_out=h_out, rotate=rotate, fmt=fmt)
    rh = orc.gated_residual(x, d, gate)
    rc, rs = orc.quantize_norm(rh, "adarms", scale=sc, eps=1e-6, flags=_oflags(orc, rotate, fmt))
    assert np.array_equal(host(h), rh)
    assert np.array_equal(host(q.codes), rc) and np.array_equal(host(q.sf), rs)


@pytest.mark.parametrize("opt,scales", [("rot", "amax"), ("e0m3", "amax"), ("rot_e0m3", "amax"), ("rot", "mse")])
@pytest.mark.parametrize("inter", [False, True])
def test_weight_quantizer_options_bit_exact(orc, opt, scales, inter):
    rotate, fmt = FLAGS[opt]
    N, K = (512, 1024) if scales == "amax" else (128, 512)
    w = synth.bf16_normal(synth.seed_of(72, synth.W0), (N, K), 0.0, 0.02)
    w[3, 17] = synth.f32_to_bf16_bits(np.array([0.7], np.float32))[0]  # one outlier
    q = nvfp4.quantize_weight(dev_bf16(w), interleave_gate_up=inter, scales=scales, rotate=rotate, fmt=fmt)
    rc, rs, g = orc.quantize_weight_ex(w, inter, flags=_oflags(orc, rotate, fmt), mse=scales == "mse")
    assert np.float32(q.global_scale) == np.float32(g)
    assert np.array_equal(host(q.codes), rc)
    assert np.array_equal(host(q.sf), rs)


def test_weight_quantizer_rejects_mse_with_e0m3():
    import torch
    w = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nvfp4.NVFP4Error) as err:
        nvfp4.quantize_weight(w, scales="mse", fmt="e0m3")
    assert err.value.status == 1


def test_norm_quantizer_rejects_unknown_flags():
    import torch
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    q = nvfp4.empty_fp4(4, 64)
    st = nvfp4.lib().nvfp4_quantize_norm_ex(C.c_void_p(x.data_ptr()), 0, 4, 64, 64, 0, None, None, None, None,
                                            1e-6, 1.0, 8, C.c_void_p(q.codes.data_ptr()),
                                            C.c_void_p(q.sf.data_ptr()), None)
    assert st == 1


# ---- GEMMs on rotated operands --------------------------------------------------------------
def _rotated_operands(orc, wl, M, N, K, inter=False):
    x = synth.bf16_normal(synth.seed_of(wl, synth.X), (M, K))
    w = synth.bf16_normal(synth.seed_of(wl, synth.W0), (N, K), 0.0, 0.02)
    ac, asf = orc.quantize_norm(x, "none", flags=orc.ROTATE)
    wc, wsf, gw = orc.quantize_weight_ex(w, inter, flags=orc.ROTATE)
    return x, w, (ac, asf, 1.0), (wc, wsf, gw)


@pytest.mark.parametrize("M,N,K,epi", [(41, 4608, 1536, "bias"), (41, 1536, 6144, "bias_residual"),
                                       (50, 2560, 1024, "none"), (50, 1024, 4096, "residual"),
                                       (968, 2560, 2048, "none")])
def test_rotated_gemm_against_oracle(orc, M, N, K, epi):
    """Rotated operands (quantized by the oracle), the default GEMM schedule: the GEMM bar
    against the oracle's GEMM of the same codes, and close to the unrotated x w^T."""
    wl = 73
    x, w, (ac, asf, ga), (wc, wsf, gw) = _rotated_operands(orc, wl, M, N, K)
    bias = synth.bf16_normal(synth.seed_of(wl, synth.BIAS0), (N,), 0.0, 0.01) if "bias" in epi else None
    res = synth.bf16_normal(synth.seed_of(wl, synth.RESIDUAL), (M, N)) if "residual" in epi else None
    sel = None if M <= 128 else [0, 1, 127, 128, 500, 967]
    ref = orc.gemm(ac, asf, ga, M, wc, wsf, gw, N, K, epi=epi, bias=bias, residual=res, rows=sel)["v"]
    out = nvfp4.gemm(to_gpu_fp4(ac, asf, ga, M, K), to_gpu_fp4(wc, wsf, gw, N, K), epi,
                     bias=dev_bf16(bias) if bias is not None else None,
                     residual=dev_bf16(res) if res is not None else None)
    got = host(out) if sel is None else host(out)[sel]
    check_gemm_bf16(got, ref, what=("rotated", M, N, K, epi))
    # the rotation is inert on the product: the unrotated fp64 x w^T (+ terms) is close
    xs = synth.bf16_bits_to_f32(x).astype(np.float64)
    if sel is not None:
        xs = xs[sel]
    plain = xs @ synth.bf16_bits_to_f32(w).astype(np.float64).T
    if bias is not None:
        plain = plain + synth.bf16_bits_to_f32(bias).astype(np.float64)
    if res is not None:
        rr = synth.bf16_bits_to_f32(res).astype(np.float64)
        plain = plain + (rr if sel is None else rr[sel])
    g = got.astype(np.uint32) << 16
    g = g.view(np.float32).astype(np.float64)
    cos = (g * plain).sum() / np.sqrt((g * g).sum() * (plain * plain).sum())
    assert cos > 0.99, cos


@pytest.mark.parametrize("M,N,K,epi", [(41, 6144, 1536, "bias_gelu_rht"), (50, 8192, 1024, "geglu_rht"),
                                       (300, 1024, 768, "geglu_rht"), (41, 512, 512, "bias_gelu_rht")])
def test_rotated_fp4_epilogues_against_oracle(orc, M, N, K, epi):
    """The rotated FP4-output epilogues (default schedule; M = 300 on the many-row kernel)
    under the FP4-output acceptance rule, with h the fp64 rotation of the oracle's h."""
    wl = 74
    _, _, (ac, asf, ga), (wc, wsf, gw) = _rotated_operands(orc, wl, M, N, K, inter=epi.startswith("geglu"))
    bias = synth.bf16_normal(synth.seed_of(wl, synth.BIAS0), (N,), 0.0, 0.01) if epi.startswith("bias") else None
    sel = None if M <= 128 else [0, 5, 127, 128, 255, 299]
    ref = orc.gemm(ac, asf, ga, M, wc, wsf, gw, N, K, epi=epi, bias=bias, rows=sel)
    out = nvfp4.gemm(to_gpu_fp4(ac, asf, ga, M, K), to_gpu_fp4(wc, wsf, gw, N, K), epi,
                     bias=dev_bf16(bias) if bias is not None else None)
    n_out = N // 2 if epi.startswith("geglu") else N
    check_fp4_output(orc, host(out.codes), host(out.sf), ref["codes"], ref["sf"], ref["h"], 1.0, M, n_out,
                     what=(M, N, K, epi), sel=sel)


def test_rotated_chain_gpu_quantized(orc):
    """The rotated decoder MLP chain on the GPU: rotated AdaRMS -> FP4 and rotated weights
    (bit-exact with the oracle), gate/up -> GeGLU -> rotated FP4 (the FP4-output rule), and
    the down GEMM on the GPU's rotated weights (the GEMM bar)."""
    M, H, F, wl = 50, 1024, 2048, 75
    x = synth.bf16_normal(synth.seed_of(wl, synth.X), (M, H))
    sc = synth.bf16_normal(synth.seed_of(wl, synth.MOD_SCALE), (H,), 0.0, 0.1)
    w1 = synth.bf16_normal(synth.seed_of(wl, synth.W0), (2 * F, H), 0.0, 0.02)
    w2 = synth.bf16_normal(synth.seed_of(wl, synth.W0 + 1), (H, F), 0.0, 0.02)
    a = nvfp4.quantize_norm(dev_bf16(x), "adarms", scale=dev_bf16(sc), eps=1e-6, rotate=True)
    q1 = nvfp4.quantize_weight(dev_bf16(w1), interleave_gate_up=True, rotate=True)
    q2 = nvfp4.quantize_weight(dev_bf16(w2), rotate=True)
    u = nvfp4.gemm(a, q1, "geglu_rht")
    ac, asf = orc.quantize_norm(x, "adarms", scale=sc, eps=1e-6, flags=orc.ROTATE)
    c1, s1, g1 = orc.quantize_weight_ex(w1, True, flags=orc.ROTATE)
    c2, s2, g2 = orc.quantize_weight_ex(w2, False, flags=orc.ROTATE)
    assert np.array_equal(host(a.codes), ac) and np.array_equal(host(a.sf), asf)
    assert np.array_equal(host(q1.codes), c1) and np.float32(q1.global_scale) == np.float32(g1)
    assert np.array_equal(host(q2.codes), c2) and np.array_equal(host(q2.sf), s2)
    r1 = orc.gemm(ac, asf, 1.0, M, c1, s1, g1, 2 * F, H, epi="geglu_rht")
    check_fp4_output(orc, host(u.codes), host(u.sf), r1["codes"], r1["sf"], r1["h"], 1.0, M, F, what="chain u")
    # the down GEMM on the GPU's rotated weights, fed the oracle's rotated u
    y = nvfp4.gemm(to_gpu_fp4(r1["codes"], r1["sf"], 1.0, M, F), q2, "residual", residual=dev_bf16(x))
    ref = orc.gemm(r1["codes"], r1["sf"], 1.0, M, c2, s2, g2, H, F, epi="residual", residual=x)["v"]
    check_gemm_bf16(host(y), ref, what="chain y")
    nvfp4.device_status()
