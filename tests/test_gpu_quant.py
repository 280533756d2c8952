"""GPU parity of the norm -> NVFP4 front-end and the weight quantizer against the oracle.

Encodings are compared byte for byte.  The acceptance bar allows fused-norm code
mismatches only within one fp32 ulp of a rounding boundary, at most 1e-4 of the elements;
the kernel's fp64 row statistics make them identical in practice, which is asserted too
where it holds by construction (plain quantizer, weights)."""
import numpy as np
import pytest

from parity import dev_bf16, dev_f32, host
from vla_action_head_b200 import nvfp4, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _probe():
    nvfp4.probe()


def _gpu_qn(x, kind, params, eps, g):
    xd = dev_f32(x) if x.dtype == np.float32 else dev_bf16(x)
    pd = {k: (dev_bf16(v) if v is not None else None) for k, v in params.items()}
    q = nvfp4.quantize_norm(xd, kind, eps=eps, global_scale=g, **pd)
    return host(q.codes), host(q.sf)


def _crafted_blocks():
    """fp32 blocks exercising every E2M1 tie (amax 3 -> S = 0.5), +-1 ulp around them,
    signed zeros, E4M3 ties of the block scale, subnormal and saturated scales."""
    rows = []
    ties = np.array([0.125, 0.375, 0.625, 0.875, 1.25, 1.75, 2.5], np.float32)
    for t in ties:
        for v in (t, np.nextafter(t, np.float32(9)), np.nextafter(t, np.float32(0))):
            b = np.zeros(16, np.float32)
            b[0] = 3.0
            b[1:8] = v
            b[8:15] = -v
            b[15] = -1e-9
            rows.append(b)
    b = np.full(16, -0.0, np.float32)
    b[0] = 3.0
    rows.append(b)
    rows.append(np.full(16, -0.0, np.float32))
    for a in (6.375, 7.125, 2592.0, 6000.0, 1e-4, 0.0146484375 * 6, 0.0029296875 * 6, 448 * 6 * 1.5):
        b = np.linspace(-a, a, 16).astype(np.float32)
        rows.append(b)
    rng = np.random.default_rng(0)
    r = rng.standard_normal((256, 16)).astype(np.float32)
    r *= np.exp(rng.uniform(-12, 9, (256, 1))).astype(np.float32)
    out = np.concatenate([np.stack(rows), r]).astype(np.float32)
    pad = (-len(out)) % 4
    return np.concatenate([out, np.zeros((pad, 16), np.float32)])


@pytest.mark.parametrize("g", [1.0, 0.37, 2.0 ** -20])
def test_quantizer_canary_bit_exact(orc, g):
    blocks = _crafted_blocks()
    x = blocks.reshape(-1, 64)  # 4 blocks per row
    c, s = _gpu_qn(x, "none", {}, 0.0, g)
    rc, rs = orc.quantize_rows(x, g)
    assert np.array_equal(c, rc), np.argwhere(c != rc)[:8]
    assert np.array_equal(s, rs)


def _params(wl, K, kind):
    p = {}
    if kind == "layernorm":
        p["gamma"] = synth.bf16_normal(synth.seed_of(wl, synth.GAMMA), (K,), 1.0, 0.1)
        p["beta"] = synth.bf16_normal(synth.seed_of(wl, synth.BETA), (K,), 0.0, 0.1)
    elif kind == "rmsnorm":
        p["gamma"] = synth.bf16_normal(synth.seed_of(wl, synth.GAMMA), (K,), 1.0, 0.1)
    elif kind == "adaln":
        p["scale"] = synth.bf16_normal(synth.seed_of(wl, synth.MOD_SCALE), (K,), 0.0, 0.1)
        p["shift"] = synth.bf16_normal(synth.seed_of(wl, synth.MOD_SHIFT), (K,), 0.0, 0.1)
    elif kind == "adarms":
        p["scale"] = synth.bf16_normal(synth.seed_of(wl, synth.MOD_SCALE), (K,), 0.0, 0.1)
    return p


CASES = [  # (workload id, M, K, kind, eps): the configs' front-ends plus ragged / edge shapes
    (1, 41, 256, "layernorm", 1e-5),
    (2, 41, 1536, "adaln", 1e-6),
    (2, 41, 1536, "layernorm", 1e-5),
    (2, 41, 1536, "none", 0.0),
    (3, 50, 1024, "adarms", 1e-6),
    (3, 50, 2048, "none", 0.0),
    (4, 968, 2048, "rmsnorm", 1e-6),
    (7, 1, 16, "layernorm", 1e-5),
    (7, 3, 48, "rmsnorm", 1e-6),
    (7, 129, 4096, "adaln", 1e-6),
    (7, 33, 6144, "adarms", 1e-6),
    (7, 5, 16384, "layernorm", 1e-5),
    (7, 2, 32768, "rmsnorm", 1e-6),
]


@pytest.mark.parametrize("wl,M,K,kind,eps", CASES)
def test_quantize_norm_matches_oracle(orc, wl, M, K, kind, eps):
    x = synth.bf16_normal(synth.seed_of(wl, synth.X), (M, K))
    p = _params(wl, K, kind)
    c, s = _gpu_qn(x, kind, p, eps, 1.0)
    rc, rs = orc.quantize_norm(x, kind, eps=eps, g=1.0, **p)
    frac = (c != rc).mean()
    assert frac <= 1e-4, frac
    assert np.array_equal(s == rs, np.ones_like(s, bool)) or (s != rs).mean() <= 1e-4
    assert np.array_equal(c, rc) and np.array_equal(s, rs)  # fp64 statistics: exact in practice


@pytest.mark.parametrize("kind", ["layernorm", "rmsnorm", "adaln", "adarms"])
def test_fused_equals_two_step_on_gpu(orc, kind):
    """The fused front-end equals norm -> fp32 y -> plain quantizer, both on the GPU; and
    the GPU's fp32 y equals the oracle's."""
    M, K = 50, 1024
    x = synth.bf16_normal(synth.seed_of(9, synth.X), (M, K))
    p = _params(9, K, kind)
    pd = {k: dev_bf16(v) for k, v in p.items()}
    xd = dev_bf16(x)
    fused = nvfp4.quantize_norm(xd, kind, eps=1e-6, **pd)
    y = nvfp4.norm_f32(xd, kind, eps=1e-6, **pd)
    two = nvfp4.quantize_norm(y, "none")
    assert np.array_equal(host(fused.codes), host(two.codes))
    assert np.array_equal(host(fused.sf), host(two.sf))
    y_ref = orc.norm_rows(x, kind, eps=1e-6, **p)
    assert np.array_equal(host(y), y_ref)


def test_edge_rows(orc):
    """Constant rows (LayerNorm -> zero block), +-1e4 outliers, 1e-4-magnitude rows
    (subnormal block scales), all-zero rows."""
    K = 256
    rows = [np.full(K, 3.25), np.zeros(K), synth.normal(5, K) * 1e-4, synth.normal(6, K)]
    rows[3][7] = 1e4
    rows[3][100] = -1e4
    x = synth.f32_to_bf16_bits(np.stack(rows).astype(np.float32))
    for kind in ("layernorm", "none", "rmsnorm"):
        c, s = _gpu_qn(x, kind, {}, 1e-5, 1.0)
        rc, rs = orc.quantize_norm(x, kind, eps=1e-5, g=1.0)
        assert np.array_equal(c, rc) and np.array_equal(s, rs), kind


def test_empty_is_noop():
    import torch
    x = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    out = nvfp4.empty_fp4(1, 64)
    out.codes.fill_(0xAB)
    st = nvfp4.lib().nvfp4_quantize_norm(x.data_ptr(), 0, 0, 64, 64, 0, None, None, None, None, 0.0, 1.0,
                                         out.codes.data_ptr(), out.sf.data_ptr(), None)
    torch.cuda.synchronize()
    assert st == 0 and int(out.codes[0, 0]) == 0xAB


@pytest.mark.parametrize("N,K,inter", [(512, 256, False), (6144, 1536, False), (8192, 1024, True),
                                       (64, 48, False)])
def test_weight_quantizer_matches_oracle(orc, N, K, inter):
    w = synth.bf16_normal(synth.seed_of(5, synth.W0), (N, K), 0.0, 0.02)
    q = nvfp4.quantize_weight(dev_bf16(w), interleave_gate_up=inter)
    rc, rs, rg = orc.quantize_weight(w, interleave_gate_up=inter)
    assert np.float32(q.global_scale) == np.float32(rg)
    assert np.array_equal(host(q.codes), rc)
    assert np.array_equal(host(q.sf), rs)


def _weights(kind, seed, N, K):
    """bf16 weights: Gaussian, heavy-tailed (a few large values per row), or Gaussian rows
    of very different magnitudes (small blocks take subnormal E4M3 scales)."""
    w = synth.bf16_normal(synth.seed_of(seed, synth.W0), (N, K), 0.0, 0.02)
    f = synth.bf16_bits_to_f32(w)
    if kind == "outliers":
        f[:, ::37] *= 25.0
    elif kind == "row_scales":
        f *= np.logspace(-6, 0, N, dtype=np.float32)[:, None]
    return synth.f32_to_bf16_bits(f) if kind != "gauss" else w


@pytest.mark.parametrize("N,K,inter,kind", [(64, 256, False, "gauss"), (130, 1024, True, "gauss"),
                                            (48, 2048, False, "outliers"), (96, 512, False, "row_scales"),
                                            (256, 4096, True, "gauss"), (16, 48, False, "gauss")])
def test_weight_mse_scales_match_oracle(orc, N, K, inter, kind):
    """MSE-searched block scales: codes, scale bytes and global scale bit for bit."""
    w = _weights(kind, 6, N, K)
    q = nvfp4.quantize_weight(dev_bf16(w), interleave_gate_up=inter, scales="mse")
    rc, rs, rg = orc.quantize_weight_mse(w, interleave_gate_up=inter)
    assert np.float32(q.global_scale) == np.float32(rg)
    assert np.array_equal(host(q.sf), rs)
    assert np.array_equal(host(q.codes), rc)


def test_weight_mse_never_worse_than_amax(orc):
    """On the device results: per block, dequantized squared error of the MSE scales is at
    most that of the amax scales; the two differ on most blocks of Gaussian weights."""
    N, K = 128, 1024
    w = _weights("gauss", 7, N, K)
    wd = dev_bf16(w)
    qa = nvfp4.quantize_weight(wd)
    qm = nvfp4.quantize_weight(wd, scales="mse")
    wf = synth.bf16_bits_to_f32(w).astype(np.float64)
    da = orc.dequantize(host(qa.codes), host(qa.sf), qa.global_scale, N, K)
    dm = orc.dequantize(host(qm.codes), host(qm.sf), qm.global_scale, N, K)
    ea = ((wf - da) ** 2).reshape(N, K // 16, 16).sum(-1)
    em = ((wf - dm) ** 2).reshape(N, K // 16, 16).sum(-1)
    assert np.all(em <= ea * (1 + 1e-12) + 1e-300)
    assert (em < ea).mean() > 0.3


def test_weight_mse_rejects_bad_scales_argument():
    with pytest.raises(ValueError):
        nvfp4.quantize_weight(dev_bf16(synth.bf16_normal(1, (16, 64))), scales="max")
