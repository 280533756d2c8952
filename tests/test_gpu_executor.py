"""The layer executor (one cooperative launch per program) against the oracle and against
the standalone calls.  Norm ops are byte-exact; GEMM ops meet the GEMM bar; whole layers
and stacks agree with the standalone path within the GEMM bar."""
import numpy as np
import pytest

from parity import bf16_to_f64, check_fp4_output, check_gemm_bf16, dev_bf16, host, to_gpu_fp4
from vla_action_head_b200 import layers, nvfp4, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _probe():
    nvfp4.probe()


def _run_prog(ops):
    import torch
    prog = nvfp4.Program(ops)
    prog.run()
    torch.cuda.synchronize()
    nvfp4.device_status()
    return prog


@pytest.mark.parametrize("kind,K", [("layernorm", 1536), ("adaln", 1536), ("adarms", 1024), ("none", 2048),
                                    ("rmsnorm", 256)])
def test_norm_op_matches_oracle(orc, kind, K):
    M = 41
    x = synth.bf16_normal(synth.seed_of(21, synth.X), (M, K))
    p = {}
    if kind in ("layernorm", "rmsnorm"):
        p["gamma"] = synth.bf16_normal(synth.seed_of(21, synth.GAMMA), (K,), 1.0, 0.1)
    if kind == "layernorm":
        p["beta"] = synth.bf16_normal(synth.seed_of(21, synth.BETA), (K,), 0.0, 0.1)
    if kind in ("adaln", "adarms"):
        p["scale"] = synth.bf16_normal(synth.seed_of(21, synth.MOD_SCALE), (K,), 0.0, 0.1)
    if kind == "adaln":
        p["shift"] = synth.bf16_normal(synth.seed_of(21, synth.MOD_SHIFT), (K,), 0.0, 0.1)
    out = nvfp4.empty_fp4(M, K)
    pd = {k: dev_bf16(v) for k, v in p.items()}
    xd = dev_bf16(x)
    _run_prog([nvfp4.op_norm(xd, out, kind, eps=1e-6, **pd)])
    rc, rs = orc.quantize_norm(x, kind, eps=1e-6, **p)
    assert np.array_equal(host(out.codes), rc) and np.array_equal(host(out.sf), rs)


@pytest.mark.parametrize("M,N,K,epi", [(41, 4608, 1536, "bias"), (41, 1536, 1536, "bias_residual"),
                                       (41, 6144, 1536, "bias_gelu"), (41, 1536, 6144, "bias_residual"),
                                       (50, 2560, 1024, "none"), (50, 8192, 1024, "geglu"),
                                       (50, 1024, 4096, "residual"), (1, 512, 256, "bias"), (64, 256, 96, "bias")])
def test_gemm_op_matches_oracle(orc, M, N, K, epi):
    import torch
    x = synth.bf16_normal(synth.seed_of(22, synth.X), (M, K))
    w = synth.bf16_normal(synth.seed_of(22, synth.W0), (N, K), 0.0, 0.02)
    ac, asf = orc.quantize_norm(x, "none")
    wc, wsf, gw = orc.quantize_weight(w, interleave_gate_up=(epi == "geglu"))
    uses_bias = epi in ("bias", "bias_residual", "bias_gelu")
    uses_res = epi in ("residual", "bias_residual")
    bias = synth.bf16_normal(synth.seed_of(22, synth.BIAS0), (N,), 0.0, 0.01) if uses_bias else None
    res = synth.bf16_normal(synth.seed_of(22, synth.RESIDUAL), (M, N)) if uses_res else None
    ref = orc.gemm(ac, asf, 1.0, M, wc, wsf, gw, N, K, epi=epi, bias=bias, residual=res)
    A, W = to_gpu_fp4(ac, asf, 1.0, M, K), to_gpu_fp4(wc, wsf, gw, N, K)
    if epi in ("bias_gelu", "geglu"):
        n_out = N // 2 if epi == "geglu" else N
        out = nvfp4.empty_fp4(M, n_out)
    else:
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    _run_prog([nvfp4.op_gemm(A, W, epi, bias=dev_bf16(bias) if uses_bias else None,
                             residual=dev_bf16(res) if uses_res else None, out=out)])
    if epi in ("bias_gelu", "geglu"):
        check_fp4_output(orc, host(out.codes), host(out.sf), ref["codes"], ref["sf"], ref["h"], 1.0, M,
                         out.K, what=(M, N, K, epi))
    else:
        check_gemm_bf16(host(out), ref["v"], what=(M, N, K, epi))


def _stack_compare(cls, n_layers, M, H, ctx_dim):
    import torch
    ws = nvfp4.Workspace("cuda")
    lays = [cls(layer=i, ws=ws) for i in range(n_layers)]
    x0 = synth.bf16_normal_torch(synth.seed_of(23, synth.X), (M, H), device="cuda")
    ctx = synth.bf16_normal_torch(synth.seed_of(23, synth.CONTEXT), (M, ctx_dim), device="cuda")
    # standalone calls
    a = [x0.clone(), torch.empty_like(x0)]
    for i, lay in enumerate(lays):
        lay.forward(a[i % 2], ctx, a[(i + 1) % 2])
    ref = host(a[n_layers % 2]).copy()
    # the same stack as one program
    b = [x0.clone(), torch.empty_like(x0)]
    ops = []
    for i, lay in enumerate(lays):
        ops += lay.ops(b[i % 2], ctx, b[(i + 1) % 2])
    prog = _run_prog(ops)
    got = host(b[n_layers % 2])
    check_gemm_bf16(got, bf16_to_f64(ref), what=(cls.__name__, n_layers))
    # a second run of the same program gives the same bytes
    b[0].copy_(x0)
    prog.run()
    torch.cuda.synchronize()
    assert np.array_equal(host(b[n_layers % 2]), got)


def test_dit_layer_program_matches_standalone():
    _stack_compare(layers.DiTLayer, 1, 41, 1536, 1536)


def test_dit_stack_program_matches_standalone():
    _stack_compare(layers.DiTLayer, 4, 41, 1536, 1536)


def test_action_expert_stack_program_matches_standalone():
    _stack_compare(layers.ActionExpertLayer, 3, 50, 1024, 2048)
