"""Grouped NVFP4 GEMM: independent problems in one launch of the grouped kernel ("GROOT N1.7
update: Thor NVFP4 + FA4 performance tier", §What is in the tier: the 32 per-frame
cross-attention K/V projections run as NVFP4 GEMMs).  Every problem meets the GEMM bar
against the oracle and the group agrees with the standalone calls; groups the grouped kernel
does not take run as standalone launches, and programs with dependent or norm ops are
refused."""
import numpy as np
import pytest

from parity import bf16_to_f64, check_fp4_output, check_gemm_bf16, dev_bf16, host, to_gpu_fp4
from vla_action_head_b200 import nvfp4, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _probe():
    nvfp4.probe()


def _problem(orc, g, M, N, K, with_bias):
    x = synth.bf16_normal(synth.seed_of(40 + g, synth.CONTEXT), (M, K))
    w = synth.bf16_normal(synth.seed_of(40 + g, synth.W0), (N, K), 0.0, 0.02)
    ac, asf = orc.quantize_norm(x, "none")
    wc, wsf, gw = orc.quantize_weight(w)
    bias = synth.bf16_normal(synth.seed_of(40 + g, synth.BIAS0), (N,), 0.0, 0.01) if with_bias else None
    ref = orc.gemm(ac, asf, 1.0, M, wc, wsf, gw, N, K, epi="bias" if with_bias else "none", bias=bias)
    return x, (ac, asf), (wc, wsf, gw), bias, ref


def _sync():
    import torch
    torch.cuda.synchronize()
    nvfp4.device_status()


@pytest.mark.parametrize("with_bias", [False, True])
def test_grouped_mixed_shapes_match_oracle(orc, with_bias):
    """Problems of different M, N and K (tiles of 64 and 128 columns, ragged K) in one group."""
    import torch
    shapes = [(41, 1536, 1536), (50, 1024, 2048), (1, 512, 256), (64, 2560, 1024), (17, 256, 96),
              (41, 3072, 1536), (33, 640, 4096)]
    probs, refs = [], []
    for g, (M, N, K) in enumerate(shapes):
        _, (ac, asf), (wc, wsf, gw), bias, ref = _problem(orc, g, M, N, K, with_bias)
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        probs.append((to_gpu_fp4(ac, asf, 1.0, M, K), to_gpu_fp4(wc, wsf, gw, N, K), out,
                      dev_bf16(bias) if with_bias else None))
        refs.append(ref["v"])
    grp = nvfp4.GroupedGemm(probs, epi="bias" if with_bias else "none")
    assert grp.prog.kind == 1  # the grouped kernel
    grp.run()
    _sync()
    for g, (p, ref) in enumerate(zip(probs, refs)):
        check_gemm_bf16(host(p[2]), ref, what=("grouped", g, shapes[g]))


@pytest.mark.parametrize("epi", ["residual", "bias_gelu", "geglu", "bias_gelu_rht", "geglu_rht"])
def test_grouped_kernel_epilogues(orc, epi):
    """The grouped kernel's other epilogue kinds, including FP4 outputs, on problems of
    different M (one above 128 rows: two m-tiles) and K."""
    import torch
    shapes = [(41, 1024, 1536), (150, 512, 512), (8, 256, 2048)]
    probs, refs = [], []
    for g, (M, N, K) in enumerate(shapes):
        x = synth.bf16_normal(synth.seed_of(90 + g, synth.CONTEXT), (M, K))
        w = synth.bf16_normal(synth.seed_of(90 + g, synth.W0), (N, K), 0.0, 0.02)
        ac, asf = orc.quantize_norm(x, "none")
        wc, wsf, gw = orc.quantize_weight(w, interleave_gate_up=epi.startswith("geglu"))
        bias = (synth.bf16_normal(synth.seed_of(90 + g, synth.BIAS0), (N,), 0.0, 0.01)
                if epi.startswith("bias_gelu") else None)
        res = synth.bf16_normal(synth.seed_of(90 + g, synth.RESIDUAL), (M, N)) if epi == "residual" else None
        ref = orc.gemm(ac, asf, 1.0, M, wc, wsf, gw, N, K, epi=epi, bias=bias, residual=res)
        A, W = to_gpu_fp4(ac, asf, 1.0, M, K), to_gpu_fp4(wc, wsf, gw, N, K)
        if "gelu" in epi or "geglu" in epi:
            out = nvfp4.empty_fp4(M, N // 2 if epi.startswith("geglu") else N)
        else:
            out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        probs.append(nvfp4.op_gemm(A, W, epi, bias=dev_bf16(bias) if bias is not None else None,
                                   residual=dev_bf16(res) if res is not None else None, out=out))
        refs.append((ref, out, M, N, K))
    prog = nvfp4.Program(probs)
    assert prog.prog.kind == 1
    prog.run()
    _sync()
    for ref, out, M, N, K in refs:
        if "gelu" in epi or "geglu" in epi:
            check_fp4_output(orc, host(out.codes), host(out.sf), ref["codes"], ref["sf"], ref["h"], 1.0, M, out.K,
                             what=(M, N, K, epi))
        else:
            check_gemm_bf16(host(out), ref["v"], what=(M, N, K, epi))


def test_groups_the_kernel_does_not_take_run_as_standalone_launches(orc):
    """A problem with N % 128 != 0 keeps the group off the grouped kernel: GroupedGemm runs
    each problem as an nvfp4_gemm launch."""
    import torch
    probs, refs = [], []
    for g, (M, N, K) in enumerate([(41, 192, 512), (41, 256, 512)]):
        _, (ac, asf), (wc, wsf, gw), _, ref = _problem(orc, 30 + g, M, N, K, False)
        out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
        probs.append((to_gpu_fp4(ac, asf, 1.0, M, K), to_gpu_fp4(wc, wsf, gw, N, K), out))
        refs.append(ref["v"])
    grp = nvfp4.GroupedGemm(probs)
    assert grp.prog is None
    grp.run()
    _sync()
    for p, ref in zip(probs, refs):
        check_gemm_bf16(host(p[2]), ref, what="standalone group")


def test_grouped_cross_kv_32_matches_standalone(orc):
    """32 projections of one shared context, as the K and V of 16 cross-attention layers;
    checked against the oracle on a sample of problems and against the standalone GEMM on all."""
    import torch
    M, N, K, G = 41, 1536, 1536, 32
    ctx = synth.bf16_normal(synth.seed_of(60, synth.CONTEXT), (M, K))
    ac, asf = orc.quantize_norm(ctx, "none")
    A = to_gpu_fp4(ac, asf, 1.0, M, K)
    probs, refs = [], {}
    for g in range(G):
        w = synth.bf16_normal(synth.seed_of(60 + g, synth.W0), (N, K), 0.0, 0.02)
        wc, wsf, gw = orc.quantize_weight(w)
        if g in (0, 13, 31):
            refs[g] = orc.gemm(ac, asf, 1.0, M, wc, wsf, gw, N, K, epi="none")["v"]
        probs.append((A, to_gpu_fp4(wc, wsf, gw, N, K), torch.empty((M, N), dtype=torch.bfloat16, device="cuda")))
    grp = nvfp4.GroupedGemm(probs)
    assert grp.prog.kind == 1
    grp.run()
    _sync()
    for g, ref in refs.items():
        check_gemm_bf16(host(probs[g][2]), ref, what=("cross-kv", g))
    for g, (a, w, out) in enumerate(probs):
        alone = nvfp4.gemm(a, w, "none")
        _sync()
        check_gemm_bf16(host(out), bf16_to_f64(host(alone)), what=("vs standalone", g))
    # replays give the same bytes
    first = [host(p[2]).copy() for p in probs]
    for p in probs:
        p[2].zero_()
    grp.run()
    _sync()
    assert all(np.array_equal(host(p[2]), f) for p, f in zip(probs, first))


def test_program_refuses_dependent_and_norm_ops(orc):
    """nvfp4_program_build takes independent GEMM ops only: an op that names another op, a
    norm op, or mixed epilogues are refused (NVFP4_ERR_UNSUPPORTED_SHAPE)."""
    import torch
    M, N, K = 8, 256, 256
    _, (ac, asf), (wc, wsf, gw), _, _ = _problem(orc, 0, M, N, K, False)
    A, W = to_gpu_fp4(ac, asf, 1.0, M, K), to_gpu_fp4(wc, wsf, gw, N, K)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    dep_op = nvfp4.op_gemm(A, W, "none", out=out)
    dep_op.dep = 0  # "the previous op"
    norm_op = nvfp4.op_gemm(A, W, "none", out=out)
    norm_op.type = 0
    mixed = nvfp4.op_gemm(A, W, "bias", bias=torch.zeros(N, dtype=torch.bfloat16, device="cuda"), out=out)
    for bad in ([nvfp4.op_gemm(A, W, "none", out=out), dep_op], [norm_op],
                [nvfp4.op_gemm(A, W, "none", out=out), mixed]):
        with pytest.raises(nvfp4.NVFP4Error) as err:
            nvfp4.Program(bad)
        assert err.value.status == 2
