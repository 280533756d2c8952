"""GPU parity of the gated residual front-end (nvfp4_residual_quantize_norm) against the
oracle: h = bf16(x + gate * d), then the norm -> NVFP4 of h ("Pi0.5 Thor NVFP4 End-to-End
Results", §Implemented Path: gated residual update + AdaRMSNorm + gate output + NVFP4/SFA in
one launch).  The stored residual stream h and the FP4 codes and scales are bit-exact."""
import numpy as np
import pytest
import torch

from parity import dev_bf16, host
from vla_action_head_b200 import nvfp4, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _probe():
    nvfp4.probe()


def _case(orc, M, K, kind, wl=40, gate=True, shift=True, in_place=False):
    s = lambda tid: synth.seed_of(wl, tid)  # noqa: E731
    x = synth.bf16_normal(s(synth.X), (M, K))
    d = synth.bf16_normal(s(synth.CONTEXT), (M, K))
    g = synth.bf16_normal(s(synth.RESIDUAL), (K,), 0.0, 0.5) if gate else None
    sc = synth.bf16_normal(s(synth.MOD_SCALE), (K,), 0.0, 0.1)
    sh = synth.bf16_normal(s(synth.MOD_SHIFT), (K,), 0.0, 0.1) if shift else None
    ga = synth.bf16_normal(s(synth.GAMMA), (K,), 1.0, 0.1)
    be = synth.bf16_normal(s(synth.BETA), (K,), 0.0, 0.1)
    kw = dict(gamma=ga, beta=be, scale=sc, shift=sh, eps=1e-6)
    rh, rc, rs = orc.residual_quantize_norm(x, d, g, kind, **kw)
    xg = dev_bf16(x)
    h_out = xg if in_place else None
    h, q = nvfp4.residual_quantize_norm(xg, dev_bf16(d), dev_bf16(g) if gate else None, kind,
                                        **{k: (dev_bf16(v) if v is not None else None) for k, v in kw.items()
                                           if k != "eps"}, eps=1e-6, h_out=h_out)
    torch.cuda.synchronize()
    assert np.array_equal(host(h).view(np.uint16), rh), (M, K, kind)
    assert np.array_equal(host(q.codes), rc), (M, K, kind)
    assert np.array_equal(host(q.sf), rs), (M, K, kind)


@pytest.mark.parametrize("kind", ["adarms", "rmsnorm", "layernorm", "adaln", "none"])
@pytest.mark.parametrize("M,K", [(50, 1024), (41, 1536), (1, 16), (33, 48), (129, 4096), (200, 2048)])
def test_residual_front_end_matches_oracle(orc, kind, M, K):
    _case(orc, M, K, kind)


def test_residual_front_end_variants(orc):
    _case(orc, 50, 1024, "adarms", gate=False)      # gate NULL reads 1
    _case(orc, 50, 1024, "adarms", shift=False)     # AdaRMS without shift
    _case(orc, 50, 1024, "adarms", in_place=True)   # h written over x
    _case(orc, 968, 2048, "rmsnorm", wl=41)         # one warp per row


def test_residual_front_end_rejects_bad_args():
    L = nvfp4.lib()
    x = torch.zeros((4, 64), dtype=torch.bfloat16, device="cuda")
    st = L.nvfp4_residual_quantize_norm(x.data_ptr(), None, None, 4, 64, 64, 64, 64, 0, None, None, None, None,
                                        1e-6, 1.0, x.data_ptr(), x.data_ptr(), x.data_ptr(), None)
    assert st == 1  # no d


def test_gated_action_expert_layer_against_oracle(orc):
    """One layer of the gated stack: the attention-output GEMM (no residual epilogue) against
    the oracle's fp64 GEMM, then the second front-end exactly, given the GPU's GEMM output."""
    from parity import check_gemm_bf16
    from vla_action_head_b200 import layers
    lay = layers.GatedActionExpertLayer(device="cuda")
    M, H, A = lay.M, lay.H, lay.A
    x = synth.bf16_normal_torch(synth.seed_of(42, synth.X), (M, H), device="cuda")
    ctx = synth.bf16_normal_torch(synth.seed_of(42, synth.CONTEXT), (M, A), device="cuda")
    r = x.clone()
    lay.forward(r, None, None, ctx)
    torch.cuda.synchronize()
    cq, cs = orc.quantize_norm(host(ctx), "none")
    assert np.array_equal(host(lay.ctx_q.codes), cq) and np.array_equal(host(lay.ctx_q.sf), cs)
    v = orc.gemm(cq, cs, 1.0, M, host(lay.o.w.codes), host(lay.o.w.sf), lay.o.w.global_scale, H, A, epi="none")["v"]
    check_gemm_bf16(host(lay.d_o), v, what="gated layer attention-output")
    rh, rc, rs = orc.residual_quantize_norm(host(x), host(lay.d_o), host(lay.g1), "adarms", scale=host(lay.s2),
                                            shift=host(lay.t2), eps=1e-6)
    assert np.array_equal(host(r), rh)
    assert np.array_equal(host(lay.a2.codes), rc) and np.array_equal(host(lay.a2.sf), rs)
    # a second layer consumes (d_out, g2) in its first front-end
    lay2 = layers.GatedActionExpertLayer(layer=1, device="cuda")
    r_before = host(r).copy()
    d_out = host(lay.d_out).copy()
    lay2.forward(r, lay.d_out, lay.g2, ctx)
    torch.cuda.synchronize()
    rh1, rc1, rs1 = orc.residual_quantize_norm(r_before, d_out, host(lay.g2), "adarms", scale=host(lay2.s1),
                                               shift=host(lay2.t1), eps=1e-6)
    assert np.array_equal(host(lay2.a1.codes), rc1) and np.array_equal(host(lay2.a1.sf), rs1)
