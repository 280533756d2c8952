"""NVFP4 layer compositions of the hot path, built only from the C-ABI calls.

Each layer quantizes its weights once at construction (nvfp4_quantize_weight) and its
forward issues the norm -> FP4 front-ends and the block-scaled GEMMs with fused
epilogues into preallocated buffers, so a forward can be captured in a CUDA graph.

  DiTLayer           DiT block at M tokens, hidden H, FFN F ("GROOT N1.7 update: Thor
                     NVFP4 + FA4 performance tier", §What is in the tier): AdaLN->FP4,
                     fused QKV (+bias), attention-output (+bias+residual), pre-FFN
                     LayerNorm->FP4, FFN up (+bias, tanh-GELU -> FP4), FFN down
                     (+bias+residual).
  ActionExpertLayer  Pi0.5 action-expert decoder layer ("Pi0.5 Thor NVFP4 End-to-End
                     Results", §Implemented Path, §Fused GeGLU FFN in the Decoder):
                     AdaRMSNorm->FP4, QKV, attention-output (+residual), AdaRMSNorm->FP4,
                     gate/up with GeGLU -> FP4 (pairwise-interleaved weights), down
                     (+residual).
  GatedActionExpertLayer  the same layer with the gated residual updates fused into the
                     norm front-ends (nvfp4_residual_quantize_norm).
  PrefillLayer       backbone-shaped prefill layer at M = 968: RMSNorm->FP4, QKV,
                     RMSNorm->FP4, gate/up GeGLU -> FP4, down (+residual).

Attention itself is not part of the linear path: the attention-output GEMM reads a
caller-supplied bf16 context tensor (quantized with the plain quantizer), which stands in
for the attention result.
"""
import torch

from . import nvfp4, synth


class Linear:
    """NVFP4 weight [N, K] (+ optional bf16 bias), quantized once from bf16 with amax or
    MSE-searched block scales."""

    def __init__(self, w_bf16, bias=None, interleave_gate_up=False, scales="amax"):
        self.N, self.K = w_bf16.shape
        self.w = nvfp4.quantize_weight(w_bf16.contiguous(), interleave_gate_up=interleave_gate_up, scales=scales)
        self.bias = bias

    def weight_bytes(self):
        return self.w.codes.numel() + self.w.sf.numel()


def _rand(seed, shape, mean, std, device):
    return synth.bf16_normal_torch(seed, shape, mean, std, device=device)


class DiTLayer:
    def __init__(self, M=41, H=1536, F=6144, wl=2, layer=0, device="cuda", ws=None):
        s = lambda tid: synth.seed_of(wl, 100 * layer + tid)  # noqa: E731
        d = device
        self.M, self.H, self.F = M, H, F
        self.ada_scale = _rand(s(synth.MOD_SCALE), (H,), 0.0, 0.1, d)
        self.ada_shift = _rand(s(synth.MOD_SHIFT), (H,), 0.0, 0.1, d)
        self.ln_gamma = _rand(s(synth.GAMMA), (H,), 1.0, 0.1, d)
        self.ln_beta = _rand(s(synth.BETA), (H,), 0.0, 0.1, d)
        self.qkv = Linear(_rand(s(synth.W0), (3 * H, H), 0, 0.02, d), _rand(s(synth.BIAS0), (3 * H,), 0, 0.01, d))
        self.o = Linear(_rand(s(synth.W0 + 1), (H, H), 0, 0.02, d), _rand(s(synth.BIAS0 + 1), (H,), 0, 0.01, d))
        self.up = Linear(_rand(s(synth.W0 + 2), (F, H), 0, 0.02, d), _rand(s(synth.BIAS0 + 2), (F,), 0, 0.01, d))
        self.down = Linear(_rand(s(synth.W0 + 3), (H, F), 0, 0.02, d), _rand(s(synth.BIAS0 + 3), (H,), 0, 0.01, d))
        self.ws = ws or nvfp4.Workspace(d)
        # activations
        self.a1 = nvfp4.empty_fp4(M, H, d)
        self.ctx_q = nvfp4.empty_fp4(M, H, d)
        self.a2 = nvfp4.empty_fp4(M, H, d)
        self.u = nvfp4.empty_fp4(M, F, d)
        self.qkv_out = torch.empty((M, 3 * H), dtype=torch.bfloat16, device=d)
        self.h = torch.empty((M, H), dtype=torch.bfloat16, device=d)

    def linears(self):
        return [self.qkv, self.o, self.up, self.down]

    def forward(self, x, context, y):
        """x, context: bf16 [M, H]; writes the layer output into y (bf16 [M, H])."""
        nvfp4.quantize_norm(x, "adaln", scale=self.ada_scale, shift=self.ada_shift, eps=1e-6, out=self.a1)
        nvfp4.gemm(self.a1, self.qkv.w, "bias", bias=self.qkv.bias, out=self.qkv_out, workspace=self.ws)
        nvfp4.quantize_norm(context, "none", out=self.ctx_q)
        nvfp4.gemm(self.ctx_q, self.o.w, "bias_residual", bias=self.o.bias, residual=x, out=self.h, workspace=self.ws)
        nvfp4.quantize_norm(self.h, "layernorm", gamma=self.ln_gamma, beta=self.ln_beta, eps=1e-5, out=self.a2)
        nvfp4.gemm(self.a2, self.up.w, "bias_gelu", bias=self.up.bias, out=self.u, workspace=self.ws)
        nvfp4.gemm(self.u, self.down.w, "bias_residual", bias=self.down.bias, residual=self.h, out=y,
                   workspace=self.ws)
        return y

    launches = 7


class ActionExpertLayer:
    # The decoder projections take MSE-searched block scales by default ("Pi0.5 Thor NVFP4
    # End-to-End Results", §E0M3 Uniform-INT4 Decoder Weights: NVFP4 "(MSE, default)").
    def __init__(self, M=50, H=1024, A=2048, F=4096, wl=3, layer=0, device="cuda", ws=None, weight_scales="mse"):
        s = lambda tid: synth.seed_of(wl, 100 * layer + tid)  # noqa: E731
        d = device
        self.M, self.H, self.A, self.F = M, H, A, F
        self.scale1 = _rand(s(synth.MOD_SCALE), (H,), 0.0, 0.1, d)
        self.scale2 = _rand(s(synth.MOD_SHIFT), (H,), 0.0, 0.1, d)
        self.qkv = Linear(_rand(s(synth.W0), (2560, H), 0, 0.02, d), scales=weight_scales)
        self.o = Linear(_rand(s(synth.W0 + 1), (H, A), 0, 0.02, d), scales=weight_scales)
        self.gate_up = Linear(_rand(s(synth.W0 + 2), (2 * F, H), 0, 0.02, d), interleave_gate_up=True,
                              scales=weight_scales)
        self.down = Linear(_rand(s(synth.W0 + 3), (H, F), 0, 0.02, d), scales=weight_scales)
        self.ws = ws or nvfp4.Workspace(d)
        self.a1 = nvfp4.empty_fp4(M, H, d)
        self.ctx_q = nvfp4.empty_fp4(M, A, d)
        self.a2 = nvfp4.empty_fp4(M, H, d)
        self.u = nvfp4.empty_fp4(M, F, d)
        self.qkv_out = torch.empty((M, 2560), dtype=torch.bfloat16, device=d)
        self.h = torch.empty((M, H), dtype=torch.bfloat16, device=d)

    def linears(self):
        return [self.qkv, self.o, self.gate_up, self.down]

    def forward(self, x, context, y):
        """x: bf16 [M, H]; context: bf16 [M, A]; writes the output into y (bf16 [M, H])."""
        nvfp4.quantize_norm(x, "adarms", scale=self.scale1, eps=1e-6, out=self.a1)
        nvfp4.gemm(self.a1, self.qkv.w, "none", out=self.qkv_out, workspace=self.ws)
        nvfp4.quantize_norm(context, "none", out=self.ctx_q)
        nvfp4.gemm(self.ctx_q, self.o.w, "residual", residual=x, out=self.h, workspace=self.ws)
        nvfp4.quantize_norm(self.h, "adarms", scale=self.scale2, eps=1e-6, out=self.a2)
        nvfp4.gemm(self.a2, self.gate_up.w, "geglu", out=self.u, workspace=self.ws)
        nvfp4.gemm(self.u, self.down.w, "residual", residual=self.h, out=y, workspace=self.ws)
        return y

    launches = 7


class GatedActionExpertLayer:
    """Pi0.5 action-expert decoder layer with the gated residual updates moved into the norm
    front-ends ("Pi0.5 Thor NVFP4 End-to-End Results", §Implemented Path: gated residual update
    + Pi0.5 AdaRMSNorm + gate output + NVFP4/SFA in one launch before Gate+Up and the next
    layer's QKV).  The residual stream r is updated in place:

      r = r + g_in * d_in;  a1 = AdaRMS(r)(1 + s1) + t1 -> FP4    (front-end 1; d_in from the
                                                                    previous layer's down)
      QKV; context -> FP4; d_o = O(context)                        (bf16, no residual)
      r = r + g1 * d_o;     a2 = AdaRMS(r)(1 + s2) + t2 -> FP4     (front-end 2)
      u = GeGLU(gate_up(a2)) -> FP4;  d_out = down(u)              (bf16, no residual)

    forward returns (d_out, g2): the next layer's front-end 1 applies r += g2 * d_out."""

    def __init__(self, M=50, H=1024, A=2048, F=4096, wl=6, layer=0, device="cuda", ws=None, weight_scales="mse"):
        s = lambda tid: synth.seed_of(wl, 100 * layer + tid)  # noqa: E731
        d = device
        self.M, self.H, self.A, self.F = M, H, A, F
        self.s1 = _rand(s(synth.MOD_SCALE), (H,), 0.0, 0.1, d)
        self.t1 = _rand(s(synth.MOD_SHIFT), (H,), 0.0, 0.1, d)
        self.s2 = _rand(s(synth.GAMMA), (H,), 0.0, 0.1, d)
        self.t2 = _rand(s(synth.BETA), (H,), 0.0, 0.1, d)
        self.g1 = _rand(s(synth.RESIDUAL), (H,), 0.0, 0.5, d)
        self.g2 = _rand(s(synth.RESIDUAL + 1), (H,), 0.0, 0.5, d)
        self.qkv = Linear(_rand(s(synth.W0), (2560, H), 0, 0.02, d), scales=weight_scales)
        self.o = Linear(_rand(s(synth.W0 + 1), (H, A), 0, 0.02, d), scales=weight_scales)
        self.gate_up = Linear(_rand(s(synth.W0 + 2), (2 * F, H), 0, 0.02, d), interleave_gate_up=True,
                              scales=weight_scales)
        self.down = Linear(_rand(s(synth.W0 + 3), (H, F), 0, 0.02, d), scales=weight_scales)
        self.ws = ws or nvfp4.Workspace(d)
        self.a1 = nvfp4.empty_fp4(M, H, d)
        self.ctx_q = nvfp4.empty_fp4(M, A, d)
        self.a2 = nvfp4.empty_fp4(M, H, d)
        self.u = nvfp4.empty_fp4(M, F, d)
        self.qkv_out = torch.empty((M, 2560), dtype=torch.bfloat16, device=d)
        self.d_o = torch.empty((M, H), dtype=torch.bfloat16, device=d)
        self.d_out = torch.empty((M, H), dtype=torch.bfloat16, device=d)

    def linears(self):
        return [self.qkv, self.o, self.gate_up, self.down]

    def forward(self, r, d_in, g_in, context):
        """r: bf16 [M, H] residual stream (updated in place); d_in, g_in: the previous layer's
        down output and gate (d_in None: a plain AdaRMS front-end for the first layer)."""
        if d_in is None:
            nvfp4.quantize_norm(r, "adarms", scale=self.s1, shift=self.t1, eps=1e-6, out=self.a1)
        else:
            nvfp4.residual_quantize_norm(r, d_in, g_in, "adarms", scale=self.s1, shift=self.t1, eps=1e-6,
                                         h_out=r, out=self.a1)
        nvfp4.gemm(self.a1, self.qkv.w, "none", out=self.qkv_out, workspace=self.ws)
        nvfp4.quantize_norm(context, "none", out=self.ctx_q)
        nvfp4.gemm(self.ctx_q, self.o.w, "none", out=self.d_o, workspace=self.ws)
        nvfp4.residual_quantize_norm(r, self.d_o, self.g1, "adarms", scale=self.s2, shift=self.t2, eps=1e-6,
                                     h_out=r, out=self.a2)
        nvfp4.gemm(self.a2, self.gate_up.w, "geglu", out=self.u, workspace=self.ws)
        nvfp4.gemm(self.u, self.down.w, "none", out=self.d_out, workspace=self.ws)
        return self.d_out, self.g2

    launches = 7


class PrefillLayer:
    def __init__(self, M=968, H=2048, F=16384, wl=4, layer=0, device="cuda", ws=None):
        s = lambda tid: synth.seed_of(wl, 100 * layer + tid)  # noqa: E731
        d = device
        self.M, self.H, self.F = M, H, F
        self.gamma1 = _rand(s(synth.GAMMA), (H,), 1.0, 0.1, d)
        self.gamma2 = _rand(s(synth.BETA), (H,), 1.0, 0.1, d)
        self.qkv = Linear(_rand(s(synth.W0), (2560, H), 0, 0.02, d))
        self.gate_up = Linear(_rand(s(synth.W0 + 2), (2 * F, H), 0, 0.02, d), interleave_gate_up=True)
        self.down = Linear(_rand(s(synth.W0 + 3), (H, F), 0, 0.02, d))
        self.ws = ws or nvfp4.Workspace(d)
        self.a1 = nvfp4.empty_fp4(M, H, d)
        self.a2 = nvfp4.empty_fp4(M, H, d)
        self.u = nvfp4.empty_fp4(M, F, d)
        self.qkv_out = torch.empty((M, 2560), dtype=torch.bfloat16, device=d)

    def linears(self):
        return [self.qkv, self.gate_up, self.down]

    def forward(self, x, context, y):
        nvfp4.quantize_norm(x, "rmsnorm", gamma=self.gamma1, eps=1e-6, out=self.a1)
        nvfp4.gemm(self.a1, self.qkv.w, "none", out=self.qkv_out, workspace=self.ws)
        nvfp4.quantize_norm(x, "rmsnorm", gamma=self.gamma2, eps=1e-6, out=self.a2)
        nvfp4.gemm(self.a2, self.gate_up.w, "geglu", out=self.u, workspace=self.ws)
        nvfp4.gemm(self.u, self.down.w, "residual", residual=x, out=y, workspace=self.ws)
        return y

    launches = 5

    def flops(self):
        M = self.M
        return 2.0 * M * (2560 * self.H + 2 * self.F * self.H + self.H * self.F)
