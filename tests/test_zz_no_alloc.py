"""nvfp4_gemm_noalloc: the GEMM entry point for callers that cannot allocate device memory
(its split-K workspace is a fixed buffer inside the library).  Called through the C ABI
on operands the oracle quantized, and checked against the oracle's fp64 GEMM and against
nvfp4_gemm (which takes a caller-allocated workspace) on two calls in a row: the second
call finds the first call's leftovers in the shared buffer."""
import ctypes as C

import pytest

from parity import bf16_to_f64, check_gemm_bf16, dev_bf16, host, to_gpu_fp4
from vla_action_head_b200 import nvfp4, synth

pytestmark = pytest.mark.gpu


def _operands(orc, M, N, K, wl):
    x = synth.bf16_normal(synth.seed_of(wl, synth.X), (M, K))
    w = synth.bf16_normal(synth.seed_of(wl, synth.W0), (N, K), 0.0, 0.02)
    bias = synth.bf16_normal(synth.seed_of(wl, synth.BIAS0), (N,), 0.0, 0.01)
    res = synth.bf16_normal(synth.seed_of(wl, synth.RESIDUAL), (M, N))
    ac, asf = orc.quantize_norm(x, "none", g=1.0)
    wc, wsf, gw = orc.quantize_weight(w)
    return (ac, asf, 1.0), (wc, wsf, gw), bias, res


def _call(fn, a, w, M, N, K, epi, bias, res, out, extra):
    ta, tw = a.c(), w.c()
    stream = C.c_void_p(__import__("torch").cuda.current_stream().cuda_stream)
    args = [C.byref(ta), C.byref(tw), M, N, K, nvfp4.EPI[epi], C.c_void_p(bias.data_ptr()),
            C.c_void_p(res.data_ptr()), res.stride(0), C.c_void_p(out.data_ptr()), out.stride(0), None, None,
            1.0]
    return fn(*(args + extra + [stream]))


@pytest.mark.parametrize("M,N,K", [(41, 1536, 6144), (50, 1024, 4096), (41, 4608, 1536)])
def test_noalloc_matches_oracle_and_gemm_twice(orc, M, N, K):
    import torch
    nvfp4.probe()
    L = nvfp4.lib()
    # these shapes run split-K through the workspace, so the fixed scratch is exercised
    assert L.nvfp4_gemm_workspace_bytes_ex(M, N, K, 0, -1) > 0
    (ac, asf, ga), (wc, wsf, gw), bias_h, res_h = _operands(orc, M, N, K, 41)
    ref_orc = orc.gemm(ac, asf, ga, M, wc, wsf, gw, N, K, epi="bias_residual", bias=bias_h, residual=res_h)["v"]
    a, w = to_gpu_fp4(ac, asf, ga, M, K), to_gpu_fp4(wc, wsf, gw, N, K)
    bias, res = dev_bf16(bias_h), dev_bf16(res_h)
    need = L.nvfp4_gemm_workspace_bytes(M, N, K)
    ws = torch.zeros(max(need, 16), dtype=torch.uint8, device="cuda")
    ref = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = _call(L.nvfp4_gemm, a, w, M, N, K, "bias_residual", bias, res, ref,
               [C.c_void_p(ws.data_ptr()), C.c_size_t(need)])
    assert st == 0
    for _ in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = _call(L.nvfp4_gemm_noalloc, a, w, M, N, K, "bias_residual", bias, res, out, [])
        assert st == 0, L.nvfp4_status_string(st)
        torch.cuda.synchronize()
        check_gemm_bf16(host(out), ref_orc, what=("noalloc vs oracle", M, N, K))
        check_gemm_bf16(host(out), bf16_to_f64(host(ref)), what=("noalloc vs nvfp4_gemm", M, N, K))
    nvfp4.device_status()


def test_noalloc_rejects_oversized_workspace(orc):
    """A shape whose split-K workspace exceeds the fixed buffer is refused, not run."""
    import torch
    nvfp4.probe()
    L = nvfp4.lib()
    M, N, K = 128, 1024, 16384
    need = L.nvfp4_gemm_workspace_bytes_ex(M, N, K, 0, -1)
    assert need > (4 << 20)
    (ac, asf, ga), (wc, wsf, gw), bias_h, res_h = _operands(orc, M, N, K, 42)
    a, w = to_gpu_fp4(ac, asf, ga, M, K), to_gpu_fp4(wc, wsf, gw, N, K)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = _call(L.nvfp4_gemm_noalloc, a, w, M, N, K, "bias_residual", dev_bf16(bias_h), dev_bf16(res_h), out, [])
    assert st == 4 and L.nvfp4_status_string(st) == b"workspace missing or too small"


def test_noalloc_rejected_call_leaves_the_buffer_alone(orc):
    """An invalid call (here: no bias for a bias epilogue) returns INVALID_ARG before it
    clears any ticket, so it cannot disturb the shared buffer; a valid call then runs."""
    import torch
    nvfp4.probe()
    L = nvfp4.lib()
    M, N, K = 41, 1536, 6144
    (ac, asf, ga), (wc, wsf, gw), bias_h, res_h = _operands(orc, M, N, K, 43)
    a, w = to_gpu_fp4(ac, asf, ga, M, K), to_gpu_fp4(wc, wsf, gw, N, K)
    res = dev_bf16(res_h)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    ta, tw = a.c(), w.c()
    stream = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = L.nvfp4_gemm_noalloc(C.byref(ta), C.byref(tw), M, N, K, nvfp4.EPI["bias_residual"], None,
                              C.c_void_p(res.data_ptr()), res.stride(0), C.c_void_p(out.data_ptr()), out.stride(0),
                              None, None, 1.0, stream)
    assert st == 1  # invalid argument
    bias = dev_bf16(bias_h)
    st = _call(L.nvfp4_gemm_noalloc, a, w, M, N, K, "bias_residual", bias, res, out, [])
    assert st == 0
    torch.cuda.synchronize()
    rows = [0, 20, 40]
    ref = orc.gemm(ac, asf, ga, M, wc, wsf, gw, N, K, epi="bias_residual", bias=bias_h, residual=res_h, rows=rows)
    check_gemm_bf16(host(out)[rows], ref["v"], what="noalloc after a rejected call")
    nvfp4.device_status()
