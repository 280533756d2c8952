"""nvfp4_gemm_noalloc: the GEMM entry point for callers that cannot allocate device memory
(its split-K workspace is a fixed buffer inside the library).  Checked through the C ABI
against nvfp4_gemm, which takes a caller-allocated workspace, on two calls in a row (the
second call finds the first call's leftovers in the shared buffer)."""
import ctypes as C

import pytest

from parity import bf16_to_f64, check_gemm_bf16, host
from vla_action_head_b200 import nvfp4, synth

pytestmark = pytest.mark.gpu


def _operands(M, N, K, wl):
    import torch
    x = synth.bf16_normal_torch(synth.seed_of(wl, synth.X), (M, K), device="cuda")
    w = synth.bf16_normal_torch(synth.seed_of(wl, synth.W0), (N, K), 0, 0.02, device="cuda")
    bias = synth.bf16_normal_torch(synth.seed_of(wl, synth.BIAS0), (N,), 0, 0.01, device="cuda")
    res = synth.bf16_normal_torch(synth.seed_of(wl, synth.RESIDUAL), (M, N), device="cuda")
    a = nvfp4.quantize_norm(x, "none")
    wq = nvfp4.quantize_weight(w)
    torch.cuda.synchronize()
    return a, wq, bias, res


def _call(fn, a, w, M, N, K, epi, bias, res, out, extra):
    ta, tw = a.c(), w.c()
    stream = C.c_void_p(__import__("torch").cuda.current_stream().cuda_stream)
    args = [C.byref(ta), C.byref(tw), M, N, K, nvfp4.EPI[epi], C.c_void_p(bias.data_ptr()),
            C.c_void_p(res.data_ptr()), res.stride(0), C.c_void_p(out.data_ptr()), out.stride(0), None, None,
            1.0]
    return fn(*(args + extra + [stream]))


@pytest.mark.parametrize("M,N,K", [(41, 1536, 6144), (50, 1024, 4096), (41, 4608, 1536)])
def test_noalloc_matches_gemm_twice(M, N, K):
    import torch
    nvfp4.probe()
    L = nvfp4.lib()
    # these shapes run split-K through the workspace, so the fixed scratch is exercised
    assert L.nvfp4_gemm_workspace_bytes_ex(M, N, K, 0, -1) > 0
    a, w, bias, res = _operands(M, N, K, 41)
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
        check_gemm_bf16(host(out), bf16_to_f64(host(ref)), what=("noalloc", M, N, K))
    nvfp4.device_status()


def test_noalloc_rejects_oversized_workspace():
    """A shape whose split-K workspace exceeds the fixed buffer is refused, not run."""
    import torch
    nvfp4.probe()
    L = nvfp4.lib()
    M, N, K = 128, 1024, 16384
    need = L.nvfp4_gemm_workspace_bytes_ex(M, N, K, 0, -1)
    assert need > (4 << 20)
    a, w, bias, res = _operands(M, N, K, 42)
    out = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    st = _call(L.nvfp4_gemm_noalloc, a, w, M, N, K, "bias_residual", bias, res, out, [])
    assert st == 4 and L.nvfp4_status_string(st) == b"workspace missing or too small"
