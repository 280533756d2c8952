"""Python binding of libnvfp4.so (include/nvfp4.h).

Argument marshalling only: torch supplies device memory and the current CUDA stream; every
step of the computation runs in the library's sm_100a kernels.  There is no fallback: if
the library is missing or the device is not sm_100, calls raise.

Raw entry points keep their C names (`nvfp4_quantize_norm`, `nvfp4_quantize_weight`,
`nvfp4_gemm`, ...) and take plain integers / pointers.  The lower-case helpers
(`quantize_norm`, `quantize_weight`, `gemm`, ...) accept torch tensors and allocate outputs.
"""
import ctypes as C
import os
import re
from dataclasses import dataclass
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("NVFP4_LIB") or os.path.join(HERE, "libnvfp4.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "nvfp4.h")

NORM = {"none": 0, "layernorm": 1, "rmsnorm": 2, "adaln": 3, "adarms": 4}
EPI = {"none": 0, "bias": 1, "residual": 2, "bias_residual": 3, "bias_gelu": 4, "geglu": 5,
       "bias_gelu_rht": 6, "geglu_rht": 7}
QUANT_ROTATE, QUANT_E0M3, QUANT_MSE = 1, 2, 4  # nvfp4_quant_flags
IN_BF16, IN_FP32 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "misaligned",
          4: "workspace", 5: "unsupported device", 6: "CUDA error", 7: "timeout"}


class NVFP4Error(RuntimeError):
    def __init__(self, call, status, detail=""):
        super().__init__(f"{call} failed: {status} ({STATUS.get(status, '?')}){detail}")
        self.status = status


class _Tensor(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("sf", C.c_void_p), ("global_scale", C.c_float),
                ("rows", C.c_int), ("K", C.c_int)]


class _Op(C.Structure):
    _fields_ = [("type", C.c_int), ("M", C.c_int), ("N", C.c_int), ("K", C.c_int),
                ("x", C.c_void_p), ("ldx", C.c_int), ("norm", C.c_int),
                ("gamma", C.c_void_p), ("beta", C.c_void_p), ("mod_scale", C.c_void_p),
                ("mod_shift", C.c_void_p), ("eps", C.c_float),
                ("A", _Tensor), ("W", _Tensor), ("epi", C.c_int), ("bias", C.c_void_p),
                ("residual", C.c_void_p), ("ldr", C.c_int), ("out_bf16", C.c_void_p), ("ldo", C.c_int),
                ("out_codes", C.c_void_p), ("out_sf", C.c_void_p), ("out_global_scale", C.c_float),
                ("dep", C.c_int)]


class _Program(C.Structure):
    _fields_ = [("buffer", C.c_void_p), ("bytes", C.c_size_t), ("n_ops", C.c_int), ("grid", C.c_int),
                ("cluster", C.c_int), ("ops_offset", C.c_size_t), ("maps_offset", C.c_size_t),
                ("done_offset", C.c_size_t), ("waits", C.c_int), ("kind", C.c_int), ("epi", C.c_int),
                ("tiles", C.c_int)]


_lib = None
P, I, F, SZ = C.c_void_p, C.c_int, C.c_float, C.c_size_t


def lib():
    """Loads libnvfp4.so (built in-tree by vla_action_head_b200.build; NVFP4_LIB overrides
    the path, e.g. to compare builds)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: run vla_action_head_b200.build.build()")
        L = C.CDLL(LIB_PATH)
        sig = {
            "nvfp4_probe": (I, []),
            "nvfp4_status_string": (C.c_char_p, [I]),
            "nvfp4_last_cuda_error_string": (C.c_char_p, []),
            "nvfp4_sf_bytes": (SZ, [I, I]),
            "nvfp4_sf_offset": (SZ, [I, I, I]),
            "nvfp4_sf_zero": (I, [P, I, I, P]),
            "nvfp4_gemm_workspace_bytes": (SZ, [I, I, I]),
            "nvfp4_gemm_workspace_bytes_ex": (SZ, [I, I, I, I, I]),
            "nvfp4_get_device_status": (I, [P]),
            "nvfp4_set_gemm_trace": (I, [P, SZ]),
            "nvfp4_gemm_trace_words": (SZ, [I, I, I, I]),
            "nvfp4_mma_rate": (I, [I, I, I, P, P]),
            "nvfp4_quantize_norm": (I, [P, I, I, I, I, I, P, P, P, P, F, F, P, P, P]),
            "nvfp4_residual_quantize_norm": (I, [P, P, P, I, I, I, I, I, I, P, P, P, P, F, F, P, P, P, P]),
            "nvfp4_norm_f32": (I, [P, I, I, I, I, I, P, P, P, P, F, P, P]),
            "nvfp4_quantize_weight": (I, [P, I, I, I, I, P, P, C.POINTER(C.c_float), P, P]),
            "nvfp4_quantize_weight_mse": (I, [P, I, I, I, I, P, P, C.POINTER(C.c_float), P, P]),
            "nvfp4_quantize_weight_ex": (I, [P, I, I, I, I, I, P, P, C.POINTER(C.c_float), P, P]),
            "nvfp4_quantize_norm_ex": (I, [P, I, I, I, I, I, P, P, P, P, F, F, I, P, P, P]),
            "nvfp4_residual_quantize_norm_ex": (I, [P, P, P, I, I, I, I, I, I, P, P, P, P, F, F, I, P, P, P,
                                                    P]),
            "nvfp4_gemm": (I, [C.POINTER(_Tensor), C.POINTER(_Tensor), I, I, I, I, P, P, I, P, I, P, P,
                               F, P, SZ, P]),
            "nvfp4_program_bytes": (SZ, [I]),
            "nvfp4_program_build": (I, [C.POINTER(_Op), I, P, SZ, C.POINTER(_Program)]),
            "nvfp4_program_run": (I, [C.POINTER(_Program), P]),
            "nvfp4_gemm_noalloc": (I, [C.POINTER(_Tensor), C.POINTER(_Tensor), I, I, I, I, P, P, I, P, I, P,
                                       P, F, P]),
            "nvfp4_gemm_ex": (I, [C.POINTER(_Tensor), C.POINTER(_Tensor), I, I, I, I, P, P, I, P, I, P,
                                  P, F, P, SZ, I, I, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def header_functions():
    """Names of the functions include/nvfp4.h declares."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:nvfp4_status|size_t|const char \*)\s*(nvfp4_\w+)\(", txt, re.M)))


def _check(call, st):
    if st != 0:
        detail = ""
        if STATUS.get(st) == "CUDA error":
            detail = ": " + lib().nvfp4_last_cuda_error_string().decode()
        raise NVFP4Error(call, st, detail)


# ---- torch-facing helpers ---------------------------------------------------------------
def _torch():
    import torch
    return torch


def _ptr(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _stream():
    return C.c_void_p(_torch().cuda.current_stream().cuda_stream)


@dataclass
class NVFP4Tensor:
    """FP4 codes [rows, K/2] (uint8), scale bytes (uint8, nvfp4_sf_bytes), global scale."""
    codes: "object"
    sf: "object"
    global_scale: float
    rows: int
    K: int

    def c(self):
        return _Tensor(self.codes.data_ptr(), self.sf.data_ptr(), self.global_scale, self.rows, self.K)


def sf_bytes(rows, K):
    return int(lib().nvfp4_sf_bytes(rows, K))


def empty_fp4(rows, K, device="cuda", global_scale=1.0):
    """Output buffers for an FP4 tensor; the scale buffer is zeroed (padding must be 0)."""
    torch = _torch()
    codes = torch.empty((rows, K // 2), dtype=torch.uint8, device=device)
    sf = torch.zeros(sf_bytes(rows, K), dtype=torch.uint8, device=device)
    return NVFP4Tensor(codes, sf, global_scale, rows, K)


def _qflags(rotate, fmt):
    if fmt not in ("e2m1", "e0m3"):
        raise ValueError(f"fmt must be 'e2m1' or 'e0m3', got {fmt!r}")
    return (QUANT_ROTATE if rotate else 0) | (QUANT_E0M3 if fmt == "e0m3" else 0)


def quantize_norm(x, kind="none", gamma=None, beta=None, scale=None, shift=None, eps=1e-6,
                  global_scale=1.0, out: Optional[NVFP4Tensor] = None, rotate=False, fmt="e2m1") -> NVFP4Tensor:
    """rotate: Hadamard-rotate each 16-element block before quantizing; fmt "e0m3": uniform
    INT4 elements (a storage format; the GEMM reads E2M1)."""
    torch = _torch()
    M, K = x.shape
    dt = IN_FP32 if x.dtype == torch.float32 else IN_BF16
    if out is None:
        out = empty_fp4(M, K, x.device, global_scale)
    flags = _qflags(rotate, fmt)
    args = (_ptr(x), dt, M, K, x.stride(0), NORM[kind], _ptr(gamma), _ptr(beta), _ptr(scale), _ptr(shift), eps,
            global_scale)
    if flags:
        st = lib().nvfp4_quantize_norm_ex(*args, flags, _ptr(out.codes), _ptr(out.sf), _stream())
    else:
        st = lib().nvfp4_quantize_norm(*args, _ptr(out.codes), _ptr(out.sf), _stream())
    _check("nvfp4_quantize_norm", st)
    out.global_scale = global_scale
    return out


def residual_quantize_norm(x, d, gate, kind="adarms", gamma=None, beta=None, scale=None, shift=None, eps=1e-6,
                           global_scale=1.0, h_out=None, out: Optional[NVFP4Tensor] = None, rotate=False, fmt="e2m1"):
    """h = bf16(x + gate * d) (gate None: 1), stored to h_out (may be x itself), then the norm
    `kind` -> NVFP4 of h.  Returns (h_out, NVFP4Tensor)."""
    torch = _torch()
    M, K = x.shape
    if h_out is None:
        h_out = torch.empty((M, K), dtype=torch.bfloat16, device=x.device)
    if out is None:
        out = empty_fp4(M, K, x.device, global_scale)
    flags = _qflags(rotate, fmt)
    args = (_ptr(x), _ptr(d), _ptr(gate), M, K, x.stride(0), d.stride(0), h_out.stride(0), NORM[kind], _ptr(gamma),
            _ptr(beta), _ptr(scale), _ptr(shift), eps, global_scale)
    if flags:
        st = lib().nvfp4_residual_quantize_norm_ex(*args, flags, _ptr(h_out), _ptr(out.codes), _ptr(out.sf),
                                                   _stream())
    else:
        st = lib().nvfp4_residual_quantize_norm(*args, _ptr(h_out), _ptr(out.codes), _ptr(out.sf), _stream())
    _check("nvfp4_residual_quantize_norm", st)
    out.global_scale = global_scale
    return h_out, out


def norm_f32(x, kind, gamma=None, beta=None, scale=None, shift=None, eps=1e-6, out=None):
    torch = _torch()
    M, K = x.shape
    dt = IN_FP32 if x.dtype == torch.float32 else IN_BF16
    if out is None:
        out = torch.empty((M, K), dtype=torch.float32, device=x.device)
    st = lib().nvfp4_norm_f32(_ptr(x), dt, M, K, x.stride(0), NORM[kind], _ptr(gamma), _ptr(beta),
                              _ptr(scale), _ptr(shift), eps, _ptr(out), _stream())
    _check("nvfp4_norm_f32", st)
    return out


_scratch = {}


def quantize_weight(w, interleave_gate_up=False, scales="amax", rotate=False, fmt="e2m1") -> NVFP4Tensor:
    """bf16 W [N, K] -> NVFP4; scales "amax" (block amax / 6) or "mse" (the scale byte of
    least block squared error); rotate: Hadamard-rotated blocks; fmt "e0m3": uniform INT4."""
    if scales not in ("amax", "mse"):
        raise ValueError(f"scales must be 'amax' or 'mse', got {scales!r}")
    flags = _qflags(rotate, fmt) | (QUANT_MSE if scales == "mse" else 0)
    torch = _torch()
    N, K = w.shape
    out = empty_fp4(N, K, w.device)
    dev = w.device.index if w.device.index is not None else torch.cuda.current_device()
    if dev not in _scratch:
        _scratch[dev] = torch.zeros(256, dtype=torch.uint8, device=w.device)
    g = C.c_float(0.0)
    if flags & (QUANT_ROTATE | QUANT_E0M3):
        name = "nvfp4_quantize_weight_ex"
        st = lib().nvfp4_quantize_weight_ex(_ptr(w), N, K, w.stride(0), int(bool(interleave_gate_up)), flags,
                                            _ptr(out.codes), _ptr(out.sf), C.byref(g), _ptr(_scratch[dev]),
                                            _stream())
    else:
        name = "nvfp4_quantize_weight" if scales == "amax" else "nvfp4_quantize_weight_mse"
        st = getattr(lib(), name)(_ptr(w), N, K, w.stride(0), int(bool(interleave_gate_up)), _ptr(out.codes),
                                  _ptr(out.sf), C.byref(g), _ptr(_scratch[dev]), _stream())
    _check(name, st)
    out.global_scale = g.value
    return out


class Workspace:
    """Caller-owned GEMM workspace: zeroed once when (re)allocated, reused across calls."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = None

    def get(self, nbytes):
        torch = _torch()
        if nbytes == 0:
            return None, 0
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=self.device)
        return self.buf, self.buf.numel()


_default_ws = {}


def gemm(a: NVFP4Tensor, w: NVFP4Tensor, epi="none", bias=None, residual=None, out=None,
         out_global_scale=1.0, workspace: Optional[Workspace] = None, block_n=0, splits=0):
    """a: M x K, w: N x K.  bf16 epilogues return bf16 [M, N]; FP4 epilogues an NVFP4Tensor.

    workspace: split-K scratch (counters + fp32 partials), grown on demand.  Without one the
    device's shared default is used, which is right for GEMMs issued on one stream; GEMMs
    that may run concurrently (several streams) each need their own Workspace."""
    torch = _torch()
    M, N, K = a.rows, w.rows, a.K
    e = EPI[epi]
    fp4 = e in (4, 5, 6, 7)
    if out is None:
        if fp4:
            out = empty_fp4(M, N // 2 if e in (5, 7) else N, a.codes.device, out_global_scale)
        else:
            out = torch.empty((M, N), dtype=torch.bfloat16, device=a.codes.device)
    if workspace is None:
        dev = a.codes.device.index if a.codes.device.index is not None else torch.cuda.current_device()
        workspace = _default_ws.setdefault(dev, Workspace(a.codes.device))
    need = lib().nvfp4_gemm_workspace_bytes_ex(M, N, K, block_n, splits)
    ws, ws_bytes = workspace.get(need)
    ta, tw = a.c(), w.c()
    ldr = residual.stride(0) if residual is not None else 0
    if fp4:
        st = lib().nvfp4_gemm_ex(C.byref(ta), C.byref(tw), M, N, K, e, _ptr(bias), _ptr(residual), ldr,
                                 None, 0, _ptr(out.codes), _ptr(out.sf), out_global_scale, _ptr(ws),
                                 ws_bytes, block_n, splits, _stream())
        out.global_scale = out_global_scale
    else:
        st = lib().nvfp4_gemm_ex(C.byref(ta), C.byref(tw), M, N, K, e, _ptr(bias), _ptr(residual), ldr,
                                 _ptr(out), out.stride(0), None, None, 1.0, _ptr(ws), ws_bytes, block_n,
                                 splits, _stream())
    _check("nvfp4_gemm", st)
    return out


def probe():
    _check("nvfp4_probe", lib().nvfp4_probe())


def device_status():
    """Raises NVFP4Error(TIMEOUT) if a kernel's bounded wait expired since the last check."""
    _check("nvfp4_get_device_status", lib().nvfp4_get_device_status(_stream()))


def mma_rate(n=256, mode=0, ksteps=64):
    """Diagnostics: SM cycles per K step of 256 (four block-scaled MMAs of 128 x n x 64; mode 1
    adds the step's scale-atom copies from the same thread), as (issued, completed)."""
    issue, done = C.c_double(), C.c_double()
    _check("nvfp4_mma_rate", lib().nvfp4_mma_rate(n, mode, ksteps, C.byref(issue), C.byref(done)))
    return issue.value, done.value


# ---- grouped GEMM ------------------------------------------------------------------------
def op_gemm(a: NVFP4Tensor, w: NVFP4Tensor, epi="none", bias=None, residual=None, out=None, out_global_scale=1.0):
    """One problem of a grouped GEMM; `out` is bf16 [M, N] or, for FP4 epilogues, an
    NVFP4Tensor.  Its inputs are ready before the launch (no dependency between problems)."""
    e = EPI[epi]
    op = _Op(type=1, M=a.rows, N=w.rows, K=a.K, A=a.c(), W=w.c(), epi=e, bias=_ptr(bias),
             residual=_ptr(residual), ldr=residual.stride(0) if residual is not None else 0, dep=-1)
    if e in (4, 5, 6, 7):
        op.out_codes, op.out_sf, op.out_global_scale = out.codes.data_ptr(), out.sf.data_ptr(), out_global_scale
    else:
        op.out_bf16, op.ldo, op.out_global_scale = out.data_ptr(), out.stride(0), 1.0
    op.keep = (a, w, bias, residual, out)  # the program only holds raw pointers
    return op


class Program:
    """A built grouped GEMM of ops (nvfp4_program_build; device buffer owned here); run()
    makes one launch.  It keeps the ops, and through them every tensor they name, alive."""

    def __init__(self, ops, device="cuda"):
        self.ops = list(ops)
        torch = _torch()
        n = len(ops)
        arr = (_Op * n)(*ops)
        nbytes = int(lib().nvfp4_program_bytes(n))
        self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        base = (self.buf.data_ptr() + 255) // 256 * 256
        self.prog = _Program()
        _check("nvfp4_program_build", lib().nvfp4_program_build(arr, n, C.c_void_p(base), nbytes, C.byref(self.prog)))
        self.n_ops = n

    def run(self):
        _check("nvfp4_program_run", lib().nvfp4_program_run(C.byref(self.prog), _stream()))


class GroupedGemm:
    """A grouped NVFP4 GEMM: independent problems (a_g, w_g, out_g[, bias_g]), each taking
    the same epilogue kind; problems may differ in M, N and K.  When every N is a multiple of
    128 one launch of the grouped kernel runs them all, streaming the problems' weights back
    to back (`program`, whose built handle is `prog`); otherwise the problems run as standalone
    nvfp4_gemm launches (`program` and `prog` are None)."""

    def __init__(self, problems, epi="none", device="cuda", workspace: Optional["Workspace"] = None):
        self.problems = [(pr[0], pr[1], pr[2], pr[3] if len(pr) > 3 else None) for pr in problems]
        self.epi = epi
        self.workspace = workspace
        self.program = self.prog = None
        if all(w.rows % 128 == 0 for _, w, _, _ in self.problems):
            self.program = Program([op_gemm(a, w, epi, bias=b, out=o) for a, w, o, b in self.problems],
                                   device=device)
            self.prog = self.program.prog

    def run(self):
        if self.program is not None:
            self.program.run()
            return
        for a, w, o, b in self.problems:
            gemm(a, w, self.epi, bias=b, out=o, workspace=self.workspace)
