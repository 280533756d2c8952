"""Host-side checks of the C ABI (no GPU needed): the library loads and exports every
function include/nvfp4.h declares, its layout helpers agree with the oracle, and argument
validation rejects bad calls before touching the device."""
import ctypes as C

import pytest

from vla_action_head_b200 import build, nvfp4


@pytest.fixture(scope="module")
def L():
    build.build()
    return nvfp4.lib()


def test_exports_every_declared_function(L):
    names = nvfp4.header_functions()
    assert {"nvfp4_quantize_norm", "nvfp4_quantize_weight", "nvfp4_gemm"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for s in range(8):
        assert L.nvfp4_status_string(s)
    assert L.nvfp4_status_string(99) == b"unknown status"


def test_sf_layout_matches_oracle(L, orc):
    for rows, K in ((1, 16), (41, 1536), (130, 4320), (968, 2048), (300, 96)):
        assert L.nvfp4_sf_bytes(rows, K) == orc.sf_bytes(rows, K)
        for r in range(0, rows, max(1, rows // 37)):
            for b in range(0, K // 16, max(1, K // 16 // 23)):
                assert L.nvfp4_sf_offset(r, b, K) == orc.sf_offset(r, b, K)


def test_workspace_sizes(L):
    assert L.nvfp4_gemm_workspace_bytes_ex(968, 2560, 2048, 256, 1) == 0
    assert L.nvfp4_gemm_workspace_bytes_ex(41, 1536, 6144, 128, 4) == 0  # reduced in a cluster
    ws = L.nvfp4_gemm_workspace_bytes_ex(41, 1536, 6144, 128, -4)  # reduced through the workspace
    assert ws >= 4 * 41 * 1536 * 4
    assert L.nvfp4_gemm_workspace_bytes_ex(41, 1536, 6144, 0, -1) > 0
    assert L.nvfp4_gemm_workspace_bytes_ex(41, 1536, 6144, 96, 1) == 0  # N % 96 != 0
    # many rows: 64 tiles of 128 x 256 on 148 SMs, K = 16384 split in two through the
    # workspace (the fixed 16 KiB counter region, then two fp32 partials of 8 whole 128-row
    # tiles x N)
    region = 16384
    assert L.nvfp4_gemm_workspace_bytes(968, 2048, 16384) == region + 2 * 1024 * 2048 * 4
    assert L.nvfp4_gemm_workspace_bytes(968, 32768, 2048) == 0  # 1024 tiles: no split
    assert L.nvfp4_gemm_workspace_bytes(968, 2560, 2048) == 0  # 80 tiles, 8 K tiles: no split
    # 8 tiles of 128 x 128 and 32 K tiles: split in two
    assert L.nvfp4_gemm_workspace_bytes(256, 512, 8192) == region + 2 * 256 * 512 * 4
    assert L.nvfp4_gemm_workspace_bytes(129, 512, 8192) == region + 2 * 256 * 512 * 4  # whole tiles
    # the one-tile kernel's partials (splits x M x N) also start after the counter region
    assert L.nvfp4_gemm_workspace_bytes_ex(41, 1536, 6144, 64, -12) == region + 12 * 41 * 1536 * 4
    # 128 tiles of 128 x 128 cover the SMs at 16 K tiles: no split
    assert L.nvfp4_gemm_workspace_bytes(968, 2048, 4096) == 0
    assert L.nvfp4_gemm_workspace_bytes(256, 256, 512) == 0  # 2 K tiles: a split does not pay


def _t(codes=0x1000, sf=0x2000, g=1.0, rows=4, K=64):
    return nvfp4._Tensor(codes, sf, g, rows, K)


def test_gemm_validation(L):
    A, W = _t(rows=4, K=64), _t(rows=64, K=64)
    out = C.c_void_p(0x3000)
    g = L.nvfp4_gemm
    ok_args = dict(epi=0, bias=None, res=None, ldr=0, out=out, ldo=64)

    def call(a=A, w=W, M=4, N=64, K=64, epi=0, bias=None, res=None, ldr=0, out=out, ldo=64,
             oc=None, osf=None, og=1.0, ws=None, wsb=0):
        return g(C.byref(a) if a is not None else None, C.byref(w) if w is not None else None, M, N, K,
                 epi, bias, res, ldr, out, ldo, oc, osf, og, ws, wsb, None)

    assert call(a=None) == 1
    assert call(M=5) == 1                      # A->rows != M
    assert call(epi=9) == 1
    assert call(N=32, w=_t(rows=32, K=64)) == 2          # N % 64
    assert call(K=48, a=_t(rows=4, K=48), w=_t(rows=64, K=48)) == 2  # K % 32
    assert call(epi=1) == 1                    # bias required
    assert call(epi=2) == 1                    # residual required
    assert call(epi=4) == 1                    # FP4 epilogue needs out_codes / out_sf
    assert call(a=_t(g=0.0)) == 1              # global scale out of range
    assert call(a=_t(g=float("inf"))) == 1
    assert call(ldo=60) == 1                   # ldo < N
    assert call(out=C.c_void_p(0x3008)) == 3   # misaligned output
    assert call(a=_t(codes=0x1004)) == 3       # misaligned codes
    assert call(ldo=68) == 3                   # ld not a multiple of 8
    # valid arguments reach the device check: no GPU here
    assert call() in (5, 6)
    # M == 0 is a no-op: valid shapes and scales are enough (no pointer is read, no device
    # call is made), while a malformed call with M == 0 is still rejected
    empty = _t(rows=0, K=64, codes=0, sf=0)
    assert call(a=empty, M=0, out=None, ldo=0, epi=3) == 0
    assert call(a=empty, M=0, epi=9) == 1
    assert call(a=empty, M=0, N=32, w=_t(rows=32, K=64)) == 2


def test_mma_rate_validation(L):
    out1, out2 = C.c_double(), C.c_double()
    for n, mode, ksteps in ((96, 0, 64), (64, 2, 64), (128, 0, 0), (256, 1, 4097)):
        assert L.nvfp4_mma_rate(n, mode, ksteps, C.byref(out1), C.byref(out2)) == 1
    assert L.nvfp4_mma_rate(64, 0, 64, None, C.byref(out2)) == 1


def test_norm_and_weight_validation(L):
    q = L.nvfp4_quantize_norm
    x, c, s = C.c_void_p(0x1000), C.c_void_p(0x2000), C.c_void_p(0x4000)
    assert q(None, 0, 4, 64, 64, 0, None, None, None, None, 1e-6, 1.0, c, s, None) == 1
    assert q(x, 0, 4, 72, 72, 0, None, None, None, None, 1e-6, 1.0, c, s, None) == 2  # K % 16
    assert q(x, 0, 4, 64, 60, 0, None, None, None, None, 1e-6, 1.0, c, s, None) == 1  # ldx < K
    assert q(x, 0, 4, 64, 64, 7, None, None, None, None, 1e-6, 1.0, c, s, None) == 1  # kind
    assert q(x, 0, 4, 64, 64, 0, None, None, None, None, 1e-6, -1.0, c, s, None) == 1  # scale
    assert q(C.c_void_p(0x1002), 0, 4, 64, 64, 0, None, None, None, None, 1e-6, 1.0, c, s, None) == 3
    assert q(x, 0, 4, 64, 64, 0, None, None, None, None, 1e-6, 1.0, c, s, None) in (5, 6)
    w = L.nvfp4_quantize_weight
    gs = C.c_float()
    assert w(x, 64, 64, 64, 0, c, s, None, x, None) == 1
    assert w(x, 63, 64, 64, 1, c, s, C.byref(gs), x, None) == 2  # interleave needs even N
    assert w(x, 64, 64, 64, 0, c, s, C.byref(gs), x, None) in (5, 6)


def test_default_schedules_of_the_workload_gemms(L):
    """The latency model's picks for the small-M GEMMs of the benchmarked layers, as CTA
    counts (trace words / 8) on a 148-SM device: the choices the in-chain A/B measurements
    settled on (64-wide tiles; the DiT FFN-down GEMM on 6 splits, one CTA per SM, rather
    than 8).  Host logic only: no device call is made for M <= 64."""
    if L.nvfp4_gemm_trace_words(41, 4608, 1536, 1) == 0:
        pytest.skip("schedule query unavailable")
    picks = {  # (M, N, K, epilogue) -> CTAs
        (41, 4608, 1536, 1): 72 * 2,   # DiT qkv: 64-wide x 2 splits
        (41, 1536, 1536, 3): 24 * 6,   # DiT attention-out: 64 x 6
        (41, 6144, 1536, 4): 96 * 2,   # DiT FFN-up (bias+GELU -> FP4): 64 x 2
        (41, 1536, 6144, 3): 24 * 6,   # DiT FFN-down: 64 x 6 (K tiles >= 16: <= one CTA per SM)
        (50, 2560, 1024, 0): 40 * 4,   # action-expert qkv: 64 x 4
        (50, 1024, 2048, 2): 16 * 8,   # action-expert attention-out
        (50, 8192, 1024, 5): 128,      # action-expert gate/up (GeGLU)
        (50, 1024, 4096, 2): 16 * 8,   # action-expert down
    }
    for (M, N, K, epi), ctas in picks.items():
        assert L.nvfp4_gemm_trace_words(M, N, K, epi) == 8 * ctas, (M, N, K, epi)

