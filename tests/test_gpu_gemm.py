"""GPU parity of the block-scaled NVFP4 GEMM and its fused epilogues against the oracle.

Operands are quantized by the oracle and uploaded, so the GEMM is checked alone: bf16
outputs meet the acceptance bar (relative error <= 1e-2 where |ref| > 1e-2 max|ref|,
cosine >= 0.99999); FP4 outputs meet the boundary-only mismatch bar in parity.py.  Every
tile width (64/128/256) and several split-K factors are pinned explicitly, over shapes
that span several tiles and ragged M / K tails."""
import numpy as np
import pytest

from parity import check_fp4_output, check_gemm_bf16, dev_bf16, host, to_gpu_fp4
from vla_action_head_b200 import nvfp4, synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _probe():
    nvfp4.probe()


def _operands(orc, wl, M, N, K, inter=False):
    x = synth.bf16_normal(synth.seed_of(wl, synth.X), (M, K))
    w = synth.bf16_normal(synth.seed_of(wl, synth.W0), (N, K), 0.0, 0.02)
    ac, asf = orc.quantize_norm(x, "none", g=1.0)
    wc, wsf, gw = orc.quantize_weight(w, interleave_gate_up=inter)
    return (ac, asf, 1.0), (wc, wsf, gw)


def _run(orc, M, N, K, epi, bn=0, sp=0, wl=11, g_out=1.0, geglu_bias=False, rows=None):
    """rows: compare only these output rows (the oracle computes just them)."""
    (ac, asf, ga), (wc, wsf, gw) = _operands(orc, wl, M, N, K)
    uses_bias = epi in ("bias", "bias_residual", "bias_gelu") or (epi == "geglu" and geglu_bias)
    uses_res = epi in ("residual", "bias_residual")
    bias = synth.bf16_normal(synth.seed_of(wl, synth.BIAS0), (N,), 0.0, 0.01) if uses_bias else None
    res = synth.bf16_normal(synth.seed_of(wl, synth.RESIDUAL), (M, N)) if uses_res else None
    ref = orc.gemm(ac, asf, ga, M, wc, wsf, gw, N, K, epi=epi, bias=bias, residual=res, g_out=g_out, rows=rows)
    A = to_gpu_fp4(ac, asf, ga, M, K)
    W = to_gpu_fp4(wc, wsf, gw, N, K)
    out = nvfp4.gemm(A, W, epi, bias=dev_bf16(bias) if uses_bias else None,
                     residual=dev_bf16(res) if uses_res else None, out_global_scale=g_out,
                     block_n=bn, splits=sp)
    if epi in ("bias_gelu", "geglu"):
        n_out = N // 2 if epi == "geglu" else N
        return check_fp4_output(orc, host(out.codes), host(out.sf), ref["codes"], ref["sf"], ref["h"],
                                g_out, M, n_out, what=(M, N, K, epi, bn, sp), sel=rows)
    got = host(out) if rows is None else host(out)[rows]
    return check_gemm_bf16(got, ref["v"], what=(M, N, K, epi, bn, sp))


SHAPES = [(41, 512, 256), (1, 64, 64), (7, 192, 96), (50, 256, 1024), (130, 384, 320), (300, 256, 512),
          (41, 1536, 1536)]


@pytest.mark.parametrize("M,N,K", SHAPES)
def test_default_schedule_bias(orc, M, N, K):
    _run(orc, M, N, K, "bias")


# Every GEMM of the benchmarked workloads at its full size, through the DEFAULT schedule
# (the one bench.py times: latency-model tile width and split factor at M <= 128, the
# persistent kernel above), against the oracle.  Row samples where the oracle would take
# long; the samples include the first and last rows and the M tail.
CONFIG_GEMMS = [
    # tiny: 41 x 256 -> 512 + bias
    (41, 512, 256, "bias", None),
    # DiT layer at M = 41, hidden 1536, FFN 6144
    (41, 4608, 1536, "bias", None),
    (41, 1536, 1536, "bias_residual", None),
    (41, 6144, 1536, "bias_gelu", None),
    (41, 1536, 6144, "bias_residual", None),
    # action-expert layer at M = 50, width 1024, context 2048, gated MLP 2 x 4096
    (50, 2560, 1024, "none", None),
    (50, 1024, 2048, "residual", None),
    (50, 8192, 1024, "geglu", None),
    (50, 1024, 4096, "residual", None),
    # prefill layer at M = 968, width 2048, MLP 2 x 16384
    (968, 2560, 2048, "none", [0, 1, 127, 128, 517, 895, 896, 967]),
    (968, 32768, 2048, "geglu", [0, 200, 895, 967]),
    (968, 2048, 16384, "residual", [0, 128, 767, 967]),
]


@pytest.mark.parametrize("M,N,K,epi,rows", CONFIG_GEMMS, ids=[f"{m}x{n}x{k}-{e}" for m, n, k, e, _ in CONFIG_GEMMS])
def test_config_gemms_default_schedule(orc, M, N, K, epi, rows):
    _run(orc, M, N, K, epi, wl=50, rows=rows)


@pytest.mark.parametrize("M", [1, 16, 41, 128, 512, 968])
def test_m_sweep_default_schedule(orc, M):
    """The M sweep on the 1536 -> 6144 GEMM (+bias), default schedule."""
    rows = None if M <= 128 else sorted({0, 1, 127, 128, M // 2, M - 1})
    _run(orc, M, 6144, 1536, "bias", wl=51, rows=rows)


@pytest.mark.parametrize("bn", [64, 128, 256])
@pytest.mark.parametrize("sp", [1, 2, 3, -2, -3])
def test_every_tile_and_split(orc, bn, sp):
    """sp > 0: split-K reduced in a cluster over DSMEM; sp < 0: through the workspace."""
    _run(orc, 41, 512, 768, "bias_residual", bn=bn, sp=sp)
    _run(orc, 64, 512, 768, "bias", bn=bn, sp=sp)
    _run(orc, 100, 256, 1024, "none", bn=bn, sp=sp)
    _run(orc, 130, 256, 1024, "none", bn=bn, sp=sp)


@pytest.mark.parametrize("sp", [4, 6, 8, -12])
def test_deep_splits(orc, sp):
    _run(orc, 41, 1536, 6144, "bias_residual", bn=64, sp=sp)
    _run(orc, 50, 1024, 4096, "residual", bn=128, sp=sp)


@pytest.mark.parametrize("epi", ["none", "bias", "residual", "bias_residual", "bias_gelu", "geglu"])
@pytest.mark.parametrize("M,sp", [(41, 1), (41, 2), (41, -4), (200, 1)])
def test_epilogues(orc, epi, M, sp):
    _run(orc, M, 512, 512, epi, bn=128, sp=sp)


@pytest.mark.parametrize("g_out", [1.0, 0.02])
def test_geglu_with_bias_and_scale(orc, g_out):
    _run(orc, 50, 1024, 1024, "geglu", bn=256, sp=1, g_out=g_out, geglu_bias=True)
    _run(orc, 50, 1024, 1024, "bias_gelu", bn=64, sp=2, g_out=g_out)


def test_k_tail_zero_padding(orc):
    """K % 64 == 32: the last MMA K step reads TMA zero-fill and zero scale padding."""
    _run(orc, 41, 128, 96, "bias", bn=64, sp=1)
    _run(orc, 41, 128, 4320, "bias", bn=128, sp=2)


@pytest.mark.parametrize("M,bn,sp", [(80, 0, 0), (80, 64, 2), (80, 128, 1), (200, 0, 0)])
def test_extreme_block_scales(orc, M, bn, sp):
    """Operands whose blocks take subnormal, normal and saturated UE4M3 scales.  Activation
    rows of magnitude 1e-2 .. 1e2 in five bands (with g = 1 the 1e-2 band's block scales are
    E4M3 subnormals) and two rows with +-1e4 outliers (saturated scales: the other values of
    those blocks round to small codes or zero); weight rows spanning 1e-6 .. 1 of the
    tensor's amax in four bands (below ~3.5e-5 of the amax a block's scale is subnormal).
    The tensor core must decode every scale byte as the format defines it, which is how the
    oracle decodes it; the output is checked block by block (activation band x weight
    band, outlier rows apart), so that small values are not hidden behind large ones.
    M = 200 runs the persistent kernel (256-wide tiles, two W scale groups per stage)."""
    N, K = 256, 1024
    outl = [3, 42]
    band = np.arange(M) % 5
    x = synth.bf16_bits_to_f32(synth.bf16_normal(synth.seed_of(61, synth.X), (M, K)))
    x = x * (10.0 ** (band - 2.0))[:, None].astype(np.float32)
    x[3, 17], x[3, 500], x[42, 1000] = 1e4, -1e4, 1e4
    w = synth.bf16_bits_to_f32(synth.bf16_normal(synth.seed_of(61, synth.W0), (N, K), 0.0, 0.02))
    w = w * np.logspace(-6, 0, N, dtype=np.float32)[:, None]
    xb, wb = synth.f32_to_bf16_bits(x), synth.f32_to_bf16_bits(w)
    ac, asf = orc.quantize_norm(xb, "none", g=1.0)
    wc, wsf, gw = orc.quantize_weight(wb)
    # the operands do take subnormal (0 < byte < 8) and saturated (0x7E) scale bytes
    assert ((asf > 0) & (asf < 8)).any() and (asf == 0x7E).any() and ((wsf > 0) & (wsf < 8)).any()
    ref = orc.gemm(ac, asf, 1.0, M, wc, wsf, gw, N, K, epi="none")["v"]
    got = host(nvfp4.gemm(to_gpu_fp4(ac, asf, 1.0, M, K), to_gpu_fp4(wc, wsf, gw, N, K), "none",
                          block_n=bn, splits=sp))
    for b in range(5):
        rows = np.array([r for r in np.nonzero(band == b)[0] if r not in outl])
        for c in range(4):
            cols = np.arange(c * N // 4, (c + 1) * N // 4)
            check_gemm_bf16(got[np.ix_(rows, cols)], ref[np.ix_(rows, cols)], what=("band", b, c, bn, sp))
    for r in outl:
        check_gemm_bf16(got[[r]], ref[[r]], what=("outlier row", r, bn, sp))


def test_zero_activations_give_bias(orc):
    M, N, K = 41, 256, 512
    ac = np.zeros((M, K // 2), np.uint8)
    asf = np.zeros(orc.sf_bytes(M, K), np.uint8)
    (_, _, _), (wc, wsf, gw) = _operands(orc, 12, M, N, K)
    bias = synth.bf16_normal(3, (N,), 0.0, 0.5)
    out = nvfp4.gemm(to_gpu_fp4(ac, asf, 1.0, M, K), to_gpu_fp4(wc, wsf, gw, N, K), "bias",
                     bias=dev_bf16(bias))
    assert np.array_equal(host(out), np.broadcast_to(bias, (M, N)))


@pytest.mark.parametrize("sp", [6, -6])
def test_determinism_split_k(orc, sp):
    (ac, asf, ga), (wc, wsf, gw) = _operands(orc, 13, 41, 1536, 6144)
    A, W = to_gpu_fp4(ac, asf, ga, 41, 6144), to_gpu_fp4(wc, wsf, gw, 1536, 6144)
    o1 = host(nvfp4.gemm(A, W, "none", block_n=128, splits=sp))
    o2 = host(nvfp4.gemm(A, W, "none", block_n=128, splits=sp))
    assert np.array_equal(o1, o2)


def test_cluster_and_workspace_reductions_agree(orc):
    """Both reductions add the partials in split order, so they agree bit for bit."""
    (ac, asf, ga), (wc, wsf, gw) = _operands(orc, 14, 41, 1536, 6144)
    A, W = to_gpu_fp4(ac, asf, ga, 41, 6144), to_gpu_fp4(wc, wsf, gw, 1536, 6144)
    o1 = host(nvfp4.gemm(A, W, "none", block_n=64, splits=6))
    o2 = host(nvfp4.gemm(A, W, "none", block_n=64, splits=-6))
    assert np.array_equal(o1, o2)


def test_device_status_clean():
    nvfp4.device_status()


# The default schedule for many rows runs a persistent kernel: one CTA per SM walking
# 128 x 256 or 128 x 128 tiles; an explicit (block_n, splits) runs the one-tile-per-CTA kernel.
@pytest.mark.parametrize("epi", ["none", "bias", "residual", "bias_residual", "bias_gelu", "geglu"])
@pytest.mark.parametrize("N,rows", [(512, None), (10240, [0, 5, 127, 128, 255, 256, 299])])
def test_persistent_epilogues(orc, epi, N, rows):
    """N = 512 runs 128-wide tiles (12 of them), N = 10240 256-wide ones (120); M = 300
    leaves the last 128-row tile 44 valid rows."""
    _run(orc, 300, N, 768, epi, rows=rows)


def test_persistent_multi_tile_and_tails(orc):
    """More tiles than SMs (each CTA walks several), the M tail of 968 = 7 * 128 + 72,
    and a last K tile with an odd number of 64-wide blocks (K = 4160)."""
    rows = [0, 1, 63, 127, 128, 500, 767, 895, 896, 900, 960, 967]
    _run(orc, 968, 5120, 1024, "none", rows=rows)
    _run(orc, 968, 2048, 4160, "residual", rows=rows)
    _run(orc, 968, 4096, 512, "geglu", rows=rows)


@pytest.mark.parametrize("epi", ["none", "bias_residual", "bias_gelu", "geglu"])
def test_persistent_split_k(orc, epi):
    """Fewer output tiles than SMs and a long K: the many-row kernel splits K in two through
    the workspace (M = 256, N = 512, K = 8192: 8 tiles of 128 x 128, 16 units, split 0 of 19
    K tiles and split 1 of 13).  The second split of a tile to arrive adds the other's
    partial to its own."""
    assert nvfp4.lib().nvfp4_gemm_workspace_bytes(256, 512, 8192) > 0  # the split schedule
    _run(orc, 256, 512, 8192, epi, rows=[0, 1, 77, 127, 128, 200, 255])


def test_persistent_split_k_odd_k_tail(orc):
    """Two unequal splits over an odd number of K tiles whose last one is ragged (K = 8320:
    33 K tiles, the last of 128 elements): split 0 takes 20, split 1 the other 13."""
    assert nvfp4.lib().nvfp4_gemm_workspace_bytes(256, 512, 8320) > 0
    _run(orc, 256, 512, 8320, "bias_residual", rows=[0, 3, 127, 128, 254, 255])


@pytest.mark.parametrize("epi", ["residual", "geglu"])
def test_persistent_split_k_one_row_tail(orc, epi):
    """M = 129: the second 128-row tile holds one valid row (lane 0 of the first epilogue
    warp), so the staged bf16 stores and the split partials must skip the other 127."""
    assert nvfp4.lib().nvfp4_gemm_workspace_bytes(129, 512, 8192) > 0
    _run(orc, 129, 512, 8192, epi, rows=[0, 64, 127, 128])


def test_persistent_split_k_prefill_down(orc):
    """The prefill down projection: 968 x 2048 x 16384 + residual, 64 tiles of 128 x 256,
    K split in two (128 units), the M tail of 72 rows."""
    assert nvfp4.lib().nvfp4_gemm_workspace_bytes(968, 2048, 16384) > 0
    _run(orc, 968, 2048, 16384, "residual", rows=[0, 127, 128, 500, 895, 896, 967])


def test_persistent_split_k_deterministic_and_tickets_reset(orc):
    """Two runs give the same bytes whichever split arrives last, and every ticket word is
    zero again afterwards (the workspace is reusable without clearing)."""
    import torch
    M, N, K = 968, 2048, 16384
    (ac, asf, ga), (wc, wsf, gw) = _operands(orc, 36, M, N, K)
    A, W = to_gpu_fp4(ac, asf, ga, M, K), to_gpu_fp4(wc, wsf, gw, N, K)
    ws = nvfp4.Workspace(torch.device("cuda"))
    o1 = host(nvfp4.gemm(A, W, "none", workspace=ws))
    o2 = host(nvfp4.gemm(A, W, "none", workspace=ws))
    torch.cuda.synchronize()
    nvfp4.device_status()
    assert np.array_equal(o1, o2)
    need = nvfp4.lib().nvfp4_gemm_workspace_bytes(M, N, K)
    buf, _ = ws.get(need)
    tickets = host(buf[:16384].view(torch.int32))  # the whole counter region
    assert not tickets.any()


def test_workspace_shared_across_shapes(orc):
    """One workspace serves split-K GEMMs of different shapes in turn: the one-tile kernel's
    partials (many splits, few tiles) never land where the many-row kernel (64 tiles) keeps
    its counters, so the later GEMM still finds its counters zero."""
    import torch
    ws = nvfp4.Workspace(torch.device("cuda"))
    (ac, asf, ga), (wc, wsf, gw) = _operands(orc, 38, 41, 1536, 6144)
    A, W = to_gpu_fp4(ac, asf, ga, 41, 6144), to_gpu_fp4(wc, wsf, gw, 1536, 6144)
    nvfp4.gemm(A, W, "none", workspace=ws, block_n=64, splits=-12)  # partials over 3 MB
    M, N, K = 968, 2048, 16384
    (ac, asf, ga), (wc, wsf, gw) = _operands(orc, 39, M, N, K)
    A, W = to_gpu_fp4(ac, asf, ga, M, K), to_gpu_fp4(wc, wsf, gw, N, K)
    rows = [0, 300, 967]
    got = host(nvfp4.gemm(A, W, "none", workspace=ws))[rows]
    torch.cuda.synchronize()
    nvfp4.device_status()
    ref = orc.gemm(ac, asf, ga, M, wc, wsf, gw, N, K, epi="none", rows=rows)
    check_gemm_bf16(got, ref["v"], what="split-K after another shape's partials")


def test_split_k_wait_expires_and_context_survives(orc):
    """Failure detection without a GPU fault.  Every tile's arrival ticket is preset to 1, as
    if a split had arrived and never published its partial: both real splits of each tile
    then take the reducer's role and wait for a partial that nobody writes.  The bounded wait
    expires (about 2 s), the kernel records a timeout and returns, and the host reads
    NVFP4_ERR_TIMEOUT.  The same GEMM then runs correctly on a cleared workspace."""
    import torch
    M, N, K = 256, 512, 8192
    L = nvfp4.lib()
    need = L.nvfp4_gemm_workspace_bytes(M, N, K)
    assert need > 16384  # the 16 KiB counter region (8 tiles use 64 bytes of it), then the partials
    (ac, asf, ga), (wc, wsf, gw) = _operands(orc, 37, M, N, K)
    A, W = to_gpu_fp4(ac, asf, ga, M, K), to_gpu_fp4(wc, wsf, gw, N, K)
    ws = nvfp4.Workspace(torch.device("cuda"))
    buf, _ = ws.get(need)
    buf[:256].view(torch.int32)[0::2] = 1  # arrival tickets; the published counts stay 0
    nvfp4.gemm(A, W, "none", workspace=ws)
    torch.cuda.synchronize()
    with pytest.raises(nvfp4.NVFP4Error) as err:
        nvfp4.device_status()
    assert err.value.status == 7  # timeout
    nvfp4.device_status()  # read and cleared
    buf.zero_()
    rows = [0, 100, 255]
    ref = orc.gemm(ac, asf, ga, M, wc, wsf, gw, N, K, epi="none", rows=rows)
    got = host(nvfp4.gemm(A, W, "none", workspace=ws))[rows]
    torch.cuda.synchronize()
    nvfp4.device_status()
    check_gemm_bf16(got, ref["v"], what=("after timeout", M, N, K))


def test_mma_rate_diagnostic():
    """The MMA issue-rate diagnostic (nvfp4_mma_rate) runs at every width and both modes, its
    completion count is at least its issue count, the scale copies add cycles (mode 1 over
    mode 0), and a 256-wide MMA is not cheaper than a 64-wide one."""
    rates = {}
    for n in (64, 128, 256):
        for mode in (0, 1):
            issue, done = nvfp4.mma_rate(n, mode, 64)
            assert 10.0 < issue <= done < 1e6, (n, mode, issue, done)
            rates[n, mode] = done
    for n in (64, 128, 256):
        assert rates[n, 1] > rates[n, 0]
    assert rates[256, 0] >= rates[64, 0]
