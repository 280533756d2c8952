"""Shared helpers of the GPU parity tests: host<->device marshalling and the acceptance
checks.  Expected values always come from the oracle (oracle/), never from the GPU."""
import numpy as np

E2M1_BOUNDS = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])


def dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).cuda().view(torch.bfloat16)


def dev_u8(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.uint8)).cuda()


def dev_f32(a):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).cuda()


def host(t):
    import torch
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def bf16_to_f64(bits):
    return (np.ascontiguousarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_gpu_fp4(codes, sf, g, rows, K):
    from vla_action_head_b200 import nvfp4
    return nvfp4.NVFP4Tensor(dev_u8(codes), dev_u8(sf), float(g), rows, K)


def check_gemm_bf16(out_bits, ref, what=""):
    """Acceptance of a bf16 GEMM output against the oracle's fp64 value: per-element relative
    error <= 1e-2 wherever |ref| > 1e-2 max|ref|, and cosine >= 0.99999."""
    got = bf16_to_f64(out_bits)
    assert got.shape == ref.shape, what
    assert np.all(np.isfinite(got)), what
    big = np.abs(ref) > 1e-2 * np.abs(ref).max()
    rel = np.abs(got - ref)[big] / np.abs(ref)[big]
    assert rel.size == 0 or rel.max() <= 1e-2, (what, float(rel.max()))
    cos = (got * ref).sum() / np.sqrt((got * got).sum() * (ref * ref).sum() + 1e-300)
    assert cos >= 0.99999 or np.abs(ref).max() == 0, (what, float(cos))
    return float(cos)


def _unpack(codes):
    c = np.ascontiguousarray(codes, np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c & 15
    out[..., 1::2] = c >> 4
    return out


E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
NEAR = 2.0 ** -10  # relative distance to a rounding boundary that fp32-vs-fp64 h may cross


def _e4m3_bounds(orc):
    """Midpoints between consecutive finite non-negative UE4M3 values (0x00..0x7E): the
    points where round-to-nearest of t = a / (6 g) changes its scale byte."""
    vals = orc.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)
    return 0.5 * (vals[1:] + vals[:-1])


def _near(x, bounds):
    """|x| within NEAR (relative) of one of `bounds` (positive), elementwise."""
    x = np.abs(np.asarray(x, np.float64))
    return np.min(np.abs(x[..., None] - bounds) / bounds, axis=-1) <= NEAR


def _codes_valid(gc, h, S):
    """Whether every code of gc [.., 16] is a correct E2M1 rounding of h / S: the nearest grid
    magnitude (ties and values within NEAR of a boundary may take either neighbour), the
    sign of h unless the magnitude is 0; S == 0 (zero scale) requires all-zero codes."""
    mag = (gc & 7).astype(np.int64)
    sgn = (gc >> 3).astype(np.int64)
    Sx = np.broadcast_to(np.asarray(S, np.float64)[..., None], h.shape)
    v = np.abs(h) / np.where(Sx == 0, 1.0, Sx)
    lo = np.clip(np.searchsorted(E2M1_GRID, v, side="right") - 1, 0, 7)  # grid point <= v
    hi = np.minimum(lo + 1, 7)
    dlo, dhi = v - E2M1_GRID[lo], E2M1_GRID[hi] - v
    nearest = np.where(dhi < dlo, hi, lo)
    nearest = np.where(v >= 6.0, 7, nearest)  # satfinite
    other = np.where(nearest == lo, hi, lo)
    ok_mag = (mag == nearest) | ((mag == other) & _near(v, E2M1_BOUNDS))
    ok_sgn = (mag == 0) | (sgn == (h < 0))
    ok = ok_mag & ok_sgn
    return np.where(Sx == 0, gc == 0, ok)


def check_fp4_output(orc, gpu_codes, gpu_sf, ref_codes, ref_sf, h_ref, g_out, rows, K, what="", sel=None):
    """Acceptance of an FP4-output epilogue (tanh-GELU / GeGLU) against the oracle, whose
    activation h is fp64 while the kernel's is fp32 (a few fp32 ulps apart):
      - scale bytes: equal, or one E4M3 step apart in <= 1e-3 of the blocks, and only where
        the oracle's t = a / (6 g_out) (a = max |fp32(h)| of the block) lies within 2^-10
        (relative) of an E4M3 rounding boundary;
      - every GPU code, in every block, is an E2M1 rounding of h / S_gpu with the GPU's own
        block scale S_gpu: the nearest grid value, or its other neighbour where h / S_gpu is
        within 2^-10 of a rounding boundary; the sign of h unless the code is zero;
      - in blocks with equal scales, codes that differ from the oracle's <= 1e-3 of the
        elements.
    sel: only these rows of the `rows`-row outputs are compared (h_ref holds just them)."""
    nblk = K // 16
    gs = orc.sf_gather(gpu_sf, rows, K).astype(np.int32)
    rs = orc.sf_gather(ref_sf, rows, K).astype(np.int32)
    if sel is not None:
        gs, rs = gs[sel], rs[sel]
        gpu_codes = np.ascontiguousarray(np.asarray(gpu_codes).reshape(rows, -1)[sel])
        ref_codes = np.ascontiguousarray(np.asarray(ref_codes).reshape(rows, -1)[sel])
        rows = len(sel)
    h = np.asarray(h_ref, np.float64).reshape(rows, nblk, 16)
    dif = np.abs(gs - rs)
    assert dif.max() <= 1, (what, "scale bytes differ by more than one step")
    assert (dif != 0).mean() <= 1e-3, (what, float((dif != 0).mean()))
    if (dif != 0).any():
        a = np.abs(h.astype(np.float32).astype(np.float64)).max(axis=-1)
        t = a / (6.0 * float(np.float32(g_out)))
        off = (dif != 0) & ~_near(t, _e4m3_bounds(orc))
        assert not off.any(), (what, "scale byte differs away from an E4M3 rounding boundary", int(off.sum()))
    gc = _unpack(gpu_codes).reshape(rows, nblk, 16)
    rc = _unpack(ref_codes).reshape(rows, nblk, 16)
    S_gpu = orc.e4m3_decode(gs.astype(np.uint8)).astype(np.float64) * g_out
    valid = _codes_valid(gc, h, S_gpu)
    assert valid.all(), (what, "GPU code is not an E2M1 rounding of h / S_gpu", int((~valid).sum()))
    same = (dif == 0)
    mism = (gc != rc) & same[:, :, None]
    frac = mism.sum() / max(1, same.sum() * 16)
    assert frac <= 1e-3, (what, float(frac))
    return float(frac)
