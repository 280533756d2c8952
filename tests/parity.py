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


def check_fp4_output(orc, gpu_codes, gpu_sf, ref_codes, ref_sf, h_ref, g_out, rows, K, what="", sel=None):
    """Acceptance of an FP4-output epilogue (tanh-GELU / GeGLU) against the oracle, whose
    activation is fp64 while the kernel's is fp32:
      - scale bytes: equal, or one E4M3 step apart, in <= 1e-3 of the blocks;
      - in blocks with equal scales, code mismatches <= 1e-3 of the elements, each at an
        oracle value h/S within 2^-10 (relative) of an E2M1 rounding boundary.
    sel: only these rows of the `rows`-row outputs are compared (h_ref holds just them)."""
    nblk = K // 16
    gs = orc.sf_gather(gpu_sf, rows, K).astype(np.int32)
    rs = orc.sf_gather(ref_sf, rows, K).astype(np.int32)
    if sel is not None:
        gs, rs = gs[sel], rs[sel]
        gpu_codes = np.ascontiguousarray(np.asarray(gpu_codes).reshape(rows, -1)[sel])
        ref_codes = np.ascontiguousarray(np.asarray(ref_codes).reshape(rows, -1)[sel])
        rows = len(sel)
    dif = np.abs(gs - rs)
    assert dif.max() <= 1, (what, "scale bytes differ by more than one step")
    assert (dif != 0).mean() <= 1e-3, (what, float((dif != 0).mean()))
    gc = _unpack(gpu_codes).reshape(rows, nblk, 16)
    rc = _unpack(ref_codes).reshape(rows, nblk, 16)
    same = (dif == 0)
    mism = (gc != rc) & same[:, :, None]
    frac = mism.sum() / max(1, same.sum() * 16)
    assert frac <= 1e-3, (what, float(frac))
    if mism.any():
        S = orc.e4m3_decode(rs.astype(np.uint8)).astype(np.float64) * g_out
        v = np.abs(h_ref.reshape(rows, nblk, 16)) / np.where(S == 0, 1, S)[:, :, None]
        near = np.min(np.abs(v[..., None] - E2M1_BOUNDS) / E2M1_BOUNDS, axis=-1) <= 2.0 ** -10
        bad = mism & ~near
        assert not bad.any(), (what, "code mismatch away from a rounding boundary", int(bad.sum()))
    return float(frac)
