"""Seeded synthetic inputs, shared by the oracle side and the CUDA side.

This module holds none of the method's arithmetic: a counter-based generator
(SplitMix64, Steele, Lea and Flood, "Fast splittable pseudorandom number generators",
OOPSLA 2014), Box-Muller normals in fp64, and fp32 -> bf16 round-to-nearest-even
packing of the drawn values.  Seeds follow 1000 * workload + tensor id.
"""
import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# tensor ids inside one workload
X, GAMMA, BETA, MOD_SCALE, MOD_SHIFT = 1, 2, 3, 4, 5
W0, BIAS0, RESIDUAL, CONTEXT = 10, 20, 30, 31


def splitmix64(seed: int, n: int) -> np.ndarray:
    """Outputs 1..n of the SplitMix64 stream started at `seed`."""
    with np.errstate(over="ignore"):
        i = np.arange(1, n + 1, dtype=np.uint64)
        z = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + i * _GAMMA
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
        return z ^ (z >> np.uint64(31))


def uniform(seed: int, n: int) -> np.ndarray:
    """Uniform fp64 in the open interval (0, 1)."""
    z = splitmix64(seed, n)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(seed: int, n: int, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """fp64 normals by Box-Muller on consecutive uniform pairs."""
    m = (n + 1) // 2
    u = uniform(seed, 2 * m)
    r = np.sqrt(-2.0 * np.log(u[0::2]))
    th = 2.0 * np.pi * u[1::2]
    z = np.empty(2 * m, np.float64)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    return mean + std * z[:n]


def f32_to_bf16_bits(x) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, np.float32).view(np.uint32)
    with np.errstate(over="ignore"):
        r = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (r >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b) -> np.ndarray:
    return (np.ascontiguousarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_normal(seed: int, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """bf16 bit patterns (uint16) of N(mean, std^2) draws, row-major `shape`."""
    n = int(np.prod(shape))
    return f32_to_bf16_bits(normal(seed, n, mean, std).astype(np.float32)).reshape(shape)


def seed_of(workload: int, tensor_id: int) -> int:
    return 1000 * workload + tensor_id


# ---- the same recipe evaluated with torch on a device (large timing inputs) ----------
def _signed(c: int) -> int:
    return c - (1 << 64) if c >= (1 << 63) else c


def bf16_normal_torch(seed: int, shape, mean: float = 0.0, std: float = 1.0, device="cuda"):
    """SplitMix64 -> Box-Muller -> bf16, computed with torch int64 / fp64 tensors on
    `device`.  Same recipe as bf16_normal; the device's log / sin / cos may differ from
    numpy's in the last fp64 bit, so a rare value can differ by one bf16 step.  Used for
    timing inputs, never for a parity comparison."""
    import torch
    n = 1
    for s in shape:
        n *= int(s)
    m = (n + 1) // 2

    def lsr(z, s):  # logical shift right of the 64-bit pattern
        return (z >> s) & ((1 << (64 - s)) - 1)

    z = torch.arange(1, 2 * m + 1, dtype=torch.int64, device=device)
    z.mul_(_signed(0x9E3779B97F4A7C15)).add_(_signed(seed & 0xFFFFFFFFFFFFFFFF))
    z = z ^ lsr(z, 30)
    z.mul_(_signed(0xBF58476D1CE4E5B9))
    z = z ^ lsr(z, 27)
    z.mul_(_signed(0x94D049BB133111EB))
    z = z ^ lsr(z, 31)
    u = (lsr(z, 11).to(torch.float64) + 0.5) * (2.0 ** -53)
    del z
    r = torch.sqrt(-2.0 * torch.log(u[0::2]))
    th = (2.0 * torch.pi) * u[1::2]
    out = torch.empty(2 * m, dtype=torch.float64, device=device)
    out[0::2] = r * torch.cos(th)
    out[1::2] = r * torch.sin(th)
    out = (mean + std * out[:n]).to(torch.float32)
    return out.to(torch.bfloat16).reshape(tuple(int(s) for s in shape))
