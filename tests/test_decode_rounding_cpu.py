"""The decode kernel's bf16 rounding argument, checked in exact rational arithmetic (CPU).

The fused RMSNorm stores bf16(x * gamma * r) with one rounding (reading R23 of the
RMSNorm Router Top-K A2AV Kernel API Reference, Parameters: the pages fix no
precision).  The kernel forms it in fp32: xg = x * gamma is exact, r = rh + rl
(two fp32), p = fl32(xg * rh); where p lies on a bf16 midpoint or one fp32 ulp
from one, the side is decided by the sign of (p - m) + fma(xg, rl, fma(xg, rh, -p)).
This test restates those steps with exact rationals standing for each IEEE
operation and checks the result against the exactly rounded value, on inputs
steered next to midpoints.  (The kernel itself is compared with the oracle on the
GPU in test_decode_gpu.py.)
"""
import random
from fractions import Fraction as F

import numpy as np


def f32(q: F) -> np.float32:
    x = np.float32(float(q))
    cands = [np.nextafter(x, np.float32(-np.inf)), x, np.nextafter(x, np.float32(np.inf))]
    return np.float32(min(cands, key=lambda c: (abs(F(float(c)) - q), int(bits(c)) & 1)))


def bits(x) -> int:
    return int(np.frombuffer(np.float32(x).tobytes(), np.uint32)[0])


def from_bits(u: int) -> np.float32:
    return np.frombuffer(np.uint32(u & 0xffffffff).tobytes(), np.float32)[0]


def bf16_exact(q: F) -> int:
    """Nearest-even bf16 (as its 16 bits) of a rational."""
    lo = bits(f32(q)) & 0xffff0000
    best = None
    for b in (lo - 0x10000, lo, lo + 0x10000):
        v = from_bits(b)
        if not np.isfinite(v):
            continue
        key = (abs(F(float(v)) - q), (b >> 16) & 1)
        if best is None or key < best[0]:
            best = (key, (b & 0xffffffff) >> 16)
    return best[1]


def kernel_steps(xg: np.float32, rh: np.float32, rl: np.float32) -> int:
    p = f32(F(float(xg)) * F(float(rh)))
    u = bits(p)
    if ((u + 0x8001) & 0xffff) < 3:
        mb = (u & 0xffff0000) | 0x8000
        m = from_bits(mb)
        inner = f32(F(float(xg)) * F(float(rh)) - F(float(p)))       # fmaf(xg, rh, -p): exact
        c = f32(F(float(xg)) * F(float(rl)) + F(float(inner)))       # fmaf(xg, rl, inner)
        d = f32(F(float(f32(F(float(p)) - F(float(m))))) + F(float(c)))
        u = mb
        if d != 0:
            u += -1 if ((bits(d) ^ mb) >> 31) else 1
    uu = bits(from_bits(u))
    return ((uu + 0x7fff + ((uu >> 16) & 1)) & 0xffffffff) >> 16     # nearest-even to bf16


def test_single_rounding_near_midpoints():
    rng = random.Random(7)
    near = 0
    for it in range(6000):
        xb = (rng.getrandbits(15) + 0x2000) << 16 | (rng.getrandbits(1) << 31)
        x = from_bits(xb)
        if not np.isfinite(x) or abs(float(x)) < 1e-20 or abs(float(x)) > 1e20:
            continue
        g = from_bits((0x3f80 + rng.randint(-20, 20)) << 16)
        xg = np.float32(x * g)  # exact: 8-bit by 8-bit significands
        if it % 3:
            # steer x*g*r onto, or within a few fp32 ulps of, a bf16 midpoint
            m = F(float(from_bits((bits(xg) & 0xffff0000) | 0x8000)))
            r = float(m / F(float(xg))) * (1 + rng.uniform(-2e-7, 2e-7))
        else:
            r = rng.uniform(0.25, 4.0)
        rh = np.float32(r)
        rl = np.float32(r - float(rh))
        if ((bits(f32(F(float(xg)) * F(float(rh)))) + 0x8001) & 0xffff) < 3:
            near += 1
        assert kernel_steps(xg, rh, rl) == bf16_exact(F(float(xg)) * F(r)), (float(xg), r)
    assert near > 1000  # the steered cases really exercise the midpoint branch
