"""Counter-based Gaussian gradient streams (the simulated workers' gradients).

Philox4x32-10 is the counter-based generator of Salmon, Moraes, Dror and
Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3" (SC 2011): a 128-bit
counter and a 64-bit key go through ten rounds; each round multiplies two
counter words by fixed odd constants, swaps the words and mixes the high
halves of the products with the other words and the key, and the key is
bumped by two Weyl constants between rounds. Its published known-answer
vectors pin this implementation (tests/test_counter_rng.py).

A gradient entry is a pure function of (worker, matrix, step, entry index),
so the CUDA library can draw the same numbers inside its kernels, and the
oracle can recompute them, without either reading the other:

* key     = (seed_base + worker, matrix_id)
* counter = (g mod 2^32, g div 2^32, step, 0) with g = entry // 4, the entry
  index flat in row-major order
* the four 32-bit outputs give two Box-Muller pairs; entry 4g + j takes the
  j-th Gaussian, times sigma.

The Box-Muller transform is evaluated in float32 with a fixed sequence of
correctly rounded operations (+, -, *, /, sqrt), so that any IEEE float32
implementation that performs the same operations gets the same bits: the
uniforms are exact multiples of 2^-24 (u1 in (0, 1]) and 2^-22 (the angle's
position inside its quadrant), ln is the series 2*atanh((f-1)/(f+1)) after
splitting off the binary exponent, and sin / cos are Taylor polynomials on
[0, pi/2) rotated into the quadrant given by the top two bits. Nothing here
is part of the optimizer's arithmetic; this module only makes inputs.
"""
from __future__ import annotations

import numpy as np

PHILOX_M0 = np.uint64(0xD2511F53)
PHILOX_M1 = np.uint64(0xCD9E8D57)
PHILOX_W0 = np.uint32(0x9E3779B9)
PHILOX_W1 = np.uint32(0xBB67AE85)
_MASK32 = np.uint64(0xFFFFFFFF)

f32 = np.float32


def philox4x32_10(ctr, key):
    """ctr: uint32 array [..., 4]; key: uint32 array [..., 2] (broadcast).
    Returns the uint32 array [..., 4] after ten rounds."""
    c = [np.asarray(ctr[..., i], dtype=np.uint32) for i in range(4)]
    k0 = np.asarray(key[..., 0], dtype=np.uint32)
    k1 = np.asarray(key[..., 1], dtype=np.uint32)
    with np.errstate(over="ignore"):
        for r in range(10):
            if r:
                k0 = (k0 + PHILOX_W0).astype(np.uint32)
                k1 = (k1 + PHILOX_W1).astype(np.uint32)
            p0 = PHILOX_M0 * c[0].astype(np.uint64)
            p1 = PHILOX_M1 * c[2].astype(np.uint64)
            hi0, lo0 = (p0 >> np.uint64(32)).astype(np.uint32), (p0 & _MASK32).astype(np.uint32)
            hi1, lo1 = (p1 >> np.uint64(32)).astype(np.uint32), (p1 & _MASK32).astype(np.uint32)
            c = [hi1 ^ c[1] ^ k0, lo1, hi0 ^ c[3] ^ k1, lo0]
    return np.stack(c, axis=-1)


# float32 constants of the transform (each the float32 nearest to the real number)
_LN2 = f32(np.log(2.0))
_HALF_PI = f32(np.pi / 2)
_SQRT2_BITS = np.uint32(0x3FB504F3)     # float32 just below sqrt(2)
_ATANH = [f32(1.0 / k) for k in (13, 11, 9, 7, 5, 3)]       # series 1 + s/3 + s^2/5 + ...
_SIN = [f32((-1.0) ** i / np.prod(np.arange(1, 2 * i + 2, dtype=np.float64))) for i in range(7)]   # 1, -1/3!, ...
_COS = [f32((-1.0) ** i / np.prod(np.arange(1, 2 * i + 1, dtype=np.float64))) for i in range(8)]   # 1, -1/2!, ...


def ln_f32(u):
    """ln(u) for float32 u in (0, 1], by a fixed sequence of float32 operations."""
    u = np.asarray(u, dtype=f32)
    bits = u.view(np.uint32)
    e = (bits >> np.uint32(23)).astype(np.int32) - 127
    fb = (bits & np.uint32(0x7FFFFF)) | np.uint32(0x3F800000)
    big = fb > _SQRT2_BITS
    fb = np.where(big, fb - np.uint32(0x00800000), fb)  # f / 2, exact
    e = e + big.astype(np.int32)
    f = fb.view(f32)
    t = (f - f32(1)) / (f + f32(1))
    s = t * t
    p = _ATANH[0]
    for c in _ATANH[1:]:
        p = p * s + c
    p = p * s + f32(1)
    lnf = f32(2) * t * p
    return e.astype(f32) * _LN2 + lnf


def sincos_quadrant(q, r):
    """cos and sin of (q + r) * pi/2 for quadrant q in 0..3 and float32 r in [0, 1)."""
    x = np.asarray(r, dtype=f32) * _HALF_PI
    s = x * x
    ps = _SIN[6]
    for c in _SIN[5::-1]:
        ps = ps * s + c
    sn = x * ps
    pc = _COS[7]
    for c in _COS[6::-1]:
        pc = pc * s + c
    cs = pc
    q = np.asarray(q)
    cos_t = np.select([q == 0, q == 1, q == 2], [cs, -sn, -cs], sn)
    sin_t = np.select([q == 0, q == 1, q == 2], [sn, cs, -sn], -cs)
    return cos_t.astype(f32), sin_t.astype(f32)


def box_muller(x0, x1):
    """Two standard normal float32 draws from two uint32 words."""
    u1 = ((x0 >> np.uint32(8)) + np.uint32(1)).astype(f32) * f32(2.0 ** -24)
    q = (x1 >> np.uint32(30)).astype(np.int32)
    r = ((x1 >> np.uint32(8)) & np.uint32(0x3FFFFF)).astype(f32) * f32(2.0 ** -22)
    rad = np.sqrt(f32(-2) * ln_f32(u1)).astype(f32)
    c, s = sincos_quadrant(q, r)
    return rad * c, rad * s


def gaussian_entries(seed_base: int, worker: int, matrix_id: int, step: int, n: int,
                     sigma: float = 1.0) -> np.ndarray:
    """The first n entries (row-major) of one worker's gradient for one matrix at one step."""
    groups = (n + 3) // 4
    g = np.arange(groups, dtype=np.uint64)
    ctr = np.stack([(g & _MASK32).astype(np.uint32), (g >> np.uint64(32)).astype(np.uint32),
                    np.full(groups, step, np.uint32), np.zeros(groups, np.uint32)], axis=-1)
    key = np.array([(seed_base + worker) & 0xFFFFFFFF, matrix_id & 0xFFFFFFFF], dtype=np.uint32)
    x = philox4x32_10(ctr, key[None, :])
    z0, z1 = box_muller(x[:, 0], x[:, 1])
    z2, z3 = box_muller(x[:, 2], x[:, 3])
    z = np.stack([z0, z1, z2, z3], axis=-1).reshape(-1)[:n]
    return (z * f32(sigma)).astype(f32)


def gaussian_matrix(seed_base: int, worker: int, matrix_id: int, step: int, shape, sigma: float = 1.0):
    r, c = shape
    return gaussian_entries(seed_base, worker, matrix_id, step, r * c, sigma).reshape(r, c)
