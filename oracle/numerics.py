"""Storage rounding, the counter-based generator and the Haar rotation (oracle side).

Test infrastructure only; see oracle/__init__.py.

Readings (the JoLT pages fix none of these):
* factors and core are stored as bf16, residual scales as fp16 (saturating at 65504);
  rounding is round-to-nearest-even from float64;
* random numbers come from SplitMix64 (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014): the key of stream `s` under seed `k`
  is mix64(k + mix64(s + 1)); word i of that stream is mix64(key + (i + 1) * gamma),
  i.e. output i of a SplitMix64 generator whose state starts at the key;
* uniforms take the top 53 bits; normals are Box-Muller pairs
  (z0, z1) = sqrt(-2 ln(1 - u1)) * (cos(2 pi u2), sin(2 pi u2)) from words 2j, 2j+1;
* the "random orthogonal rotation" of the Abstract is a Haar matrix: the Q factor of a
  D x D standard-normal matrix with the signs of R's diagonal moved into Q
  (Mezzadri, "How to generate random matrices from the classical compact groups",
  Notices AMS 2007). Stream 1 draws it; stream 2 + lt draws the sketch of layer-tensor lt.
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX_M1 = 0xBF58476D1CE4E5B9
MIX_M2 = 0x94D049BB133111EB
TWO_PI = 6.283185307179586           # float64 nearest to 2*pi
STREAM_ROTATION = 1
STREAM_SKETCH0 = 2


# ----------------------------------------------------------------------------- rounding
def round_sig(x, sig_bits: int, min_exp: int):
    """Round float64 values to `sig_bits` significant bits, round-half-even.

    `min_exp` is the exponent (of 2) of the smallest normal number; below it the grid is
    uniform with spacing 2**(min_exp - sig_bits + 1) (gradual underflow).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    xm = x[nz]
    _, e = np.frexp(xm)                       # xm = m * 2**e, 0.5 <= |m| < 1
    e = np.maximum(e - 1, min_exp)            # exponent of the leading bit, clamped to subnormal range
    q = np.ldexp(1.0, e - (sig_bits - 1))     # grid spacing at this binade
    out[nz] = np.round(xm / q) * q            # xm / q is exact (power-of-two scale); np.round is half-even
    out[~np.isfinite(x)] = x[~np.isfinite(x)]
    return out


def round_bf16(x):
    """float64 -> nearest bf16 value (8 significant bits, normal range from 2**-126)."""
    return round_sig(x, 8, -126)


def round_fp16_sat(x):
    """float64 -> nearest fp16 value, saturating at +-65504 (11 significant bits, 2**-14)."""
    r = round_sig(x, 11, -14)
    return np.clip(r, -65504.0, 65504.0)


def round_f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)


def bf16_bits(x) -> np.ndarray:
    """Bit patterns (uint16) of values already on the bf16 grid."""
    return (np.asarray(x, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint32) << 16).view(np.float32).astype(np.float64)


def fp16_bits(x) -> np.ndarray:
    return np.asarray(x, dtype=np.float16).view(np.uint16)


def fp16_from_bits(b) -> np.ndarray:
    return np.asarray(b, dtype=np.uint16).view(np.float16).astype(np.float64)


# ----------------------------------------------------------------------------- SplitMix64
def mix64(z):
    """SplitMix64 output finaliser on uint64 arrays (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX_M1)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX_M2)
        z = z ^ (z >> np.uint64(31))
    return z


def splitmix64_outputs(state: int, n: int) -> np.ndarray:
    """First n outputs of a SplitMix64 generator whose state starts at `state`."""
    i = np.arange(1, n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        s = np.uint64(state & MASK64) + i * np.uint64(GAMMA)
    return mix64(s)


def stream_key(seed: int, stream: int) -> int:
    inner = int(mix64(np.array([(stream + 1) & MASK64], dtype=np.uint64))[0])
    return int(mix64(np.array([(seed + inner) & MASK64], dtype=np.uint64))[0])


def stream_words(seed: int, stream: int, start: int, n: int) -> np.ndarray:
    """Words start .. start+n-1 of stream `stream` under `seed`."""
    key = stream_key(seed, stream)
    i = np.arange(start + 1, start + n + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        s = np.uint64(key) + i * np.uint64(GAMMA)
    return mix64(s)


def uniform53(w) -> np.ndarray:
    return (np.asarray(w, dtype=np.uint64) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def gaussians(seed: int, stream: int, n: int) -> np.ndarray:
    """Normals 0 .. n-1 of a stream: element n is component n % 2 of Box-Muller pair n // 2."""
    npairs = (n + 1) // 2
    w = stream_words(seed, stream, 0, 2 * npairs)
    u1 = uniform53(w[0::2])
    u2 = uniform53(w[1::2])
    r = np.sqrt(-2.0 * np.log(1.0 - u1))
    th = TWO_PI * u2
    z = np.empty(2 * npairs)
    z[0::2] = r * np.cos(th)
    z[1::2] = r * np.sin(th)
    return z[:n]


# ----------------------------------------------------------------------------- rotation
def haar_rotation(seed: int, D: int) -> np.ndarray:
    """Seeded Haar-random orthogonal D x D matrix Pi (float64)."""
    G = gaussians(seed, STREAM_ROTATION, D * D).reshape(D, D)
    Q, R = np.linalg.qr(G)
    sgn = np.where(np.diag(R) < 0, -1.0, 1.0)
    return Q * sgn[None, :]


def hadamard_matrix(D: int) -> np.ndarray:
    """Sylvester Hadamard matrix (D a power of two): H[i, j] = (-1)^popcount(i & j)."""
    assert D > 0 and D & (D - 1) == 0
    i = np.arange(D)
    par = np.zeros((D, D), dtype=np.int64)
    a = i[:, None] & i[None, :]
    while a.any():
        par ^= a & 1
        a = a >> 1
    return np.where(par == 1, -1.0, 1.0)


def hadamard_signs(seed: int, D: int) -> np.ndarray:
    """Random signs of the randomized Hadamard rotation: s_i = -1 when the top bit of word i of
    the rotation stream is set, +1 otherwise."""
    w = stream_words(seed, STREAM_ROTATION, 0, D)
    return np.where((w >> np.uint64(63)) == 1, -1.0, 1.0)


def hadamard_rotation(seed: int, D: int) -> np.ndarray:
    """Randomized Hadamard rotation Pi = diag(s) H / sqrt(D) (float64)."""
    return hadamard_signs(seed, D)[:, None] * hadamard_matrix(D) / np.sqrt(D)


def rotation_matrix(seed: int, D: int, kind: str = "haar") -> np.ndarray:
    """The codec's rotation: Haar (default) or randomized Hadamard."""
    return hadamard_rotation(seed, D) if kind == "hadamard" else haar_rotation(seed, D)


def sketch_matrix(seed: int, lt: int, HD: int, l: int) -> np.ndarray:
    """Gaussian sketch Omega (HD x l) of layer-tensor lt, entries rounded to bf16."""
    z = gaussians(seed, STREAM_SKETCH0 + lt, HD * l).reshape(HD, l)
    return round_bf16(z)
