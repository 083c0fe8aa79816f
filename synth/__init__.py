"""Seeded synthetic inputs for the separated-quantization linear layer.

This module holds no arithmetic of the method itself: it only draws the
weights W and the activations x that both the CUDA path and the CPU oracle
consume.  Every value is a pure function of (seed, stream, element index),
so any row of any matrix can be regenerated on its own, and the device
generator in ``synth_dev.cu`` reproduces the same float32 bits on the GPU.

Definition (shared by both implementations, written independently):

* SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; the constants of Vigna's public-domain
  ``splitmix64.c``): ``mix(z)`` is the output finalizer, the n-th output of
  a generator whose state starts at ``key`` is ``mix(key + (n+1)*GAMMA)``.
* ``key(seed, stream) = mix(seed*GAMMA + stream*STREAM_MUL + STREAM_ADD)``.
* ``u = ((word >> 11) + 0.5) * 2**-53``, a binary64 uniform in (0, 1).
* Laplace(0, b) by the inverse CDF; N(0, 1) by Box-Muller (one output per
  pair of words).  The logarithm and cosine they need are evaluated with
  explicit series in plain binary64 operations (no FMA, fixed order), so the
  host and the device round every step identically: ln m via the atanh
  series on m in [sqrt(1/2), sqrt(2)), cos via its Taylor series on
  [0, pi/2] after exact reduction in the turn domain.
"""
from __future__ import annotations

import numpy as np

MASK64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15
MIX1 = 0xBF58476D1CE4E5B9
MIX2 = 0x94D049BB133111EB
STREAM_MUL = 0xD1B54A32D192ED03
STREAM_ADD = 0x632BE59BD9B4E019

LN2 = float.fromhex("0x1.62e42fefa39efp-1")
SQRT_HALF = float.fromhex("0x1.6a09e667f3bcdp-1")
TWO_PI = float.fromhex("0x1.921fb54442d18p+2")

# stream ids
STREAM_W = 1
STREAM_W_HEAVY = 2
STREAM_X = 3
STREAM_XCAL = 4
STREAM_OUTLIER_CH = 5

_ATANH_TERMS = 12   # odd powers up to z^23
_COS_TERMS = 12     # even powers up to theta^22


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * np.uint64(MIX1)
    z = (z ^ (z >> np.uint64(27))) * np.uint64(MIX2)
    return z ^ (z >> np.uint64(31))


def _mix_int(z: int) -> int:
    z &= MASK64
    z = ((z ^ (z >> 30)) * MIX1) & MASK64
    z = ((z ^ (z >> 27)) * MIX2) & MASK64
    return z ^ (z >> 31)


def key(seed: int, stream: int) -> int:
    return _mix_int(seed * GAMMA + stream * STREAM_MUL + STREAM_ADD)


def words(k: int, counters) -> np.ndarray:
    c = np.asarray(counters, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(k) + (c + np.uint64(1)) * np.uint64(GAMMA)
        return _mix(z)


def uniform(k: int, counters) -> np.ndarray:
    w = words(k, counters)
    return ((w >> np.uint64(11)).astype(np.float64) + 0.5) * 2.0 ** -53


def _atanh_coeffs():
    return [1.0 / (2 * i + 1) for i in range(_ATANH_TERMS)]


def _cos_coeffs():
    d = [1.0]
    for k in range(1, _COS_TERMS):
        d.append(d[-1] / float(-(2 * k - 1) * (2 * k)))
    return d


_CA = _atanh_coeffs()
_CC = _cos_coeffs()


def ln(y: np.ndarray) -> np.ndarray:
    """Natural log of positive normal binary64 values, fixed op sequence."""
    y = np.asarray(y, np.float64)
    m, e = np.frexp(y)
    low = m < SQRT_HALF
    m = np.where(low, m * 2.0, m)
    e = np.where(low, e - 1, e).astype(np.float64)
    z = (m - 1.0) / (m + 1.0)
    z2 = z * z
    p = np.full_like(z, _CA[-1])
    for c in reversed(_CA[:-1]):
        p = p * z2
        p = p + c
    return e * LN2 + (z + z) * p


def cos_turn(u: np.ndarray) -> np.ndarray:
    """cos(2*pi*u) for u in (0, 1), fixed op sequence."""
    u = np.asarray(u, np.float64)
    v = np.where(u >= 0.5, u - 1.0, u)
    a = np.abs(v)
    flip = a > 0.25
    a = np.where(flip, 0.5 - a, a)
    th = a * TWO_PI
    t2 = th * th
    p = np.full_like(th, _CC[-1])
    for c in reversed(_CC[:-1]):
        p = p * t2
        p = p + c
    return np.where(flip, -p, p)


def laplace(k: int, counters, b: float) -> np.ndarray:
    """Laplace(0, b) in binary64 by the inverse CDF."""
    u = uniform(k, counters)
    v = u - 0.5
    a = np.abs(v)
    mag = -ln(1.0 - (a + a))
    t = b * mag
    return np.where(v >= 0.0, t, -t)


def gauss(k: int, counters) -> np.ndarray:
    """N(0, 1) in binary64 by Box-Muller, words 2i and 2i+1 per output i."""
    c = np.asarray(counters, dtype=np.uint64)
    u1 = uniform(k, c * np.uint64(2))
    u2 = uniform(k, c * np.uint64(2) + np.uint64(1))
    r = np.sqrt(-2.0 * ln(u1))
    return r * cos_turn(u2)


# ---- matrices --------------------------------------------------------------

def laplace_matrix(seed: int, N: int, K: int, b: float, rows=None) -> np.ndarray:
    """float32 [len(rows)][K] of Laplace(0, b); element (r, j) uses counter r*K + j."""
    rows = np.arange(N) if rows is None else np.asarray(rows)
    ctr = rows.astype(np.uint64)[:, None] * np.uint64(K) + np.arange(K, dtype=np.uint64)[None, :]
    return laplace(key(seed, STREAM_W), ctr, b).astype(np.float32)


def gauss_heavy_matrix(seed: int, N: int, K: int, sigma: float, heavy_frac: float,
                       heavy_mul: float, rows=None) -> np.ndarray:
    """float32 N(0, sigma^2) where a heavy_frac share of entries is multiplied by heavy_mul."""
    rows = np.arange(N) if rows is None else np.asarray(rows)
    ctr = rows.astype(np.uint64)[:, None] * np.uint64(K) + np.arange(K, dtype=np.uint64)[None, :]
    t = sigma * gauss(key(seed, STREAM_W), ctr)
    if heavy_frac > 0.0:
        hv = uniform(key(seed, STREAM_W_HEAVY), ctr) < heavy_frac
        t = np.where(hv, t * heavy_mul, t)
    return t.astype(np.float32)


def outlier_channels(seed: int, K: int, n_o: int) -> np.ndarray:
    """n_o distinct channels by a partial Fisher-Yates shuffle, sorted ascending."""
    k = key(seed, STREAM_OUTLIER_CH)
    perm = list(range(K))
    w = words(k, np.arange(max(n_o, 1), dtype=np.uint64))
    for i in range(n_o):
        j = i + int(w[i]) % (K - i)
        perm[i], perm[j] = perm[j], perm[i]
    return np.array(sorted(perm[:n_o]), dtype=np.int32)


def channel_factors(K: int, channels, factor: float) -> np.ndarray:
    f = np.ones(K, np.float32)
    f[np.asarray(channels, dtype=np.int64)] = np.float32(factor)
    return f


def activation_matrix(seed: int, stream: int, M: int, K: int, factors: np.ndarray,
                      rows=None) -> np.ndarray:
    """float32 [M][K] of N(0, 1) times a per-channel factor; (t, j) uses counter t*K + j."""
    rows = np.arange(M) if rows is None else np.asarray(rows)
    ctr = rows.astype(np.uint64)[:, None] * np.uint64(K) + np.arange(K, dtype=np.uint64)[None, :]
    g = gauss(key(seed, stream), ctr)
    f = np.asarray(factors, np.float32).astype(np.float64)[None, :]
    return np.where(f != 1.0, g * f, g).astype(np.float32)
