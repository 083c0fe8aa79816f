"""CPU checks of the two arithmetic claims the activation kernels rely on,
against the oracle and exact arithmetic (no GPU):

1. The token scale computed as one binary32 division, a / 127, equals the
   oracle's float(a / 127.0) (binary64 quotient rounded to binary32).
2. The kernels' rounding decision (k = floor(|v| * (1/s)) in binary32, then
   code k + 1 iff (k + 1/2) s - |v| <= 0, a sign the fused multiply-add keeps
   exactly) equals round-half-away-from-zero of |v| / s, as the oracle
   quantizer computes it, midpoints included.

The decision is restated here with numpy binary32 operations; the sign of
(k + 1/2) s - |v| is taken in binary64, where (k + 1/2) s is exact and the
subtraction keeps the sign of the exact difference.
"""
import numpy as np

import oracle


def test_scale_binary32_division_equals_oracle_rounding():
    rng = np.random.default_rng(11)
    # three whole binades, every subnormal, and random finite bit patterns
    parts = [np.arange(1, 1 << 23, dtype=np.uint32).view(np.float32)]
    for e in (-3, 0, 9):
        b = np.array([2.0 ** e], np.float32).view(np.uint32)[0]
        parts.append((b + np.arange(1 << 23, dtype=np.uint32)).view(np.float32))
    parts.append(rng.integers(0, 0x7F7FFFFF, 4_000_000, dtype=np.uint64).astype(np.uint32).view(np.float32))
    a = np.concatenate(parts)
    fast = a / np.float32(127.0)
    ref = (a.astype(np.float64) / 127.0).astype(np.float32)
    assert np.array_equal(fast.view(np.uint32), ref.view(np.uint32))
    # and the oracle's own routine on a sample
    for x in a[:: len(a) // 2000]:
        assert oracle.scale_from_absmax(float(x)).view(np.uint32) == np.float32(x / np.float32(127.0)).view(np.uint32)


def _kernel_decision(v: np.ndarray, s: np.float32) -> np.ndarray:
    """Codes by the kernels' binary32 procedure (common case 2^-100 < s, |v| < 2^100)."""
    av = np.abs(v).astype(np.float32)
    rinv = np.float32(1.0) / s
    k = np.floor(av * rinv).astype(np.float32)
    d = (k.astype(np.float64) + 0.5) * np.float64(s) - av.astype(np.float64)
    q = np.where(d <= 0.0, k + np.float32(1.0), k)
    q = np.minimum(q, np.float32(127.0)).astype(np.int64)
    return np.where(v < 0, -q, q)


def test_rounding_decision_equals_oracle_quantizer():
    rng = np.random.default_rng(12)
    checked = 0
    for trial in range(400):
        a = np.float32(rng.choice([1e-20, 1e-3, 0.7, 1.0, 3.0, 50.0, 1e5, 1e20]) * rng.uniform(0.5, 2.0))
        s = a / np.float32(127.0)
        v = rng.uniform(-1.0, 1.0, 64).astype(np.float32) * a
        # exact half-steps (k + 1/2) s where representable, and their neighbours
        k = rng.integers(0, 127, 32)
        mids = ((k + 0.5) * np.float64(s)).astype(np.float32)
        v = np.concatenate([v, mids, np.nextafter(mids, np.float32(0)), np.nextafter(mids, np.float32(np.inf)),
                            -mids, np.array([a, -a, 0.0], np.float32)])
        got = _kernel_decision(v, s)
        ref = np.array([oracle.quantize(float(x), float(s)) for x in v])
        assert np.array_equal(got, ref), (a, v[got != ref][:4])
        checked += v.size
    assert checked > 50_000
