"""Plain CPU oracle for the separated-quantization decode linear layer.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg are the only callers.  The product path
(``decode_matvec_sq_b200``) never imports this package.

The arithmetic lives in ``sq_oracle.c`` (single-threaded C, binary64 and
int64, no FMA contraction); this module only marshals numpy arrays through
ctypes.  Each wrapper names the page section it follows; the C header lists
the sources in full.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "sq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libsq_oracle.so")
# A prebuilt variant of the oracle may be named here; the mutation tests use
# it to load deliberately broken copies in a child process.
_LIB_OVERRIDE = os.environ.get("SQ_ORACLE_LIB")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into ``oracle/libsq_oracle.so``."""
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < max(os.path.getmtime(_SRC),
                                          os.path.getmtime(os.path.join(_HERE, "sq_oracle.h"))))
    if force or stale:
        tmp = _LIB_PATH + ".tmp.%d" % os.getpid()
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB_OVERRIDE:
                lib = ctypes.CDLL(_LIB_OVERRIDE)
            else:
                build()
                lib = ctypes.CDLL(_LIB_PATH)
            i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
            lib.sqo_quantize.argtypes = [dbl, ctypes.c_float]
            lib.sqo_quantize.restype = i32
            lib.sqo_scale_from_absmax.argtypes = [dbl]
            lib.sqo_scale_from_absmax.restype = ctypes.c_float
            lib.sqo_quantize_groups.argtypes = [vp, i64, i32, vp, vp]
            lib.sqo_trunk_threshold.argtypes = [vp, i64, i32, vp]
            lib.sqo_decompose.argtypes = [vp, i64, i64, i32, i32, vp, vp, vp, vp, vp, vp]
            lib.sqo_calibrate.argtypes = [vp, i64, i64, i32, vp]
            lib.sqo_quantize_act.argtypes = [vp, i64, i64, vp, i32, vp, vp, vp]
            lib.sqo_accumulate.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp]
            lib.sqo_trunk_popcount.argtypes = [i64, i64, i64, vp, vp, vp, vp]
            lin = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp, i32, vp]
            lib.sqo_linear.argtypes = lin
            lib.sqo_linear_naive.argtypes = lin
            lib.sqo_linear_trunk.argtypes = [i64, i64, i64, vp, vp, vp, vp, vp, vp, vp, i32, vp]
            lib.sqo_sparsify_residual.argtypes = [vp, i64, i32, i32, vp, vp, vp]
            lib.sqo_quantize_groups_asym.argtypes = [vp, i64, i32, vp, vp, vp]
            lib.sqo_linear_asym.argtypes = [i64, i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                            vp, i32, vp]
            lib.sqo_abs_dot.argtypes = [i64, i64, i64, vp, vp, vp]
            lib.sqo_layer_sq_error.argtypes = [i64, i64, i32, vp, vp, vp, vp, vp, vp, vp, vp]
            lib.sqo_plain_sq_error.argtypes = [i64, i64, i32, vp, vp]
            lib.sqo_e2m1_value.argtypes = [i32]
            lib.sqo_e2m1_value.restype = dbl
            lib.sqo_e2m1_round.argtypes = [dbl]
            lib.sqo_e2m1_round.restype = i32
            lib.sqo_ue4m3_value.argtypes = [i32]
            lib.sqo_ue4m3_value.restype = dbl
            lib.sqo_ue4m3_round.argtypes = [dbl]
            lib.sqo_ue4m3_round.restype = i32
            lib.sqo_nvfp4_quantize.argtypes = [vp, i64, i64, i32, vp, vp, vp]
            lib.sqo_nvfp4_quantize.restype = i32
            lib.sqo_nvfp4_linear.argtypes = [i64, i64, i64, vp, vp, ctypes.c_float, vp, vp, vp, vp]
            lib.sqo_nvfp4_linear.restype = i32
            for name in ("sqo_quantize_groups", "sqo_trunk_threshold", "sqo_decompose",
                         "sqo_calibrate", "sqo_quantize_act", "sqo_accumulate",
                         "sqo_trunk_popcount", "sqo_linear", "sqo_linear_naive", "sqo_linear_trunk",
                         "sqo_sparsify_residual", "sqo_quantize_groups_asym", "sqo_linear_asym",
                         "sqo_abs_dot", "sqo_layer_sq_error", "sqo_plain_sq_error"):
                getattr(lib, name).restype = i32
            _lib = lib
    return _lib


class OracleError(RuntimeError):
    pass


def _ck(rc: int, name: str, allow_nonfinite: bool = False) -> int:
    if rc == 1:
        raise OracleError(f"{name}: invalid argument")
    if rc == 2 and not allow_nonfinite:
        raise OracleError(f"{name}: non-finite input")
    return rc


def _p(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(np.asarray(a, dtype=dtype))


def n_groups(K: int, G: int) -> int:
    return (K + G - 1) // G


# ---- scalar quantizer ([P3] s3.1, [P2] absmax) -------------------------------

def quantize(v: float, s: float) -> int:
    """Q(v, s) = clip(round_half_away(v / s), +-127); 0 when s == 0."""
    return int(_load().sqo_quantize(float(v), float(np.float32(s))))


def scale_from_absmax(a: float) -> np.float32:
    """s = (float)(a / 127) ([P3] s3.1 step 2, divide convention)."""
    return np.float32(_load().sqo_scale_from_absmax(float(a)))


def quantize_groups(r, G: int):
    """One residual row, symmetric INT8 per group of G ([P2] Q4_K blocks)."""
    r = _c(r, np.float64)
    K = r.shape[0]
    q = np.zeros(K, np.int8)
    s = np.zeros(n_groups(K, G), np.float32)
    _ck(_load().sqo_quantize_groups(_p(r), K, G, _p(q), _p(s)), "quantize_groups")
    return q, s


def trunk_threshold(w, P: int) -> np.float32:
    """Nearest-rank P-th percentile of |w| ([P1] s5.2)."""
    w = _c(w, np.float32)
    tau = np.zeros(1, np.float32)
    _ck(_load().sqo_trunk_threshold(_p(w), w.shape[0], int(P), _p(tau)), "trunk_threshold")
    return tau[0]


# ---- offline decomposition ([P1] s2.1, s5.3, s6.2) --------------------------

def decompose(W, G: int = 128, P: int = -1, want_residual: bool = False):
    """Unpacked decomposition of W[N][K]: dict of sign, mask, alpha, q, s (and res)."""
    W = _c(W, np.float32)
    N, K = W.shape
    out = dict(sign=np.zeros((N, K), np.uint8), mask=np.zeros((N, K), np.uint8),
               alpha=np.zeros(N, np.float32), q=np.zeros((N, K), np.int8),
               s=np.zeros((N, n_groups(K, G)), np.float32))
    res = np.zeros((N, K), np.float64) if want_residual else None
    rc = _load().sqo_decompose(_p(W), N, K, G, int(P), _p(out["sign"]), _p(out["mask"]),
                               _p(out["alpha"]), _p(res), _p(out["q"]), _p(out["s"]))
    out["status"] = _ck(rc, "decompose", allow_nonfinite=True)
    if want_residual:
        out["res"] = res
    out["G"] = G
    return out


# ---- calibration and activations ([P1] s2.2, [P2] dynamic quantization) -----

def sparsify_residual(r, G: int, Ps: int):
    """One residual row r[K] (float64): drop the entries at or below the
    nearest-rank Ps-th percentile of |r| (strict > keeps), quantize the kept
    ones by groups ([P1] s3.3, sparse residual).  Returns keep, q, s."""
    r = _c(r, np.float64)
    K = r.shape[0]
    keep = np.zeros(K, np.uint8)
    q = np.zeros(K, np.int8)
    s = np.zeros(n_groups(K, G), np.float32)
    _ck(_load().sqo_sparsify_residual(_p(r), K, G, Ps, _p(keep), _p(q), _p(s)), "sparsify_residual")
    return keep, q, s


def decompose_sparse(W, G: int = 128, P: int = -1, Ps: int = 60):
    """decompose() with the residual sparsified row by row (keys as
    decompose, plus keep [N][K] uint8)."""
    d = decompose(W, G=G, P=P, want_residual=True)
    N, K = d["res"].shape
    keep = np.zeros((N, K), np.uint8)
    q = np.zeros_like(d["q"])
    s = np.zeros_like(d["s"])
    for r in range(N):
        keep[r], q[r], s[r] = sparsify_residual(d["res"][r], G, Ps)
    d = dict(d, q=q, s=s, keep=keep)
    return d


def quantize_groups_asym(r, G: int):
    """One residual row, asymmetric INT8 per group: own min/max, scale and
    zero-point ([P1] s2 pitfalls, [P3] asymmetric quantization).  q, s, z."""
    r = _c(r, np.float64)
    K = r.shape[0]
    q = np.zeros(K, np.int8)
    s = np.zeros(n_groups(K, G), np.float32)
    z = np.zeros(n_groups(K, G), np.int32)
    _ck(_load().sqo_quantize_groups_asym(_p(r), K, G, _p(q), _p(s), _p(z)), "quantize_groups_asym")
    return q, s, z


def decompose_asym(W, G: int = 128, P: int = -1):
    """decompose() with asymmetric residual groups (keys as decompose, plus z)."""
    d = decompose(W, G=G, P=P, want_residual=True)
    N = d["res"].shape[0]
    q, s = np.zeros_like(d["q"]), np.zeros_like(d["s"])
    z = np.zeros(d["s"].shape, np.int32)
    for r in range(N):
        q[r], s[r], z[r] = quantize_groups_asym(d["res"][r], G)
    return dict(d, q=q, s=s, z=z)


def linear_asym(d, xq, sx, xout, idx):
    """y = sx*(alpha*T + sum_g s_g*(R_g - z_g*S_g)) + sum_i What*xout (binary64)."""
    xq = _c(xq, np.int8)
    M, K = xq.shape
    N = d["sign"].shape[0]
    idx = _c(idx, np.int32)
    n = idx.shape[0]
    sx = _c(sx, np.float32)
    xout = _c(xout, np.float32).reshape(M, n) if n else np.zeros((M, 1), np.float32)
    y = np.zeros((M, N), np.float64)
    _ck(_load().sqo_linear_asym(M, N, K, d["G"], _p(d["sign"]), _p(d["mask"]), _p(d["alpha"]),
                                _p(d["q"]), _p(d["s"]), _p(_c(d["z"], np.int32)), _p(xq), _p(sx),
                                _p(xout), _p(idx) if n else None, n, _p(y)), "linear_asym")
    return y


def calibrate(X, k: int) -> np.ndarray:
    X = _c(X, np.float32)
    T, K = X.shape
    idx = np.zeros(k, np.int32)
    _ck(_load().sqo_calibrate(_p(X), T, K, int(k), _p(idx)), "calibrate", allow_nonfinite=True)
    return idx


def quantize_act(x, idx):
    x = _c(x, np.float32)
    if x.ndim == 1:
        x = x[None, :]
    M, K = x.shape
    idx = _c(idx, np.int32)
    n = idx.shape[0]
    xq = np.zeros((M, K), np.int8)
    sx = np.zeros(M, np.float32)
    xout = np.zeros((M, max(n, 1)), np.float32)
    _ck(_load().sqo_quantize_act(_p(x), M, K, _p(idx) if n else None, n, _p(xq), _p(sx),
                                 _p(xout)), "quantize_act", allow_nonfinite=True)
    return xq, sx, xout[:, :n]


# ---- accumulators and output ([P1] s2.3, s3.3) -------------------------------

def accumulate(d, xq):
    xq = _c(xq, np.int8)
    M, K = xq.shape
    N = d["sign"].shape[0]
    G = d["G"]
    T = np.zeros((M, N), np.int64)
    R = np.zeros((M, N, n_groups(K, G)), np.int64)
    _ck(_load().sqo_accumulate(M, N, K, G, _p(d["sign"]), _p(d["mask"]), _p(d["q"]), _p(xq),
                               _p(T), _p(R)), "accumulate")
    return T, R


def trunk_popcount(d, xq):
    xq = _c(xq, np.int8)
    M, K = xq.shape
    N = d["sign"].shape[0]
    T = np.zeros((M, N), np.int64)
    _ck(_load().sqo_trunk_popcount(M, N, K, _p(d["sign"]), _p(d["mask"]), _p(xq), _p(T)),
        "trunk_popcount")
    return T


def _linear(fn, d, xq, sx, xout, idx):
    xq = _c(xq, np.int8)
    M, K = xq.shape
    N = d["sign"].shape[0]
    idx = _c(idx, np.int32)
    n = idx.shape[0]
    sx = _c(sx, np.float32)
    xout = _c(xout, np.float32).reshape(M, n) if n else np.zeros((M, 1), np.float32)
    y = np.zeros((M, N), np.float64)
    _ck(fn(M, N, K, d["G"], _p(d["sign"]), _p(d["mask"]), _p(d["alpha"]), _p(d["q"]),
           _p(d["s"]), _p(xq), _p(sx), _p(xout), _p(idx) if n else None, n, _p(y)), "linear")
    return y


def linear(d, xq, sx, xout, idx):
    """Factored y = sx*(alpha*T + sum_g s_g*R_g) + sum_i What*xout (binary64)."""
    return _linear(_load().sqo_linear, d, xq, sx, xout, idx)


def linear_naive(d, xq, sx, xout, idx):
    """Second route: y = sum_j What_j * xhat_j (binary64)."""
    return _linear(_load().sqo_linear_naive, d, xq, sx, xout, idx)


def linear_trunk(d, xq, sx, xout, idx):
    """Trunk-only y = sx*alpha*T + sum_i Wt*xout, Wt = m*alpha*(2b-1): the
    residual path skipped ([P1] s3.3, binary64)."""
    xq = _c(xq, np.int8)
    M, K = xq.shape
    N = d["sign"].shape[0]
    idx = _c(idx, np.int32)
    n = idx.shape[0]
    sx = _c(sx, np.float32)
    xout = _c(xout, np.float32).reshape(M, n) if n else np.zeros((M, 1), np.float32)
    y = np.zeros((M, N), np.float64)
    _ck(_load().sqo_linear_trunk(M, N, K, _p(d["sign"]), _p(d["mask"]), _p(d["alpha"]), _p(xq),
                                 _p(sx), _p(xout), _p(idx) if n else None, n, _p(y)),
        "linear_trunk")
    return y


def abs_dot(W, x):
    """Tolerance scale sum_j |W_rj x_tj| from the original fp32 values, [M][N]."""
    W = _c(W, np.float32)
    x = _c(x, np.float32)
    if x.ndim == 1:
        x = x[None, :]
    M, K = x.shape
    N = W.shape[0]
    out = np.zeros((M, N), np.float64)
    _ck(_load().sqo_abs_dot(M, N, K, _p(W), _p(x), _p(out)), "abs_dot")
    return out


def reference_forward(W, x, idx, G: int = 128, P: int = -1):
    """Whole path on the CPU: decompose, split activations, output."""
    d = decompose(W, G=G, P=P)
    xq, sx, xout = quantize_act(x, idx)
    y = linear(d, xq, sx, xout, idx)
    return d, (xq, sx, xout), y


def layer_sq_error(d, W) -> float:
    """sum over the layer of (W - What)^2 for decomposition d (symmetric, or
    asymmetric when d has "z"), binary64 ([P1] s2.3: the fallback measure)."""
    W = _c(W, np.float32)
    N, K = W.shape
    z = d.get("z")
    out = np.zeros(1, np.float64)
    _ck(_load().sqo_layer_sq_error(N, K, d["G"], _p(W), _p(_c(d["sign"], np.uint8)),
                                   _p(_c(d["mask"], np.uint8)), _p(_c(d["alpha"], np.float32)),
                                   _p(_c(d["q"], np.int8)), _p(_c(d["s"], np.float32)),
                                   None if z is None else _p(_c(z, np.int32)), _p(out)),
        "layer_sq_error")
    return float(out[0])


def plain_sq_error(W, G: int = 128) -> float:
    """The same error for plain symmetric INT8 groups of W (no trunk)."""
    W = _c(W, np.float32)
    N, K = W.shape
    out = np.zeros(1, np.float64)
    _ck(_load().sqo_plain_sq_error(N, K, G, _p(W), _p(out)), "plain_sq_error")
    return float(out[0])


def choose_fallback(W, P: int = -1, G: int = 128) -> bool:
    """The per-layer rule ([P1] s2.3, last paragraph: a layer that gains
    nothing from the split falls back to plain 8-bit): fall back when plain
    INT8 groups reconstruct W at least as well as the split does."""
    return plain_sq_error(W, G) <= layer_sq_error(decompose(W, G=G, P=P), W)


# ---- NVFP4 prefill format (the ISTA-DASLab page on separated quantization,
# paragraphs 2-4: hardware-native NVFP4 for prefill).  The format's reading is
# in sq_oracle.h.

def e2m1_value(code: int) -> float:
    return float(_load().sqo_e2m1_value(int(code)))


def e2m1_round(v: float) -> int:
    return int(_load().sqo_e2m1_round(float(v)))


def ue4m3_value(code: int) -> float:
    return float(_load().sqo_ue4m3_value(int(code)))


def ue4m3_round(v: float) -> int:
    return int(_load().sqo_ue4m3_round(float(v)))


def nvfp4_quantize(X, per_row: bool):
    """X [R][K] -> dict(codes [R][K] uint8 (one E2M1 code per byte), scales
    [R][ceil(K/16)] uint8 (UE4M3), g [R] float32 (per row) or [1] (per
    tensor))."""
    X = _c(X, np.float32)
    R, K = X.shape
    codes = np.zeros((R, K), np.uint8)
    scales = np.zeros((R, (K + 15) // 16), np.uint8)
    g = np.zeros(R if per_row else 1, np.float32)
    _ck(_load().sqo_nvfp4_quantize(_p(X), R, K, int(bool(per_row)), _p(codes), _p(scales), _p(g)),
        "sqo_nvfp4_quantize")
    return {"codes": codes, "scales": scales, "g": g}


def nvfp4_linear(w, x):
    """y [M][N] (binary64) = sum_j What_rj * xhat_tj for a per-tensor
    quantized weight w and per-token quantized activations x."""
    wc, ws = _c(w["codes"], np.uint8), _c(w["scales"], np.uint8)
    xc, xs, gx = _c(x["codes"], np.uint8), _c(x["scales"], np.uint8), _c(x["g"], np.float32)
    N, K = wc.shape
    M = xc.shape[0]
    y = np.zeros((M, N), np.float64)
    _ck(_load().sqo_nvfp4_linear(M, N, K, _p(wc), _p(ws), float(w["g"][0]), _p(xc), _p(xs),
                                 _p(gx), _p(y)), "sqo_nvfp4_linear")
    return y
