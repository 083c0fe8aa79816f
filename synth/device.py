"""Device-side generation of the synthetic inputs (same bits as the host).

Wraps ``libsqsynth.so`` (synth_dev.cu).  Used to create full-size weights and
activations directly in device memory; the host functions of :mod:`synth`
regenerate any subset of rows for the CPU oracle.
"""
from __future__ import annotations

import ctypes
import os

import synth

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsqsynth.so")
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m decode_matvec_sq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        u64, i64, dbl, vp = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
        L.synth_fill_laplace.argtypes = [vp, i64, u64, u64, dbl, vp]
        L.synth_fill_laplace.restype = ctypes.c_int
        L.synth_fill_gauss.argtypes = [vp, i64, i64, u64, u64, dbl, u64, dbl, dbl, vp, vp]
        L.synth_fill_gauss.restype = ctypes.c_int
        _lib = L
    return _lib


def _stream():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def fill_weights(layer, out, row0: int = 0):
    """out[rows][K] (float32 device) <- rows [row0, row0 + rows) of the layer's W."""
    rows, K = out.shape
    assert K == layer.K and out.is_contiguous()
    ctr0 = row0 * K
    n = rows * K
    if layer.w_kind == "laplace":
        rc = lib().synth_fill_laplace(ctypes.c_void_p(out.data_ptr()), n, ctr0,
                                      synth.key(layer.seed, synth.STREAM_W), layer.w_scale, _stream())
    else:
        rc = lib().synth_fill_gauss(ctypes.c_void_p(out.data_ptr()), n, K, ctr0,
                                    synth.key(layer.seed, synth.STREAM_W), layer.w_scale,
                                    synth.key(layer.seed, synth.STREAM_W_HEAVY), layer.heavy_frac,
                                    layer.heavy_mul, None, _stream())
    if rc != 0:
        raise RuntimeError(f"synth device fill failed ({rc})")
    return out


def fill_activations(layer, out, stream_id: int = synth.STREAM_X, factors=None, row0: int = 0):
    """out[M][K] (float32 device) <- N(0,1) activations times the channel factors."""
    import torch
    M, K = out.shape
    if factors is None:
        factors = torch.from_numpy(layer.factors()).to(out.device)
    rc = lib().synth_fill_gauss(ctypes.c_void_p(out.data_ptr()), M * K, K, row0 * K,
                                synth.key(layer.seed, stream_id), 1.0, 0, 0.0, 1.0,
                                ctypes.c_void_p(factors.data_ptr()), _stream())
    if rc != 0:
        raise RuntimeError(f"synth device fill failed ({rc})")
    return out
