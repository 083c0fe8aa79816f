"""Python binding of libsq, the separated-quantization decode linear layer.

Argument marshalling only: every step of the path runs in the CUDA kernels of
``libsq.so`` (include/sq.h).  PyTorch provides device memory and the stream.
There is no CPU fallback: importing works without a GPU (so the library can
be inspected), but every call needs the built library and an sm_100 device,
and fails loudly otherwise.

Method (m.lqnn.cn/news/241359, sections 2.1-2.3): W ~ alpha_r*sign(W) + W_res
with an INT8 group residual, activations split into cached fp32 outlier
channels and per-token INT8 codes, and one fused kernel summing the trunk
(bit operations), the residual (integer products) and the outliers.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libsq.so")
HEADER = os.path.join(os.path.dirname(PKG_DIR), "include", "sq.h")

SQ_LAUNCH_PDL = 1
SQ_TRUNK_ONLY = 2
SQ_LAYOUT_ROWS = 0
SQ_LAYOUT_TILES = 1
SQ_LAYOUT_TILES_SPARSE = 2
SQ_LAYOUT_TILES_ASYM = 3

STATUS = {
    0: "SQ_OK", 1: "SQ_ERR_INVALID_ARG", 2: "SQ_ERR_SHAPE", 3: "SQ_ERR_ALIGN",
    4: "SQ_ERR_UNSUPPORTED_DEVICE", 5: "SQ_ERR_CUDA", 6: "SQ_ERR_NONFINITE",
    7: "SQ_ERR_TIMEOUT", 8: "SQ_ERR_WORKSPACE",
}
STATUS_CODE = {v: k for k, v in STATUS.items()}


class SQError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        self.name = STATUS.get(code, f"status {code}")
        super().__init__(f"{where}: {self.name}")


class SqPackedWeight(ctypes.Structure):
    _fields_ = [
        ("N", ctypes.c_int32), ("K", ctypes.c_int32), ("group_size", ctypes.c_int32),
        ("layout", ctypes.c_int32), ("sign_stride", ctypes.c_int32), ("res_stride", ctypes.c_int32),
        ("scale_stride", ctypes.c_int32),
        ("sign_bits", ctypes.c_void_p), ("mask_bits", ctypes.c_void_p),
        ("alpha", ctypes.c_void_p), ("res_q", ctypes.c_void_p), ("res_scale", ctypes.c_void_p),
        ("keep_bits", ctypes.c_void_p), ("res_bytes", ctypes.c_void_p),
        ("res_zero", ctypes.c_void_p),
    ]


class SqNvfp4Matrix(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int32), ("K", ctypes.c_int32), ("per_row", ctypes.c_int32),
        ("rows_pad", ctypes.c_int32), ("code_stride", ctypes.c_int32), ("sf_chunks", ctypes.c_int32),
        ("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("g", ctypes.c_void_p),
    ]


_lib = None


def lib():
    """The loaded libsq.so; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m decode_matvec_sq_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, u32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_uint32, ctypes.c_size_t
    pw = ctypes.POINTER(SqPackedWeight)
    nm = ctypes.POINTER(SqNvfp4Matrix)
    sig = {
        "sq_nvfp4_bytes": ([i32, i32, i32], sz),
        "sq_nvfp4_view": ([vp, i32, i32, i32, nm], ctypes.c_int),
        "sq_nvfp4_quantize": ([vp, nm, vp, vp], ctypes.c_int),
        "sq_nvfp4_linear": ([nm, nm, vp, vp, vp], ctypes.c_int),
        "sq_testing_nvfp4_stalled": ([nm, nm, vp, i32, ctypes.c_uint64, vp, vp], ctypes.c_int),
        "sq_testing_mma_peak": ([i32, i32, ctypes.POINTER(ctypes.c_double), vp, vp], ctypes.c_int),
        "sq_testing_read_peak": ([vp, ctypes.c_uint64, i32, ctypes.POINTER(ctypes.c_double), vp], ctypes.c_int),
        "sq_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "sq_device_check": ([], ctypes.c_int),
        "sq_packed_bytes": ([i32, i32, i32, i32, i32], sz),
        "sq_packed_view": ([vp, i32, i32, i32, i32, i32, pw], ctypes.c_int),
        "sq_decompose_pack": ([vp, i32, i32, i32, pw, vp, vp], ctypes.c_int),
        "sq_decompose_pack_sparse": ([vp, i32, i32, i32, i32, pw, vp, vp], ctypes.c_int),
        "sq_residual_errors_scratch_bytes": ([i32], sz),
        "sq_residual_errors": ([vp, pw, vp, vp, sz, vp, vp], ctypes.c_int),
        "sq_decompose_pack_auto": ([vp, i32, i32, i32, pw, vp, sz, vp, vp, vp, vp], ctypes.c_int),
        "sq_calibrate_outliers": ([vp, i32, i32, i32, vp, vp, vp], ctypes.c_int),
        "sq_quantize_act": ([vp, i32, i32, vp, i32, vp, vp, vp, vp, u32, vp], ctypes.c_int),
        "sq_linear_workspace_bytes": ([pw, i32], sz),
        "sq_quantize_linear_workspace_bytes": ([pw, i32, i32], sz),
        "sq_quantize_linear_tokens_per_pass": ([pw, i32], i32),
        "sq_linear_tokens_per_pass": ([pw, u32], i32),
        "sq_linear": ([pw, vp, vp, vp, vp, i32, i32, vp, vp, sz, vp, u32, vp], ctypes.c_int),
        "sq_linear_accumulators": ([pw, vp, vp, vp, vp, i32, i32, vp, vp, vp, vp, sz, vp, u32, vp],
                                   ctypes.c_int),
        "sq_linear_noalloc": ([pw, vp, vp, vp, vp, i32, i32, vp, vp, u32, vp], ctypes.c_int),
        "sq_quantize_linear": ([pw, vp, i32, vp, i32, vp, vp, sz, vp, u32, vp], ctypes.c_int),
        "sq_testing_prefill_stalled": ([pw, vp, vp, vp, vp, i32, i32, vp, i32, ctypes.c_uint64, vp,
                                        vp], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        fn = getattr(L, name)
        fn.argtypes = args
        fn.restype = res
    _lib = L
    return L


def _ck(rc: int, where: str) -> None:
    if rc != 0:
        raise SQError(rc, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def round_up(a: int, b: int) -> int:
    return ceil_div(a, b) * b


def device_check() -> None:
    _ck(lib().sq_device_check(), "sq_device_check")


# ---- packed weights ------------------------------------------------------------

def default_layout(group_size: int) -> int:
    """The tensor-core layout for group size 128, the row layout otherwise."""
    return SQ_LAYOUT_TILES if group_size == 128 else SQ_LAYOUT_ROWS


@dataclass
class PackedWeight:
    """A packed weight in one device allocation (``buf``) with its C view.
    The array accessors return the raw arrays in the weight's layout
    (include/sq.h documents both layouts)."""
    N: int
    K: int
    group_size: int
    with_mask: bool
    layout: int
    buf: object                 # torch.uint8 device tensor
    view: SqPackedWeight

    @property
    def nbytes(self) -> int:
        return int(self.buf.numel())

    @property
    def tiled(self) -> bool:
        return self.layout in (SQ_LAYOUT_TILES, SQ_LAYOUT_TILES_SPARSE, SQ_LAYOUT_TILES_ASYM)

    @property
    def rows(self) -> int:
        """Rows of every array: N, or N padded to 16 in the tiled layouts."""
        return round_up(self.N, 16) if self.tiled else self.N

    def _arr(self, field: str, dtype, shape):
        import torch
        base = self.buf.data_ptr()
        off = getattr(self.view, field) - base
        count = 1
        for s in shape:
            count *= s
        itemsize = torch.empty(0, dtype=dtype).element_size()
        return self.buf[off:off + count * itemsize].view(dtype).view(*shape)

    def sign_bits(self):
        import torch
        return self._arr("sign_bits", torch.int32, (self.rows, self.view.sign_stride))

    def mask_bits(self):
        import torch
        if not self.with_mask:
            return None
        return self._arr("mask_bits", torch.int32, (self.rows, self.view.sign_stride))

    def alpha(self):
        import torch
        return self._arr("alpha", torch.float32, (self.rows,))[:self.N]

    def res_q(self):
        import torch
        return self._arr("res_q", torch.int8, (self.rows, self.view.res_stride))

    def res_scale(self):
        import torch
        return self._arr("res_scale", torch.float32, (self.rows, self.view.scale_stride))

    def res_zero(self):
        """Zero-points of the asymmetric residual, indexed like res_scale."""
        import torch
        if self.layout != SQ_LAYOUT_TILES_ASYM:
            return None
        return self._arr("res_zero", torch.int32, (self.rows, self.view.scale_stride))

    def keep_bits(self):
        import torch
        if self.layout != SQ_LAYOUT_TILES_SPARSE:
            return None
        return self._arr("keep_bits", torch.int32, (self.rows, self.view.sign_stride))

    def res_bytes(self):
        """Packed code bytes of every tile (sparse layout)."""
        import torch
        if self.layout != SQ_LAYOUT_TILES_SPARSE:
            return None
        tiles = (self.rows // 16) * (self.view.res_stride // 128)
        return self._arr("res_bytes", torch.int32, (tiles,))


def packed_bytes(N: int, K: int, group_size: int = 128, with_mask: bool = False,
                 layout: int = None) -> int:
    if layout is None:
        layout = default_layout(group_size)
    return int(lib().sq_packed_bytes(N, K, group_size, int(with_mask), layout))


def alloc_packed(N: int, K: int, group_size: int = 128, with_mask: bool = False,
                 layout: int = None, device=None) -> PackedWeight:
    import torch
    if layout is None:
        layout = default_layout(group_size)
    nbytes = packed_bytes(N, K, group_size, with_mask, layout)
    if nbytes == 0:
        raise SQError(STATUS_CODE["SQ_ERR_SHAPE"], "sq_packed_bytes")
    buf = torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")
    v = SqPackedWeight()
    _ck(lib().sq_packed_view(_ptr(buf), N, K, group_size, int(with_mask), layout,
                             ctypes.byref(v)), "sq_packed_view")
    return PackedWeight(N, K, group_size, with_mask, layout, buf, v)


def decompose_pack(W, trunk_percent: int = -1, group_size: int = 128, layout: int = None,
                   out: PackedWeight = None, status=None, stream=None) -> PackedWeight:
    """Offline split of W[N][K] (float32, device) into the packed form
    (default layout: tiles for group size 128, rows otherwise)."""
    N, K = W.shape
    if out is None:
        out = alloc_packed(N, K, group_size, trunk_percent > 0, layout, device=W.device)
    _ck(lib().sq_decompose_pack(_ptr(W), N, K, trunk_percent, ctypes.byref(out.view),
                                _ptr(status), _stream(stream)), "sq_decompose_pack")
    return out


def decompose_pack_sparse(W, residual_percent: int, trunk_percent: int = -1,
                          out: PackedWeight = None, status=None, stream=None) -> PackedWeight:
    """sq_decompose_pack with the residual entries at or below the per-row
    residual_percent-th percentile of |r| dropped, into SQ_LAYOUT_TILES_SPARSE."""
    N, K = W.shape
    if out is None:
        out = alloc_packed(N, K, 128, trunk_percent > 0, SQ_LAYOUT_TILES_SPARSE, device=W.device)
    _ck(lib().sq_decompose_pack_sparse(_ptr(W), N, K, trunk_percent, residual_percent,
                                       ctypes.byref(out.view), _ptr(status), _stream(stream)),
        "sq_decompose_pack_sparse")
    return out


def residual_errors(W, pw: PackedWeight, status=None, stream=None):
    """(err_split, err_plain): sum over the layer of (W - What)^2 for the
    packed weight and for plain symmetric INT8 groups of W (binary64, on the
    device; include/sq.h sq_residual_errors).  Reads the two numbers back."""
    import torch
    err = torch.zeros(2, dtype=torch.float64, device=W.device)
    nb = int(lib().sq_residual_errors_scratch_bytes(pw.N))
    scratch = torch.empty(nb, dtype=torch.uint8, device=W.device)
    _ck(lib().sq_residual_errors(_ptr(W), ctypes.byref(pw.view), _ptr(err), _ptr(scratch), nb,
                                 _ptr(status), _stream(stream)), "sq_residual_errors")
    e = err.cpu().tolist()
    return e[0], e[1]


def decompose_pack_auto(W, trunk_percent: int = -1, layout: int = None, status=None, stream=None):
    """The split with the per-layer fallback (include/sq.h
    sq_decompose_pack_auto): plain INT8 groups (an empty trunk) when they
    reconstruct W at least as well as the split.  Returns (packed weight,
    fell_back).  Synchronous."""
    import torch
    N, K = W.shape
    out = alloc_packed(N, K, 128, True, layout, device=W.device)
    nb = int(lib().sq_residual_errors_scratch_bytes(N)) + 256
    scratch = torch.empty(nb, dtype=torch.uint8, device=W.device)
    fell = ctypes.c_int32(0)
    _ck(lib().sq_decompose_pack_auto(_ptr(W), N, K, trunk_percent, ctypes.byref(out.view),
                                     _ptr(scratch), nb, ctypes.byref(fell), None, _ptr(status),
                                     _stream(stream)), "sq_decompose_pack_auto")
    if not out.view.mask_bits:
        out.with_mask = False
    return out, bool(fell.value)


def calibrate_outliers(X, k: int, out=None, status=None, stream=None):
    """Top-k channels of X[T][K] by max |x| (ties: lower channel), ascending int32."""
    import torch
    T, K = X.shape
    idx = out if out is not None else torch.empty(k, dtype=torch.int32, device=X.device)
    _ck(lib().sq_calibrate_outliers(_ptr(X), T, K, k, _ptr(idx), _ptr(status), _stream(stream)),
        "sq_calibrate_outliers")
    return idx


def quantize_act(x, idx, xq=None, sx=None, x_out=None, status=None, pdl: bool = False,
                 stream=None):
    """x[M][K] float32 -> (xq [M][roundup(K,128)] int8, sx [M], x_out [M][n_out])."""
    import torch
    M, K = x.shape
    n = 0 if idx is None else int(idx.numel())
    dev = x.device
    if xq is None:
        xq = torch.empty(M, round_up(K, 128), dtype=torch.int8, device=dev)
    if sx is None:
        sx = torch.empty(M, dtype=torch.float32, device=dev)
    if x_out is None:
        x_out = torch.empty(M, max(n, 1), dtype=torch.float32, device=dev)
    _ck(lib().sq_quantize_act(_ptr(x), M, K, _ptr(idx) if n else None, n, _ptr(xq), _ptr(sx),
                              _ptr(x_out) if n else None, _ptr(status),
                              SQ_LAUNCH_PDL if pdl else 0, _stream(stream)), "sq_quantize_act")
    return xq, sx, x_out


def workspace_bytes(pw: PackedWeight, M: int = 1) -> int:
    return int(lib().sq_linear_workspace_bytes(ctypes.byref(pw.view), M))


def workspace_counters(ws, pw: PackedWeight, M: int = 1):
    """The per-row arrival counters inside a workspace (they end every call at zero)."""
    base = workspace_bytes(pw, M) - round_up(4 * pw.N, 256)
    return ws[base: base + 4 * pw.N]


def new_workspace(pw: PackedWeight, M: int = 1, device=None):
    """A zero-filled workspace for sq_linear (zero once; calls keep it zeroed)."""
    import torch
    return torch.zeros(max(workspace_bytes(pw, M), 16), dtype=torch.uint8,
                       device=device or pw.buf.device)


def fused_workspace_bytes(pw: PackedWeight, M: int = 1, n_out: int = 0) -> int:
    """Workspace with which quantize_linear may run the activation split once
    and the linear layer on its codes (where that is faster)."""
    return int(lib().sq_quantize_linear_workspace_bytes(ctypes.byref(pw.view), M, n_out))


def new_fused_workspace(pw: PackedWeight, M: int = 1, n_out: int = 0, device=None):
    """A zero-filled workspace of fused_workspace_bytes."""
    import torch
    return torch.zeros(max(fused_workspace_bytes(pw, M, n_out), 16), dtype=torch.uint8,
                       device=device or pw.buf.device)


def _flags(pdl: bool, trunk_only: bool = False) -> int:
    return (SQ_LAUNCH_PDL if pdl else 0) | (SQ_TRUNK_ONLY if trunk_only else 0)


def linear(pw: PackedWeight, xq, sx, x_out, idx, y=None, workspace=None, status=None,
           pdl: bool = False, stream=None, trunk_only: bool = False):
    """y[M][N] = fused trunk + residual + outlier product (float32).
    The weight's layout picks the kernel: tiles -> tensor cores, rows -> dp4a.
    trunk_only (tiles): the residual path skipped."""
    import torch
    M = xq.shape[0]
    n = 0 if idx is None else int(idx.numel())
    if y is None:
        y = torch.empty(M, pw.N, dtype=torch.float32, device=xq.device)
    if workspace is None:
        workspace = new_workspace(pw, M)
    _ck(lib().sq_linear(ctypes.byref(pw.view), _ptr(xq), _ptr(sx), _ptr(x_out) if n else None,
                        _ptr(idx) if n else None, n, M, _ptr(y), _ptr(workspace),
                        workspace.numel(), _ptr(status), _flags(pdl, trunk_only),
                        _stream(stream)), "sq_linear")
    return y


def quantize_linear(pw: PackedWeight, x, idx, y=None, workspace=None, status=None,
                    pdl: bool = False, stream=None, trunk_only: bool = False):
    """y[M][N] from fp32 activations x[M][K]: the activation split and the
    linear layer in one kernel (tiled layout), or, for larger M * K with a
    workspace of fused_workspace_bytes, the split once and the linear layer."""
    import torch
    M = x.shape[0]
    n = 0 if idx is None else int(idx.numel())
    if y is None:
        y = torch.empty(M, pw.N, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = new_fused_workspace(pw, M, n)
    _ck(lib().sq_quantize_linear(ctypes.byref(pw.view), _ptr(x), M, _ptr(idx) if n else None, n,
                                 _ptr(y), _ptr(workspace), workspace.numel(), _ptr(status),
                                 _flags(pdl, trunk_only), _stream(stream)), "sq_quantize_linear")
    return y


# the fixed scratch size of sq_linear_noalloc (include/sq.h)
NOALLOC_SCRATCH_BYTES = 16 << 20


def linear_noalloc(pw: PackedWeight, xq, sx, x_out, idx, y, status=None, pdl: bool = False,
                   stream=None, trunk_only: bool = False):
    """sq_linear with the library's fixed device scratch instead of a workspace
    (for callers that cannot allocate device memory at call time).  y [M][N]
    float32 is the caller's.  Calls on one device must not overlap in time."""
    M = xq.shape[0]
    n = 0 if idx is None else int(idx.numel())
    _ck(lib().sq_linear_noalloc(ctypes.byref(pw.view), _ptr(xq), _ptr(sx),
                                _ptr(x_out) if n else None, _ptr(idx) if n else None, n, M,
                                _ptr(y), _ptr(status), _flags(pdl, trunk_only), _stream(stream)),
        "sq_linear_noalloc")
    return y


def testing_prefill_stalled(pw: PackedWeight, xq, sx, x_out, idx, y, skip_group: int,
                            wait_ns: int, status=None, stream=None):
    """include/sq_testing.h: the prefill kernel with its waits limited to
    wait_ns and channel group skip_group's operands never requested (-1:
    none), so that its bounded waits run out (tests of the wind-down path)."""
    M = xq.shape[0]
    n = 0 if idx is None else int(idx.numel())
    _ck(lib().sq_testing_prefill_stalled(ctypes.byref(pw.view), _ptr(xq), _ptr(sx),
                                         _ptr(x_out) if n else None, _ptr(idx) if n else None, n,
                                         M, _ptr(y), skip_group, wait_ns, _ptr(status),
                                         _stream(stream)),
        "sq_testing_prefill_stalled")
    return y


def linear_accumulators(pw: PackedWeight, xq, sx, x_out, idx, workspace=None, status=None,
                        stream=None):
    """(y, T [M][N] int32, R [M][N][ceil(K/G)] int32) from the decode kernel."""
    import torch
    M = xq.shape[0]
    n = 0 if idx is None else int(idx.numel())
    dev = xq.device
    ng = ceil_div(pw.K, pw.group_size)
    y = torch.full((M, pw.N), float("nan"), dtype=torch.float32, device=dev)
    T = torch.empty(M, pw.N, dtype=torch.int32, device=dev)
    R = torch.empty(M, pw.N, ng, dtype=torch.int32, device=dev)
    if workspace is None:
        workspace = new_workspace(pw, M)
    _ck(lib().sq_linear_accumulators(ctypes.byref(pw.view), _ptr(xq), _ptr(sx),
                                     _ptr(x_out) if n else None, _ptr(idx) if n else None, n, M,
                                     _ptr(y), _ptr(T), _ptr(R), _ptr(workspace),
                                     workspace.numel(), _ptr(status), _flags(False),
                                     _stream(stream)), "sq_linear_accumulators")
    return y, T, R


# ---- NVFP4 prefill (format separation; include/sq.h documents the format) ----

@dataclass
class Nvfp4Matrix:
    """An NVFP4 matrix [rows][K] in one device allocation with its C view."""
    rows: int
    K: int
    per_row: bool
    buf: object                 # torch.uint8 device tensor
    view: SqNvfp4Matrix

    def _arr(self, field: str, dtype, count: int):
        import torch
        off = getattr(self.view, field) - self.buf.data_ptr()
        itemsize = torch.empty(0, dtype=dtype).element_size()
        return self.buf[off:off + count * itemsize].view(dtype)

    def codes(self):
        """[rows_pad][code_stride] uint8, two E2M1 codes a byte."""
        import torch
        v = self.view
        return self._arr("codes", torch.uint8, v.rows_pad * v.code_stride).view(v.rows_pad,
                                                                                v.code_stride)

    def scales(self):
        """The UE4M3 scale chunks, flat: [rows_pad/128 * sf_chunks * 512] uint8."""
        import torch
        v = self.view
        return self._arr("scales", torch.uint8, (v.rows_pad // 128) * v.sf_chunks * 512)

    def g(self):
        """Second-level scales: [rows] (per row) or [1] (per tensor)."""
        import torch
        return self._arr("g", torch.float32, self.view.rows_pad if self.per_row else 1)[
            :self.rows if self.per_row else 1]


def alloc_nvfp4(rows: int, K: int, per_row: bool, device=None) -> Nvfp4Matrix:
    import torch
    nbytes = lib().sq_nvfp4_bytes(rows, K, int(per_row))
    if nbytes == 0:
        raise SQError(STATUS_CODE["SQ_ERR_SHAPE"], "sq_nvfp4_bytes")
    buf = torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")
    v = SqNvfp4Matrix()
    _ck(lib().sq_nvfp4_view(_ptr(buf), rows, K, int(per_row), ctypes.byref(v)), "sq_nvfp4_view")
    return Nvfp4Matrix(rows, K, bool(per_row), buf, v)


def nvfp4_quantize(X, per_row: bool, out: Nvfp4Matrix = None, status=None,
                   stream=None) -> Nvfp4Matrix:
    """X[rows][K] (float32, device) -> NVFP4 (per tensor for a weight, per
    row for activations)."""
    rows, K = X.shape
    if out is None:
        out = alloc_nvfp4(rows, K, per_row, device=X.device)
    _ck(lib().sq_nvfp4_quantize(_ptr(X), ctypes.byref(out.view), _ptr(status), _stream(stream)),
        "sq_nvfp4_quantize")
    return out


def nvfp4_linear(w: Nvfp4Matrix, x: Nvfp4Matrix, y=None, status=None, stream=None):
    """y [x.rows][w.rows] float32 = dequantized x @ dequantized w^T on the
    block-scaled tensor cores."""
    import torch
    if y is None:
        y = torch.empty(x.rows, w.rows, dtype=torch.float32, device=x.buf.device)
    _ck(lib().sq_nvfp4_linear(ctypes.byref(w.view), ctypes.byref(x.view), _ptr(y), _ptr(status),
                              _stream(stream)), "sq_nvfp4_linear")
    return y


def testing_nvfp4_stalled(w: Nvfp4Matrix, x: Nvfp4Matrix, y, skip_stage: int, wait_ns: int,
                          status=None, stream=None):
    """include/sq_testing.h: sq_nvfp4_linear with one channel stage never
    requested and every wait limited to wait_ns (tests of the timeout path)."""
    _ck(lib().sq_testing_nvfp4_stalled(ctypes.byref(w.view), ctypes.byref(x.view), _ptr(y), skip_stage,
                                       wait_ns, _ptr(status), _stream(stream)), "sq_testing_nvfp4_stalled")


def testing_read_peak(buf, iters: int = 20, stream=None) -> float:
    """include/sq_testing.h: bytes per second of read-only sweeps of a CUDA
    tensor `buf` (contiguous, 16-byte aligned, size a multiple of 16)."""
    if not buf.is_cuda or not buf.is_contiguous():
        raise SQError(STATUS_CODE["SQ_ERR_INVALID_ARG"], "sq_testing_read_peak: a contiguous CUDA tensor")
    out = ctypes.c_double(0.0)
    nbytes = buf.numel() * buf.element_size()
    _ck(lib().sq_testing_read_peak(buf.data_ptr(), nbytes, iters, ctypes.byref(out), _stream(stream)),
        "sq_testing_read_peak")
    return out.value


def testing_mma_peak(kind: int, iters: int = 4000, status=None, stream=None) -> float:
    """include/sq_testing.h: the measured dense tensor-core rate in ops/s
    (kind 0: int8 MMA, 1: NVFP4 block-scaled MMA)."""
    out = ctypes.c_double(0.0)
    _ck(lib().sq_testing_mma_peak(kind, iters, ctypes.byref(out), _ptr(status), _stream(stream)),
        "sq_testing_mma_peak")
    return out.value
