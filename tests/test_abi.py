"""C-ABI checks that need no GPU: the libraries load, every function declared
in include/sq.h is exported, the host-only layout calls agree with the
documented strides, and host-side validation rejects bad arguments before
any device work."""
import ctypes
import os
import re

import pytest

import decode_matvec_sq_b200 as sq

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared(header):
    text = open(header, encoding="utf-8").read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    names = re.findall(r"\b(sq_[a-z_0-9]+)\s*\(", text)
    return sorted(set(names))


@pytest.fixture(scope="module")
def L():
    import torch  # noqa: F401  (loads the CUDA runtime the library links against)
    from decode_matvec_sq_b200 import build
    build.build_libsq()
    return sq.lib()


def test_every_declared_symbol_is_exported(L):
    import glob
    names = []
    for h in sorted(glob.glob(os.path.join(ROOT, "include", "*.h"))):
        names += _declared(h)
    assert "sq_testing_prefill_stalled" in names
    assert {"sq_decompose_pack", "sq_calibrate_outliers", "sq_quantize_act", "sq_linear"} <= set(names)
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/sq.h but not exported"


def test_oracle_exports_its_header():
    import oracle
    oracle.build()
    lib = ctypes.CDLL(os.path.join(ROOT, "oracle", "libsq_oracle.so"))
    for n in re.findall(r"\b(sqo_[a-z_0-9]+)\s*\(", open(os.path.join(ROOT, "oracle", "sq_oracle.h")).read()):
        assert hasattr(lib, n)


def test_status_strings(L):
    for code in range(9):
        assert L.sq_status_string(code)
    assert L.sq_status_string(99) == b"unknown status"


@pytest.mark.parametrize("N,K,G,mask,layout", [
    (1, 1, 128, 0, 0), (7, 33, 32, 1, 0), (512, 512, 128, 0, 0), (12288, 4096, 128, 0, 0),
    (8192, 28672, 64, 1, 0), (1, 1, 128, 0, 1), (7, 33, 128, 1, 1), (12288, 4096, 128, 0, 1),
    (4096, 11008, 128, 1, 1), (8192, 28672, 128, 0, 1), (7, 33, 128, 0, 2), (12288, 4096, 128, 1, 2),
    (4096, 11008, 128, 0, 2), (7, 33, 128, 1, 3), (12288, 4096, 128, 0, 3)])
def test_packed_view_layout(L, N, K, G, mask, layout):
    nbytes = L.sq_packed_bytes(N, K, G, mask, layout)
    assert nbytes > 0
    base = 1 << 40  # a fake 256-aligned address: the view call does not touch memory
    v = sq.SqPackedWeight()
    assert L.sq_packed_view(ctypes.c_void_p(base), N, K, G, mask, layout, ctypes.byref(v)) == 0
    assert v.layout == layout
    if layout == sq.SQ_LAYOUT_ROWS:
        rows = N
        assert v.sign_stride == sq.round_up(sq.ceil_div(K, 32), 4)
        assert v.res_stride == sq.round_up(K, 16)
        assert v.scale_stride == sq.round_up(sq.ceil_div(K, G), 4)
    else:
        rows = sq.round_up(N, 16)
        assert v.res_stride == sq.round_up(K, 128)
        assert v.sign_stride == v.res_stride // 32 and v.scale_stride == v.res_stride // 128
    spans = [(v.sign_bits, rows * v.sign_stride * 4), (v.alpha, sq.round_up(rows, 8) * 4),
             (v.res_q, rows * v.res_stride), (v.res_scale, rows * v.scale_stride * 4)]
    if mask:
        spans.append((v.mask_bits, rows * v.sign_stride * 4))
    else:
        assert v.mask_bits is None
    if layout == sq.SQ_LAYOUT_TILES_SPARSE:
        tiles = rows // 16 * (v.res_stride // 128)
        spans += [(v.keep_bits, rows * v.sign_stride * 4), (v.res_bytes, tiles * 4)]
    else:
        assert v.keep_bits is None and v.res_bytes is None
    if layout == sq.SQ_LAYOUT_TILES_ASYM:
        spans.append((v.res_zero, rows * v.scale_stride * 4))
    else:
        assert v.res_zero is None
    spans.sort()
    for (a, la), (b, _) in zip(spans, spans[1:]):
        assert a % 256 == 0 and a + la <= b
    assert spans[-1][0] + spans[-1][1] <= base + nbytes


def test_packed_view_rejects(L):
    v = sq.SqPackedWeight()
    assert L.sq_packed_view(ctypes.c_void_p((1 << 40) + 16), 8, 8, 128, 0, 0, ctypes.byref(v)) == 3
    assert L.sq_packed_view(ctypes.c_void_p(1 << 40), 8, 8, 48, 0, 0, ctypes.byref(v)) == 2
    assert L.sq_packed_view(ctypes.c_void_p(1 << 40), 0, 8, 128, 0, 0, ctypes.byref(v)) == 2
    assert L.sq_packed_view(None, 8, 8, 128, 0, 0, ctypes.byref(v)) == 1
    assert L.sq_packed_view(ctypes.c_void_p(1 << 40), 8, 8, 128, 0, 4, ctypes.byref(v)) == 1
    # the sparse tiled layout: group size 128 only
    assert L.sq_packed_view(ctypes.c_void_p(1 << 40), 8, 8, 64, 0, 2, ctypes.byref(v)) == 2
    # the tiled layout: group size 128 only, K <= 131072
    assert L.sq_packed_view(ctypes.c_void_p(1 << 40), 8, 8, 64, 0, 1, ctypes.byref(v)) == 2
    assert L.sq_packed_view(ctypes.c_void_p(1 << 40), 8, 131073, 128, 0, 1, ctypes.byref(v)) == 2
    assert L.sq_packed_bytes(8, 8, 100, 0, 0) == 0
    assert L.sq_packed_bytes(8, 8, 64, 0, 1) == 0


def test_host_validation_before_device_work(L):
    """Each of these returns from the host checks; no kernel is launched."""
    v = sq.SqPackedWeight()
    L.sq_packed_view(ctypes.c_void_p(1 << 40), 64, 256, 128, 0, 1, ctypes.byref(v))
    p = ctypes.c_void_p(1 << 41)
    bad = ctypes.c_void_p((1 << 41) + 4)
    # sq_linear(w, xq, sx, x_out, idx, n_out, M, y, ws, ws_bytes, status, flags, stream)
    assert L.sq_linear(None, p, p, p, p, 1, 1, p, p, 1 << 20, None, 0, None) == 1
    assert L.sq_linear(ctypes.byref(v), None, p, p, p, 1, 1, p, p, 1 << 20, None, 0, None) == 1
    assert L.sq_linear(ctypes.byref(v), p, p, p, p, 1, 0, p, p, 1 << 20, None, 0, None) == 2
    assert L.sq_linear(ctypes.byref(v), bad, p, p, p, 1, 1, p, p, 1 << 20, None, 0, None) == 3
    assert L.sq_linear(ctypes.byref(v), p, p, p, p, 1, 1, p, p, 1 << 20, None, 8, None) == 1
    assert L.sq_linear(ctypes.byref(v), p, p, p, p, 1, 1, p, p, 1 << 20, None, 4, None) == 1
    # SQ_TRUNK_ONLY (2) needs the tiled layout
    vr = sq.SqPackedWeight()
    L.sq_packed_view(ctypes.c_void_p(1 << 40), 64, 256, 128, 0, 0, ctypes.byref(vr))
    assert L.sq_linear(ctypes.byref(vr), p, p, p, p, 1, 1, p, p, 1 << 20, None, 2, None) == 1
    assert L.sq_linear(ctypes.byref(vr), p, p, p, p, 1, 1, p, p, 1 << 20, None, 3, None) == 1
    w3 = sq.SqPackedWeight.from_buffer_copy(v)
    w3.layout = 5
    assert L.sq_linear(ctypes.byref(w3), p, p, p, p, 1, 1, p, p, 1 << 20, None, 0, None) == 1
    assert L.sq_linear(ctypes.byref(v), p, p, None, p, 1, 1, p, p, 1 << 20, None, 0, None) == 1
    w2 = sq.SqPackedWeight.from_buffer_copy(v)
    w2.res_stride = 100
    assert L.sq_linear(ctypes.byref(w2), p, p, p, p, 1, 1, p, p, 1 << 20, None, 0, None) == 2
    # accumulators: neither PDL nor the trunk-only mode is accepted
    for flags in (1, 2):
        assert L.sq_linear_accumulators(ctypes.byref(v), p, p, p, p, 1, 1, p, p, p, p, 1 << 20, None,
                                        flags, None) == 1
    # sq_quantize_linear(w, x, M, idx, n_out, y, ws, ws_bytes, status, flags, stream): unknown flag
    assert L.sq_quantize_linear(ctypes.byref(v), p, 1, p, 1, p, p, 1 << 20, None, 4, None) == 1
    assert L.sq_decompose_pack(None, 64, 256, -1, ctypes.byref(v), None, None) == 1
    assert L.sq_decompose_pack(p, 64, 256, 0, ctypes.byref(v), None, None) == 1
    assert L.sq_decompose_pack(p, 64, 256, 60, ctypes.byref(v), None, None) == 1  # no mask array
    assert L.sq_decompose_pack(p, 65, 256, -1, ctypes.byref(v), None, None) == 2
    # sq_quantize_act(x, M, K, idx, n_out, xq, sx, x_out, status, flags, stream)
    assert L.sq_quantize_act(p, 1, 256, p, -1, p, p, p, None, 0, None) == 2
    assert L.sq_quantize_act(p, 1, 256, None, 3, p, p, p, None, 0, None) == 1
    assert L.sq_quantize_act(p, 1, 256, p, 3, bad, p, p, None, 0, None) == 3
    assert L.sq_calibrate_outliers(p, 64, 256, 0, p, None, None) == 2
    assert L.sq_calibrate_outliers(p, 64, 256, 300, p, None, None) == 2


def test_product_path_does_not_import_oracle():
    """The package and its native sources never reach into oracle/."""
    pkg = os.path.join(ROOT, "decode_matvec_sq_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                text = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert "oracle" not in text.replace("no CPU fallback", ""), f


def test_fused_tokens_per_pass(L):
    """Tokens per fused pass follow the shared-memory arithmetic of
    include/sq.h: a ring of two 2560-byte slots (2816 with a mask) per warp,
    16 warps; an outlier table of K/32*8 bytes; per token roundup(K,128) +
    4*roundup(n,4) + 8192 bytes; 227 KiB in all.  Host-only: no device."""
    def view(N, K, mask=False, layout=1):
        v = sq.SqPackedWeight()
        assert L.sq_packed_view(ctypes.c_void_p(1 << 40), N, K, 128, int(mask), layout, ctypes.byref(v)) == 0
        return v
    for K, n, mask, want in [(4096, 20, False, 8), (11008, 55, False, 7), (28672, 72, False, 3),
                             (28672, 72, True, 3), (65536, 0, False, 1), (131072, 0, False, 0)]:
        assert L.sq_quantize_linear_tokens_per_pass(ctypes.byref(view(64, K, mask)), n) == want, (K, n)
    assert L.sq_quantize_linear_tokens_per_pass(ctypes.byref(view(64, 4096, layout=0)), 20) == 0
    assert L.sq_quantize_linear_tokens_per_pass(ctypes.byref(view(64, 4096)), -1) == 0
    assert L.sq_quantize_linear_tokens_per_pass(None, 0) == 0


def test_linear_tokens_per_pass(L):
    """Tokens per weight read of sq_linear follow the shared-memory arithmetic:
    16 when 16 tokens' partial sums (8192 bytes each) + the outlier table
    (roundup(K,128)/4 bytes) + 16 + a ring of two slots per warp (16 warps;
    2560 bytes, 2816 with a mask or for the sparse / asymmetric residual,
    3072 for both; six 256-byte slots, 512 with a mask, in the trunk-only
    mode) fit in 227 KiB - 256; else 8.  The row layout: 4.  Host-only."""
    def view(K, mask=False, layout=1):
        v = sq.SqPackedWeight()
        assert L.sq_packed_view(ctypes.c_void_p(1 << 40), 64, K, 128, int(mask), layout, ctypes.byref(v)) == 0
        return v
    for K, mask, layout, flags, want in [
            (4096, False, 1, 0, 16), (28672, False, 1, 0, 16), (65536, False, 1, 0, 16),
            (81920, False, 1, 0, 8), (43904, True, 1, 0, 16), (44032, True, 1, 0, 8),
            (43904, False, 2, 0, 16), (44032, False, 3, 0, 8), (11008, True, 2, 0, 16),
            (11264, True, 2, 0, 8), (11264, True, 3, 0, 8), (28672, True, 3, 0, 8),
            (81920, True, 1, 2, 16), (4096, False, 0, 0, 4), (4096, False, 0, 2, 0)]:
        assert L.sq_linear_tokens_per_pass(ctypes.byref(view(K, mask, layout)), flags) == want, \
            (K, mask, layout, flags)
    assert L.sq_linear_tokens_per_pass(ctypes.byref(view(4096)), 1) == 0  # PDL is not a pass flag
    assert L.sq_linear_tokens_per_pass(None, 0) == 0


def test_decompose_pack_auto_host_checks(L):
    """sq_decompose_pack_auto refuses, before any device work: a weight view
    without a mask array (the fallback's empty trunk needs one), the sparse
    layout, and a scratch below sq_residual_errors_scratch_bytes(N) + 256."""
    p = ctypes.c_void_p(1 << 40)
    def view(mask, layout=1):
        v = sq.SqPackedWeight()
        assert L.sq_packed_view(ctypes.c_void_p(1 << 41), 64, 512, 128, int(mask), layout, ctypes.byref(v)) == 0
        return v
    need = L.sq_residual_errors_scratch_bytes(64) + 256
    fell = ctypes.c_int32(7)
    assert L.sq_decompose_pack_auto(p, 64, 512, -1, ctypes.byref(view(False)), p, need, ctypes.byref(fell),
                                    None, None, None) == 1
    assert L.sq_decompose_pack_auto(p, 64, 512, -1, ctypes.byref(view(True, 2)), p, need, None, None, None,
                                    None) == 1
    assert L.sq_decompose_pack_auto(p, 64, 512, -1, ctypes.byref(view(True)), p, need - 1, None, None, None,
                                    None) == 8
    assert fell.value == 7  # untouched on a refusal


def test_nvfp4_view_arithmetic(L):
    """sq_nvfp4_bytes / sq_nvfp4_view: codes [roundup(rows,128)][roundup(K,256)/2],
    scale chunks [rows_pad/128][roundup(K,256)/64][512], g [rows_pad] floats per
    row or 2 per tensor, each piece 256-byte aligned; bad arguments refused.
    Host-only: no device memory is touched."""
    def r256(v):
        return -(-v // 256) * 256
    for rows, K, per_row in [(1, 16, 0), (130, 300, 1), (2048, 4096, 1), (14336, 4096, 0)]:
        rp, k256 = -(-rows // 128) * 128, r256(K)
        codes = r256(rp * k256 // 2)
        scales = r256(rp // 128 * (k256 // 64) * 512)
        gb = r256(rp * 4 if per_row else 8)
        assert L.sq_nvfp4_bytes(rows, K, per_row) == codes + scales + gb
        v = sq.SqNvfp4Matrix()
        base = 1 << 40
        assert L.sq_nvfp4_view(ctypes.c_void_p(base), rows, K, per_row, ctypes.byref(v)) == 0
        assert (v.rows, v.K, v.per_row, v.rows_pad) == (rows, K, per_row, rp)
        assert (v.code_stride, v.sf_chunks) == (k256 // 2, k256 // 64)
        assert (v.codes, v.scales, v.g) == (base, base + codes, base + codes + scales)
    v = sq.SqNvfp4Matrix()
    assert L.sq_nvfp4_bytes(0, 16, 0) == 0 and L.sq_nvfp4_bytes(4, 16, 2) == 0
    assert L.sq_nvfp4_view(ctypes.c_void_p((1 << 40) + 16), 4, 16, 0, ctypes.byref(v)) == 3
    assert L.sq_nvfp4_view(None, 4, 16, 0, ctypes.byref(v)) == 1
    assert L.sq_nvfp4_view(ctypes.c_void_p(1 << 40), 4, 0, 0, ctypes.byref(v)) == 2
    # quantize / linear refuse bad views before any device work
    assert L.sq_nvfp4_quantize(None, None, None, None) == 1
    w, x = sq.SqNvfp4Matrix(), sq.SqNvfp4Matrix()
    assert L.sq_nvfp4_view(ctypes.c_void_p(1 << 40), 64, 512, 0, ctypes.byref(w)) == 0
    assert L.sq_nvfp4_view(ctypes.c_void_p(1 << 41), 8, 512, 1, ctypes.byref(x)) == 0
    p = ctypes.c_void_p(1 << 42)
    assert L.sq_nvfp4_linear(ctypes.byref(x), ctypes.byref(x), p, None, None) == 1  # weight per row
    assert L.sq_nvfp4_linear(ctypes.byref(w), ctypes.byref(x), None, None, None) == 1
    x.code_stride += 128
    assert L.sq_nvfp4_linear(ctypes.byref(w), ctypes.byref(x), p, None, None) == 2


def test_missing_library_fails_loudly():
    """Without the built CUDA library every entry point raises: there is no
    CPU fallback.  Run in a child process so this process keeps its loaded
    library."""
    import subprocess
    import sys
    code = ("import decode_matvec_sq_b200 as sq\n"
            "sq.LIB_PATH = '/nonexistent/libsq.so'\n"
            "sq._lib = None\n"
            "try:\n"
            "    sq.packed_bytes(64, 256)\n"
            "except ImportError as e:\n"
            "    print('raised', 'missing' in str(e))\n")
    r = subprocess.run([sys.executable, "-c", code], cwd=os.path.dirname(os.path.dirname(__file__)),
                       capture_output=True, text=True, timeout=120)
    assert r.returncode == 0 and r.stdout.strip() == "raised True", r.stdout + r.stderr


def test_device_entry_points_refuse_without_a_device(L):
    """On a machine with no usable sm_100 device the device check fails with
    a status, not a silent fallback (this CPU machine has none)."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is visible")
    assert L.sq_device_check() != 0


C_PROGRAM = r"""
#include <stdio.h>
#include "sq.h"
int main(void) {
  sq_packed_weight v;
  size_t b = sq_packed_bytes(64, 256, 128, 0, SQ_LAYOUT_TILES);
  int rc = sq_packed_view((void *)(1ull << 40), 64, 256, 128, 0, SQ_LAYOUT_TILES, &v);
  int bad = sq_linear(NULL, NULL, NULL, NULL, NULL, 0, 1, NULL, NULL, 0, NULL, 0u, NULL);
  printf("%zu %d %d %d %s\n", b, rc, v.layout, bad, sq_status_string(SQ_ERR_INVALID_ARG));
  return 0;
}
"""


def test_header_is_plain_c_and_links(tmp_path):
    """include/sq.h compiles as pedantic C11 with warnings as errors, and a C
    host program links against libsq.so and makes host-only calls."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    src = tmp_path / "t.c"
    src.write_text(C_PROGRAM)
    exe = tmp_path / "t"
    libdir = os.path.dirname(sq.LIB_PATH)
    subprocess.run(["gcc", "-std=c11", "-Wall", "-Wextra", "-pedantic", "-Werror",
                    "-I" + os.path.join(root, "include"), str(src), "-L" + libdir, "-lsq",
                    "-Wl,-rpath," + libdir, "-o", str(exe)], check=True, capture_output=True)
    out = subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.split()
    assert int(out[0]) == L_bytes() and out[1] == "0" and out[2] == "1" and out[3] == "1"


def L_bytes() -> int:
    return sq.packed_bytes(64, 256, 128, False, sq.SQ_LAYOUT_TILES)


def test_probe_host_checks(L):
    """The peak probes refuse, before any device work: a null output or
    buffer, a buffer not 16-byte aligned, a size that is not a positive
    multiple of 16, an iteration count out of range, an unknown MMA kind."""
    buf = ctypes.c_void_p(1 << 41)
    out = ctypes.c_double(-1.0)
    rp = L.sq_testing_read_peak
    assert rp(None, 1 << 20, 10, ctypes.byref(out), None) == 1
    assert rp(buf, 1 << 20, 10, None, None) == 1
    assert rp(ctypes.c_void_p((1 << 41) + 8), 1 << 20, 10, ctypes.byref(out), None) == 3
    for nbytes in (0, 8, 40):
        assert rp(buf, nbytes, 10, ctypes.byref(out), None) == 2
    for iters in (0, 1001):
        assert rp(buf, 1 << 20, iters, ctypes.byref(out), None) == 2
    mp = L.sq_testing_mma_peak
    assert mp(2, 100, ctypes.byref(out), None, None) == 1
    assert mp(0, 100, None, None, None) == 1
    for iters in (0, 100001):
        assert mp(1, iters, ctypes.byref(out), None, None) == 2
    assert out.value == -1.0  # untouched on a refusal
