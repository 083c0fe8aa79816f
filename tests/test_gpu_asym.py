"""Parity of the asymmetric residual (SQ_LAYOUT_TILES_ASYM) and of the
per-layer fallback measure with the oracle.

"1-bit量化不是玄学，以往掉点是机制问题" section 2 (pitfalls): the residual gets its
own min/max, scale and zero-point; section 2.3 (last paragraph): a layer that
gains nothing from the split falls back to plain 8-bit.  Bit for bit: sign /
mask bits, alpha, codes in [-128, 127], group scales and zero-points, the
int32 trunk and group accumulators, the two binary64 reconstruction errors.
y within 1e-5 * sum_j |W_rj x_j| of oracle.linear_asym.
"""
import numpy as np
import pytest
import torch

import decode_matvec_sq_b200 as sq
import oracle
from tests import packed_layout
import synth.device as sdev
from synth import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def built(cuda_device):
    from decode_matvec_sq_b200 import build
    build.build_all()
    sq.device_check()
    yield


def _bits(words, K):
    b = np.unpackbits(np.ascontiguousarray(words).view(np.uint8), axis=1, bitorder="little")
    return b[:, :K], b[:, K:]


def check_asym_packed(pw, d, rows=None):
    K = pw.K
    u = packed_layout.unpack(pw, rows)
    sign, pad = _bits(u["sign"], K)
    assert np.array_equal(sign, d["sign"]) and not pad.any(), "sign bits"
    if pw.with_mask:
        mask, pad = _bits(u["mask"], K)
        assert np.array_equal(mask, d["mask"]) and not pad.any(), "mask bits"
    assert np.array_equal(u["alpha"].view(np.uint32), d["alpha"].view(np.uint32)), "alpha"
    assert np.array_equal(u["q"][:, :K], d["q"]), "residual codes"
    ng = d["s"].shape[1]
    assert np.array_equal(u["s"][:, :ng].view(np.uint32), d["s"].view(np.uint32)), "group scales"
    assert np.array_equal(u["z"][:, :ng], d["z"]), "zero-points"
    if rows is None:
        assert packed_layout.pad_rows_are_zero(pw)


@pytest.mark.parametrize("N,K", [(16, 128), (40, 129), (513, 300), (64, 4096), (24, 11008),
                                 (8, 28672)])
@pytest.mark.parametrize("P", [-1, 60])
def test_asym_parity(N, K, P):
    rng = np.random.default_rng(N * 17 + K + P)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    W[0, : min(K, 200)] = np.abs(W[0, : min(K, 200)]) + 0.01  # one-sided groups: z far from 0
    M, n = 3, min(9, K)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n, replace=False)).astype(np.int32)
    x[:, idx] *= 30.0
    Wd, xd = torch.from_numpy(W).cuda(), torch.from_numpy(x).cuda()
    idxd = torch.from_numpy(idx).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(Wd, trunk_percent=P, layout=sq.SQ_LAYOUT_TILES_ASYM, status=st)
    xq, sx, xo = sq.quantize_act(xd, idxd, status=st)
    y, T, R = sq.linear_accumulators(pw, xq, sx, xo, idxd, status=st)
    y2 = sq.linear(pw, xq, sx, xo, idxd, status=st)
    y3 = sq.quantize_linear(pw, xd, idxd, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    d = oracle.decompose_asym(W, P=P)
    check_asym_packed(pw, d)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    oT, oR = oracle.accumulate(d, oxq)
    assert np.array_equal(T.cpu().numpy().astype(np.int64), oT), "trunk accumulators"
    assert np.array_equal(R.cpu().numpy().astype(np.int64), oR), "group accumulators"
    ref = oracle.linear_asym(d, oxq, osx, oxo, idx)
    bound = oracle.abs_dot(W, x)
    for v in (y, y2, y3):
        err = np.abs(v.cpu().numpy().astype(np.float64) - ref)
        assert np.all(err <= TOL * bound), float((err / bound).max())
    assert torch.equal(y2, y3), "fused split + linear == two kernels"


@pytest.mark.parametrize("mid", [0, 3])
def test_asym_stack_layers_sampled(mid):
    """The 7B-shaped stack's linears at batch 1 with PDL, sampled rows."""
    L = wl.config2_layer(7, mid)
    Wd = sdev.fill_weights(L, torch.empty(L.N, L.K, device="cuda"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(Wd, layout=sq.SQ_LAYOUT_TILES_ASYM, status=st)
    del Wd
    x, idx = L.activations(), L.planted_channels()
    y = sq.quantize_linear(pw, torch.from_numpy(x).cuda(), torch.from_numpy(idx).cuda(),
                           status=st, pdl=True)
    torch.cuda.synchronize()
    assert st.item() == 0
    rows = np.array(sorted(set(np.random.default_rng(mid).choice(L.N, 40, replace=False).tolist())
                           | {0, L.N - 1}))
    Wr = L.weights(rows=rows)
    d = oracle.decompose_asym(Wr)
    check_asym_packed(pw, d, rows)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    ref = oracle.linear_asym(d, oxq, osx, oxo, idx)
    got = y[:, torch.as_tensor(rows, device="cuda")].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= TOL * oracle.abs_dot(Wr, x))


@pytest.mark.parametrize("layout,G", [(sq.SQ_LAYOUT_ROWS, 32), (sq.SQ_LAYOUT_ROWS, 128),
                                      (sq.SQ_LAYOUT_TILES, 128), (sq.SQ_LAYOUT_TILES_ASYM, 128)])
@pytest.mark.parametrize("P", [-1, 60])
def test_residual_errors_bit_exact(layout, G, P):
    rng = np.random.default_rng(G + P + layout)
    W = rng.laplace(0, 0.02, (37, 300)).astype(np.float32)
    Wd = torch.from_numpy(W).cuda()
    pw = sq.decompose_pack(Wd, trunk_percent=P, group_size=G, layout=layout)
    e_split, e_plain = sq.residual_errors(Wd, pw)
    d = oracle.decompose_asym(W, G=G, P=P) if layout == sq.SQ_LAYOUT_TILES_ASYM else \
        oracle.decompose(W, G=G, P=P)
    assert e_split == oracle.layer_sq_error(d, W)
    assert e_plain == oracle.plain_sq_error(W, G)


def test_fallback_decisions_match_the_oracle():
    """The three pinned situations: binary rows on an exact grid (tie: fall
    back), the stack's Laplace weights (keep the split), weights on their
    own INT8 grid (fall back)."""
    rng = np.random.default_rng(5)
    signs = rng.choice([-1.0, 1.0], size=(3, 256))
    c = (127.0 * np.array([2.0 ** -8, 2.0 ** -10, 2.0 ** -6]))[:, None]
    W_tie = (c * signs).astype(np.float32)
    W_stack = wl.config2_layer(0, 0).weights(rows=np.arange(16))
    k = rng.integers(-127, 128, size=(4, 256))
    k[:, 0], k[:, 128] = 127, -127
    W_grid = (np.repeat(rng.uniform(1e-3, 1e-2, size=(4, 2)), 128, axis=1) * k).astype(np.float32)
    for W, want in ((W_tie, True), (W_stack, False), (W_grid, True)):
        assert oracle.choose_fallback(W) == want
        pw, fell = sq.decompose_pack_auto(torch.from_numpy(W).cuda())
        assert fell == want
        d = oracle.decompose(W, P=100 if want else -1)
        u = packed_layout.unpack(pw)
        assert np.array_equal(u["q"][:, :W.shape[1]], d["q"])
        assert np.array_equal(u["alpha"].view(np.uint32), d["alpha"].view(np.uint32))
