"""Parity of the sparse-residual path (SQ_LAYOUT_TILES_SPARSE) with the oracle.

"1-bit量化不是玄学，以往掉点是机制问题" section 3.3: the residual entries near
zero are dropped (50-70 % of them) and the rest stored sparsely.  The oracle's
reading (oracle.decompose_sparse): per row, theta = the nearest-rank Ps-th
percentile of |r|, keep |r| > theta, the kept entries quantized by groups.
Bit for bit: sign / mask bits, alpha, keep bits, codes (read back from the
packed stream), group scales, the packed byte counts, the int32 trunk and
group accumulators.  y within 1e-5 * sum_j |W_rj x_j|.
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


def check_sparse_packed(pw, d, rows=None):
    K = pw.K
    u = packed_layout.unpack(pw, rows)
    sign, sign_pad = _bits(u["sign"], K)
    assert np.array_equal(sign, d["sign"]) and not sign_pad.any(), "sign bits"
    if pw.with_mask:
        mask, mask_pad = _bits(u["mask"], K)
        assert np.array_equal(mask, d["mask"]) and not mask_pad.any(), "mask bits"
    keep, keep_pad = _bits(u["keep"], K)
    assert np.array_equal(keep, d["keep"]), "keep bits"
    assert not keep_pad.any(), "keep pad bits"
    assert np.array_equal(u["alpha"].view(np.uint32), d["alpha"].view(np.uint32)), "alpha"
    assert np.array_equal(u["q"][:, :K], d["q"]), "residual codes"
    assert not u["q"][:, K:].any()
    ng = d["s"].shape[1]
    assert np.array_equal(u["s"][:, :ng].view(np.uint32), d["s"].view(np.uint32)), "group scales"
    assert u["res_bytes_ok"], "packed byte counts"
    if rows is None:
        assert packed_layout.pad_rows_are_zero(pw)


@pytest.mark.parametrize("N,K", [(16, 128), (40, 129), (513, 300), (64, 4096), (24, 11008),
                                 (17, 2048), (8, 28672)])
@pytest.mark.parametrize("Ps", [50, 60, 70])
@pytest.mark.parametrize("P", [-1, 60])
def test_sparse_parity(N, K, Ps, P):
    rng = np.random.default_rng(N * 31 + K + Ps + P)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    M, n = 3, min(9, K)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n, replace=False)).astype(np.int32)
    x[:, idx] *= 30.0
    Wd, xd = torch.from_numpy(W).cuda(), torch.from_numpy(x).cuda()
    idxd = torch.from_numpy(idx).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack_sparse(Wd, Ps, trunk_percent=P, status=st)
    xq, sx, xo = sq.quantize_act(xd, idxd, status=st)
    y, T, R = sq.linear_accumulators(pw, xq, sx, xo, idxd, status=st)
    y2 = sq.linear(pw, xq, sx, xo, idxd, status=st)
    y3 = sq.quantize_linear(pw, xd, idxd, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    d = oracle.decompose_sparse(W, P=P, Ps=Ps)
    check_sparse_packed(pw, d)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    oT, oR = oracle.accumulate(d, oxq)
    assert np.array_equal(T.cpu().numpy().astype(np.int64), oT), "trunk accumulators"
    assert np.array_equal(R.cpu().numpy().astype(np.int64), oR), "group accumulators"
    ref = oracle.linear(d, oxq, osx, oxo, idx)
    bound = oracle.abs_dot(W, x)
    for v in (y, y2, y3):
        err = np.abs(v.cpu().numpy().astype(np.float64) - ref)
        assert np.all(err <= TOL * bound), float((err / bound).max())
    assert torch.equal(y2, y3), "fused split + linear == two kernels"


@pytest.mark.parametrize("mid", [0, 1, 2, 3])
@pytest.mark.parametrize("Ps", [50, 60, 70])
def test_sparse_stack_layers_sampled(mid, Ps):
    """The 7B-shaped stack's linears (layer 5) at batch 1 with PDL: sampled
    rows of the packed weight and of y against the oracle, and the sparsity
    the pages give (about Ps % of the residual entries dropped)."""
    L = wl.config2_layer(5, mid)
    Wd = sdev.fill_weights(L, torch.empty(L.N, L.K, device="cuda"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack_sparse(Wd, Ps, status=st)
    del Wd
    x, idx = L.activations(), L.planted_channels()
    xd, idxd = torch.from_numpy(x).cuda(), torch.from_numpy(idx).cuda()
    y = sq.quantize_linear(pw, xd, idxd, status=st, pdl=True)
    torch.cuda.synchronize()
    assert st.item() == 0
    rng = np.random.default_rng(Ps + mid)
    rows = np.array(sorted(set(rng.choice(L.N, 40, replace=False).tolist()) | {0, L.N - 1}))
    Wr = L.weights(rows=rows)
    d = oracle.decompose_sparse(Wr, Ps=Ps)
    check_sparse_packed(pw, d, rows)
    assert abs(1.0 - d["keep"].mean() - Ps / 100.0) < 0.01
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    ref = oracle.linear(d, oxq, osx, oxo, idx)
    got = y[:, torch.as_tensor(rows, device="cuda")].cpu().numpy().astype(np.float64)
    bound = oracle.abs_dot(Wr, x)
    assert np.all(np.abs(got - ref) <= TOL * bound)
    # the decode kernel reads the kept codes only
    nb = pw.res_bytes()
    assert int(nb.sum().item()) <= (1 - Ps / 100.0 + 0.02) * pw.rows * pw.view.res_stride + 16 * nb.numel()


def test_sparse_trunk_only_and_rejections():
    """The trunk-only mode ignores the residual: equal to the dense weight's
    trunk-only output.  sq_decompose_pack refuses the sparse layout and the
    sparse call refuses percentages outside 1..99."""
    rng = np.random.default_rng(3)
    W = torch.from_numpy(rng.laplace(0, 0.02, (48, 512)).astype(np.float32)).cuda()
    x = torch.randn(2, 512, device="cuda")
    pd = sq.decompose_pack(W)
    ps = sq.decompose_pack_sparse(W, 60)
    xq, sx, xo = sq.quantize_act(x, None)
    assert torch.equal(sq.linear(pd, xq, sx, xo, None, trunk_only=True),
                       sq.linear(ps, xq, sx, xo, None, trunk_only=True))
    with pytest.raises(sq.SQError) as e:
        sq.decompose_pack(W, out=sq.alloc_packed(48, 512, layout=sq.SQ_LAYOUT_TILES_SPARSE))
    assert e.value.name == "SQ_ERR_INVALID_ARG"
    for bad in (0, 100):
        with pytest.raises(sq.SQError) as e:
            sq.decompose_pack_sparse(W, bad)
        assert e.value.name == "SQ_ERR_INVALID_ARG"
