"""The decode kernel's two-group pass: up to 16 tokens share one read of the
weights (two MMA B operands per tile).

Against the oracle: the int32 trunk and group accumulators bit for bit and y
within 1e-5 * sum_j |W_rj x_j|, for 9..16 tokens, the dense, sparse and
asymmetric residuals, with and without the threshold trunk's mask.  Against
the one-group pass: every token's y is summed in the same order whichever
pass it sits in, so a 16-token call equals two 8-token calls bit for bit.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_matvec_sq_b200 as sq
import oracle

pytestmark = pytest.mark.gpu

TOL = 1e-5


@pytest.fixture(scope="module", autouse=True)
def built(cuda_device):
    from decode_matvec_sq_b200 import build
    build.build_all()
    sq.device_check()
    yield


def _pack(W, layout, P):
    Wd = torch.from_numpy(W).cuda()
    if layout == sq.SQ_LAYOUT_TILES_SPARSE:
        return sq.decompose_pack_sparse(Wd, 60, trunk_percent=P)
    return sq.decompose_pack(Wd, trunk_percent=P, layout=layout)


def _oracle_d(W, layout, P):
    if layout == sq.SQ_LAYOUT_TILES_SPARSE:
        return oracle.decompose_sparse(W, P=P, Ps=60)
    if layout == sq.SQ_LAYOUT_TILES_ASYM:
        return oracle.decompose_asym(W, P=P)
    return oracle.decompose(W, P=P)


def _case(N, K, M, n, seed):
    rng = np.random.default_rng(seed)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n, replace=False)).astype(np.int32)
    x[:, idx] *= 30.0
    return W, x, idx


@pytest.mark.parametrize("layout", [sq.SQ_LAYOUT_TILES, sq.SQ_LAYOUT_TILES_SPARSE,
                                    sq.SQ_LAYOUT_TILES_ASYM])
@pytest.mark.parametrize("P", [-1, 60])
@pytest.mark.parametrize("N,K,M", [(40, 300, 9), (513, 1000, 13), (64, 4096, 16), (24, 11008, 16)])
def test_sixteen_token_pass_matches_the_oracle(layout, P, N, K, M):
    W, x, idx = _case(N, K, M, min(9, K), seed=N + K + M + P + 7 * layout)
    pw = _pack(W, layout, P)
    assert sq.lib().sq_linear_tokens_per_pass(ctypes.byref(pw.view), 0) == 16
    idxd = torch.from_numpy(idx).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    xq, sx, xo = sq.quantize_act(torch.from_numpy(x).cuda(), idxd, status=st)
    y, T, R = sq.linear_accumulators(pw, xq, sx, xo, idxd, status=st)
    y2 = sq.linear(pw, xq, sx, xo, idxd, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    d = _oracle_d(W, layout, P)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    oT, oR = oracle.accumulate(d, oxq)
    assert np.array_equal(T.cpu().numpy().astype(np.int64), oT), "trunk accumulators"
    assert np.array_equal(R.cpu().numpy().astype(np.int64), oR), "group accumulators"
    ref = (oracle.linear_asym if layout == sq.SQ_LAYOUT_TILES_ASYM else oracle.linear)(
        d, oxq, osx, oxo, idx)
    bound = oracle.abs_dot(W, x)
    for v in (y, y2):
        err = np.abs(v.cpu().numpy().astype(np.float64) - ref)
        assert np.all(err <= TOL * bound), float((err / bound).max())


@pytest.mark.parametrize("layout", [sq.SQ_LAYOUT_TILES, sq.SQ_LAYOUT_TILES_SPARSE,
                                    sq.SQ_LAYOUT_TILES_ASYM])
@pytest.mark.parametrize("P", [-1, 60])
@pytest.mark.parametrize("trunk", [False, True])
def test_sixteen_tokens_equal_two_passes_of_eight(layout, P, trunk):
    """4096 x 4096 (rows shared between CTAs and warps): one 16-token launch
    against tokens 0..7 and 8..15 launched apart; and 12 tokens against 8 + 4."""
    W, x, idx = _case(4096, 4096, 16, 20, seed=layout * 10 + P)
    pw = _pack(W, layout, P)
    idxd = torch.from_numpy(idx).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    xq, sx, xo = sq.quantize_act(torch.from_numpy(x).cuda(), idxd, status=st)
    y16 = sq.linear(pw, xq, sx, xo, idxd, status=st, trunk_only=trunk)
    y12 = sq.linear(pw, xq[:12], sx[:12], xo[:12], idxd, status=st, trunk_only=trunk)
    parts = [sq.linear(pw, xq[a:b], sx[a:b], xo[a:b], idxd, status=st, trunk_only=trunk)
             for a, b in ((0, 8), (8, 16), (8, 12))]
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(y16, torch.cat(parts[:2]))
    assert torch.equal(y12, torch.cat([parts[0], parts[2]]))


def test_seventeen_tokens_take_two_passes():
    """17 tokens: a 16-token pass and a 1-token pass, each bit-equal to the
    same tokens launched alone; the PDL flag changes nothing."""
    W, x, idx = _case(1000, 2048, 17, 5, seed=17)
    pw = _pack(W, sq.SQ_LAYOUT_TILES, -1)
    idxd = torch.from_numpy(idx).cuda()
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    xq, sx, xo = sq.quantize_act(torch.from_numpy(x).cuda(), idxd, status=st)
    y = sq.linear(pw, xq, sx, xo, idxd, status=st)
    yp = sq.linear(pw, xq, sx, xo, idxd, status=st, pdl=True)
    a = sq.linear(pw, xq[:16], sx[:16], xo[:16], idxd, status=st)
    b = sq.linear(pw, xq[16:], sx[16:], xo[16:], idxd, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(y, torch.cat([a, b])) and torch.equal(y, yp)
