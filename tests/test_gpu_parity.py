"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer and byte outputs (sign and mask bits, alpha, residual codes and
scales, activation codes, outlier indices, the int32 trunk and group
accumulators) must match bit for bit.  The float output y must satisfy
|y - y_ref| <= 1e-5 * sum_j |W_rj * x_j| (original fp32 W and x), per element.
Small shapes compare every element; full-size workloads compare sampled rows
that the oracle recomputes from regenerated inputs.
"""
import ctypes

import numpy as np
import pytest
import torch

import decode_matvec_sq_b200 as sq
import oracle
from tests import packed_layout
import synth
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


def _bits(words: np.ndarray, K: int):
    """uint32 words in row bit order -> (bits of channels < K, pad bits)."""
    bits = np.unpackbits(np.ascontiguousarray(words).view(np.uint8), axis=1, bitorder="little")
    return bits[:, :K], bits[:, K:]


def _layout(tc: bool, G: int = 128) -> int:
    return sq.SQ_LAYOUT_TILES if (tc and G == 128) else sq.SQ_LAYOUT_ROWS


def check_packed(pw: sq.PackedWeight, d: dict, rows=None):
    """GPU packed weight (optionally only `rows`) == oracle decomposition d,
    read back in row order from either layout; pads are zero."""
    K = pw.K
    u = packed_layout.unpack(pw, rows)
    sign, sign_pad = _bits(u["sign"], K)
    assert np.array_equal(sign, d["sign"]), "sign bits"
    assert not sign_pad.any(), "sign pad bits"
    if pw.with_mask:
        mask, mask_pad = _bits(u["mask"], K)
        assert np.array_equal(mask, d["mask"]), "mask bits"
        assert not mask_pad.any()
    else:
        assert d["mask"].all()
    assert np.array_equal(u["alpha"].view(np.uint32), d["alpha"].view(np.uint32)), "alpha"
    assert np.array_equal(u["q"][:, :K], d["q"]), "residual codes"
    assert not u["q"][:, K:].any()
    ng = d["s"].shape[1]
    assert np.array_equal(u["s"][:, :ng].view(np.uint32), d["s"].view(np.uint32)), "group scales"
    assert not u["s"][:, ng:].any()
    if rows is None:
        assert packed_layout.pad_rows_are_zero(pw), "pad rows of the tiled layout"


def check_y(y, y_ref, bound, what="y"):
    err = np.abs(y.astype(np.float64) - y_ref)
    ok = err <= TOL * bound
    assert ok.all(), f"{what}: {int((~ok).sum())} of {ok.size} outside tolerance; worst " \
                     f"{float((err / np.maximum(bound, 1e-300)).max()):.3e}"


def run_path(W: np.ndarray, x: np.ndarray, idx: np.ndarray, P=-1, G=128, pdl=False, tc=True):
    Wd = torch.from_numpy(W).cuda()
    xd = torch.from_numpy(x).cuda()
    idxd = torch.from_numpy(idx.astype(np.int32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(Wd, trunk_percent=P, group_size=G, layout=_layout(tc, G), status=status)
    act = sq.quantize_act(xd, idxd, status=status, pdl=pdl)
    xq, sx, xo = act
    y, T, R = sq.linear_accumulators(pw, xq, sx, xo, idxd, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return pw, act, (y, T, R)


def full_compare(W, x, idx, P=-1, G=128, tc=True):
    pw, act, (y, T, R) = run_path(W, x, idx, P, G, tc=tc)
    xq, sx, xo = act
    d = oracle.decompose(W, G=G, P=P)
    check_packed(pw, d)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    K = W.shape[1]
    assert np.array_equal(xq.cpu().numpy()[:, :K], oxq)
    assert not xq.cpu().numpy()[:, K:].any()
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), osx.view(np.uint32))
    if len(idx):
        assert np.array_equal(xo.cpu().numpy()[:, :len(idx)], oxo)
    oT, oR = oracle.accumulate(d, oxq)
    assert np.array_equal(T.cpu().numpy().astype(np.int64), oT), "trunk accumulators"
    assert np.array_equal(R.cpu().numpy().astype(np.int64), oR), "group accumulators"
    y_ref = oracle.linear(d, oxq, osx, oxo, idx)
    check_y(y.cpu().numpy(), y_ref, oracle.abs_dot(W, x))
    return pw, y


# ---- generators ------------------------------------------------------------------

def test_device_generator_matches_host():
    L1 = wl.config1()
    Wd = sdev.fill_weights(L1, torch.empty(L1.N, L1.K, device="cuda"))
    assert np.array_equal(Wd.cpu().numpy().view(np.uint32), L1.weights().view(np.uint32))
    L3 = wl.config3()[1]
    Wd = sdev.fill_weights(L3, torch.empty(16, L3.K, device="cuda"), row0=100)
    assert np.array_equal(Wd.cpu().numpy().view(np.uint32),
                          L3.weights(rows=np.arange(100, 116)).view(np.uint32))
    L2 = wl.config2_layer(3, 3)
    xd = sdev.fill_activations(L2, torch.empty(4, L2.K, device="cuda"))
    assert np.array_equal(xd.cpu().numpy().view(np.uint32), L2.activations(M=4).view(np.uint32))
    Xd = sdev.fill_activations(L2, torch.empty(wl.CAL_TOKENS, L2.K, device="cuda"), synth.STREAM_XCAL)
    assert np.array_equal(Xd.cpu().numpy().view(np.uint32), L2.calibration().view(np.uint32))


# ---- offline pack ------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(1, 8), (7, 33), (8, 100), (13, 128), (9, 129), (64, 512),
                                 (513, 300), (16, 4096), (3, 1000)])
@pytest.mark.parametrize("G,layout", [(32, 0), (64, 0), (128, 0), (128, 1)])
@pytest.mark.parametrize("P", [-1, 60])
def test_pack_parity_shapes(N, K, G, layout, P):
    rng = np.random.default_rng(N * 1000 + K + G + P)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    W[0, : min(K, 5)] = np.array([0.0, -0.0, 1e-30, -1e-30, 0.5], np.float32)[: min(K, 5)]
    if N > 2:
        W[1] = 0.0                                   # all-zero row: alpha 0, codes 0
        W[2, : K // 2] = np.round(W[2, : K // 2], 2)  # ties for the percentile
    pw = sq.decompose_pack(torch.from_numpy(W).cuda(), trunk_percent=P, group_size=G, layout=layout)
    torch.cuda.synchronize()
    check_packed(pw, oracle.decompose(W, G=G, P=P))


@pytest.mark.parametrize("P", [1, 50, 99, 100])
def test_pack_threshold_percentiles(P):
    rng = np.random.default_rng(P)
    W = rng.laplace(0, 0.02, (37, 777)).astype(np.float32)
    W[5] = np.round(W[5], 3)
    pw = sq.decompose_pack(torch.from_numpy(W).cuda(), trunk_percent=P)
    torch.cuda.synchronize()
    check_packed(pw, oracle.decompose(W, P=P))


def test_pack_nonfinite_status():
    W = np.ones((4, 64), np.float32)
    W[2, 7] = np.inf
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.decompose_pack(torch.from_numpy(W).cuda(), status=st)
    torch.cuda.synchronize()
    assert st.item() == sq.STATUS_CODE["SQ_ERR_NONFINITE"]


# ---- calibration and activation split ----------------------------------------------

@pytest.mark.parametrize("layer", [wl.config1(), wl.config2_layer(0, 0), wl.config2_layer(0, 3),
                                   wl.config3()[1]])
def test_calibrate_parity(layer):
    X = layer.calibration()
    idx = sq.calibrate_outliers(torch.from_numpy(X).cuda(), layer.n_out)
    torch.cuda.synchronize()
    ref = oracle.calibrate(X, layer.n_out)
    assert np.array_equal(idx.cpu().numpy(), ref)
    assert np.array_equal(ref, layer.planted_channels())


def test_calibrate_ties():
    rng = np.random.default_rng(9)
    X = np.round(rng.standard_normal((16, 1000)) * 3).astype(np.float32)
    for k in (1, 7, 100, 1000):
        idx = sq.calibrate_outliers(torch.from_numpy(X).cuda(), k)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), oracle.calibrate(X, k)), k


@pytest.mark.parametrize("M,K,n", [(1, 512, 4), (3, 100, 0), (2, 33, 5), (5, 4096, 20),
                                   (1, 11008, 55), (16, 8192, 20), (1, 1, 0)])
def test_quantize_act_parity(M, K, n):
    rng = np.random.default_rng(M * K + n)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n, replace=False)).astype(np.int32)
    x[:, idx] *= 40.0
    if M > 1:
        x[1] = 0.0                                  # zero token
    if K >= 8:
        # exact midpoints: absmax 127 gives s = 1, values k + 0.5 tie
        x[0, :8] = np.array([127.0, 2.5, -2.5, 0.5, -0.5, 126.5, -126.5, 1.5], np.float32)
        x[0, idx] = np.where(idx < 8, 0.0, x[0, idx])
    xq, sx, xo = sq.quantize_act(torch.from_numpy(x).cuda(),
                                 torch.from_numpy(idx).cuda() if n else None)
    torch.cuda.synchronize()
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    assert np.array_equal(xq.cpu().numpy()[:, :K], oxq)
    assert not xq.cpu().numpy()[:, K:].any()
    assert np.array_equal(sx.cpu().numpy().view(np.uint32), osx.view(np.uint32))
    if n:
        assert np.array_equal(xo.cpu().numpy(), oxo)


def test_quantize_act_large_k():
    """K beyond the range the kernel keeps in registers (re-read path)."""
    rng = np.random.default_rng(12)
    K = 40000
    x = rng.standard_normal((2, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, 50, replace=False)).astype(np.int32)
    act = sq.quantize_act(torch.from_numpy(x).cuda(), torch.from_numpy(idx).cuda())
    torch.cuda.synchronize()
    oxq, osx, _ = oracle.quantize_act(x, idx)
    assert np.array_equal(act[0].cpu().numpy()[:, :K], oxq)


def test_quantize_act_random_midpoints():
    """Values on exact half-steps of many different scales."""
    rng = np.random.default_rng(4)
    M, K = 64, 256
    a = rng.uniform(0.1, 100.0, M).astype(np.float32)
    s = (a.astype(np.float64) / 127.0).astype(np.float32)
    k = rng.integers(0, 127, (M, K))
    x = ((k + 0.5) * s[:, None].astype(np.float64)).astype(np.float32)
    x *= rng.choice([-1, 1], (M, K)).astype(np.float32)
    x[:, 0] = a
    xq, sx, _ = sq.quantize_act(torch.from_numpy(x).cuda(), None)
    torch.cuda.synchronize()
    oxq, osx, _ = oracle.quantize_act(x, np.zeros(0, np.int32))
    assert np.array_equal(sx.cpu().numpy(), osx)
    assert np.array_equal(xq.cpu().numpy()[:, :K], oxq)


# ---- fused linear: small shapes, every element --------------------------------------

@pytest.mark.parametrize("N,K,M,n", [(1, 8, 1, 0), (7, 33, 1, 2), (8, 100, 2, 3), (513, 300, 1, 6),
                                     (64, 512, 3, 4), (16, 4096, 4, 20), (33, 1000, 5, 9),
                                     (40, 129, 8, 1), (20, 300, 8, 3), (24, 11008, 1, 55), (8, 28672, 1, 72),
                                     (100, 2048, 16, 10)])
@pytest.mark.parametrize("P", [-1, 60])
@pytest.mark.parametrize("tc", [False, True])
def test_linear_parity_small(N, K, M, n, P, tc):
    rng = np.random.default_rng(N + K + M + n + P)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n, replace=False)).astype(np.int32)
    x[:, idx] *= 30.0
    full_compare(W, x, idx, P=P, tc=tc)


@pytest.mark.parametrize("G", [32, 64])
def test_linear_parity_group_sizes(G):
    rng = np.random.default_rng(G)
    W = rng.laplace(0, 0.02, (50, 1500)).astype(np.float32)
    x = rng.standard_normal((2, 1500)).astype(np.float32)
    idx = np.array([0, 31, 32, 700, 1499], np.int32)
    full_compare(W, x, idx, G=G)


@pytest.mark.parametrize("tc", [False, True])
def test_linear_degenerate(tc):
    rng = np.random.default_rng(0)
    W = np.zeros((9, 64), np.float32)
    x = rng.standard_normal((1, 64)).astype(np.float32)
    full_compare(W, x, np.array([3], np.int32), tc=tc)          # zero weights: y = 0
    W = rng.laplace(0, 0.02, (9, 64)).astype(np.float32)
    full_compare(W, np.zeros((2, 64), np.float32), np.array([3], np.int32), tc=tc)  # zero tokens
    x = np.zeros((1, 64), np.float32)
    x[0, 3] = 7.0                                         # only the outlier channel is live
    full_compare(W, x, np.array([3], np.int32), tc=tc)
    full_compare(W[:1, :1], np.ones((1, 1), np.float32), np.zeros(0, np.int32), tc=tc)


@pytest.mark.parametrize("tc", [False, True])
def test_linear_deterministic_and_split_rows(tc):
    """N=8, K=28672: one row block split over many warps (partials + fixup)."""
    rng = np.random.default_rng(1)
    W = rng.laplace(0, 0.02, (8, 28672)).astype(np.float32)
    x = rng.standard_normal((1, 28672)).astype(np.float32)
    idx = np.sort(rng.choice(28672, 72, replace=False)).astype(np.int32)
    Wd, xd, idxd = (torch.from_numpy(a).cuda() for a in (W, x, idx))
    pw = sq.decompose_pack(Wd, layout=_layout(tc))
    act = sq.quantize_act(xd, idxd)
    xq, sx, xo = act
    ws = sq.new_workspace(pw, 1)
    ys = []
    for _ in range(5):
        y = torch.full((1, 8), float("nan"), device="cuda")
        ys.append(sq.linear(pw, xq, sx, xo, idxd, y=y, workspace=ws).cpu().numpy())
    torch.cuda.synchronize()
    for y in ys[1:]:
        assert np.array_equal(y.view(np.uint32), ys[0].view(np.uint32))
    assert not sq.workspace_counters(ws, pw).any().item(), "arrival counters left zero-filled"
    d = oracle.decompose(W)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    check_y(ys[0], oracle.linear(d, oxq, osx, oxo, idx), oracle.abs_dot(W, x))


def test_linear_errors():
    W = torch.randn(16, 256, device="cuda")
    pw = sq.decompose_pack(W)
    xq, sx, xo = sq.quantize_act(torch.randn(1, 256, device="cuda"), None)
    small = torch.zeros(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(sq.SQError) as e:
        sq.linear(pw, xq, sx, xo, None, workspace=small)
    assert e.value.name == "SQ_ERR_WORKSPACE"
    y = torch.empty(2, 17, device="cuda")
    with pytest.raises(sq.SQError) as e:
        sq.linear(pw, xq, sx, xo, None, y=y.view(-1)[1:17].view(1, 16))
    assert e.value.name == "SQ_ERR_ALIGN"
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = torch.randn(1, 256, device="cuda")
    x[0, 5] = float("nan")
    sq.quantize_act(x, None, status=st)
    torch.cuda.synchronize()
    assert st.item() == sq.STATUS_CODE["SQ_ERR_NONFINITE"]
    st.zero_()
    bad_idx = torch.tensor([5, 3], dtype=torch.int32, device="cuda")
    sq.quantize_act(torch.randn(1, 256, device="cuda"), bad_idx, status=st)
    torch.cuda.synchronize()
    assert st.item() == sq.STATUS_CODE["SQ_ERR_INVALID_ARG"]


# ---- the five workloads ------------------------------------------------------------

@pytest.mark.parametrize("tc", [False, True])
def test_config1_full_pipeline(tc):
    """512 x 512, batch 1, top-4 calibrated outliers: every output element."""
    L = wl.config1()
    X = torch.from_numpy(L.calibration()).cuda()
    idx = sq.calibrate_outliers(X, L.n_out)
    W, x = L.weights(), L.activations()
    torch.cuda.synchronize()
    assert np.array_equal(idx.cpu().numpy(), L.planted_channels())
    full_compare(W, x, idx.cpu().numpy(), tc=tc)


@pytest.mark.parametrize("tc", [False, True])
def test_config4_threshold_full(tc):
    """4096 -> 14336 threshold trunk (per-row 60th percentile), batch 1, every row."""
    L = wl.config4()
    W, x, idx = L.weights(), L.activations(), L.planted_channels()
    full_compare(W, x, idx, P=L.trunk_percent, tc=tc)


def _sampled_layer(L, M, rows, pdl=False, tc=True):
    """Full-size layer generated on the device; oracle on sampled rows."""
    Wd = sdev.fill_weights(L, torch.empty(L.N, L.K, device="cuda"))
    Xc = sdev.fill_activations(L, torch.empty(wl.CAL_TOKENS, L.K, device="cuda"), synth.STREAM_XCAL)
    xd = sdev.fill_activations(L, torch.empty(M, L.K, device="cuda"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(Wd, trunk_percent=L.trunk_percent, layout=_layout(tc), status=st)
    del Wd
    idx = sq.calibrate_outliers(Xc, L.n_out, status=st)
    xq, sx, xo = sq.quantize_act(xd, idx, status=st, pdl=pdl)
    y, T, R = sq.linear_accumulators(pw, xq, sx, xo, idx, status=st)
    y2 = torch.full_like(y, float("nan"))
    sq.linear(pw, xq, sx, xo, idx, y=y2, status=st, pdl=pdl)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(y, y2)
    idx_h = idx.cpu().numpy()
    assert np.array_equal(idx_h, oracle.calibrate(L.calibration(), L.n_out))
    Wr = L.weights(rows=rows)
    x = L.activations(M=M)
    d = oracle.decompose(Wr, P=L.trunk_percent)
    check_packed(pw, d, rows=rows)
    oxq, osx, oxo = oracle.quantize_act(x, idx_h)
    assert np.array_equal(xq.cpu().numpy()[:, :L.K], oxq)
    oT, oR = oracle.accumulate(d, oxq)
    rt = torch.as_tensor(rows, device="cuda")
    assert np.array_equal(T[:, rt].cpu().numpy().astype(np.int64), oT)
    assert np.array_equal(R[:, rt].cpu().numpy().astype(np.int64), oR)
    check_y(y[:, rt].cpu().numpy(), oracle.linear(d, oxq, osx, oxo, idx_h), oracle.abs_dot(Wr, x))


def _rows(N, n=96, seed=0):
    rng = np.random.default_rng(seed)
    r = set(rng.choice(N, n, replace=False).tolist()) | {0, 1, 7, 8, N // 2, N - 9, N - 8, N - 1}
    return np.array(sorted(r))


@pytest.mark.parametrize("M", [1, 2, 4, 8, 16])
@pytest.mark.parametrize("which", [0, 1])
@pytest.mark.parametrize("tc", [False, True])
def test_config3_batch_sweep_sampled(M, which, tc):
    L = wl.config3(M)[which]
    _sampled_layer(L, M, _rows(L.N, seed=M + which), tc=tc)


@pytest.mark.parametrize("layer", [0, 31])
@pytest.mark.parametrize("mid", [0, 1, 2, 3])
@pytest.mark.parametrize("tc", [False, True])
def test_config2_stack_layers_sampled(layer, mid, tc):
    L = wl.config2_layer(layer, mid)
    _sampled_layer(L, 1, _rows(L.N, seed=layer * 4 + mid), pdl=True, tc=tc)


# ---- launch modes ----------------------------------------------------------------

def test_pdl_chain_in_cuda_graph_matches_plain():
    """quantize -> linear pairs launched with PDL inside a captured graph."""
    layers = [wl.config2_layer(0, m) for m in range(4)] + [wl.config1()]
    pws, xs, idxs, ys_plain = [], [], [], []
    for L in layers:
        Wd = sdev.fill_weights(L, torch.empty(L.N, L.K, device="cuda"))
        pws.append(sq.decompose_pack(Wd))
        xs.append(sdev.fill_activations(L, torch.empty(1, L.K, device="cuda")))
        idxs.append(torch.from_numpy(L.planted_channels()).cuda())
    ws = sq.new_workspace(max(pws, key=lambda p: p.N), 1)
    bufs = [sq.quantize_act(x, i) for x, i in zip(xs, idxs)]
    ys = [torch.empty(1, p.N, device="cuda") for p in pws]
    for p, a, i, y in zip(pws, bufs, idxs, ys):
        y.fill_(float("nan"))
        ys_plain.append(sq.linear(p, a[0], a[1], a[2], i, y=y, workspace=ws).clone())
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for p, x, i, a, y in zip(pws, xs, idxs, bufs, ys):
                sq.quantize_act(x, i, xq=a[0], sx=a[1], x_out=a[2], pdl=True)
                sq.linear(p, a[0], a[1], a[2], i, y=y, workspace=ws, pdl=True)
    for _ in range(3):
        for y in ys:
            y.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        for y, yp in zip(ys, ys_plain):
            assert torch.equal(y, yp)
    for p in pws:
        assert not sq.workspace_counters(ws, p).any().item()


@pytest.mark.parametrize("tc", [False, True])
def test_shared_workspace_across_shapes(tc):
    """One workspace serving layers of different N, called in interleaved
    order: every row is written every time and matches the oracle."""
    layers = [wl.config2_layer(1, m) for m in (0, 2, 1, 3)] + [wl.config1()]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    items = []
    for L in layers:
        Wd = sdev.fill_weights(L, torch.empty(L.N, L.K, device="cuda"))
        pw = sq.decompose_pack(Wd, layout=_layout(tc))
        del Wd
        idx = torch.from_numpy(L.planted_channels()).cuda()
        x = sdev.fill_activations(L, torch.empty(1, L.K, device="cuda"))
        items.append((L, pw, idx, sq.quantize_act(x, idx, status=st)))
    ws = torch.zeros(max(sq.workspace_bytes(pw, 1) for _, pw, _, _ in items), dtype=torch.uint8,
                     device="cuda")
    outs = {}
    for rep in range(3):
        for L, pw, idx, a in items[::(1 if rep % 2 == 0 else -1)]:
            y = torch.full((1, L.N), float("nan"), device="cuda")
            sq.linear(pw, a[0], a[1], a[2], idx, y=y, workspace=ws, status=st)
            torch.cuda.synchronize()
            assert not torch.isnan(y).any().item(), f"{L.name}: rows not written"
            if L.name in outs:
                assert torch.equal(outs[L.name], y), f"{L.name}: not reproducible"
            outs[L.name] = y
    assert st.item() == 0
    for L, pw, idx, _ in items:
        assert not sq.workspace_counters(ws, pw).any().item()
        rows = _rows(L.N, n=48, seed=L.N)
        Wr, x = L.weights(rows=rows), L.activations()
        d = oracle.decompose(Wr)
        oxq, osx, oxo = oracle.quantize_act(x, L.planted_channels())
        y_ref = oracle.linear(d, oxq, osx, oxo, L.planted_channels())
        check_y(outs[L.name][:, torch.as_tensor(rows, device="cuda")].cpu().numpy(), y_ref,
                oracle.abs_dot(Wr, x), L.name)


@pytest.mark.parametrize("tc", [False, True])
@pytest.mark.parametrize("N,K", [(16, 129), (40, 256), (3, 3000), (17, 2048)])
def test_fewer_work_units_than_warps(N, K, tc):
    """Tiny layers: more warps than units of work; rows split between warps
    must still be finished on every call (two calls in a row, NaN-prefilled)."""
    rng = np.random.default_rng(N * K)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((2, K)).astype(np.float32)
    pw = sq.decompose_pack(torch.from_numpy(W).cuda(), layout=_layout(tc))
    act = sq.quantize_act(torch.from_numpy(x).cuda(), None)
    ws = sq.new_workspace(pw, 2)
    d = oracle.decompose(W)
    oxq, osx, oxo = oracle.quantize_act(x, np.zeros(0, np.int32))
    y_ref = oracle.linear(d, oxq, osx, oxo, np.zeros(0, np.int32))
    for _ in range(2):
        y = torch.full((2, N), float("nan"), device="cuda")
        sq.linear(pw, act[0], act[1], act[2], None, y=y, workspace=ws)
        torch.cuda.synchronize()
        check_y(y.cpu().numpy(), y_ref, oracle.abs_dot(W, x))
        assert not sq.workspace_counters(ws, pw, 2).any().item()


# ---- fused activation split + linear --------------------------------------------

def _fused_vs_two_step(W, x, idx, P=-1, pdl=False):
    """sq_quantize_linear == sq_quantize_act + sq_linear bit for bit, and
    within the tolerance of the oracle."""
    Wd, xd = torch.from_numpy(W).cuda(), torch.from_numpy(x).cuda()
    idxd = torch.from_numpy(idx.astype(np.int32)).cuda() if len(idx) else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(Wd, trunk_percent=P, layout=sq.SQ_LAYOUT_TILES, status=st)
    xq, sx, xo = sq.quantize_act(xd, idxd, status=st)
    M, n = x.shape[0], len(idx)
    ws = sq.new_workspace(pw, M)
    y2 = torch.full((M, W.shape[0]), float("nan"), device="cuda")
    sq.linear(pw, xq, sx, xo, idxd, y=y2, workspace=ws, status=st)
    # the fused kernel (a workspace for sq_linear), then with a workspace that
    # also lets the call take the staged route (split once + linear)
    assert sq.fused_workspace_bytes(pw, M, n) > sq.workspace_bytes(pw, M)
    for ws in (ws, sq.new_fused_workspace(pw, M, n)):
        for _ in range(2):  # twice: the arrival counters are left zero
            y1 = torch.full_like(y2, float("nan"))
            sq.quantize_linear(pw, xd, idxd, y=y1, workspace=ws, status=st, pdl=pdl)
            torch.cuda.synchronize()
            assert st.item() == 0
            assert np.array_equal(y1.cpu().numpy().view(np.uint32), y2.cpu().numpy().view(np.uint32))
        assert not sq.workspace_counters(ws, pw, M).any().item()
    d = oracle.decompose(W, P=P)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    check_y(y1.cpu().numpy(), oracle.linear(d, oxq, osx, oxo, idx), oracle.abs_dot(W, x))


@pytest.mark.parametrize("N,K,M,n", [(1, 8, 1, 0), (7, 33, 1, 2), (40, 129, 8, 1), (20, 300, 3, 3),
                                     (513, 300, 1, 6), (64, 4096, 1, 20), (24, 11008, 1, 55),
                                     (8, 28672, 2, 72), (16, 28672, 5, 72), (100, 2048, 16, 10),
                                     (33, 1000, 13, 9)])
@pytest.mark.parametrize("P", [-1, 60])
def test_quantize_linear_parity(N, K, M, n, P):
    rng = np.random.default_rng(7 * N + K + M + n + P)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n, replace=False)).astype(np.int32)
    x[:, idx] *= 30.0
    if M > 1:
        x[1] = 0.0  # a zero token
    _fused_vs_two_step(W, x, idx, P=P)


def test_quantize_linear_config2_layers():
    """Full-size stack shapes, batch 1, with PDL."""
    for mid in range(4):
        L = wl.config2_layer(2, mid)
        rows = _rows(L.N, n=64, seed=mid)
        Wd = sdev.fill_weights(L, torch.empty(L.N, L.K, device="cuda"))
        pw = sq.decompose_pack(Wd)
        del Wd
        x = L.activations()
        idx = L.planted_channels()
        xd, idxd = torch.from_numpy(x).cuda(), torch.from_numpy(idx).cuda()
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        y = sq.quantize_linear(pw, xd, idxd, status=st, pdl=True)
        xq, sx, xo = sq.quantize_act(xd, idxd, status=st)
        y2 = sq.linear(pw, xq, sx, xo, idxd, status=st)
        torch.cuda.synchronize()
        assert st.item() == 0 and torch.equal(y, y2)
        Wr = L.weights(rows=rows)
        d = oracle.decompose(Wr)
        oxq, osx, oxo = oracle.quantize_act(x, idx)
        check_y(y[:, torch.as_tensor(rows, device="cuda")].cpu().numpy(),
                oracle.linear(d, oxq, osx, oxo, idx), oracle.abs_dot(Wr, x), L.name)


def test_quantize_linear_status_and_errors():
    W = torch.randn(32, 256, device="cuda")
    pw = sq.decompose_pack(W)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    x = torch.randn(2, 256, device="cuda")
    x[1, 9] = float("inf")
    sq.quantize_linear(pw, x, None, status=st)
    torch.cuda.synchronize()
    assert st.item() == sq.STATUS_CODE["SQ_ERR_NONFINITE"]
    st.zero_()
    sq.quantize_linear(pw, torch.randn(1, 256, device="cuda"),
                       torch.tensor([7, 7], dtype=torch.int32, device="cuda"), status=st)
    torch.cuda.synchronize()
    assert st.item() == sq.STATUS_CODE["SQ_ERR_INVALID_ARG"]
    pr = sq.decompose_pack(W, layout=sq.SQ_LAYOUT_ROWS)
    with pytest.raises(sq.SQError) as e:
        sq.quantize_linear(pr, torch.randn(1, 256, device="cuda"), None)
    assert e.value.name == "SQ_ERR_SHAPE"


# ---- trunk-only mode (residual path skipped) ------------------------------------

@pytest.mark.parametrize("N,K,M,n,P", [(1, 8, 1, 0, -1), (40, 129, 8, 1, -1), (20, 300, 3, 3, 60),
                                       (513, 300, 1, 6, -1), (64, 4096, 2, 20, 60),
                                       (24, 11008, 1, 55, -1), (16, 28672, 4, 72, -1)])
def test_trunk_only_parity(N, K, M, n, P):
    """sq_linear with SQ_TRUNK_ONLY against the oracle's trunk-only output,
    and sq_quantize_linear (fused kernel and staged route) bit for bit
    against it."""
    rng = np.random.default_rng(3 * N + K + 5 * M + n + P)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n, replace=False)).astype(np.int32)
    x[:, idx] *= 30.0
    Wd, xd = torch.from_numpy(W).cuda(), torch.from_numpy(x).cuda()
    idxd = torch.from_numpy(idx).cuda() if n else None
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(Wd, trunk_percent=P, layout=sq.SQ_LAYOUT_TILES, status=st)
    xq, sx, xo = sq.quantize_act(xd, idxd, status=st)
    y = sq.linear(pw, xq, sx, xo, idxd, status=st, trunk_only=True)
    for ws in (sq.new_workspace(pw, M), sq.new_fused_workspace(pw, M, n)):
        y1 = torch.full_like(y, float("nan"))
        sq.quantize_linear(pw, xd, idxd, y=y1, workspace=ws, status=st, trunk_only=True)
        torch.cuda.synchronize()
        assert np.array_equal(y1.cpu().numpy().view(np.uint32), y.cpu().numpy().view(np.uint32))
    assert st.item() == 0
    d = oracle.decompose(W, P=P)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    ref = oracle.linear_trunk(d, oxq, osx, oxo, idx)
    xh = oxq.astype(np.float64) * osx.astype(np.float64)[:, None]
    xh[:, idx] = x[:, idx]
    trunk_hat = d["mask"] * d["alpha"].astype(np.float64)[:, None]
    bound = np.abs(xh) @ trunk_hat.T
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= 1e-5 * bound + 1e-30), float((err / np.maximum(bound, 1e-30)).max())
    # the full output differs from it by the residual path
    assert not torch.equal(y, sq.linear(pw, xq, sx, xo, idxd, status=st)) or not d["q"].any()


def test_trunk_only_rejected_for_row_layout():
    W = torch.randn(32, 256, device="cuda")
    pr = sq.decompose_pack(W, layout=sq.SQ_LAYOUT_ROWS)
    xq, sx, xo = sq.quantize_act(torch.randn(1, 256, device="cuda"), None)
    with pytest.raises(sq.SQError) as e:
        sq.linear(pr, xq, sx, xo, None, trunk_only=True)
    assert e.value.name == "SQ_ERR_INVALID_ARG"


def test_quantize_linear_staged_route_status():
    """The staged route (M * roundup(K,128) > 16 KiB) reports the same device
    findings as the fused kernel: non-finite x, a bad index list."""
    W = torch.randn(48, 8192, device="cuda")
    pw = sq.decompose_pack(W)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ws = sq.new_fused_workspace(pw, 4, 2)
    x = torch.randn(4, 8192, device="cuda")
    x[3, 100] = float("nan")
    sq.quantize_linear(pw, x, torch.tensor([5, 9], dtype=torch.int32, device="cuda"), workspace=ws,
                       status=st)
    torch.cuda.synchronize()
    assert st.item() == sq.STATUS_CODE["SQ_ERR_NONFINITE"]
    st.zero_()
    sq.quantize_linear(pw, torch.randn(4, 8192, device="cuda"),
                       torch.tensor([9, 5], dtype=torch.int32, device="cuda"), workspace=ws, status=st)
    torch.cuda.synchronize()
    assert st.item() == sq.STATUS_CODE["SQ_ERR_INVALID_ARG"]


def test_fused_workspace_query():
    """The staged-route workspace follows the arithmetic of include/sq.h."""
    L = sq.lib()
    r = lambda a: -(-a // 256) * 256
    w = sq.SqPackedWeight()
    assert L.sq_packed_view(ctypes.c_void_p(1 << 40), 300, 8192, 128, 0, 1, ctypes.byref(w)) == 0
    for M, n in [(1, 0), (4, 20), (16, 72)]:
        got = L.sq_quantize_linear_workspace_bytes(ctypes.byref(w), M, n)
        assert got == r(L.sq_linear_workspace_bytes(ctypes.byref(w), M)) + r(M * 8192) + r(4 * M) + r(4 * M * n)
    assert L.sq_quantize_linear_workspace_bytes(ctypes.byref(w), 0, 0) == 0


# ---- prefill: many tokens on tcgen05 (row layout, M >= 64) --------------------------

@pytest.mark.parametrize("N,K,M,n,P", [(64, 128, 128, 2, -1), (100, 300, 200, 5, -1), (64, 129, 64, 1, 60),
                                       (130, 1024, 257, 9, -1), (64, 4096, 128, 20, 60),
                                       (192, 2048, 384, 70, -1)])
def test_prefill_parity(N, K, M, n, P):
    """Exact T and R_g, y within tolerance, on ragged tokens, rows and channels."""
    rng = np.random.default_rng(N * 7 + K + M + n)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n, replace=False)).astype(np.int32)
    x[:, idx] *= 30.0
    x[3] = 0.0  # a zero token
    Wd, xd, idxd = (torch.from_numpy(a).cuda() for a in (W, x, idx))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(Wd, trunk_percent=P, layout=sq.SQ_LAYOUT_ROWS, status=st)
    xq, sx, xo = sq.quantize_act(xd, idxd, status=st)
    y, T, R = sq.linear_accumulators(pw, xq, sx, xo, idxd, status=st)
    y2 = sq.linear(pw, xq, sx, xo, idxd, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0, sq.STATUS.get(st.item())
    d = oracle.decompose(W, P=P)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    oT, oR = oracle.accumulate(d, oxq)
    assert np.array_equal(T.cpu().numpy().astype(np.int64), oT), "trunk accumulators"
    assert np.array_equal(R.cpu().numpy().astype(np.int64), oR), "group accumulators"
    y_ref = oracle.linear(d, oxq, osx, oxo, idx)
    bound = oracle.abs_dot(W, x)
    check_y(y.cpu().numpy(), y_ref, bound)
    check_y(y2.cpu().numpy(), y_ref, bound)


def test_prefill_config5_sampled():
    """M = 2048 tokens x 4096 -> 14336 (the prefill workload): every token of
    sampled rows against the oracle."""
    L = wl.config5()
    Wd = sdev.fill_weights(L, torch.empty(L.N, L.K, device="cuda"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(Wd, layout=sq.SQ_LAYOUT_ROWS, status=st)
    del Wd
    xd = sdev.fill_activations(L, torch.empty(L.M, L.K, device="cuda"))
    idx = torch.from_numpy(L.planted_channels()).cuda()
    xq, sx, xo = sq.quantize_act(xd, idx, status=st)
    y = sq.linear(pw, xq, sx, xo, idx, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    rows = _rows(L.N, n=40, seed=5)
    Wr = L.weights(rows=rows)
    x = L.activations(M=L.M)
    d = oracle.decompose(Wr)
    oxq, osx, oxo = oracle.quantize_act(x, L.planted_channels())
    assert np.array_equal(xq.cpu().numpy()[:, :L.K], oxq)
    check_y(y[:, torch.as_tensor(rows, device="cuda")].cpu().numpy(),
            oracle.linear(d, oxq, osx, oxo, L.planted_channels()), oracle.abs_dot(Wr, x))
