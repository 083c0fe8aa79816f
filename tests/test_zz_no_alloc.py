"""sq_linear_noalloc: the decode linear layer with the library's fixed device
scratch instead of a caller workspace.  Two calls in a row must agree with
sq_linear on the same inputs within the y tolerance (1e-5 * sum_j |W_rj x_j|);
the second call also shows that the first left the arrival counters zero.
Self-contained: passes alone in a fresh process and after the other tests."""
import ctypes

import numpy as np
import pytest

import decode_matvec_sq_b200 as sq

torch = pytest.importorskip("torch")

TOL = 1e-5


def _inputs(N, K, M, n_out, seed):
    rng = np.random.default_rng(seed)
    W = rng.laplace(0.0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n_out, replace=False)).astype(np.int32)
    x[:, idx] *= 30.0
    return W, x, idx


def _bound(W, x):
    return np.abs(x.astype(np.float64)) @ np.abs(W.astype(np.float64)).T  # [M][N]


@pytest.mark.gpu
@pytest.mark.parametrize("N,K,M,n_out,P,layout", [
    (512, 512, 1, 4, -1, 1),           # the single-layer workload's shape
    (4096, 4096, 1, 20, -1, 1),        # rows shared between warps and CTAs
    (1000, 1000, 3, 9, 60, 1),         # threshold trunk, ragged K, 3 tokens
    (777, 2048, 5, 10, -1, 0),         # row layout: CUDA-core kernel, two passes
])
def test_noalloc_matches_sq_linear_twice(cuda_device, N, K, M, n_out, P, layout):
    W, x, idx = _inputs(N, K, M, n_out, seed=N + K + M)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(torch.from_numpy(W).cuda(), trunk_percent=P, layout=layout, status=st)
    idxd = torch.from_numpy(idx).cuda()
    xq, sx, xo = sq.quantize_act(torch.from_numpy(x).cuda(), idxd, status=st)
    y_ref = sq.linear(pw, xq, sx, xo, idxd, status=st)
    ys = []
    for _ in range(2):
        y = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        sq.linear_noalloc(pw, xq, sx, xo, idxd, y, status=st)
        ys.append(y)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = y_ref.cpu().numpy().astype(np.float64)
    bound = _bound(W, x)
    for y in ys:
        err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
        assert np.isfinite(err).all()
        assert (err <= TOL * bound).all(), float((err / bound).max())
        # the same kernel on the same inputs: the scratch must not change the sums
        assert torch.equal(y, y_ref)


@pytest.mark.gpu
def test_noalloc_reuse_across_sizes_is_exact(cuda_device):
    """The row layout (CUDA-core kernel, rows split between CTAs finished
    through per-row counters in the scratch): a large layer, a small one, then
    the large one again through the one shared array, each bit-equal to
    sq_linear with a workspace of its own.  A counter left non-zero by one
    call would change the next call's finishing order or sums."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    cases = {}
    for name, (N, K, M, n_out) in {"large": (6000, 4096, 2, 20), "small": (40, 512, 1, 3)}.items():
        W, x, idx = _inputs(N, K, M, n_out, seed=N + 7)
        pw = sq.decompose_pack(torch.from_numpy(W).cuda(), layout=0, status=st)
        idxd = torch.from_numpy(idx).cuda()
        act = sq.quantize_act(torch.from_numpy(x).cuda(), idxd, status=st)
        cases[name] = (pw, idxd, act, sq.linear(pw, *act, idxd, status=st), (M, N))
    for name in ("large", "small", "large", "small"):
        pw, idxd, act, y_ref, shape = cases[name]
        y = torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        sq.linear_noalloc(pw, *act, idxd, y, status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert torch.equal(y, y_ref), name


@pytest.mark.gpu
def test_noalloc_rejects_a_stream_of_another_device(cuda_device):
    """Only checkable with two devices; on one it checks the same-device path
    with an explicit (non-default) stream."""
    W, x, idx = _inputs(64, 256, 1, 2, seed=3)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(torch.from_numpy(W).cuda(), layout=1, status=st)
    idxd = torch.from_numpy(idx).cuda()
    act = sq.quantize_act(torch.from_numpy(x).cuda(), idxd, status=st)
    y_ref = sq.linear(pw, *act, idxd, status=st)
    s = torch.cuda.Stream()
    y = torch.full((1, 64), float("nan"), dtype=torch.float32, device="cuda")
    with torch.cuda.stream(s):
        sq.linear_noalloc(pw, *act, idxd, y, status=st)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    if torch.cuda.device_count() > 1:
        with torch.cuda.device(1):
            other = torch.cuda.Stream()
        with pytest.raises(sq.SQError) as e:
            sq.linear_noalloc(pw, *act, idxd, y, status=st, stream=other)
        assert e.value.name == "SQ_ERR_INVALID_ARG"


@pytest.mark.gpu
def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    """More rows than the fixed scratch has counters for: SQ_ERR_WORKSPACE from
    the host checks, before any device work (the view's pointers are never
    dereferenced)."""
    L = sq.lib()
    N, K = 8_000_000, 128
    v = sq.SqPackedWeight()
    assert L.sq_packed_view(ctypes.c_void_p(1 << 40), N, K, 128, 0, 1, ctypes.byref(v)) == 0
    need = L.sq_linear_workspace_bytes(ctypes.byref(v), 1)
    assert need > sq.NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(1 << 41)
    rc = L.sq_linear_noalloc(ctypes.byref(v), p, p, None, None, 0, 1, p, None, 0, None)
    assert rc == 8 and L.sq_status_string(rc)  # SQ_ERR_WORKSPACE


@pytest.mark.gpu
def test_noalloc_trunk_only_matches_sq_linear(cuda_device):
    """The trunk-only flag passes through the no-allocation entry point."""
    W, x, idx = _inputs(1000, 1000, 3, 9, seed=5)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(torch.from_numpy(W).cuda(), layout=1, status=st)
    idxd = torch.from_numpy(idx).cuda()
    xq, sx, xo = sq.quantize_act(torch.from_numpy(x).cuda(), idxd, status=st)
    y_ref = sq.linear(pw, xq, sx, xo, idxd, status=st, trunk_only=True)
    y = torch.full((3, 1000), float("nan"), dtype=torch.float32, device="cuda")
    sq.linear_noalloc(pw, xq, sx, xo, idxd, y, status=st, trunk_only=True)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(y, y_ref)
