"""Parity of the NVFP4 prefill path (format separation) with the oracle.

The ISTA-DASLab page on separated quantization (paragraphs 2-4): prefill in
the hardware's native NVFP4.  Bit for bit: the E2M1 codes, the UE4M3 block
scales and the second-level scales of sq_nvfp4_quantize, per tensor (a
weight) and per row (activations), pads included.  y of sq_nvfp4_linear
(tcgen05 kind::mxf4nvf4, fp32 accumulation) within 1e-5 * sum_j |W_rj x_tj|
of oracle.nvfp4_linear (binary64).
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


def check_quantized(m, d, X):
    rows, K = X.shape
    u = packed_layout.unpack_nvfp4(m)
    assert np.array_equal(u["codes"][:rows, :K], d["codes"]), "codes"
    nb = d["scales"].shape[1]
    assert np.array_equal(u["scales"][:rows, :nb], d["scales"]), "block scales"
    assert not u["codes"][rows:].any() and not u["codes"][:, K:].any(), "code pads"
    assert not u["scales"][rows:].any() and not u["scales"][:, nb:].any(), "scale pads"
    g = m.g().cpu().numpy()
    assert np.array_equal(g.view(np.uint32), d["g"].view(np.uint32)), "second-level scales"


def _rows_with_ties(rng, R, K):
    """Rows holding, besides noise, values exactly on the E2M1 midpoints of
    their block's step (the RNE ties) and exact block maxima."""
    X = rng.standard_normal((R, K)).astype(np.float32)
    X[:, 0] = 2688.0 * 2.0 ** -8  # g = 2^-8 exactly for every row
    for r in range(R):
        for b in range(1, K // 16):
            s = 2.0 ** int(rng.integers(-3, 4))  # an exact UE4M3 scale
            step = s * 2.0 ** -8
            blk = rng.choice([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 3.0], 16) * step
            blk *= rng.choice([-1.0, 1.0], 16)
            blk[int(rng.integers(0, 16))] = 6.0 * step
            X[r, 16 * b: 16 * b + 16] = blk
    return X


@pytest.mark.parametrize("R,K", [(1, 16), (5, 40), (130, 300), (128, 256), (257, 4096),
                                 (64, 11008), (3, 1000), (3, 20000), (2, 40000)])
@pytest.mark.parametrize("per_row", [False, True])
def test_quantize_parity(R, K, per_row):
    rng = np.random.default_rng(R * 7 + K + per_row)
    X = (rng.standard_normal((R, K)) * np.exp(rng.uniform(-4, 4, (R, 1)))).astype(np.float32)
    X[:, rng.integers(0, K, 3)] *= 25.0
    if R > 2:
        X[1] = 0.0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    m = sq.nvfp4_quantize(torch.from_numpy(X).cuda(), per_row, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    check_quantized(m, oracle.nvfp4_quantize(X, per_row), X)


@pytest.mark.parametrize("per_row", [False, True])
def test_quantize_ties_and_exact_blocks(per_row):
    rng = np.random.default_rng(11)
    X = _rows_with_ties(rng, 9, 512)
    m = sq.nvfp4_quantize(torch.from_numpy(X).cuda(), per_row)
    d = oracle.nvfp4_quantize(X, per_row)
    check_quantized(m, d, X)
    assert d["g"][0] == np.float32(2.0 ** -8)


def test_quantize_stack_weight_and_nonfinite():
    """A 7B-shaped gate_up weight (4096 -> 22016) per tensor, sampled rows;
    then a NaN sets SQ_ERR_NONFINITE."""
    L = wl.config2_layer(0, 2)
    Wd = sdev.fill_weights(L, torch.empty(L.N, L.K, device="cuda"))
    m = sq.nvfp4_quantize(Wd, False)
    rows = np.array([0, 1, 127, 128, 5000, L.N - 1])
    W = Wd.cpu().numpy()
    full = oracle.nvfp4_quantize(W, False)
    u = packed_layout.unpack_nvfp4(m, rows)
    assert np.array_equal(u["codes"][:, :L.K], full["codes"][rows])
    assert np.array_equal(u["scales"][:, :L.K // 16], full["scales"][rows])
    assert m.g().cpu().numpy()[0] == full["g"][0]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    Wd[7, 9] = float("nan")
    sq.nvfp4_quantize(Wd, False, out=m, status=st)
    x = torch.randn(4, L.K, device="cuda")
    x[2, 3] = float("inf")
    sq.nvfp4_quantize(x, True, status=st)
    torch.cuda.synchronize()
    assert st.item() == sq.STATUS_CODE["SQ_ERR_NONFINITE"]


def _linear_case(M, N, K, seed):
    rng = np.random.default_rng(seed)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    x[:, rng.integers(0, K, 4)] *= 30.0
    return W, x


@pytest.mark.parametrize("M,N,K", [(128, 128, 256), (5, 40, 300), (200, 130, 1000),
                                   (256, 384, 4096), (130, 257, 2048), (1, 1, 16)])
def test_linear_parity(M, N, K):
    W, x = _linear_case(M, N, K, seed=M + N + K)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = sq.nvfp4_quantize(torch.from_numpy(W).cuda(), False, status=st)
    a = sq.nvfp4_quantize(torch.from_numpy(x).cuda(), True, status=st)
    y = sq.nvfp4_linear(w, a, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = oracle.nvfp4_linear(oracle.nvfp4_quantize(W, False), oracle.nvfp4_quantize(x, True))
    err = np.abs(y.cpu().numpy().astype(np.float64) - ref)
    bound = oracle.abs_dot(W, x)
    assert np.all(err <= TOL * bound), float((err / bound).max())


def test_linear_exact_products():
    """Operands that NVFP4 represents exactly, with dyadic scales: g = 2^-8
    (each row's maximum 10.5 = 2688 * 2^-8 sits in block 0, where the other
    operand is 0), every other block's maximum 6 * 2^-8 (s_b = 1) and codes
    in {0, +-0.5, +-1}.  Every partial sum is exact in fp32, so y equals the
    oracle and the plain product x W^T exactly."""
    rng = np.random.default_rng(3)
    K = 512
    Wq = rng.choice([-1.0, -0.5, 0.0, 0.5, 1.0], (64, K))
    xq = rng.choice([-1.0, 0.0, 1.0], (128, K))
    Wq[:, 16::16] = 6.0
    xq[:, 16::16] = -6.0
    Wq[:, :16] = 0.0
    xq[:, :16] = 0.0
    W = (Wq * 2.0 ** -8).astype(np.float32)
    W[:, 0] = 10.5
    x = (xq * 2.0 ** -8).astype(np.float32)
    x[:, 1] = 10.5
    w = sq.nvfp4_quantize(torch.from_numpy(W).cuda(), False)
    a = sq.nvfp4_quantize(torch.from_numpy(x).cuda(), True)
    y = sq.nvfp4_linear(w, a).cpu().numpy().astype(np.float64)
    dw, dx = oracle.nvfp4_quantize(W, False), oracle.nvfp4_quantize(x, True)
    assert dw["g"][0] == np.float32(2.0 ** -8) and np.all(dx["g"] == np.float32(2.0 ** -8))
    ref = oracle.nvfp4_linear(dw, dx)
    assert np.array_equal(y, ref)
    assert np.array_equal(ref, x.astype(np.float64) @ W.astype(np.float64).T)


def test_linear_prefill_shape_sampled():
    """The prefill workload's shape (2048 tokens x 4096 -> 14336): every
    token of sampled weight rows against the oracle on those rows."""
    L = wl.config5()
    Wd = sdev.fill_weights(L, torch.empty(L.N, L.K, device="cuda"))
    xd = sdev.fill_activations(L, torch.empty(L.M, L.K, device="cuda"))
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = sq.nvfp4_quantize(Wd, False, status=st)
    a = sq.nvfp4_quantize(xd, True, status=st)
    y = sq.nvfp4_linear(w, a, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    W, x = Wd.cpu().numpy(), xd.cpu().numpy()
    del Wd, xd
    rows = np.array([0, 1, 127, 128, 7001, L.N - 1])
    wq = oracle.nvfp4_quantize(W, False)
    sub = {"codes": wq["codes"][rows], "scales": wq["scales"][rows], "g": wq["g"]}
    ref = oracle.nvfp4_linear(sub, oracle.nvfp4_quantize(x, True))
    got = y[:, torch.as_tensor(rows, device="cuda")].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(got - ref) <= TOL * oracle.abs_dot(W[rows], x))


def test_linear_rejects_mismatched_operands():
    w = sq.alloc_nvfp4(64, 512, False)
    a = sq.alloc_nvfp4(8, 256, True)
    for args in ((w, a), (a, a), (w, w)):
        with pytest.raises(sq.SQError):
            sq.nvfp4_linear(*args)


def test_mma_peak_probe_is_plausible():
    """The tensor-core probe the prefill fractions are reported against:
    int8 and NVFP4 rates on this device, between a tenth of and twice the
    nominal dense figures (4.5 and 9 P ops/s), NVFP4 above int8."""
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    i8 = sq.testing_mma_peak(0, status=st)
    f4 = sq.testing_mma_peak(1, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert 0.45e15 < i8 < 9e15 and 0.9e15 < f4 < 18e15
    assert f4 > i8
