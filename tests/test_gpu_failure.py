"""Failure detection on the GPU without a fault: a bounded wait that runs out.

The prefill kernels (int8 and NVFP4) bound every wait on their pipeline barriers.  Through the
test-only entry point of include/sq_testing.h the operands of one channel
group are never requested and every wait is limited to 1 ms: the kernel must
report SQ_ERR_TIMEOUT in the status word and wind down (drain its copies and
MMAs, free its tensor memory), leaving the context usable -- the next call on
the same stream must run and match the oracle.  Small cases only.
"""
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


def _case(N, K, M, n, seed):
    rng = np.random.default_rng(seed)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    idx = np.sort(rng.choice(K, n, replace=False)).astype(np.int32)
    x[:, idx] *= 30.0
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    pw = sq.decompose_pack(torch.from_numpy(W).cuda(), layout=sq.SQ_LAYOUT_ROWS, status=st)
    idxd = torch.from_numpy(idx).cuda()
    xq, sx, xo = sq.quantize_act(torch.from_numpy(x).cuda(), idxd, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return W, x, idx, pw, idxd, xq, sx, xo


def test_unstalled_entry_matches_sq_linear():
    """skip_group = -1: every operand requested; the result is sq_linear's."""
    W, x, idx, pw, idxd, xq, sx, xo = _case(64, 512, 128, 4, seed=1)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y_ref = sq.linear(pw, xq, sx, xo, idxd, status=st)
    y = torch.full_like(y_ref, float("nan"))
    sq.testing_prefill_stalled(pw, xq, sx, xo, idxd, y, -1, 1_000_000_000, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(y, y_ref)


@pytest.mark.parametrize("N,K,M,skip", [(64, 512, 128, 1), (64, 512, 128, 0), (130, 1024, 256, 5)])
def test_stalled_group_times_out_and_the_context_survives(N, K, M, skip):
    W, x, idx, pw, idxd, xq, sx, xo = _case(N, K, M, 3, seed=N + K + skip)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.zeros(M, N, device="cuda")
    sq.testing_prefill_stalled(pw, xq, sx, xo, idxd, y, skip, 1_000_000, status=st)
    torch.cuda.synchronize()  # returns: the kernel wound down
    assert st.item() == sq.STATUS_CODE["SQ_ERR_TIMEOUT"]
    # the same stream, the next call: runs and is right
    st.zero_()
    y2 = sq.linear(pw, xq, sx, xo, idxd, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    d = oracle.decompose(W)
    oxq, osx, oxo = oracle.quantize_act(x, idx)
    ref = oracle.linear(d, oxq, osx, oxo, idx)
    err = np.abs(y2.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= TOL * oracle.abs_dot(W, x))


def test_stalled_entry_rejects_bad_arguments():
    W, x, idx, pw, idxd, xq, sx, xo = _case(64, 512, 128, 2, seed=9)
    y = torch.zeros(128, 64, device="cuda")
    for skip, wait in [(4, 1000), (-2, 1000), (0, 0), (0, 2_000_000_000)]:
        with pytest.raises(sq.SQError) as e:
            sq.testing_prefill_stalled(pw, xq, sx, xo, idxd, y, skip, wait)
        assert e.value.name == "SQ_ERR_INVALID_ARG"
    with pytest.raises(sq.SQError) as e:  # too few tokens for the prefill kernel
        sq.testing_prefill_stalled(pw, xq[:8], sx[:8], xo[:8], idxd, y, -1, 1000)
    assert e.value.name == "SQ_ERR_SHAPE"


def _nvfp4_case(N, K, M, seed):
    rng = np.random.default_rng(seed)
    W = rng.laplace(0, 0.02, (N, K)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    w = sq.nvfp4_quantize(torch.from_numpy(W).cuda(), False, status=st)
    a = sq.nvfp4_quantize(torch.from_numpy(x).cuda(), True, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    return W, x, w, a


def test_nvfp4_unstalled_entry_matches_linear():
    W, x, w, a = _nvfp4_case(256, 1024, 256, seed=2)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y_ref = sq.nvfp4_linear(w, a, status=st)
    y = torch.full_like(y_ref, float("nan"))
    sq.testing_nvfp4_stalled(w, a, y, -1, 1_000_000_000, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(y, y_ref)


@pytest.mark.parametrize("N,K,M,skip", [(256, 1024, 256, 1), (256, 1024, 256, 0), (130, 2048, 300, 7)])
def test_nvfp4_stalled_stage_times_out_and_the_context_survives(N, K, M, skip):
    """The persistent block-scaled GEMM: one 256-channel stage never
    requested, 1 ms waits -> SQ_ERR_TIMEOUT, the CTAs drain their copies and
    MMAs and free tensor memory; the next call on the stream is right."""
    W, x, w, a = _nvfp4_case(N, K, M, seed=N + K + skip)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = torch.zeros(M, N, device="cuda")
    sq.testing_nvfp4_stalled(w, a, y, skip, 1_000_000, status=st)
    torch.cuda.synchronize()
    assert st.item() == sq.STATUS_CODE["SQ_ERR_TIMEOUT"]
    st.zero_()
    y2 = sq.nvfp4_linear(w, a, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = oracle.nvfp4_linear(oracle.nvfp4_quantize(W, False), oracle.nvfp4_quantize(x, True))
    err = np.abs(y2.cpu().numpy().astype(np.float64) - ref)
    assert np.all(err <= TOL * oracle.abs_dot(W, x))


def test_nvfp4_stalled_entry_rejects_bad_arguments():
    W, x, w, a = _nvfp4_case(64, 512, 8, seed=4)
    y = torch.zeros(8, 64, device="cuda")
    for skip, wait in [(2, 1000), (-2, 1000), (0, 0), (0, 2_000_000_000)]:
        with pytest.raises(sq.SQError) as e:
            sq.testing_nvfp4_stalled(w, a, y, skip, wait)
        assert e.value.name == "SQ_ERR_INVALID_ARG"
