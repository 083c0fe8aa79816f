"""The timed decode step as a whole against the oracle.

bench.py times one CUDA graph per token: the 128 linears of the 7B-shaped
stack, each one fused launch (activation split + linear) chained with
programmatic dependent launch and sharing one workspace.  This replays that
same graph (bench.Stack) twice and checks sampled rows of every one of the
128 outputs against the oracle, element by element, at the stated tolerance
|y - y_ref| <= 1e-5 * sum_j |W_rj x_j|.
"""
import numpy as np
import pytest
import torch

import oracle
from synth import workloads as wl

pytestmark = pytest.mark.gpu

TOL = 1e-5


def _rows(N, n, seed):
    rng = np.random.default_rng(seed)
    r = set(rng.choice(N, n, replace=False).tolist()) | {0, 15, 16, N - 1}
    return np.array(sorted(r))


@pytest.mark.parametrize("fused", [True, False])
def test_bench_stack_graph_matches_oracle(cuda_device, fused):
    import bench
    import decode_matvec_sq_b200 as sq
    from decode_matvec_sq_b200 import build
    build.build_all()
    sq.device_check()
    layers = wl.config2(32)
    stack = bench.Stack(layers, cuda_device, pdl=True, fused=fused)
    g = stack.capture()
    stack.y_all.fill_(float("nan"))
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert stack.status.item() == 0
    assert not torch.isnan(stack.y_all).any().item(), "an output row was not written"
    y_all = stack.y_all.cpu().numpy()
    worst, off = 0.0, 0
    for i, L in enumerate(layers):
        rows = _rows(L.N, 6, seed=i)
        W, x, idx = L.weights(rows=rows), L.activations(), L.planted_channels()
        d = oracle.decompose(W)
        xq, sx, xo = oracle.quantize_act(x, idx)
        ref = oracle.linear(d, xq, sx, xo, idx)[0]
        bound = oracle.abs_dot(W, x)[0]
        got = y_all[off + rows].astype(np.float64)
        err = np.abs(got - ref) / np.maximum(bound, 1e-300)
        assert np.all(err <= TOL), f"{L.name}: worst {err.max():.3e}"
        worst = max(worst, float(err.max()))
        off += L.N
    del g
