"""Host-side logic of bench.py that needs no GPU: the algorithmic byte
accounting, the rank helpers on a world-size-2 gloo group, and the CPU
reference arm launched the way the multi-GPU bench is (torchrun, 2 ranks)."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from synth import workloads as wl  # noqa: E402
from tests.conftest import read_golden  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_bytes_per_weight_matches_page_example():
    # m.lqnn.cn/news/241359, section 3.2: 0.125 * 0.7 + 1 * 0.3 = 0.3875 byte
    rows = read_golden("bytes_per_weight_example.txt")
    shares = [(float(v[0]), float(v[1])) for k, v in rows if k == "share"]
    assert len(shares) == 2
    assert bench.bytes_per_weight(shares) == pytest.approx(0.3875, abs=1e-12)


def test_stack_step_bytes():
    """Packed weights of the 7B-shaped stack: 1/8 + 1 + 4/128 + 4/K bytes per
    weight; plus per token xq, sx, x_out, idx, y and the activation split."""
    layers = wl.config2(32)
    shapes = {(4096, 12288, 20), (4096, 4096, 20), (4096, 22016, 20), (11008, 4096, 55)}
    assert {(L.K, L.N, L.n_out) for L in layers} == shapes
    w = sum(L.N * L.K for L in layers)
    assert w == 32 * (4096 * 12288 + 4096 * 4096 + 4096 * 22016 + 11008 * 4096)
    packed = sum(bench.linear_weight_bytes(L) for L in layers)
    closed = sum(L.N * (L.K / 8 + L.K + 4 * L.K / 128 + 4) for L in layers)
    assert packed == pytest.approx(closed, rel=1e-9)  # K multiple of 128: no padding
    total = bench.step_bytes(layers)
    assert 7.49e9 < packed < total < 7.52e9


def _gloo_worker(rank, world, port, out_dir):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        m = bench.max_over_ranks(1.5 * (rank + 1), world, "cpu")
        bench.barrier(world)
        with open(os.path.join(out_dir, f"r{rank}.txt"), "w") as f:
            f.write(repr(m))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo(tmp_path):
    import torch.multiprocessing as mp
    mp.start_processes(_gloo_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2,
                       start_method="spawn", join=True)
    for r in range(2):
        assert float(open(tmp_path / f"r{r}.txt").read()) == 3.0


def test_max_over_ranks_single_rank_is_identity():
    assert bench.max_over_ranks(2.25, 1, "cpu") == 2.25
    bench.barrier(1)


def test_reference_arm_under_torchrun_two_ranks():
    """Rank 0 alone times the oracle and prints one JSON line; rank 1 exits 0
    without work."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node", "2",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()),
           os.path.join(ROOT, "bench.py"), "--impl", "reference", "--gpus", "2",
           "--steps", "1", "--warmup", "3", "--oracle-rows", "4"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    p = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=600, env=env)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [l for l in p.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, p.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["n_gpus"] == 2
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] == 1
    assert d["cpu_baseline"]["host_nproc"] == os.cpu_count() >= 1
    assert isinstance(d["cpu_baseline"]["host_cpu"], str)
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["value"] == d["value"] > 0
    assert d["metric"] == bench.METRIC and d["higher_is_better"] is True


def test_single_layer_workload_cases():
    """The single-layer workloads cover the 512 x 512 layer hot and cold, the
    70B-shaped pair at every batch of its sweep, and the threshold layer; every
    cold case rotates over at least twice the L2 capacity of weights."""
    single = bench.layer_cases("single")
    assert [c[3] for c in single][0] == 1
    L, copies = single[1][1], single[1][3]
    assert copies * L.packed_bytes >= 2 * bench.L2_BYTES
    mlp = bench.layer_cases("mlp70b")
    assert sorted({c[2] for c in mlp}) == [1, 2, 4, 8, 16]
    assert {(c[1].K, c[1].N) for c in mlp} == {(8192, 28672), (28672, 8192)}
    assert all(c[3] * c[1].packed_bytes >= 2 * bench.L2_BYTES for c in mlp)
    (label, L, M, copies), = bench.layer_cases("threshold")
    assert L.trunk_percent == 60 and M == 1 and copies * L.packed_bytes >= 2 * bench.L2_BYTES


def test_trunk_workload_cases():
    """The trunk-only workload covers the stack's four shapes at batch 1, each
    rotating over at least twice the L2 capacity of sign bits and row scales."""
    cases = bench.layer_cases("trunk")
    assert [(c[1].K, c[1].N) for c in cases] == [(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)]
    for label, L, M, copies in cases:
        assert M == 1 and copies * bench.trunk_weight_bytes(L) >= 2 * bench.L2_BYTES
        # sign bits (1/8 byte per weight of the padded tile grid) + 4 bytes per padded row
        assert bench.trunk_weight_bytes(L) == (-(-L.N // 16) * 16) * (-(-L.K // 128) * 16 + 4)


@pytest.mark.parametrize("n", [1, 4, 7, 8, 15, 16, 20, 40, 128, 129])
def test_e2e_bounds_cover_every_linear_once(n):
    """The end-to-end graph's copy groups: for inputs and for outputs,
    strictly increasing starts from 0 to the linear count; from 16 linears up
    the first input group is two linears, the last output group two, and no
    output group is longer than 32 linears."""
    h2d, d2h = bench.e2e_bounds(n)
    for b in (h2d, d2h):
        assert b[0] == 0 and b[-1] == n
        assert all(x < y for x, y in zip(b, b[1:]))
    if n >= 16:
        assert h2d[1] == 2 and d2h[-2] == n - 2
        assert all(y - x <= 32 for x, y in zip(d2h, d2h[1:]))
