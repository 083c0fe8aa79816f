#!/usr/bin/env python3
"""Benchmark: batch-1 decode of the Llama-2-7B-shaped separated-quantization stack.

One step = one token through 32 layers x {qkv 4096->12288, o 4096->4096,
gate_up 4096->22016, down 11008->4096}: for each of the 128 linears the
activation split and the linear layer in one kernel (sq_quantize_linear;
--two-kernels: sq_quantize_act then sq_linear), all in one CUDA graph with
programmatic dependent launch.  Weights are packed once
(offline) and resident in HBM; the 7.5 GB they take per step exceed the
126 MB L2 many times over, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sq|reference]

Prints ONE JSON line (rank 0).  With N > 1 (torchrun) every rank runs its own
replica of the stack (weak scaling, no collective on the data path); the step
time is the max over ranks.  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload (host cores, no GPU).
"""
from __future__ import annotations

import argparse
import json
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode sq_linear HBM GB/s (% of 8 TB/s) and µs/token for 7B-shaped stack, batch 1"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ---- algorithmic traffic ----------------------------------------------------------

def bytes_per_weight(shares) -> float:
    """Sum of share * bytes over the parts of a weight (the pages' accounting:
    0.125 * 0.7 + 1 * 0.3 = 0.3875 for a 30 % 8-bit residual)."""
    return sum(s * b for s, b in shares)


def linear_weight_bytes(L) -> int:
    """Packed-weight bytes the fused linear must read: sign (and mask) bits,
    INT8 codes, fp32 group scales and the fp32 row scale."""
    return L.packed_bytes


def linear_act_bytes(L, M=1) -> int:
    """Per call of the linear beyond the weights: xq, sx, x_out, idx in; y out."""
    return M * (L.K + 4 + 4 * L.n_out + 4 * L.N) + 4 * L.n_out


def quantize_bytes(L, M=1) -> int:
    """Per call of the activation split: x and idx in; xq, sx, x_out out."""
    return M * (4 * L.K + L.K + 4 + 4 * L.n_out) + 4 * L.n_out


def fused_launch_bytes(L, M=1) -> int:
    """One launch of the fused kernel: packed weights, x and idx in, y out."""
    return L.packed_bytes + M * (4 * L.K + 4 * L.N) + 4 * L.n_out


def step_bytes(layers, M=1) -> int:
    return sum(linear_weight_bytes(L) + linear_act_bytes(L, M) + quantize_bytes(L, M) for L in layers)


# ---- helpers ----------------------------------------------------------------------

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS = 1590.0
INT8_PER_BF16 = 2.0  # nominal dense int8 : bf16 tensor throughput (4.5 : 2.25 P/s)


FP4_PER_BF16 = 4.0  # nominal dense fp4 : bf16 tensor throughput (9 : 2.25 P/s)


def load_fp4_peak():
    """Dense NVFP4 tensor peak in TFLOP/s: the measured cuBLAS bf16 burst
    figure times the nominal fp4/bf16 ratio."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]) * FP4_PER_BF16, "measured bf16 x nominal fp4/bf16 ratio"
    except Exception:
        return FALLBACK_BF16_TFLOPS * FP4_PER_BF16, "fallback bf16 x nominal fp4/bf16 ratio"


def host_info():
    """The host the oracle baseline ran on: logical CPUs and the CPU model."""
    model = platform.processor() or ""
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_nproc": os.cpu_count(), "host_cpu": model}


def read_probe(device, nbytes: int = 2 << 30, iters: int = 10):
    """The device's pure-read HBM rate in GB/s (sq_testing_read_peak over a
    buffer 16x the L2), the decode kernels' second denominator."""
    import torch
    import decode_matvec_sq_b200 as sq
    buf = torch.zeros(nbytes, dtype=torch.uint8, device=device)
    gbs = sq.testing_read_peak(buf, iters=iters) / 1e9
    del buf
    torch.cuda.empty_cache()
    return round(gbs, 1)


def probe_peak(kind: int) -> float:
    """The dense tensor-core rate measured on this device by the library's
    probe (sq_testing_mma_peak): kind 0 int8, 1 NVFP4; T ops/s."""
    import decode_matvec_sq_b200 as sq
    return sq.testing_mma_peak(kind) / 1e12


def load_int8_peak():
    """Dense int8 tensor peak in T int-ops/s: the measured cuBLAS bf16 burst
    figure times the nominal int8/bf16 ratio."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["bf16_tflops"]) * INT8_PER_BF16, "measured bf16 x nominal int8/bf16 ratio"
    except Exception:
        return FALLBACK_BF16_TFLOPS * INT8_PER_BF16, "fallback bf16 x nominal int8/bf16 ratio"


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(prefix="sq_clocks_", suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.dev), "--query-gpu=" + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        except OSError:
            pass
        finally:
            try:
                os.unlink(self.path)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = [num(r[2]) for r in rows if num(r[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def barrier(world: int) -> None:
    """Every rank reaches this point before any goes on (no-op on one rank)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int, device) -> float:
    """The largest of the ranks' values (the step time of the slowest rank)."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---- CPU oracle baseline -----------------------------------------------------------

def oracle_sample(rows: int = 256, layers_idx=(0,)):
    """A bounded sample of the stack for the CPU oracle: the first `rows` rows of
    each linear of the given layers (inputs generated on the host)."""
    import numpy as np
    from synth import workloads as wl
    import oracle
    sample = []
    for l in layers_idx:
        for mid in range(4):
            L = wl.config2_layer(l, mid)
            n = min(rows, L.N)
            W = L.weights(rows=np.arange(n))
            d = oracle.decompose(W)
            sample.append((L, n, d, L.activations(), L.planted_channels(), W))
    return sample


def time_oracle(sample, min_seconds: float | None = None, passes: int | None = None):
    """Times oracle.quantize_act + oracle.linear over the sample (one thread):
    exactly `passes` passes, or as many as fill `min_seconds`."""
    import oracle
    done, t0 = 0, time.perf_counter()
    while True:
        for L, n, d, x, idx, _ in sample:
            xq, sx, xo = oracle.quantize_act(x, idx)
            oracle.linear(d, xq, sx, xo, idx)
        done += 1
        el = time.perf_counter() - t0
        if passes is not None and done >= passes:
            break
        if passes is None and el >= (min_seconds or 0.0):
            break
    per_pass = el / done
    nbytes = 0
    for L, n, d, x, idx, _ in sample:
        Ls = L.with_(N=n)
        nbytes += linear_weight_bytes(Ls) + linear_act_bytes(Ls) + quantize_bytes(Ls)
    return nbytes / per_pass / 1e9, per_pass, done, nbytes


def oracle_parity(sample, ys):
    """The oracle's y for the sampled rows against the GPU's y of the same
    linears (ys[i] [1][N], device): max |y - y_ref| / sum_j |W_rj x_j| and
    whether it is within the 1e-5 tolerance."""
    import numpy as np
    import oracle
    worst, rows = 0.0, 0
    for (L, n, d, x, idx, W), y in zip(sample, ys):
        xq, sx, xo = oracle.quantize_act(x, idx)
        ref = oracle.linear(d, xq, sx, xo, idx)
        bound = oracle.abs_dot(W, x)
        got = y[:, :n].cpu().numpy().astype(np.float64)
        worst = max(worst, float((np.abs(got - ref) / np.maximum(bound, 1e-300)).max()))
        rows += n
    return {"rows": rows, "max_err_over_bound": worst, "tolerance": 1e-5, "ok": worst <= 1e-5}


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    sample = oracle_sample(rows=args.oracle_rows)
    time_oracle(sample, passes=args.warmup)
    gbs, per_pass, passes, nbytes = time_oracle(sample, passes=args.steps)
    desc = (f"first {args.oracle_rows} rows of each of the 4 linears of layer 0 "
            f"({nbytes / 1e6:.1f} MB of algorithmic traffic per pass); quantize_act + linear, "
            f"batch 1")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(per_pass * 1e3, 3), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "int8+f64", "data": "synthetic",
        "config": config_dict(args),
        "cpu_baseline": {"value": round(gbs, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
                         "sample": desc, **host_info()},
        "e2e": {"value": round(gbs, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_dict(args):
    return {"workload": "llama-2-7b-shaped decode linear stack, batch 1: "
                        f"{args.layers} layers x {{qkv 4096->12288, o 4096->4096, "
                        "gate_up 4096->22016, down 11008->4096}, W Laplace(0,0.02), "
                        "x N(0,1) with 0.5% channels x30",
            "layers": args.layers, "tokens": 1, "group_size": 128,
            "l2": "inputs larger than L2 (packed weights of the stack, ~7.5 GB per step)",
            "parallelism": "replicas" if args.gpus > 1 else "single"}


# ---- GPU arm -----------------------------------------------------------------------

class Stack:
    def __init__(self, layers, device, pdl=True, fused=True):
        import torch
        import decode_matvec_sq_b200 as sq
        import synth
        import synth.device as sdev
        self.layers = layers
        self.pdl = pdl
        self.fused = fused
        maxw = max(L.N * L.K for L in layers)
        scratch = torch.empty(maxw, dtype=torch.float32, device=device)
        cal = torch.empty(64 * max(L.K for L in layers), dtype=torch.float32, device=device)
        st = torch.zeros(1, dtype=torch.int32, device=device)
        self.status = st
        self.pws, self.idx = [], []
        xs_total = sum(L.K for L in layers)
        ys_total = sum(L.N for L in layers)
        # one contiguous x and y buffer each (e2e copies them in one transfer)
        self.x_all = torch.empty(xs_total, dtype=torch.float32, device=device)
        self.y_all = torch.empty(ys_total, dtype=torch.float32, device=device)
        self.xs, self.ys, self.bufs = [], [], []
        xo_, yo_ = 0, 0
        for L in layers:
            W = scratch[: L.N * L.K].view(L.N, L.K)
            sdev.fill_weights(L, W)
            self.pws.append(sq.decompose_pack(W, status=st))
            X = cal[: 64 * L.K].view(64, L.K)
            sdev.fill_activations(L, X, synth.STREAM_XCAL)
            self.idx.append(sq.calibrate_outliers(X, L.n_out, status=st))
            x = self.x_all[xo_: xo_ + L.K].view(1, L.K)
            sdev.fill_activations(L, x)
            self.xs.append(x)
            self.ys.append(self.y_all[yo_: yo_ + L.N].view(1, L.N))
            # keep every sub-buffer 16-byte aligned
            assert (L.K * 4) % 16 == 0 and (L.N * 4) % 16 == 0
            xo_ += L.K
            yo_ += L.N
            self.bufs.append(sq.quantize_act(x, self.idx[-1], status=st))
        torch.cuda.synchronize()
        del scratch, cal
        if st.item() != 0:
            raise RuntimeError(f"setup status {sq.STATUS.get(st.item())}")
        self.ws = sq.new_workspace(max(self.pws, key=lambda p: p.N * 1000 + p.K), 1)
        need = max(sq.workspace_bytes(p, 1) for p in self.pws)
        if self.ws.numel() < need:
            self.ws = torch.zeros(need, dtype=torch.uint8, device=device)

    @property
    def launches_per_step(self) -> int:
        return len(self.layers) * (1 if self.fused else 2)

    def step(self, pdl=None, lo=0, hi=None):
        """One token through the stack (linears lo .. hi-1): per linear, the
        activation split and the fused linear layer (one kernel, or two with
        fused=False)."""
        import decode_matvec_sq_b200 as sq
        pdl = self.pdl if pdl is None else pdl
        hi = len(self.pws) if hi is None else hi
        for pw, x, idx, a, y in list(zip(self.pws, self.xs, self.idx, self.bufs, self.ys))[lo:hi]:
            if self.fused:
                sq.quantize_linear(pw, x, idx, y=y, workspace=self.ws, status=self.status, pdl=pdl)
            else:
                sq.quantize_act(x, idx, xq=a[0], sx=a[1], x_out=a[2], status=self.status, pdl=pdl)
                sq.linear(pw, a[0], a[1], a[2], idx, y=y, workspace=self.ws, status=self.status,
                          pdl=pdl)

    def capture(self):
        import torch
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            self.step()  # warm every launch path once outside capture
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            self.step()
        torch.cuda.synchronize()
        return g


def e2e_bounds(n: int):
    """Where the end-to-end graph's copies join the compute stream.  Each join
    costs the step time (measured on B200, 7B-shaped stack, with 16-byte copies
    in the same graph shape: a wait of the compute stream for an input copy
    about 4 us, a record that releases an output copy about 2 us), so there
    are few of them:
      inputs: linears [0, 2) first (the bytes that must land before any
        compute), then [2, 12), then the rest, all on the copy stream from the
        step's start; the compute stream waits before linears 0, 2 and 12;
      outputs: back after every 32 linears and after the last two.
    Returns (input group starts, output group starts), each from 0 to n."""
    if n < 16:
        return list(range(n + 1)), list(range(n + 1))
    h2d = [0, 2, 12, n]
    d2h = [0] + list(range(32, n - 2, 32)) + [n - 2, n]
    return h2d, d2h


def capture_e2e(stack, x_host, y_host, bounds=None):
    """One end-to-end step as a CUDA graph: the stack's inputs copied in from
    pinned host memory and its outputs copied back on a copy stream, the inputs
    by groups of linears issued at the step's start and each awaited before its
    first linear, the outputs by groups sent back once their linears are done,
    while the later linears compute.  Every byte of x and y crosses each step;
    results are those of the plain step.  `bounds`: (input group starts,
    output group starts), by default e2e_bounds."""
    import torch
    n = len(stack.pws)
    h2d, d2h = e2e_bounds(n) if bounds is None else bounds
    for b in (h2d, d2h):
        assert b[0] == 0 and b[-1] == n and all(x < y for x, y in zip(b, b[1:]))
    xoff, yoff = [0], [0]
    for L in stack.layers:
        xoff.append(xoff[-1] + L.K)
        yoff.append(yoff[-1] + L.N)
    s, sc = torch.cuda.Stream(), torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        fork = torch.cuda.Event()
        fork.record(s)
        sc.wait_event(fork)
        x_in = {}
        for c in range(len(h2d) - 1):
            a, b = xoff[h2d[c]], xoff[h2d[c + 1]]
            with torch.cuda.stream(sc):
                stack.x_all[a:b].copy_(x_host[a:b], non_blocking=True)
                e = torch.cuda.Event()
                e.record(sc)
            x_in[h2d[c]] = e
        ends = set(d2h[1:])
        start = 0
        for i in range(n):
            if i in x_in:
                s.wait_event(x_in[i])
            stack.step(lo=i, hi=i + 1)
            if i + 1 in ends:
                done = torch.cuda.Event()
                done.record(s)
                sc.wait_event(done)
                a, b = yoff[start], yoff[i + 1]
                with torch.cuda.stream(sc):
                    y_host[a:b].copy_(stack.y_all[a:b], non_blocking=True)
                start = i + 1
        s.wait_stream(sc)
    torch.cuda.synchronize()
    return g, s


def run_prefill(args, world, rank, local):
    """Prefill-sized linear layer: M = 2048 tokens x 4096 -> 14336 (row layout,
    tcgen05 kernel).  One step = the activation split of the 2048 tokens and
    the linear layer.  Tensor-bound: reported in T int-ops/s, where the work
    is the trunk and residual products, 4*M*N*K int-ops."""
    import torch
    import torch.distributed as dist
    import decode_matvec_sq_b200 as sq
    from decode_matvec_sq_b200 import build
    import synth.device as sdev
    from synth import workloads as wl

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device visible (the sq path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    if rank == 0 or world == 1:
        build.build_all()
    barrier(world)
    sq.device_check()
    L = wl.config5()
    W = sdev.fill_weights(L, torch.empty(L.N, L.K, device=device))
    st = torch.zeros(1, dtype=torch.int32, device=device)
    pw = sq.decompose_pack(W, layout=sq.SQ_LAYOUT_ROWS, status=st)
    del W
    x = sdev.fill_activations(L, torch.empty(L.M, L.K, device=device))
    idx = torch.from_numpy(L.planted_channels()).to(device)
    xq, sx, xo = sq.quantize_act(x, idx, status=st)
    y = torch.empty(L.M, L.N, device=device)
    ws = sq.new_workspace(pw, L.M)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # > L2, written between steps

    def step():
        sq.quantize_act(x, idx, xq=xq, sx=sx, x_out=xo, status=st)
        sq.linear(pw, xq, sx, xo, idx, y=y, workspace=ws, status=st)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    ops = 4 * L.M * L.N * L.K
    with ClockSampler(local) as clk:
        barrier(world)
        ev = []
        for _ in range(args.steps):
            flush.fill_(1)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            c = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            sq.quantize_act(x, idx, xq=xq, sx=sx, x_out=xo, status=st)
            b.record(stream)
            sq.linear(pw, xq, sx, xo, idx, y=y, workspace=ws, status=st)
            c.record(stream)
            ev.append((a, b, c))
        torch.cuda.synchronize()
        barrier(world)
    clocks = clk.summary()
    ms_step = max_over_ranks(sum(a.elapsed_time(c) for a, b, c in ev) / len(ev), world, device)
    ms_lin = max_over_ranks(sum(b.elapsed_time(c) for a, b, c in ev) / len(ev), world, device)
    if st.item() != 0:
        raise RuntimeError(f"device status {sq.STATUS.get(st.item())}")
    peak, kind = load_int8_peak()
    probe = probe_peak(0)
    value = world * ops / (ms_step * 1e-3) / 1e12
    achieved = ops / (ms_lin * 1e-3) / 1e12
    if rank == 0:
        print(json.dumps({
            "metric": "prefill sq_linear int8 tensor T int-ops/s, 2048 tokens x 4096 -> 14336",
            "value": round(value, 1), "unit": "T int-ops/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": "prefill 2048 tokens x 4096 -> 14336, W Laplace(0,0.02), "
                                   "x N(0,1) with 0.5% channels x30",
                       "l2": "a 256 MB buffer written between steps"},
            "gpu_launches": 2 * args.steps,
            "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1),
                         "unit": "T int-ops/s", "frac": round(achieved / peak, 4), "peak_kind": kind,
                         "traffic": None, "kernel": "k_prefill (tcgen05 kind::i8)",
                         "us_per_launch": round(ms_lin * 1e3, 2),
                         "probe_peak": round(probe, 1),
                         "frac_of_probe": round(achieved / probe, 4),
                         "probe_kind": "measured on this device: back-to-back kind::i8 MMAs "
                                       "128x256x32 on every SM (sq_testing_mma_peak)"},
            "clocks": clocks,
        }), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


L2_BYTES = 126 << 20


def _time_calls(launch, replays: int) -> float:
    """Device ms per replay of a CUDA graph of launch(), on a side stream."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        launch()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        launch()
    with torch.cuda.stream(s):
        for _ in range(3):
            g.replay()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(s)
        for _ in range(replays):
            g.replay()
        b.record(s)
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / replays
    del g
    return ms


def layer_cases(workload: str):
    """(label, layer, M, weight copies) of a single-layer workload.  Cold cases
    rotate over enough copies of the packed weight that every call reads it
    from HBM; the hot case of the 512 x 512 layer reads one L2-resident copy."""
    from synth import workloads as wl
    if workload == "single":
        L = wl.config1()
        cold = -(-2 * L2_BYTES // L.packed_bytes)
        return [("512x512 hot (L2-resident)", L, 1, 1), ("512x512 cold", L, 1, cold)]
    if workload == "mlp70b":
        out = []
        for M in (1, 2, 4, 8, 16):
            for L in wl.config3(M):
                out.append((f"{L.K}->{L.N} M={M}", L, M, 2))
        return out
    if workload == "threshold":
        L = wl.config4()
        return [("4096->14336 threshold trunk P=60", L, 1, -(-2 * L2_BYTES // L.packed_bytes))]
    if workload == "asym":
        out = []
        for mid in range(4):
            L = wl.config2_layer(0, mid)
            out.append((f"{L.name.split('.')[-1]} {L.K}->{L.N} asymmetric residual",
                        L.with_(residual_percent=-1), 1, -(-2 * L2_BYTES // L.packed_bytes)))
        return out
    if workload == "sparse":
        out = []
        for Ps in (50, 60, 70):
            for mid in range(4):
                L = wl.config2_layer(0, mid)
                out.append((f"{L.name.split('.')[-1]} {L.K}->{L.N} sparse residual Ps={Ps}",
                            L.with_(residual_percent=Ps), 1,
                            -(-2 * L2_BYTES // int(L.packed_bytes * (1.2 - Ps / 100.0)))))
        return out
    if workload == "trunk":
        out = []
        for mid in range(4):
            L = wl.config2_layer(0, mid)
            out.append((f"{L.name.split('.')[-1]} {L.K}->{L.N} trunk only", L, 1,
                        -(-2 * L2_BYTES // trunk_weight_bytes(L))))
        return out
    raise ValueError(workload)


def trunk_weight_bytes(L) -> int:
    """Bytes the trunk-only mode reads of a tiled packed weight: the sign (and
    mask) bits and the row scales of the padded rows."""
    rows = -(-L.N // 16) * 16
    words = -(-L.K // 128) * 4
    planes = 2 if L.trunk_percent >= 0 else 1
    return rows * (4 * words * planes + 4)


def sparse_weight_bytes(pw) -> int:
    """Bytes the decode kernel reads of a sparse-residual weight: sign (and
    mask) and keep bits, each tile's packed kept codes (padded to 16), the
    group scales, the row scales and the per-tile byte counts."""
    rows, words, groups = pw.rows, pw.view.sign_stride, pw.view.scale_stride
    planes = 3 if pw.with_mask else 2
    nb = pw.res_bytes()
    return rows * (4 * words * planes + 4 * groups + 4) + int(nb.sum().item()) + 4 * nb.numel()


def _fused_launches(pw, M: int, L, flags: int = 0) -> int:
    """Launches of one sq_quantize_linear call with a fused_workspace_bytes
    workspace: the staged route (split + linear passes of sq_linear's pass
    size) when M > 1 and M * roundup(K, 128) > 16 KiB or when fused passes
    outnumber those passes, else one fused launch per pass."""
    import ctypes
    import decode_matvec_sq_b200 as sq
    kx = -(-L.K // 128) * 128
    per_pass = int(sq.lib().sq_quantize_linear_tokens_per_pass(ctypes.byref(pw.view), L.n_out))
    lin = int(sq.lib().sq_linear_tokens_per_pass(ctypes.byref(pw.view), flags))
    staged = M > 1 and (M * kx > (16 << 10) or -(-M // per_pass) > -(-M // lin))
    return 1 + -(-M // lin) if staged else -(-M // per_pass)


def time_layer_case(L, M, copies, trunk, st, device, warmup, reps):
    """Device ms per sq_quantize_linear call of layer L at M tokens, as a CUDA
    graph of calls rotating over `copies` copies of the packed weight (enough
    copies that every call reads its weight from HBM, unless one), and the
    call's algorithmic bytes, launches per call and calls per graph."""
    import torch
    import decode_matvec_sq_b200 as sq
    import synth.device as sdev
    W = sdev.fill_weights(L, torch.empty(L.N, L.K, device=device))
    Ps = getattr(L, "residual_percent", 0)
    if Ps > 0:
        pw = sq.decompose_pack_sparse(W, Ps, trunk_percent=L.trunk_percent, status=st)
    elif Ps < 0:  # asymmetric residual groups
        pw = sq.decompose_pack(W, trunk_percent=L.trunk_percent, layout=sq.SQ_LAYOUT_TILES_ASYM,
                               status=st)
    else:
        pw = sq.decompose_pack(W, trunk_percent=L.trunk_percent, status=st)
    del W
    pws = [pw]
    for _ in range(copies - 1):
        c = sq.alloc_packed(L.N, L.K, 128, pw.with_mask, pw.layout, device=device)
        c.buf.copy_(pw.buf)
        pws.append(c)
    idx = torch.from_numpy(L.planted_channels()).to(device)
    x = sdev.fill_activations(L, torch.empty(M, L.K, device=device))
    y = torch.empty(M, L.N, device=device)
    ws = sq.new_fused_workspace(pw, M, L.n_out)
    calls = max(copies, 20)

    def launch():
        for r in range(calls):
            sq.quantize_linear(pws[r % copies], x, idx, y=y, workspace=ws, status=st,
                               trunk_only=trunk)

    for _ in range(warmup):
        launch()
    ms = _time_calls(launch, reps) / calls
    if trunk:
        wbytes = trunk_weight_bytes(L)
    elif Ps > 0:
        wbytes = sparse_weight_bytes(pw)
    else:  # (an asymmetric residual adds its zero-points: 4 bytes per group)
        wbytes = linear_weight_bytes(L) + (4 * pw.rows * pw.view.scale_stride if Ps < 0 else 0)
    nbytes = wbytes + M * (4 * L.K + 4 * L.N) + 4 * L.n_out
    launches = _fused_launches(pw, M, L, sq.SQ_TRUNK_ONLY if trunk else 0)
    del pws, pw, ws
    torch.cuda.empty_cache()
    return ms, nbytes, launches, calls


def time_prefill_case(st, device, warmup, steps):
    """The prefill workload (2048 tokens x 4096 -> 14336, row layout): device
    ms of the activation split + linear step and of the linear alone, with a
    256 MB buffer written between steps (cold L2)."""
    import torch
    import decode_matvec_sq_b200 as sq
    import synth.device as sdev
    from synth import workloads as wl
    L = wl.config5()
    W = sdev.fill_weights(L, torch.empty(L.N, L.K, device=device))
    pw = sq.decompose_pack(W, layout=sq.SQ_LAYOUT_ROWS, status=st)
    del W
    x = sdev.fill_activations(L, torch.empty(L.M, L.K, device=device))
    idx = torch.from_numpy(L.planted_channels()).to(device)
    xq, sx, xo = sq.quantize_act(x, idx, status=st)
    y = torch.empty(L.M, L.N, device=device)
    ws = sq.new_workspace(pw, L.M)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        sq.quantize_act(x, idx, xq=xq, sx=sx, x_out=xo, status=st)
        sq.linear(pw, xq, sx, xo, idx, y=y, workspace=ws, status=st)
    torch.cuda.synchronize()
    ev = []
    for _ in range(steps):
        flush.fill_(1)
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(stream)
        sq.quantize_act(x, idx, xq=xq, sx=sx, x_out=xo, status=st)
        b.record(stream)
        sq.linear(pw, xq, sx, xo, idx, y=y, workspace=ws, status=st)
        c.record(stream)
        ev.append((a, b, c))
    torch.cuda.synchronize()
    ms_step = sum(a.elapsed_time(c) for a, b, c in ev) / len(ev)
    ms_lin = sum(b.elapsed_time(c) for a, b, c in ev) / len(ev)
    del pw, ws, flush, x, xq, y
    torch.cuda.empty_cache()
    return ms_step, ms_lin, 4 * L.M * L.N * L.K


def time_nvfp4_prefill_case(st, device, warmup, steps):
    """The prefill workload's shape (2048 tokens x 4096 -> 14336) in NVFP4
    (format separation): the weight quantized once, then per step the
    per-token activation quantizer and the block-scaled tcgen05 GEMM, with a
    256 MB buffer written between steps (cold L2).  Device ms of the step and
    of the GEMM alone, and the GEMM's 2*M*N*K flops."""
    import torch
    import decode_matvec_sq_b200 as sq
    import synth.device as sdev
    from synth import workloads as wl
    L = wl.config5()
    W = sdev.fill_weights(L, torch.empty(L.N, L.K, device=device))
    w = sq.nvfp4_quantize(W, False, status=st)
    del W
    x = sdev.fill_activations(L, torch.empty(L.M, L.K, device=device))
    a = sq.alloc_nvfp4(L.M, L.K, True, device=device)
    y = torch.empty(L.M, L.N, device=device)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        sq.nvfp4_quantize(x, True, out=a, status=st)
        sq.nvfp4_linear(w, a, y=y, status=st)
    torch.cuda.synchronize()
    ev = []
    for _ in range(steps):
        flush.fill_(1)
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        e[0].record(stream)
        sq.nvfp4_quantize(x, True, out=a, status=st)
        e[1].record(stream)
        sq.nvfp4_linear(w, a, y=y, status=st)
        e[2].record(stream)
        ev.append(e)
    torch.cuda.synchronize()
    ms_step = sum(e[0].elapsed_time(e[2]) for e in ev) / len(ev)
    ms_lin = sum(e[1].elapsed_time(e[2]) for e in ev) / len(ev)
    del w, a, x, y, flush
    torch.cuda.empty_cache()
    return ms_step, ms_lin, 2 * L.M * L.N * L.K


def run_prefill_nvfp4(args, world, rank, local):
    """NVFP4 prefill (format separation) at the prefill workload's shape.
    Tensor-bound: TFLOP/s of the GEMM's 2*M*N*K against the dense fp4 peak."""
    import torch
    import torch.distributed as dist
    import decode_matvec_sq_b200 as sq
    from decode_matvec_sq_b200 import build

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device visible (the sq path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    if rank == 0 or world == 1:
        build.build_all()
    barrier(world)
    sq.device_check()
    st = torch.zeros(1, dtype=torch.int32, device=device)
    with ClockSampler(local) as clk:
        barrier(world)
        ms_step, ms_lin, flops = time_nvfp4_prefill_case(st, device, args.warmup, args.steps)
        barrier(world)
    clocks = clk.summary()
    ms_step = max_over_ranks(ms_step, world, device)
    ms_lin = max_over_ranks(ms_lin, world, device)
    if st.item() != 0:
        raise RuntimeError(f"device status {sq.STATUS.get(st.item())}")
    peak, kind = load_fp4_peak()
    probe = probe_peak(1)
    achieved = flops / (ms_lin * 1e-3) / 1e12
    if rank == 0:
        print(json.dumps({
            "metric": "prefill NVFP4 tensor TFLOP/s, 2048 tokens x 4096 -> 14336",
            "value": round(world * flops / (ms_step * 1e-3) / 1e12, 1), "unit": "TFLOP/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "nvfp4", "data": "synthetic",
            "config": {"workload": "prefill 2048 tokens x 4096 -> 14336 in NVFP4 (E2M1, UE4M3 "
                                   "blocks of 16, per-tensor / per-token fp32 scales), W "
                                   "Laplace(0,0.02), x N(0,1) with 0.5% channels x30",
                       "l2": "a 256 MB buffer written between steps"},
            "gpu_launches": 2 * args.steps,
            "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1),
                         "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "peak_kind": kind,
                         "traffic": None, "kernel": "k_nvfp4_gemm (tcgen05 kind::mxf4nvf4)",
                         "us_per_launch": round(ms_lin * 1e3, 2),
                         "probe_peak": round(probe, 1),
                         "frac_of_probe": round(achieved / probe, 4),
                         "probe_kind": "measured on this device: back-to-back kind::mxf4nvf4 MMAs "
                                       "128x256x64 on every SM (sq_testing_mma_peak)"},
            "clocks": clocks,
        }), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def side_configs(device, warmup=3, reps=10):
    """Compact measurements of the other workloads, outside the headline's
    timed region: the 512 x 512 layer (hot and cold), the 70B-shaped MLP pair
    at batch 1..16, the threshold-trunk layer and the prefill workload."""
    import torch
    st = torch.zeros(1, dtype=torch.int32, device=device)
    out = {}
    single = {}
    for label, L, M, copies in layer_cases("single"):
        ms, nbytes, _, _ = time_layer_case(L, M, copies, False, st, device, warmup, reps)
        single["us_hot" if copies == 1 else "us_cold"] = round(ms * 1e3, 2)
    out["single_512x512_batch1"] = single
    mlp = {}
    for label, L, M, copies in layer_cases("mlp70b"):
        ms, nbytes, _, _ = time_layer_case(L, M, copies, False, st, device, warmup, reps)
        mlp.setdefault(f"M={M}", {})[f"{L.K}->{L.N}"] = {"us": round(ms * 1e3, 2),
                                                           "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}
    out["mlp70b_batch_sweep"] = mlp
    for label, L, M, copies in layer_cases("threshold"):
        ms, nbytes, _, _ = time_layer_case(L, M, copies, False, st, device, warmup, reps)
        out["threshold_4096x14336_batch1"] = {"us": round(ms * 1e3, 2),
                                              "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1)}
    ms_step, ms_lin, ops = time_prefill_case(st, device, warmup, reps)
    peak, kind = load_int8_peak()
    out["prefill_2048x4096x14336"] = {"us_step": round(ms_step * 1e3, 1),
                                       "us_linear": round(ms_lin * 1e3, 1),
                                       "t_intops_linear": round(ops / (ms_lin * 1e-3) / 1e12, 1),
                                       "frac_of_int8_peak": round(ops / (ms_lin * 1e-3) / 1e12 / peak, 4),
                                       "int8_peak_kind": kind,
                                       "frac_of_probe_int8_peak": round(ops / (ms_lin * 1e-3) / 1e12 / probe_peak(0), 4)}
    ms_step, ms_lin, flops = time_nvfp4_prefill_case(st, device, warmup, reps)
    peak, kind = load_fp4_peak()
    out["prefill_nvfp4_2048x4096x14336"] = {"us_step": round(ms_step * 1e3, 1),
                                             "us_gemm": round(ms_lin * 1e3, 1),
                                             "tflops_gemm": round(flops / (ms_lin * 1e-3) / 1e12, 1),
                                             "frac_of_fp4_peak": round(flops / (ms_lin * 1e-3) / 1e12 / peak, 4),
                                             "fp4_peak_kind": kind,
                                             "frac_of_probe_fp4_peak": round(flops / (ms_lin * 1e-3) / 1e12 / probe_peak(1), 4)}
    if st.item() != 0:
        raise RuntimeError(f"side configurations: device status {st.item()}")
    return out


def run_layers(args, world, rank, local):
    """Single-layer workloads beside the stack: the 512 x 512 layer (hot and
    cold), the 70B-shaped MLP pair at batch 1..16 and the threshold-trunk layer.
    Each call is the one-launch fused entry point (activation split + linear;
    larger batches take the split, then one decode launch per 16 tokens),
    timed as a CUDA graph of
    calls rotating over the weight copies.  GB/s = algorithmic bytes (packed
    weights once + activations + y) / device time."""
    import torch
    import decode_matvec_sq_b200 as sq
    from decode_matvec_sq_b200 import build

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device visible (the sq path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)
    if rank == 0 or world == 1:
        build.build_all()
    barrier(world)
    sq.device_check()
    st = torch.zeros(1, dtype=torch.int32, device=device)
    cases = []
    tot_ms, tot_bytes, tot_launch = 0.0, 0, 0
    with ClockSampler(local) as clk:
        for label, L, M, copies in layer_cases(args.workload):
            trunk = args.workload == "trunk"
            barrier(world)
            ms, nbytes, launches, calls = time_layer_case(L, M, copies, trunk, st, device,
                                                          args.warmup, max(1, args.steps))
            ms = max_over_ranks(ms, world, device)
            cases.append({"case": label, "M": M, "us": round(ms * 1e3, 2),
                          "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1), "launches_per_call": launches})
            tot_ms += ms
            tot_bytes += nbytes
            tot_launch += max(1, args.steps) * calls * launches  # inside the timed replays
    clocks = clk.summary()
    if st.item() != 0:
        raise RuntimeError(f"device status {sq.STATUS.get(st.item())}")
    peak, kind = load_peaks()
    achieved = tot_bytes / (tot_ms * 1e-3) / 1e9
    names = {"single": "512x512 layer, batch 1, W Laplace(0,0.02), x N(0,1) with 4 channels x50",
             "mlp70b": "70B-shaped MLP pair 8192->28672 and 28672->8192, batch 1..16, "
                       "W N(0,0.015^2) with 0.1% entries x10, x N(0,1) with 0.25% channels x40",
             "threshold": "4096->14336, batch 1, per-row 60th-percentile trunk mask, "
                          "W Laplace(0,0.02), x N(0,1) with 0.5% channels x30",
             "trunk": "trunk-only mode (residual path skipped) of the 7B-shaped stack's four "
                      "linears, batch 1, W Laplace(0,0.02), x N(0,1) with 0.5% channels x30",
             "asym": "asymmetric residual groups (own min/max, scale, zero-point) on the "
                     "7B-shaped stack's four linears, batch 1, W Laplace(0,0.02), "
                     "x N(0,1) with 0.5% channels x30",
             "sparse": "sparse residual (per-row Ps-th percentile of |r| dropped, Ps 50/60/70) on "
                       "the 7B-shaped stack's four linears, batch 1, W Laplace(0,0.02), "
                       "x N(0,1) with 0.5% channels x30; GB/s on the bytes the kernel reads"}
    if rank == 0:
        print(json.dumps({
            "metric": f"single-layer sq_quantize_linear HBM GB/s ({args.workload})",
            "value": round(world * achieved, 1), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(tot_ms, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": {"workload": names[args.workload],
                       "l2": "cold cases rotate over copies of the weight totalling >= 2x L2"},
            "gpu_launches": tot_launch,
            "cases": cases,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": round(peak, 1),
                         "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_kind": kind,
                         "traffic": None, "kernel": "k_linear_tc (activation split + decode linear)"},
            "clocks": clocks,
        }), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_gpu(args, world, rank, local):
    import torch
    import torch.distributed as dist
    import decode_matvec_sq_b200 as sq
    from decode_matvec_sq_b200 import build
    from synth import workloads as wl

    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device visible (the sq path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=device)
    if rank == 0 or world == 1:
        build.build_all()
    if world > 1:
        dist.barrier()
    sq.device_check()

    layers = wl.config2(args.layers)
    stack = Stack(layers, device, pdl=not args.no_pdl, fused=not args.two_kernels)
    graph = stack.capture()
    nbytes = step_bytes(layers)
    launches_per_step = stack.launches_per_step

    stream = torch.cuda.current_stream()
    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()

    # ---- headline: device-timed steps, inputs resident in HBM --------------------
    with ClockSampler(local) as clk:
        barrier(world)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms_total = max_over_ranks(e0.elapsed_time(e1), world, device)
    clocks = clk.summary()
    ms_step = ms_total / args.steps
    value = world * nbytes / (ms_step * 1e-3) / 1e9
    if stack.status.item() != 0:
        raise RuntimeError(f"device status {sq.STATUS.get(stack.status.item())}")

    # ---- roofline of the dominant kernel ---------------------------------------
    # Every launch of the timed graph is the decode kernel (fused: activation
    # split + linear; two-kernel mode: the linear, with the split beside it),
    # so its average duration inside the timed step is the step time divided
    # by the launches; the algorithmic bytes per launch are its own reads and
    # writes.
    peak, peak_kind = load_peaks()
    if stack.fused:
        kbytes = sum(fused_launch_bytes(L) for L in layers)
        n_kernel = len(layers)
    else:
        kbytes = sum(linear_weight_bytes(L) + linear_act_bytes(L) + quantize_bytes(L) for L in layers)
        n_kernel = 2 * len(layers)
    bytes_launch = kbytes / len(layers)
    ms_launch = ms_step / n_kernel
    achieved = kbytes / (ms_step * 1e-3) / 1e9
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "linear_traffic.json")
    if os.path.exists(tpath):
        try:
            with open(tpath) as f:
                tr = json.load(f)
            if tr.get("kernel_hash") == kernel_hash():
                traffic = tr.get("dram_bytes_per_launch_stack_avg")
        except Exception:
            traffic = None

    y_checked = [y.clone() for y in stack.ys[:4]]  # layer 0's outputs of the timed steps

    # ---- end to end through host buffers ---------------------------------------
    e2e = None
    if not args.no_e2e:
        x_host = torch.empty_like(stack.x_all, device="cpu").pin_memory()
        x_host.copy_(stack.x_all.cpu())
        y_host = torch.empty_like(stack.y_all, device="cpu").pin_memory()
        g_e2e, _ = capture_e2e(stack, x_host, y_host)
        for _ in range(2):
            g_e2e.replay()
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.steps):
            g_e2e.replay()
        b.record(stream)
        torch.cuda.synchronize()
        barrier(world)
        ms_e2e = max_over_ranks(a.elapsed_time(b), world, device) / args.steps
        # the outputs that came back equal the outputs on the device, bit for bit
        e2e_same = bool(torch.equal(y_host, stack.y_all.cpu()))
        e2e = {"value": round(world * nbytes / (ms_e2e * 1e-3) / 1e9, 1), "unit": UNIT,
               "us_per_token": round(ms_e2e * 1e3, 2),
               "h2d_bytes_per_step": int(stack.x_all.numel() * 4),
               "d2h_bytes_per_step": int(stack.y_all.numel() * 4),
               "copies": "in the step's graph on a copy stream: inputs issued at the step's start "
                         "in three groups (linears 0-1, 2-11, the rest), each awaited before its "
                         "first linear; outputs back after every 32 linears and after the last two, "
                         "while later linears run",
               "outputs_equal_device": e2e_same}

    cpu, parity = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        sample = oracle_sample(rows=args.oracle_rows)
        gbs, per_pass, passes, sbytes = time_oracle(sample, min_seconds=args.oracle_seconds)
        cpu = {"value": round(gbs, 4), "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"first {args.oracle_rows} rows of each linear of layer 0 "
                         f"({sbytes / 1e6:.1f} MB per pass, {passes} passes, "
                         f"{per_pass * 1e3:.1f} ms per pass), quantize_act + linear",
               **host_info()}
        # the oracle's outputs for that sample against the timed graph's y
        parity = oracle_parity(sample, y_checked[:len(sample)])

    side = None
    if rank == 0 and not args.no_side_configs:
        side = side_configs(device)
    read_gbs = read_probe(device) if rank == 0 else None

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 4),
            "us_per_token": round(ms_step * 1e3, 2),
            "pct_of_8tbs": round(100.0 * value / world / NOMINAL_HBM_GBS, 2),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "int8", "data": "synthetic", "config": config_dict(argparse.Namespace(
                layers=args.layers, gpus=world)),
            "bytes_per_step": nbytes, "gpu_launches": launches_per_step * args.steps,
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "peak_kind": peak_kind, "traffic": traffic,
                         "kernel": "k_linear_tc (activation split + decode linear, tensor cores)"
                                   if stack.fused else "k_linear_tc (decode linear, tensor cores)",
                         "bytes_per_launch": int(bytes_launch),
                         "us_per_launch": round(ms_launch * 1e3, 3),
                         "timing": "timed PDL graph: step time / launches per step",
                         "read_probe_peak": read_gbs,
                         "frac_of_read_probe": round(achieved / read_gbs, 4) if read_gbs else None,
                         "read_probe_kind": "measured on this device after the timed region: read-only "
                                            "sweeps of a 2 GiB buffer, 16-byte coalesced loads "
                                            "(sq_testing_read_peak)"},
            "clocks": clocks,
            "e2e": e2e,
            "cpu_baseline": cpu,
            "parity_check": parity,
            "other_workloads": side,
        }
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def kernel_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("sq_linear_tc.cu", "sq_common.cuh", "sq_internal.h", "sq_quant.cuh", "sq_layout.h"):
        with open(os.path.join(ROOT, "decode_matvec_sq_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["sq", "reference"], default="sq")
    ap.add_argument("--layers", type=int, default=32)
    ap.add_argument("--workload", choices=["decode", "prefill", "prefill_nvfp4", "single", "mlp70b",
                                           "threshold", "trunk", "sparse", "asym"],
                    default="decode",
                    help="decode: the 7B-shaped stack at batch 1 (default); prefill: "
                         "2048 tokens x 4096 -> 14336 on the tcgen05 kernel; prefill_nvfp4: the "
                         "same shape in NVFP4 (format separation); single, mlp70b, "
                         "threshold: single-layer workloads (512x512 hot/cold, the 70B-shaped "
                         "MLP pair at batch 1..16, the threshold-trunk layer); trunk: the "
                         "stack's four linears in the trunk-only mode")
    ap.add_argument("--no-pdl", action="store_true")
    ap.add_argument("--two-kernels", action="store_true",
                    help="activation split and linear layer as two kernels per linear")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-side-configs", action="store_true",
                    help="skip the compact measurements of the other workloads (512x512, "
                         "70B-shaped MLP batch sweep, threshold trunk, prefill)")
    ap.add_argument("--oracle-rows", type=int, default=256)
    ap.add_argument("--oracle-seconds", type=float, default=10.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.workload == "prefill":
        return run_prefill(args, world, rank, local)
    if args.workload == "prefill_nvfp4":
        return run_prefill_nvfp4(args, world, rank, local)
    if args.workload in ("single", "mlp70b", "threshold", "trunk", "sparse", "asym"):
        return run_layers(args, world, rank, local)
    return run_gpu(args, world, rank, local)


if __name__ == "__main__":
    sys.exit(main())
