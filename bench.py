"""Benchmark of the Monarch training step (forward + backward) on B200 GPUs.

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: forward Y = X M^T
(R stage, permutation, L stage, output permutation) and backward (dX, dR, dL).
With N > 1 (launched by torchrun, one rank per GPU) every rank runs its own
batch of the same size (weak scaling, rows sharded across ranks) and the weight
gradients are summed over ranks with NCCL all-reduce, the one exchange step of
data-parallel training.

Inputs are seeded synthetic tensors with the workload's shapes and value
distributions.  Timing: CUDA events on the launching stream around each pass;
L2 is flushed before every timed pass (untimed): a 256 MiB write, then a read of the same
buffer, so the pass starts with no useful line in L2 and without the flush's dirty lines to
write back; max over ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_diagonal_linear_b200 import synthetic  # noqa: E402

DEFAULT_WORKLOAD = "n1024_bf16"
METRIC = "Monarch fwd/bwd rows/s and TFLOP/s at 1 B200; achieved % of roofline per shape"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# fp32 FMA peak (not measured): 148 SMs x 128 FMA lanes x 2 flops x 1.965 GHz
FFMA_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def describe(name: str, w: dict) -> str:
    return ("%s: R %d blocks of %dx%d, L %d blocks of %dx%d, %d->%d, out_transpose=%d, "
            "%d rows, %s" % (name, w["nb1"], w["out1"], w["in1"], w["nb2"], w["out2"], w["in2"],
                             w["nb1"] * w["in1"], w["nb2"] * w["out2"], w["out_transpose"],
                             w["rows"], w["dtype"]))


def algorithmic(w: dict, rows: int) -> dict:
    """Algorithmic flops and HBM bytes per pass: read inputs and factors once, write
    outputs once (no intermediates, no recompute)."""
    n_in, _, n_out = synthetic.sizes(w)
    params = w["nb1"] * w["out1"] * w["in1"] + w["nb2"] * w["out2"] * w["in2"]
    es = 2 if w["dtype"] == "bf16" else 4
    return {
        "fwd": {"flops": 2.0 * rows * params,
                "bytes": float(es * (rows * n_in + params + rows * n_out))},
        "bwd": {"flops": 4.0 * rows * params,
                "bytes": float(es * (rows * n_out + 2 * rows * n_in + 2 * params))},
        "params": params,
    }


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, \
            "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_hash(files) -> str:
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, srcs) -> float | None:
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        d = json.load(open(p))[kernel]
    except Exception:
        return None
    if d.get("source_sha") != source_hash(srcs):
        return None
    return float(d["dram_bytes_per_launch_full"])


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the timed region runs."""

    REASONS = {
        "hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
        "sw_power_cap": 0x4, "hw_power_brake_slowdown": 0x80,
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(device_index)
            bus = "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - depends on the box
            self.err = repr(e)

    def _sample(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for name, bit in self.REASONS.items():
            if mask & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            try:
                self._sample()
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.ok:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [],
                    "note": "NVML unavailable"}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- oracle arm
def oracle_rate(w: dict, seed: int = 0, budget_s: float = 8.0):
    """Rows/s of the fp64 CPU oracle (forward + backward) on a bounded sample of the
    workload, all host cores.  Test infrastructure, timed as the CPU baseline."""
    import oracle
    shape = synthetic.shape_of(w)
    params = algorithmic(w, 1)["params"]
    # size the sample so one fwd+bwd pass is about budget_s / 4 at ~0.5 GFLOP/s/core
    cores = oracle.default_threads()
    per_row = 6.0 * params
    rows = int(max(cores, min(w["rows"], budget_s / 4 * 0.5e9 * cores / per_row)))
    inp = synthetic.make_inputs(w, seed=seed, rows=rows)
    X, R, L, dY = inp["X"].f64, inp["R"].f64, inp["L"].f64, inp["dY"].f64
    done, t0 = 0, time.perf_counter()
    while True:
        oracle.forward(shape, X, R, L, nthreads=cores)
        oracle.backward(shape, dY, X, R, L, nthreads=cores)
        done += rows
        if time.perf_counter() - t0 >= budget_s or done >= 64 * rows:
            break
    dt = time.perf_counter() - t0
    return {"value": done / dt, "unit": "rows/s", "cores": cores, "kind": "oracle",
            "sample": "%d rows of %s (forward+backward, fp64, %d passes, %.1f s)"
                      % (rows, w.get("name", "workload"), done // rows, dt),
            "tflops": 6.0 * params * done / dt / 1e12}


def run_reference(args, w, name):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    shape = synthetic.shape_of(w)
    params = algorithmic(w, 1)["params"]
    cores = oracle.default_threads()
    rows = int(max(cores, min(w["rows"], 1.0 * 0.5e9 * cores / (6.0 * params))))
    inp = synthetic.make_inputs(w, seed=0, rows=rows)
    X, R, L, dY = inp["X"].f64, inp["R"].f64, inp["L"].f64, inp["dY"].f64
    for _ in range(args.warmup):
        oracle.forward(shape, X, R, L)
        oracle.backward(shape, dY, X, R, L)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.forward(shape, X, R, L)
        oracle.backward(shape, dY, X, R, L)
    dt = time.perf_counter() - t0
    value = rows * args.steps / dt
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "rows/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": describe(name, w), "rows_per_step": rows,
                   "note": "fp64 CPU oracle on a bounded sample of the workload's rows"},
        "cpu_baseline": {"value": value, "unit": "rows/s", "cores": cores, "kind": "oracle",
                         "sample": "%d of %d rows per step" % (rows, w["rows"])},
        "e2e": {"value": value, "unit": "rows/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


# --------------------------------------------------------------------------- kernel paths
FWD_KERNEL = {2: "tc_rows_kernel", 3: "tc_wide_kernel", 4: "tc_bdgemm_kernel + permute_rows_kernel",
              1: "tc_fwd_kernel", 5: "tc_gemm_kernel", 6: "tc_stage_kernel"}
FWD_SOURCE = {2: "tc_rows", 3: "tc_wide", 4: "tc_split", 1: "tc_fwd"}


def stage_bytes(w: dict, rows: int) -> float:
    """Bytes the two streaming stage launches of the workspace forward must move between them:
    each reads its input rows and factor once and writes its output rows once (the middle
    vector Z is written by the first and read by the second)."""
    n_in, n_mid, n_out = synthetic.sizes(w)
    es = 2 if w["dtype"] == "bf16" else 4
    p1 = w["nb1"] * w["out1"] * w["in1"]
    p2 = w["nb2"] * w["out2"] * w["in2"]
    return float(es * (rows * (n_in + n_mid) + p1 + rows * (n_mid + n_out) + p2))


def launches(shape: dict, dtype: str, pname: str) -> int:
    """Kernels one forward or backward call launches, counted by the library itself on a
    one-row call (the count does not depend on the row count)."""
    import torch
    import block_diagonal_linear_b200 as bdl
    w = dict(shape, rows=1, dtype=dtype)
    n_in, _, n_out = synthetic.sizes(w)
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    X = torch.zeros((1, n_in), dtype=dt, device="cuda")
    R = torch.zeros((shape["nb1"], shape["out1"], shape["in1"]), dtype=dt, device="cuda")
    L = torch.zeros((shape["nb2"], shape["out2"], shape["in2"]), dtype=dt, device="cuda")
    dY = torch.zeros((1, n_out), dtype=dt, device="cuda")
    if pname == "fwd":
        n0 = bdl.kernel_launches()
        bdl.fwd_train(X, R, L, shape)
    else:
        _, saved = bdl.fwd_train(X, R, L, shape)
        torch.cuda.synchronize()
        n0 = bdl.kernel_launches()
        bdl.bwd_saved(dY, X, R, L, shape, saved)
    torch.cuda.synchronize()
    return bdl.kernel_launches() - n0


# --------------------------------------------------------------------------- per shape
PER_SHAPE = ("n256_fp32", "n1024_bf16", "r768x3072_bf16", "n4096_bf16", "nblk4_1024x4096_bf16",
             "nblk4_1024x4096_bf16_b1000")


def device_inputs(w, seed, dev):
    import torch
    inp = synthetic.make_inputs(w, seed=seed)
    out = {}
    for k in ("X", "R", "L", "dY"):
        t = inp[k]
        if t.dtype == "bf16":
            out[k] = torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)
        else:
            out[k] = torch.from_numpy(np.ascontiguousarray(t.bits)).to(dev)
    return out


class L2Flush:
    """Untimed L2 flush before a timed pass: write a buffer of at least twice the L2 size, then
    read it back.  The write evicts every line a pass could reuse; the read evicts the flush's
    own dirty lines (their write-back happens here, not inside the timed pass)."""

    def __init__(self, dev):
        import torch
        l2 = torch.cuda.get_device_properties(dev).L2_cache_size
        self.buf = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8, device=dev)

    def __call__(self):
        import torch
        self.buf.zero_()
        torch.amax(self.buf.view(torch.int32))

    def mib(self):
        return self.buf.numel() >> 20


def time_shape(name, dev, flush, peaks, reps=10, warmup=3, spin_cycles=2000000):
    """Forward and backward of one workload, each pass timed alone with CUDA events on the
    launching stream after an untimed L2 flush and GPU-side spin; averages over `reps`."""
    import torch
    import block_diagonal_linear_b200 as bdl
    w = dict(synthetic.WORKLOADS[name], name=name)
    shape = synthetic.shape_of(w)
    rows = w["rows"]
    d = device_inputs(w, seed=2000, dev=dev)
    X, R, L, dY = d["X"], d["R"], d["L"], d["dY"]
    Y = torch.empty((rows, synthetic.sizes(w)[2]), dtype=X.dtype, device=dev)
    dX, dR, dL = torch.empty_like(X), torch.empty_like(R), torch.empty_like(L)
    ws = torch.empty(max(bdl.bwd_workspace_bytes(shape, rows, w["dtype"]), 256), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream()
    # the training pair: the forward keeps the middle vector, the backward reuses it
    sb = bdl.saved_bytes(shape, rows, w["dtype"])
    saved = torch.empty(sb, dtype=torch.uint8, device=dev) if sb else None
    bdl.fwd_train(X, R, L, shape, Y=Y, saved=saved)  # the backward timings read this saved buffer
    runs = {"fwd": lambda: bdl.fwd_train(X, R, L, shape, Y=Y, saved=saved),
            "bwd": lambda: bdl.bwd_saved(dY, X, R, L, shape, saved, dX=dX, dR=dR, dL=dL, workspace=ws)}
    alg = algorithmic(w, rows)
    hbm, tpk = peaks["hbm_gbs"] * 1e9, peaks["bf16_tflops"] * 1e12
    if w["dtype"] == "f32":
        tpk = FFMA_TFLOPS * 1e12
    res = {"workload": describe(name, w), "fwd_path": bdl.fwd_ws_path(shape, w["dtype"]),
           "bwd_path": bdl.bwd_path(shape, w["dtype"])}
    for pname, fn in runs.items():
        evs, host = [], []
        for i in range(warmup + reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            flush()
            torch.cuda._sleep(spin_cycles)
            e0.record(stream)
            h0 = time.perf_counter()
            fn()
            h1 = time.perf_counter()
            e1.record(stream)
            if i >= warmup:
                evs.append((e0, e1))
                host.append(h1 - h0)
        torch.cuda.synchronize()
        ms = sum(a.elapsed_time(b) for a, b in evs) / len(evs)
        t = ms / 1e3
        a = alg[pname]
        t_roof = max(a["bytes"] / hbm, a["flops"] / tpk)
        res[pname] = {
            "ms": ms, "rows_per_s": rows / t, "tflops": a["flops"] / t / 1e12,
            "gbs": a["bytes"] / t / 1e9, "roofline_ms": t_roof * 1e3, "roofline_frac": t_roof / t,
            "bound": "hbm" if a["bytes"] / hbm >= a["flops"] / tpk else
                     ("fma" if w["dtype"] == "f32" else "tensor"),
            "launches": launches(shape, w["dtype"], pname),
            "host_enqueue_us": 1e6 * sum(host) / len(host),
            "entry": "monarch_fwd_train" if pname == "fwd" else "monarch_bwd_saved",
        }
    if bdl.last_device_status() != 0:
        raise SystemExit("device status not OK after timing %s" % name)
    del X, R, L, dY, Y, dX, dR, dL, ws, d, saved
    torch.cuda.empty_cache()
    return res


# --------------------------------------------------------------------------- GPU arm
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(synthetic.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer end-to-end timing")
    ap.add_argument("--no-per-shape", dest="per_shape", action="store_false",
                    help="skip the per-workload forward/backward timings")
    ap.add_argument("--pass", dest="only", default="step", choices=["step", "fwd", "bwd"],
                    help="time the whole step (default) or one pass only")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    name = args.workload
    w = dict(synthetic.WORKLOADS[name], name=name)

    if args.impl == "reference":
        run_reference(args, w, name)
        return

    import torch
    import torch.distributed as dist
    import block_diagonal_linear_b200 as bdl

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev_ = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev_)

    shape = synthetic.shape_of(w)
    rows = w["rows"]  # per rank (weak scaling)
    inp = synthetic.make_inputs(w, seed=1000 + rank)
    def to_dev(t):
        if t.dtype == "bf16":
            return torch.from_numpy(t.bits.view(np.int16).copy()).view(torch.bfloat16).to(dev_)
        return torch.from_numpy(np.ascontiguousarray(t.bits)).to(dev_)

    X, R, L, dY = (to_dev(inp[k]) for k in ("X", "R", "L", "dY"))
    n_in, _, n_out = synthetic.sizes(w)
    Y = torch.empty((rows, n_out), dtype=X.dtype, device=dev_)
    dX = torch.empty_like(X)
    dR = torch.empty_like(R)
    dL = torch.empty_like(L)
    ws = torch.empty(max(bdl.bwd_workspace_bytes(shape, rows, w["dtype"]), 256), dtype=torch.uint8,
                     device=dev_)
    sb = bdl.saved_bytes(shape, rows, w["dtype"])  # the forward's saved middle vector
    saved = torch.empty(sb, dtype=torch.uint8, device=dev_) if sb else None
    bdl.fwd_train(X, R, L, shape, Y=Y, saved=saved)  # a backward-only run reads this
    flush = L2Flush(dev_)
    stream = torch.cuda.current_stream()

    from block_diagonal_linear_b200 import dp

    def allreduce_grads():
        if world > 1:
            dp.allreduce_weight_grads(dR, dL)

    do_fwd = args.only in ("step", "fwd")
    do_bwd = args.only in ("step", "bwd")

    # A GPU-side spin (~1 ms) after each untimed flush lets the host enqueue the next pass
    # before the start event fires, so launch latency on the host is not timed.
    spin_cycles = 2000000

    def step(ev=None):
        if ev is not None:
            flush()
            torch.cuda._sleep(spin_cycles)
            ev[0].record(stream)
        if do_fwd:
            bdl.fwd_train(X, R, L, shape, Y=Y, saved=saved)
        if ev is not None:
            ev[1].record(stream)
            flush()
            torch.cuda._sleep(spin_cycles)
            ev[2].record(stream)
        if do_bwd:
            bdl.bwd_saved(dY, X, R, L, shape, saved, dX=dX, dR=dR, dL=dL, workspace=ws)
            allreduce_grads()
        if ev is not None:
            ev[3].record(stream)

    for _ in range(args.warmup):
        step([torch.cuda.Event(enable_timing=True) for _ in range(4)])
    torch.cuda.synchronize()
    if bdl.last_device_status() != 0:
        raise SystemExit("device status not OK after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    launches0 = bdl.kernel_launches()
    with sampler:
        for k in range(args.steps):
            step(evs[k])
        torch.cuda.synchronize()
    launches_timed = bdl.kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    bwd_ms = [e[2].elapsed_time(e[3]) for e in evs]
    tot_ms = sum(fwd_ms) + sum(bwd_ms)
    if world > 1:
        t = torch.tensor([tot_ms, sum(fwd_ms), sum(bwd_ms)], dtype=torch.float64, device=dev_)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        tot_ms, fwd_sum, bwd_sum = t.tolist()
    else:
        fwd_sum, bwd_sum = sum(fwd_ms), sum(bwd_ms)
    status = bdl.last_device_status()

    # ---- end to end through the public API with host buffers (pinned), copies timed.  Every
    # step copies its inputs in from pinned host memory and its results out; the copies and
    # the compute run on three streams with two buffer sets, so step k+1's inputs travel in
    # while step k computes and step k-1's results travel out (PCIe is full duplex).
    Xh = torch.empty_like(X, device="cpu").pin_memory()
    Xh.copy_(X)
    dYh = torch.empty_like(dY, device="cpu").pin_memory()
    dYh.copy_(dY)
    n_e2e = 0 if args.no_e2e or args.only != "step" else max(3, min(args.steps, 50))
    nbuf = 2 if n_e2e else 0
    Xe = [torch.empty_like(X) for _ in range(nbuf)]
    dYe = [torch.empty_like(dY) for _ in range(nbuf)]
    outs_d = [[torch.empty_like(t) for t in (Y, dX, dR, dL)] for _ in range(nbuf)]
    outs_h = [[torch.empty_like(t, device="cpu").pin_memory() for t in (Y, dX, dR, dL)] for _ in range(nbuf)]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev_) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(k):
        b = k % 2
        with torch.cuda.stream(s_in):
            s_in.wait_event(ev_comp[b])      # the step that last read buffer set b is done
            Xe[b].copy_(Xh, non_blocking=True)
            dYe[b].copy_(dYh, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            s_comp.wait_event(ev_out[b])     # buffer set b's previous results are copied out
            y, dx, dr, dl = outs_d[b]
            bdl.fwd_train(Xe[b], R, L, shape, Y=y, saved=saved)
            bdl.bwd_saved(dYe[b], Xe[b], R, L, shape, saved, dX=dx, dR=dr, dL=dl, workspace=ws)
            if world > 1:
                dp.allreduce_weight_grads(dr, dl)
            ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            for h, d_ in zip(outs_h[b], outs_d[b]):
                h.copy_(d_, non_blocking=True)
            ev_out[b].record(s_out)

    for k in range(2 if n_e2e else 0):
        e2e_step(k)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(n_e2e):
        e2e_step(k)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) if n_e2e else 0.0
    if world > 1:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev_)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = t.item()
    h2d = X.numel() * X.element_size() + dY.numel() * dY.element_size()
    d2h = sum(t.numel() * t.element_size() for t in (Y, dX, dR, dL))

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    peaks, peak_src = load_peaks()
    alg = algorithmic(w, rows)
    K = args.steps
    fwd_avg_s = fwd_sum / K / 1e3
    bwd_avg_s = bwd_sum / K / 1e3
    hbm = peaks["hbm_gbs"] * 1e9
    tpk = peaks["bf16_tflops"] * 1e12
    passes = {}
    for pname, t_s in (("fwd", fwd_avg_s), ("bwd", bwd_avg_s)):
        if (pname == "fwd" and not do_fwd) or (pname == "bwd" and not do_bwd):
            continue
        a = alg[pname]
        t_roof = max(a["bytes"] / hbm, a["flops"] / tpk)
        passes[pname] = {
            "ms": t_s * 1e3, "rows_per_s": rows / t_s, "tflops": a["flops"] / t_s / 1e12,
            "gbs": a["bytes"] / t_s / 1e9, "roofline_ms": t_roof * 1e3,
            "roofline_frac": t_roof / t_s,
            "bound": "hbm" if a["bytes"] / hbm >= a["flops"] / tpk else "tensor",
        }
    fpath = bdl.fwd_ws_path(shape, w["dtype"])
    bpath = bdl.bwd_path(shape, w["dtype"])
    fwd_launches = launches(shape, w["dtype"], "fwd")
    bwd_launches = launches(shape, w["dtype"], "bwd")
    # Roofline objects.  `roofline`: the forward kernel (one launch per forward pass, so the pass
    # time measured by the events is that kernel's launch duration).  `roofline_bwd`: the backward
    # pass (several launches), against the backward's algorithmic bytes and flops.
    def roof_of(pname, t_s, kname, srcs):
        a = alg[pname]
        if passes[pname]["bound"] == "hbm":
            r = {"bound": "hbm", "achieved": a["bytes"] / t_s / 1e9, "peak": peaks["hbm_gbs"],
                 "unit": "GB/s"}
        else:
            r = {"bound": "tensor", "achieved": a["flops"] / t_s / 1e12,
                 "peak": peaks["bf16_tflops"], "unit": "TFLOP/s"}
        r["frac"] = r["achieved"] / r["peak"]
        r["traffic"] = measured_traffic(kname, srcs) if srcs else None
        r["kernel"] = kname
        r["algorithmic_bytes_per_launch"] = a["bytes"]
        r["algorithmic_flops_per_launch"] = a["flops"]
        r["peak_source"] = peak_src
        return r

    roof, roof_bwd = None, None
    if do_fwd:
        kname = FWD_KERNEL.get(fpath, "gen_fwd_kernel")
        if fwd_launches > 1:
            kname += " (pass of %d kernels)" % fwd_launches
        srcs = (["block_diagonal_linear_b200/csrc/%s.cu" % FWD_SOURCE[fpath],
                 "block_diagonal_linear_b200/csrc/ptx.cuh", "block_diagonal_linear_b200/csrc/tc_common.cuh"]
                if fpath in FWD_SOURCE and fwd_launches == 1 else None)
        roof = roof_of("fwd", fwd_avg_s, kname, srcs)
        if fwd_launches == 1 and sb and roof["bound"] == "hbm":
            # the fused training forward also writes the kept middle vector: its own algorithmic
            # bytes are X, R, L read and Y, Z written
            kb = alg["fwd"]["bytes"] + sb
            roof.update({"achieved": kb / fwd_avg_s / 1e9, "algorithmic_bytes_per_launch": kb,
                         "note": "training forward kernel: X, R, L read; Y and the kept middle "
                                 "vector Z written"})
            roof["frac"] = roof["achieved"] / roof["peak"]
        if fpath == 6 and roof["bound"] == "hbm":
            # the dominant kernel is the stage kernel, launched twice per pass: its own bytes
            # (input, factor and output of each launch) over the two launches' time
            stb = stage_bytes(w, rows)
            roof.update({"achieved": stb / fwd_avg_s / 1e9, "algorithmic_bytes_per_launch": stb / 2,
                         "launches_per_pass": 2,
                         "note": "stage kernel, Z = P blockdiag(R) X then Y = P_out blockdiag(L) Z; "
                                 "pass time / 2 per launch"})
            roof["frac"] = roof["achieved"] / roof["peak"]
    if do_bwd:
        roof_bwd = roof_of("bwd", bwd_avg_s, "monarch_bwd (pass of %d kernels)" % bwd_launches, None)
    if roof is None:
        roof, roof_bwd = roof_bwd, None

    per_shape = None
    if args.per_shape and world == 1:
        per_shape = {}
        for pn in PER_SHAPE:
            per_shape[pn] = time_shape(pn, dev_, flush, peaks)

    value = world * rows * K / (tot_ms / 1e3)
    out = {
        "metric": METRIC, "value": value, "unit": "rows/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": tot_ms / K, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w["dtype"], "data": "synthetic",
        "config": {"workload": describe(name, w), "rows_per_gpu": rows,
                   "step": "forward keeping the middle vector (monarch_fwd_train) + backward reusing it "
                           "(monarch_bwd_saved: dX, dR, dL)" +
                           (" + NCCL all-reduce of dR, dL" if world > 1 else ""),
                   "l2": "flushed before every timed pass (untimed: %d MiB write, then a read of "
                         "the same buffer so no dirty flush line is written back inside the pass), "
                         "then a GPU-side spin so host launch latency is outside the timed pass"
                         % flush.mib(),
                   "parallelism": "dp%d" % world, "timed": args.only},
        "tflops": (alg["fwd"]["flops"] + alg["bwd"]["flops"]) * world * K / (tot_ms / 1e3) / 1e12,
        "passes": passes,
        "roofline": roof,
        "roofline_bwd": roof_bwd,
        "per_shape": per_shape,
        "e2e": ({"value": world * rows * n_e2e / (e2e_ms / 1e3), "unit": "rows/s",
                 "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
                 "note": "pinned host inputs in and results out every step; copies overlap the "
                         "compute of the neighbouring steps (three streams, two buffer sets)"}
                if n_e2e else None),
        "gpu_launches": launches_timed,
        "launches_per_step": {"fwd": fwd_launches if do_fwd else 0, "bwd": bwd_launches if do_bwd else 0},
        "clocks": sampler.summary(),
        "device_status": status,
    }
    if not args.no_cpu_baseline and world == 1:
        out["cpu_baseline"] = oracle_rate(w)
    print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
