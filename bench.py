#!/usr/bin/env python
"""Benchmark of the block-scaled FP4 quantization path on B200.

One step = the whole path over the 40-layer activation stack (65536 x 4096
bf16 per layer, 0.5 * Student-t(4) times per-channel LogNormal(0,1)):
  rollout side: NVFP4 amax pass + capture for all 40 layers, with guidance
                bits kept for the deepest 20 (layers 20..39);
  train side:   guided quantization of perturbed copies of layers 20..39
                against their records.
Metric: algorithmic GB/s (bytes the definition forces per element: two
reads of x for the tensor-scale pass, the code / scale / guidance writes,
the guided pass's reads and writes), as a fraction of measured HBM copy
bandwidth.  Inputs (512 MiB per layer) exceed the 126 MB L2, so no flush.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Multi-GPU (torchrun, one rank per GPU): every rank quantizes its own stack
(weak scaling, no collective on the data path); the time is the max over
ranks.  ``--impl reference`` times the CPU oracle on a bounded row sample
of the same workload instead.
"""
import argparse
import hashlib
import json
import os
import shutil
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "quantize/capture/guided GB/s and % of B200 HBM peak (1 GPU)"
FALLBACK_HBM_GBS = 6650.0
DATASHEET_HBM_GBS = 8000.0

# algorithmic bytes per element (see the module docstring)
B_AMAX = 2.0                       # read x
B_QUANT = 2.0 + 0.5 + 1.0 / 16     # read x, write codes + scale bytes
B_BITS = 1.0 / 8                   # guidance bits written by capture
B_GUIDED = 2.0 + 1.0 / 16 + 1.0 / 8 + 0.5  # read x', scales, bits; write codes


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--layers", type=int, default=40)
    p.add_argument("--deep", type=int, default=20)
    p.add_argument("--rows", type=int, default=65536)
    p.add_argument("--cols", type=int, default=4096)
    p.add_argument("--e2e-steps", type=int, default=2)
    p.add_argument("--event-every", type=int, default=10,
                   help="per-kernel CUDA events on every n-th timed step (an event between two launches "
                        "costs a few microseconds of idle GPU and stops the next launch from overlapping)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=256, help="rows per layer in the single-core oracle sample")
    p.add_argument("--cpu-mc-factor", type=int, default=8,
                   help="the all-core oracle sample is this many times the single-core one")
    p.add_argument("--ref-rows", type=int, default=256, help="rows per layer per reference step")
    p.add_argument("--train-rel", type=float, default=1e-3,
                   help="relative perturbation of the train-side copies (x' = bf16(x (1 + rel N(0,1)))); "
                        "larger values make more train values round to another codeword than the rollout's")
    p.add_argument("--suite", action="store_true",
                   help="time every call of the path on every workload (a table, not the bench line)")
    p.add_argument("--only", action="append",
                   help="with --suite: run only rows matching workload-prefix[:format[:call]] (repeatable)")
    p.add_argument("--mismatch-by-layer", action="store_true",
                   help="per layer of the stack: the diagnostics' counts of the train copy against the layer's "
                        "capture, the corrections split by direction (a table, not the bench line)")
    return p.parse_args()


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist

        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def max_over_ranks(v, world, dev):
    if world == 1:
        return v
    import torch.distributed as dist

    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- clocks
class Clocks:
    """nvidia-smi samples (every 200 ms) during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        if not shutil.which("nvidia-smi"):
            return
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        self.f = open(self.path, "w")
        self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                                      "--format=csv,noheader,nounits", "-lms", "200"],
                                     stdout=self.f, stderr=subprocess.DEVNULL)
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        for line in open(self.path):
            p = [s.strip() for s in line.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append(dict(sm=float(p[1]), max=float(p[2]), power=float(p[3]), hw=p[5], hwt=p[6],
                                 swt=p[7], pcap=p[8]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        loaded = [r for r in rows if r["power"] > 200] or rows
        reasons = set()
        for r in rows:
            for k, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                            ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[k].lower() == "active":
                    reasons.add(name)
        return dict(sm_mhz=statistics.median(r["sm"] for r in loaded), sm_max_mhz=max(r["max"] for r in rows),
                    reasons=sorted(reasons), samples=len(rows), power_w_max=max(r["power"] for r in rows))


def hbm_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash():
    """Hash of the kernel sources' code: line comments and blank lines are
    left out, so that a comment edit does not void committed counters."""
    h = hashlib.sha256()
    for rel in ("fp4_block_scaled_quantizer_b200/csrc/tf4_kernels.cuh", "fp4_block_scaled_quantizer_b200/csrc/trace_fp4.cu"):
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            for line in f:
                code = line.split("//", 1)[0].rstrip()
                if code:
                    h.update(code.encode() + b"\n")
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(p) as f:
            t = json.load(f)
    except Exception:
        return None
    e = t.get(kernel_key)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e


# ------------------------------------------------------------- workload
def make_stack(args, dev):
    from fp4_block_scaled_quantizer_b200 import workloads as W

    xs, xts = [], []
    for layer in range(args.layers):
        x = W.layer_stack_layer(layer, dev, rows=args.rows, cols=args.cols)
        xs.append(x)
        if layer >= args.layers - args.deep:
            xts.append(W.perturb(x, 1000 + layer, rel=args.train_rel))
    torch.cuda.synchronize()
    return xs, xts


def step_bytes(args):
    n = args.rows * args.cols
    deep = args.deep
    shallow = args.layers - deep
    cap = n * (args.layers * (B_AMAX + B_QUANT) + deep * B_BITS)
    gd = n * deep * B_GUIDED
    return cap + gd, n * (args.layers + deep)


def run_ours(args, world, rank, local):
    import fp4_block_scaled_quantizer_b200 as tf4
    from fp4_block_scaled_quantizer_b200 import binding as B
    from fp4_block_scaled_quantizer_b200 import build as libbuild

    libbuild.build()
    B.lib()
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    xs, xts = make_stack(args, dev)
    L, D = args.layers, args.deep
    first_deep = L - D
    n = args.rows * args.cols
    recs = [tf4.tf4_quantize_capture(xs[i], guidance=i >= first_deep) for i in range(L)]
    amax = [torch.empty(1, dtype=torch.float32, device=dev) for _ in range(L)]
    gcodes = [torch.empty(n // 2, dtype=torch.uint8, device=dev) for _ in range(D)]
    torch.cuda.synchronize()

    def new_events(count):
        return [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(count)]

    def step(ev):
        for i in range(L):
            if ev:
                ev["amax"][i][0].record(stream)
            B.tf4_segment_amax(xs[i], out=amax[i])
            if ev:
                ev["amax"][i][1].record(stream)
                ev["quant"][i][0].record(stream)
            B.tf4_quantize_capture(xs[i], guidance=i >= first_deep, amax_in=amax[i], out=recs[i])
            if ev:
                ev["quant"][i][1].record(stream)
        for j in range(D):
            if ev:
                ev["guided"][j][0].record(stream)
            B.tf4_quantize_guided(xts[j], recs[first_deep + j], out=gcodes[j])
            if ev:
                ev["guided"][j][1].record(stream)

    launches_per_step = 2 * L + D
    for _ in range(args.warmup):
        step(None)
    torch.cuda.synchronize()
    assert B.read_status(dev) == 0, "non-finite input in the workload"
    # how often a train value's nearest code differs from the rollout's (outside the timed region)
    cnt = torch.zeros(B.MISMATCH_COUNTS, dtype=torch.int64, device=dev)
    for j in range(D):
        B.tf4_mismatch_stats(xts[j], recs[first_deep + j], counts=cnt)
    mismatch_fraction = float(cnt[0].item()) / (D * n) if D else 0.0
    # per-kernel events on every event_every-th timed step, read after the timed region
    every = max(1, args.event_every)
    evs = [dict(amax=new_events(L), quant=new_events(L), guided=new_events(D)) if k % every == 0 else None
           for k in range(args.steps)]
    instrumented = [k for k in range(args.steps) if evs[k] is not None]

    clocks = Clocks(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    ms_step = max_over_ranks(ms_total / args.steps, world, dev)
    times = {k: [[a.elapsed_time(b) for a, b in e[k]] for e in evs if e is not None]
             for k in ("amax", "quant", "guided")}

    bytes_step, elems_step = step_bytes(args)
    value = world * bytes_step / (ms_step * 1e-3) / 1e9
    peak, peak_kind = hbm_peak()

    # per-kernel averages
    def avg(k):
        return statistics.mean(v for s in times[k] for v in s)

    quant_bytes = [n * (B_QUANT + (B_BITS if i >= first_deep else 0.0)) for i in range(L)]
    per_kernel = {
        "amax": dict(ms=avg("amax"), bytes=n * B_AMAX),
        "quant": dict(ms=avg("quant"), bytes=statistics.mean(quant_bytes)),
        "guided": dict(ms=avg("guided"), bytes=n * B_GUIDED),
    }
    shares = {k: sum(sum(s) for s in times[k]) for k in times}
    tot = sum(shares.values())
    calls = {}
    for k, v in per_kernel.items():
        gbs = v["bytes"] / (v["ms"] * 1e-3) / 1e9
        calls[k] = dict(us=round(v["ms"] * 1e3, 2), gbs=round(gbs, 1), frac=round(gbs / peak, 4),
                        share=round(shares[k] / tot, 4))
    dom = max(shares, key=shares.get)
    kname = {"amax": "k_amax", "quant": "k_quant (NVFP4: RTN layers 0-19, capture layers 20-39)",
             "guided": "k_guided(NVFP4)"}[dom]
    achieved = per_kernel[dom]["bytes"] / (per_kernel[dom]["ms"] * 1e-3) / 1e9
    tr = ncu_traffic(dom)
    roofline = dict(bound="hbm", kernel=kname, achieved=round(achieved, 1), peak=peak, unit="GB/s",
                    frac=round(achieved / peak, 4), peak_kind=f"{peak_kind} copy bandwidth",
                    traffic=(tr["dram_bytes_per_launch"] if tr else None),
                    algorithmic_bytes_per_launch=per_kernel[dom]["bytes"])

    out = dict(metric=METRIC, value=round(value, 1), unit="GB/s", n_gpus=world, steps=args.steps,
               warmup=args.warmup, ms_per_step=round(ms_step, 4), higher_is_better=True, scaling="weak",
               vs_baseline=None, dtype="f32", data="synthetic",
               config=dict(workload=f"layer_stack: {L} layers x {args.rows}x{args.cols} bf16 "
                                    f"(0.5*t4 x LogNormal channel scales), NVFP4 capture with guidance for "
                                    f"layers {first_deep}-{L - 1}, guided quantization of perturbed copies "
                                    f"of those layers (x (1 + {args.train_rel:g} N(0,1)))",
                           train_rel=args.train_rel, train_mismatch_fraction=round(mismatch_fraction, 6),
                           layers=L, deep_layers=D, rows=args.rows, cols=args.cols, format="NVFP4",
                           parallelism=f"dp{world} (independent stacks)",
                           l2="inputs 512 MiB per layer > 126 MB L2; no flush",
                           per_kernel_events=f"timed steps {instrumented} of {args.steps}"),
               frac_of_peak=round(value / world / peak, 4),
               frac_of_datasheet=round(value / world / DATASHEET_HBM_GBS, 4),
               elements_per_s=round(world * elems_step / (ms_step * 1e-3), 1),
               calls=calls, roofline=roofline, gpu_launches=launches_per_step * args.steps,
               clocks=clk)

    if not args.no_e2e:
        out["e2e"] = run_e2e(args, world, dev, xs, xts, recs, amax, gcodes)
    for t in (xs, xts, gcodes):
        t.clear()
    recs.clear()
    torch.cuda.empty_cache()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args, args.cpu_rows)
    return out


def run_e2e(args, world, dev, xs, xts, recs, amax, gcodes):
    """Same step through the public API with host buffers: every step copies
    the layers' inputs from pinned host memory (double-buffered on a copy
    stream) and reads every result back to pinned host memory.  With several
    ranks on one host each rank takes a 1/world share of the stack (half of
    it deep layers), so the pinned host memory stays that of one stack."""
    import psutil

    from fp4_block_scaled_quantizer_b200 import binding as B

    if world > 1:
        Lf, Df = args.layers, args.deep
        L = max(2, Lf // world)
        D = min(Df, L // 2)
        keep = list(range(L - D)) + list(range(Lf - D, Lf))  # some shallow layers, then the deepest D
        xs, recs, amax = [xs[i] for i in keep], [recs[i] for i in keep], [amax[i] for i in keep]
        xts, gcodes = xts[Df - D:], gcodes[Df - D:]
        args = argparse.Namespace(**{**vars(args), "layers": L, "deep": D})
    L, D = args.layers, args.deep
    first_deep = L - D
    n = args.rows * args.cols
    in_bytes = (L + D) * n * 2
    out_bytes = L * (n // 2 + n // 16 + 4) + D * (n // 8 + n // 2)
    local = int(os.environ.get("LOCAL_WORLD_SIZE", "1"))
    ok = psutil.virtual_memory().available >= 1.6 * (in_bytes + out_bytes) * local
    if world > 1:  # every rank takes the same branch
        import torch.distributed as dist

        f = torch.tensor([1 if ok else 0], dtype=torch.int32, device=dev)
        dist.all_reduce(f, op=dist.ReduceOp.MIN)
        ok = bool(f.item())
    if not ok:
        return dict(value=None, unit="GB/s", skipped="not enough host memory for pinned buffers")
    hx = [torch.empty_like(x, device="cpu").pin_memory() for x in xs]
    hxt = [torch.empty_like(x, device="cpu").pin_memory() for x in xts]
    for h, x in zip(hx + hxt, xs + xts):
        h.copy_(x)
    hc = [torch.empty(n // 2, dtype=torch.uint8).pin_memory() for _ in range(L)]
    hs = [torch.empty(n // 16, dtype=torch.uint8).pin_memory() for _ in range(L)]
    hst = torch.empty(L, dtype=torch.float32).pin_memory()
    hb = [torch.empty(n // 8, dtype=torch.uint8).pin_memory() for _ in range(D)]
    hg = [torch.empty(n // 2, dtype=torch.uint8).pin_memory() for _ in range(D)]
    # device staging: two input slots
    slot = [torch.empty_like(xs[0]) for _ in range(2)]
    comp = torch.cuda.current_stream(dev)
    copy = torch.cuda.Stream(dev)
    ready = [torch.cuda.Event() for _ in range(2)]
    free = [torch.cuda.Event() for _ in range(2)]
    out_stream = torch.cuda.Stream(dev)
    done = [torch.cuda.Event() for _ in range(L + D)]

    def e2e_step():
        jobs = [("cap", i) for i in range(L)] + [("gd", j) for j in range(D)]
        # prefetch first (slot 0 may still be read by the previous step)
        with torch.cuda.stream(copy):
            copy.wait_event(free[0])
            slot[0].copy_(hx[0], non_blocking=True)
            ready[0].record(copy)
        for t, (kind, i) in enumerate(jobs):
            s = t % 2
            if t + 1 < len(jobs):
                nk, ni = jobs[t + 1]
                src = hx[ni] if nk == "cap" else hxt[ni]
                with torch.cuda.stream(copy):
                    if t >= 1:
                        copy.wait_event(free[(t + 1) % 2])
                    slot[(t + 1) % 2].copy_(src, non_blocking=True)
                    ready[(t + 1) % 2].record(copy)
            comp.wait_event(ready[s])
            if kind == "cap":
                B.tf4_segment_amax(slot[s], out=amax[i])
                B.tf4_quantize_capture(slot[s], guidance=i >= first_deep, amax_in=amax[i], out=recs[i])
            else:
                B.tf4_quantize_guided(slot[s], recs[first_deep + i], out=gcodes[i])
            free[s].record(comp)
            done[t].record(comp)
            with torch.cuda.stream(out_stream):
                out_stream.wait_event(done[t])
                if kind == "cap":
                    hc[i].copy_(recs[i].codes, non_blocking=True)
                    hs[i].copy_(recs[i].scales.view(-1), non_blocking=True)
                    hst[i:i + 1].copy_(recs[i].s_t, non_blocking=True)
                    if i >= first_deep:
                        hb[i - first_deep].copy_(recs[i].bits, non_blocking=True)
                else:
                    hg[i].copy_(gcodes[i], non_blocking=True)
        comp.wait_stream(out_stream)

    for _ in range(1):
        e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(comp)
    for _ in range(args.e2e_steps):
        e2e_step()
    t1.record(comp)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(t0.elapsed_time(t1) / args.e2e_steps, world, dev)
    bytes_step, _ = step_bytes(args)
    return dict(value=round(world * bytes_step / (ms * 1e-3) / 1e9, 2), unit="GB/s", ms_per_step=round(ms, 2),
                h2d_bytes_per_step=in_bytes, d2h_bytes_per_step=out_bytes, steps=args.e2e_steps,
                layers_per_rank=L, deep_layers_per_rank=D,
                overlap="double-buffered H2D on a copy stream, D2H on a third stream")


# ---------------------------------------------------------- CPU oracle arm
def oracle_sample_step(args, rows, xs_host, xts_host):
    import oracle as O

    L, D = args.layers, args.deep
    first_deep = L - D
    recs = []
    for i in range(L):
        recs.append(O.quantize(xs_host[i], O.NVFP4, O.RTN, bits=i >= first_deep))
    for j in range(D):
        r = recs[first_deep + j]
        O.quantize_guided(xts_host[j], r["scales"], r["bits"], O.NVFP4, rec_s_t=r["s_t"])


def sample_host(args, rows):
    """The first `rows` rows of every layer (and of the perturbed copies), as
    bf16 bit patterns on the host."""
    from fp4_block_scaled_quantizer_b200 import workloads as W

    dev = "cuda" if torch.cuda.is_available() else "cpu"
    xs, xts = [], []
    for layer in range(args.layers):
        x = W.layer_stack_layer(layer, dev, rows=args.rows, cols=args.cols)
        xs.append(W.bf16_bits(x[:rows].contiguous()))
        if layer >= args.layers - args.deep:
            xts.append(W.bf16_bits(W.perturb(x, 1000 + layer, rel=args.train_rel)[:rows].contiguous()))
        del x
    return xs, xts


def cpu_baseline(args, rows):
    """The oracle on a row sample of the workload: on every host core (one
    spawned process per layer task) and, for reference, on one core."""
    import oracle as O
    from oracle.pool import OraclePool

    O.lib()
    xs, xts = sample_host(args, rows)
    t = time.perf_counter()
    oracle_sample_step(args, rows, xs, xts)
    dt1 = time.perf_counter() - t
    b1, _ = step_bytes(argparse.Namespace(**{**vars(args), "rows": rows}))
    rows_mc = rows * args.cpu_mc_factor
    xs, xts = sample_host(args, rows_mc)
    pool = OraclePool()
    try:
        t = time.perf_counter()
        pool.run(xs, xts, args.layers - args.deep)
        dtm = time.perf_counter() - t
    finally:
        pool.close()
    bm, _ = step_bytes(argparse.Namespace(**{**vars(args), "rows": rows_mc}))
    return dict(value=round(bm / dtm / 1e9, 4), unit="GB/s", cores=pool.workers, kind="oracle",
                sample=f"first {rows_mc} of {args.rows} rows of each of the {args.layers} layers "
                       f"(capture) and of the {args.deep} perturbed deep layers (guided), one process per "
                       f"layer on {pool.workers} host cores, {dtm:.1f} s",
                value_1core=round(b1 / dt1 / 1e9, 4),
                sample_1core=f"first {rows} rows of each layer, single-threaded, {dt1:.1f} s")


def run_reference(args, world, rank):
    if rank != 0:
        return None
    import oracle as O
    from oracle.pool import OraclePool

    O.lib()
    rows = args.ref_rows
    xs, xts = sample_host(args, rows)
    pool = OraclePool()
    try:
        for _ in range(args.warmup):
            pool.run(xs, xts, args.layers - args.deep)
        t = time.perf_counter()
        for _ in range(args.steps):
            pool.run(xs, xts, args.layers - args.deep)
        dt = (time.perf_counter() - t) / args.steps
    finally:
        pool.close()
    sample_args = argparse.Namespace(**{**vars(args), "rows": rows})
    b, _ = step_bytes(sample_args)
    v = round(b / dt / 1e9, 4)
    sample = (f"first {rows} of {args.rows} rows of each of the {args.layers} layers (capture) and of the "
              f"{args.deep} perturbed deep layers (guided) per step, one process per layer on {pool.workers} "
              f"host cores")
    return dict(impl="reference", metric=METRIC, value=v, unit="GB/s", n_gpus=world, steps=args.steps,
                warmup=args.warmup, ms_per_step=round(dt * 1e3, 2), higher_is_better=True, scaling="weak",
                vs_baseline=None, dtype="f64", data="synthetic",
                config=dict(workload=f"layer_stack: {args.layers} layers x {args.rows}x{args.cols} bf16, "
                                     f"NVFP4 capture + guided (row sample)", layers=args.layers,
                            rows=args.rows, cols=args.cols, format="NVFP4"),
                cpu_baseline=dict(value=v, unit="GB/s", cores=pool.workers, kind="oracle", sample=sample),
                e2e=dict(value=v, unit="GB/s", h2d_bytes_per_step=0, d2h_bytes_per_step=0))


# ------------------------------------------------------------------ suite
# algorithmic bytes per element of each call (reads the definition forces on
# a tensor larger than on-chip memory, plus the writes)
CALL_BYTES = {
    ("nvfp4", "rtn"): 4.5625, ("nvfp4", "sr"): 4.5625, ("nvfp4", "capture"): 4.6875,
    ("nvfp4", "guided"): 2.6875, ("nvfp4", "dequant"): 4.5625, ("nvfp4", "amax"): 2.0,
    ("mxfp4", "rtn"): 2.53125, ("mxfp4", "sr"): 2.53125, ("mxfp4", "capture"): 2.65625,
    ("mxfp4", "guided"): 2.65625, ("mxfp4", "dequant"): 4.53125,
    ("any", "pack"): 0.625, ("any", "unpack"): 1.125,
    ("nvfp4", "guided_fq_f32"): 6.1875, ("nvfp4", "guided_fq_bf16"): 4.1875,
    ("mxfp4", "guided_fq_f32"): 6.15625, ("mxfp4", "guided_fq_bf16"): 4.15625,
    ("nvfp4", "mismatch"): 2.5625, ("mxfp4", "mismatch"): 2.53125,
    # a stack of layers captured with guidance kept for the deeper half
    ("nvfp4", "capture_stack_half_kept"): 4.625, ("mxfp4", "capture_stack_half_kept"): 2.59375,
}
# the uniform grid uses NVFP4's container: same bytes per element
CALL_BYTES.update({("ufp4", c): v for (f, c), v in list(CALL_BYTES.items()) if f == "nvfp4"})


def run_mismatch_by_layer(args):
    """For every layer of the stack: NVFP4 capture of the layer, its train
    copy drawn as the benchmark draws it (seed 1000 + layer, --train-rel),
    and the diagnostics' counts -- nearest-rounding mismatches, adjacent or
    farther, after guidance, and the corrections guidance makes toward the
    smaller and toward the larger codeword."""
    from fp4_block_scaled_quantizer_b200 import binding as B
    from fp4_block_scaled_quantizer_b200 import build as libbuild
    from fp4_block_scaled_quantizer_b200 import workloads as W

    libbuild.build()
    dev = torch.device("cuda", 0)
    out = []
    cnt = torch.zeros(B.MISMATCH_COUNTS, dtype=torch.int64, device=dev)
    for layer in range(args.layers):
        x = W.layer_stack_layer(layer, dev, rows=args.rows, cols=args.cols)
        q = B.tf4_quantize_capture(x)
        xt = W.perturb(x, 1000 + layer, rel=args.train_rel)
        c = [int(v) for v in B.tf4_mismatch_stats(xt, q, counts=cnt.zero_()).tolist()]
        out.append(dict(layer=layer, elements=x.numel(), mismatch=c[0], adjacent=c[1], far=c[2], after_guidance=c[3],
                        toward_smaller=c[4], toward_larger=c[5]))
        del x, q, xt
    return dict(workload=f"layer_stack: {args.layers} layers x {args.rows}x{args.cols} bf16, NVFP4 capture, "
                         f"train copy x (1 + {args.train_rel:g} N(0,1))", rows=out)


def run_suite(args):
    """Every call of the path on every workload, CUDA-event timed (3 warm-up
    calls, then the mean of 10 back-to-back calls, and the median and minimum
    of 20 calls timed one by one); GB/s from the algorithmic bytes above and
    the mean."""
    from fp4_block_scaled_quantizer_b200 import binding as B
    from fp4_block_scaled_quantizer_b200 import build as libbuild
    from fp4_block_scaled_quantizer_b200 import workloads as W

    libbuild.build()
    dev = torch.device("cuda", 0)
    peak, peak_kind = hbm_peak()
    rows_out = []

    def timed(fn, reps=10):
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(reps):
            fn()
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b) / reps * 1e3  # us

    def per_call(fn, reps=20, flush=None):
        """Median and minimum of reps calls, each between its own pair of
        events (optionally after `flush`, outside the events)."""
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            if flush is not None:
                flush()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        t = sorted(a.elapsed_time(b) * 1e3 for a, b in ev)
        return dict(us_median=round(0.5 * (t[(reps - 1) // 2] + t[reps // 2]), 2), us_min=round(t[0], 2))

    only = [tuple(f.split(":")) + ("", "", "") for f in (args.only or [])]

    def sel(workload, fmt="", call=""):
        """Is (workload, format, call) selected by --only (prefix match per field)?"""
        if not only:
            return True
        return any(workload.startswith(w) and (not fmt or not f or fmt == f) and (not call or not c or call == c)
                   for w, f, c, *_ in only)

    flush_buf = []

    def timed_cold(fn, reps=10):
        """Mean time of fn with L2 flushed before each rep (a 512 MiB memset,
        outside the events)."""
        if not flush_buf:
            flush_buf.append(torch.empty(512 << 20, dtype=torch.uint8, device=dev))
        for _ in range(3):
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
        for a, b in ev:
            flush_buf[0].zero_()
            a.record()
            fn()
            b.record()
        torch.cuda.synchronize()
        return sum(a.elapsed_time(b) for a, b in ev) / reps * 1e3

    def timed_graph(fn, reps=10):
        """Mean time of fn over reps calls captured in one CUDA graph and
        replayed (back to back on the GPU, no host launch pacing)."""
        for _ in range(3):
            fn()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(reps):
                fn()
        g.replay()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        g.replay()
        b.record()
        torch.cuda.synchronize()
        del g
        return a.elapsed_time(b) / reps * 1e3

    L2_BYTES = 126e6

    def run(workload, fmt, call, n, fn, cold=False, **extra):
        if not sel(workload, fmt, call):
            return
        flush = lambda: flush_buf[0].zero_()  # noqa: E731 (timed_cold allocates flush_buf first)
        if cold:
            record(workload, fmt, call, n, timed(fn), l2="warm", **per_call(fn), **extra)
            record(workload, fmt, call, n, timed_graph(fn), l2="warm, CUDA graph", **extra)
            record(workload, fmt, call, n, timed_cold(fn), l2="cold", **per_call(fn, flush=flush), **extra)
        elif CALL_BYTES[(fmt, call)] * n < 2 * L2_BYTES:
            # a working set that back-to-back calls would find in L2: flush before each call so that
            # the figure is an HBM one
            record(workload, fmt, call, n, timed_cold(fn), l2="cold (flushed: working set < 2 x L2)",
                   **per_call(fn, flush=flush), **extra)
        else:
            record(workload, fmt, call, n, timed(fn), **per_call(fn), **extra)

    def record(workload, fmt, call, n, us, l2=None, **extra):
        gbs = CALL_BYTES[(fmt, call)] * n / (us * 1e-6) / 1e9
        if l2:
            extra["l2"] = l2
        rows_out.append(dict(workload=workload, format=fmt, call=call, elements=n, us=round(us, 2),
                             gbs=round(gbs, 1), frac=round(gbs / peak, 4),
                             elements_per_s=round(n / (us * 1e-6), 1), **extra))

    def fq_and_diag(name, fmt, q, x, xt):
        n = x.numel()
        yf = torch.empty(x.shape, dtype=torch.float32, device=dev)
        yb = torch.empty(x.shape, dtype=torch.bfloat16, device=dev)
        run(name, fmt, "guided_fq_f32", n, lambda: B.tf4_guided_fake_quant(xt, q, out=yf))
        run(name, fmt, "guided_fq_bf16", n, lambda: B.tf4_guided_fake_quant(xt, q, out=yb))
        if not sel(name, fmt, "mismatch"):
            return
        cnt = torch.zeros(B.MISMATCH_COUNTS, dtype=torch.int64, device=dev)
        us = timed(lambda: B.tf4_mismatch_stats(xt, q, counts=cnt.zero_()))
        c = [int(v) for v in B.tf4_mismatch_stats(xt, q).tolist()]
        record(name, fmt, "mismatch", n, us, counts=dict(mismatch=c[0], adjacent=c[1], far=c[2], after_guidance=c[3],
                                                        toward_smaller=c[4], toward_larger=c[5]),
               adjacent_fraction=(round(c[1] / c[0], 6) if c[0] else None))

    def nv_calls(name, x, xt, seg=None, cold=False):
        n = x.numel()
        q = B.tf4_quantize_capture(x, seg_off=seg)
        amax = B.tf4_segment_amax(x, seg)
        g = torch.empty_like(q.codes)
        out = torch.empty(x.shape, dtype=torch.float32, device=dev)
        bits = torch.empty(n // 8, dtype=torch.uint8, device=dev)
        mant = torch.empty(n, dtype=torch.uint8, device=dev)
        qr = B.tf4_quantize_rtn(x, seg_off=seg)
        run(name, "nvfp4", "amax", n, lambda: B.tf4_segment_amax(x, seg, out=amax), cold=cold)
        run(name, "nvfp4", "rtn", n, lambda: B.tf4_quantize_rtn(x, seg_off=seg, out=qr), cold=cold)
        run(name, "nvfp4", "capture", n, lambda: B.tf4_quantize_capture(x, seg_off=seg, out=q), cold=cold)
        run(name, "nvfp4", "guided", n, lambda: B.tf4_quantize_guided(xt, q, out=g), cold=cold)
        run(name, "nvfp4", "sr", n, lambda: B.tf4_quantize_sr(x, 4, seg_off=seg, out=qr), cold=cold)
        run(name, "nvfp4", "dequant", n, lambda: B.tf4_dequantize(q, out=out), cold=cold)
        rows, cols = x.shape
        run(name, "any", "pack", n, lambda: B.tf4_pack_guidance(q.codes, rows, cols, out=bits), cold=cold)
        run(name, "any", "unpack", n, lambda: B.tf4_unpack_guidance(bits, rows, cols, out=mant), cold=cold)
        fq_and_diag(name, "nvfp4", q, x, xt)
        del q, g, out, bits, mant, qr

    def uf_calls(name, x, xt, seg=None, cold=False):
        n = x.numel()
        U = B.UFP4
        q = B.tf4_quantize_capture(x, fmt=U, seg_off=seg)
        g = torch.empty_like(q.codes)
        out = torch.empty(x.shape, dtype=torch.float32, device=dev)
        qr = B.tf4_quantize_rtn(x, fmt=U, seg_off=seg)
        run(name, "ufp4", "rtn", n, lambda: B.tf4_quantize_rtn(x, fmt=U, seg_off=seg, out=qr), cold=cold)
        run(name, "ufp4", "capture", n, lambda: B.tf4_quantize_capture(x, fmt=U, seg_off=seg, out=q), cold=cold)
        run(name, "ufp4", "guided", n, lambda: B.tf4_quantize_guided(xt, q, out=g), cold=cold)
        run(name, "ufp4", "sr", n, lambda: B.tf4_quantize_sr(x, 4, fmt=U, seg_off=seg, out=qr), cold=cold)
        run(name, "ufp4", "dequant", n, lambda: B.tf4_dequantize(q, out=out), cold=cold)
        fq_and_diag(name, "ufp4", q, x, xt)
        del q, g, out, qr

    def stack_calls(name, xs, fmt, fname):
        """A stack of layers captured (deeper half keeps guidance): one
        batched call against one capture call per layer."""
        L, keep = len(xs), len(xs) // 2
        n = sum(x.numel() for x in xs)
        ob = B.tf4_quantize_capture_batched(xs, fmt=fmt, keep=keep)
        per = [B.tf4_quantize_capture(x, fmt=fmt, guidance=i >= L - keep) for i, x in enumerate(xs)]

        def per_layer():
            for i, x in enumerate(xs):
                B.tf4_quantize_capture(x, fmt=fmt, guidance=i >= L - keep, out=per[i])
        run(name, fname, "capture_stack_half_kept", n, per_layer, launch="per_layer")
        run(name, fname, "capture_stack_half_kept", n,
            lambda: B.tf4_quantize_capture_batched(xs, fmt=fmt, keep=keep, out=ob), launch="batched")
        del ob, per

    def mx_calls(name, x, xt, cold=False):
        if x.shape[1] % 32:
            return
        n = x.numel()
        q = B.tf4_quantize_capture(x, fmt=B.MXFP4)
        g = torch.empty_like(q.codes)
        out = torch.empty(x.shape, dtype=torch.float32, device=dev)
        qr = B.tf4_quantize_rtn(x, fmt=B.MXFP4)
        run(name, "mxfp4", "rtn", n, lambda: B.tf4_quantize_rtn(x, fmt=B.MXFP4, out=qr), cold=cold)
        run(name, "mxfp4", "capture", n, lambda: B.tf4_quantize_capture(x, fmt=B.MXFP4, out=q), cold=cold)
        run(name, "mxfp4", "guided", n, lambda: B.tf4_quantize_guided(xt, q, out=g), cold=cold)
        run(name, "mxfp4", "sr", n, lambda: B.tf4_quantize_sr(x, 4, fmt=B.MXFP4, out=qr), cold=cold)
        run(name, "mxfp4", "dequant", n, lambda: B.tf4_dequantize(q, out=out), cold=cold)
        fq_and_diag(name, "mxfp4", q, x, xt)
        del q, g, out, qr

    name = "reference streams (torch, 1 GiB)"
    if sel(name):
        # the measured-peak cross-check, not the library: a device copy
        buf = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
        src = torch.empty(1 << 30, dtype=torch.uint8, device=dev)
        for call, fn, bpb in (("copy (read + write)", lambda: buf.copy_(src), 2.0),):
            us = timed(fn)
            gbs = bpb * (1 << 30) / (us * 1e-6) / 1e9
            rows_out.append(dict(workload=name, format="-", call=call, elements=1 << 30, us=round(us, 2),
                                 gbs=round(gbs, 1), frac=round(gbs / peak, 4), elements_per_s=None))
        # the host link that bounds the end-to-end figure: pinned host <-> device copies (frac: none, not HBM)
        hsrc = torch.empty(1 << 30, dtype=torch.uint8).pin_memory()
        hdst = torch.empty(1 << 30, dtype=torch.uint8).pin_memory()
        side = torch.cuda.Stream(dev)

        def both():
            side.wait_stream(torch.cuda.current_stream(dev))
            with torch.cuda.stream(side):
                hdst.copy_(src, non_blocking=True)
            buf.copy_(hsrc, non_blocking=True)
            torch.cuda.current_stream(dev).wait_stream(side)

        for call, fn, bpb in (("pinned host -> device copy", lambda: buf.copy_(hsrc, non_blocking=True), 1.0),
                              ("device -> pinned host copy", lambda: hdst.copy_(src, non_blocking=True), 1.0),
                              ("both directions at once (2 x 1 GiB)", both, 2.0)):
            us = timed(fn, reps=5)
            gbs = bpb * (1 << 30) / (us * 1e-6) / 1e9
            rows_out.append(dict(workload=name, format="-", call=call, elements=1 << 30, us=round(us, 2),
                                 gbs=round(gbs, 1), frac=None, elements_per_s=None))
        del buf, src, hsrc, hdst
    name = "activation_outliers 4096x2048"
    if sel(name):
        w = W.activation_outliers(dev)
        nv_calls(name, w["x"], w["x_train"], cold=True)
        mx_calls(name, w["x"], w["x_train"], cold=True)
        uf_calls(name, w["x"], w["x_train"], cold=True)
        del w
    name = "40 layers of 4096x2048"
    if sel(name):
        xs = [W.random_bf16((4096, 2048), seed=300 + i, device=dev, outlier_frac=0.001) for i in range(40)]
        stack_calls(name, xs, B.NVFP4, "nvfp4")
        stack_calls(name, xs, B.MXFP4, "mxfp4")
        del xs
    name = "layer_stack layer 65536x4096"
    if sel(name):
        x = W.layer_stack_layer(20, dev)
        xt = W.perturb(x, 1020)
        nv_calls(name, x, xt)
        mx_calls(name, x, xt)
        uf_calls(name, x, xt)
        del x, xt
    name = "layer_stack layer 65536x4096, train copy x (1 + rel N(0,1))"
    if sel(name):
        # guided rounding, fused fake-quant and diagnostics at growing train/rollout mismatch rates
        x = W.layer_stack_layer(20, dev)
        n = x.numel()
        for fmt, fname in ((B.NVFP4, "nvfp4"), (B.MXFP4, "mxfp4"), (B.UFP4, "ufp4")):
            q = B.tf4_quantize_capture(x, fmt=fmt)
            g = torch.empty_like(q.codes)
            yf = torch.empty(x.shape, dtype=torch.float32, device=dev)
            yb = torch.empty(x.shape, dtype=torch.bfloat16, device=dev)
            cnt = torch.zeros(B.MISMATCH_COUNTS, dtype=torch.int64, device=dev)
            for rel in (0.0, 1e-3, 1e-2, 5e-2, None):
                xt = (W.perturb(x, 1020, rel=rel) if rel else x) if rel is not None else \
                    W.layer_stack_layer(21, dev)
                frac = int(B.tf4_mismatch_stats(xt, q)[0]) / n
                tag = dict(train_rel=("unrelated tensor" if rel is None else rel), mismatch_fraction=round(frac, 6))
                run(name, fname, "guided", n, lambda: B.tf4_quantize_guided(xt, q, out=g), **tag)
                run(name, fname, "guided_fq_f32", n, lambda: B.tf4_guided_fake_quant(xt, q, out=yf), **tag)
                run(name, fname, "guided_fq_bf16", n, lambda: B.tf4_guided_fake_quant(xt, q, out=yb), **tag)
                run(name, fname, "mismatch", n, lambda: B.tf4_mismatch_stats(xt, q, counts=cnt.zero_()), **tag)
                del xt
            del q, g, yf, yb
        del x
    name = "moe_dispatch 262144x2048, 128 experts"
    if sel(name):
        w = W.moe_dispatch(dev)
        nv_calls(name, w["x"], w["x_train"], seg=w["seg_off"])
        uf_calls(name, w["x"], w["x_train"], seg=w["seg_off"])
        del w
    name = "weights 8192x28672"
    if sel(name):
        x = W.weights(dev)
        nv_calls(name, x, W.perturb(x, 44))
        mx_calls(name, x, W.perturb(x, 44))
        uf_calls(name, x, W.perturb(x, 44))
        del x
    name = "kv_cache K 1048576x128"
    if sel(name):
        w = W.kv_cache(dev)
        nv_calls(name, w["k"], w["k_train"])
        mx_calls(name, w["k"], w["k_train"])
        uf_calls(name, w["k"], w["k_train"])
        del w
    torch.cuda.empty_cache()
    return dict(peak_gbs=peak, peak_kind=peak_kind, rows=rows_out)


def main():
    args = parse()
    if args.suite:
        print(json.dumps(run_suite(args)), flush=True)
        return
    if args.mismatch_by_layer:
        print(json.dumps(run_mismatch_by_layer(args)), flush=True)
        return
    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        out = run_reference(args, world, rank)
        if out is not None:
            print(json.dumps(out), flush=True)
        return
    world, rank, local = dist_setup(args)
    try:
        out = run_ours(args, world, rank, local)
        if rank == 0:
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
