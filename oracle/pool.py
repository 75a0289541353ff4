"""Runs the oracle on several layers at once, one process per layer task
(spawned processes: safe after the parent has used a GPU).

TEST INFRASTRUCTURE ONLY: the multi-core CPU baseline and reference leg of
bench.py, and the full-size parity tests.  Each task is the oracle's own
capture of one layer and, for a deep layer, its guided quantization of the
perturbed copy -- the same calls the single-threaded baseline makes,
unchanged, just spread over cores -- or one of the oracle's tensor
functions on a row range of a larger tensor (map_rows).
"""
import concurrent.futures as cf
import multiprocessing as mp
import os
import time

from . import NVFP4, RTN, dequantize, lib, mismatch_stats, quantize, quantize_guided


def _layer_task(task):
    """One layer: capture (+ guided for a deep layer).  Returns a digest of
    the outputs (sums of the code and scale bytes) so a caller can check the
    work was done."""
    x, xt = task
    lib()
    r = quantize(x, NVFP4, RTN, bits=xt is not None)
    digest = [int(r["codes"].sum()), int(r["scales"].sum())]
    if xt is not None:
        g, _ = quantize_guided(xt, r["scales"], r["bits"], NVFP4, rec_s_t=r["s_t"])
        digest.append(int(g.sum()))
    return digest


def _ready(_):
    lib()
    time.sleep(0.5)  # keeps this process busy so that every worker gets started
    return os.getpid()


def _rows_task(task):
    """One row range of a larger tensor, for the full-size parity tests:
    `kind` is one of the oracle's own tensor functions, called unchanged on
    the range (segment offsets already made relative to it, tensor scales
    given)."""
    kind, kw = task
    lib()
    fmt, seg, s_t = kw["fmt"], kw.get("seg"), kw.get("s_t")
    if kind == "capture":
        r = quantize(kw["x"], fmt, RTN, seg_off=seg, bits=True, s_t=s_t)
        return r["codes"], r["scales"], r["bits"], r["status"]
    if kind == "guided":
        return quantize_guided(kw["x"], kw["scales"], kw["bits"], fmt, rec_s_t=s_t, seg_off=seg)
    if kind == "dequant":
        rows, cols = kw["shape"]
        return dequantize(kw["codes"], kw["scales"], rows, cols, fmt, s_t=s_t, seg_off=seg)
    if kind == "mismatch":
        return mismatch_stats(kw["x"], kw["scales"], kw["codes"], fmt, rec_s_t=s_t, seg_off=seg)
    raise ValueError(kind)


class OraclePool:
    """A pool of `workers` spawned processes; run() does one step (every
    layer's capture, and the guided pass of the deep layers) across them."""

    def __init__(self, workers=None):
        self.workers = workers or max(1, min(os.cpu_count() or 1, 64))
        self.ex = cf.ProcessPoolExecutor(max_workers=self.workers, mp_context=mp.get_context("spawn"))
        list(self.ex.map(_ready, range(self.workers)))  # start every process, load the library

    def run(self, xs, xts, first_deep):
        tasks = [(x, xts[i - first_deep] if i >= first_deep else None) for i, x in enumerate(xs)]
        return list(self.ex.map(_layer_task, tasks))

    def map_rows(self, kind, tasks):
        """The oracle's `kind` on each row-range task (see _rows_task), in order."""
        return list(self.ex.map(_rows_task, [(kind, kw) for kw in tasks]))

    def close(self):
        self.ex.shutdown()
