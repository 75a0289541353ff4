"""Runs the oracle on several layers at once, one process per layer task
(spawned processes: safe after the parent has used a GPU).

TEST INFRASTRUCTURE ONLY: the multi-core CPU baseline and reference leg of
bench.py.  Each task is the oracle's own capture of one layer and, for a
deep layer, its guided quantization of the perturbed copy -- the same calls
the single-threaded baseline makes, unchanged, just spread over cores.
"""
import concurrent.futures as cf
import multiprocessing as mp
import os
import time

from . import NVFP4, RTN, lib, quantize, quantize_guided


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

    def close(self):
        self.ex.shutdown()
