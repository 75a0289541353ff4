"""Multi-rank logic on CPU with gloo (world size 2): the all-reduce MAX
exchange of the row-sharded NVFP4 path, and the bench's max-over-ranks
timing.  The CUDA calls are replaced by CPU stand-ins built on the oracle,
so only the exchange and bookkeeping are under test."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _init(rank, world, port):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))


def _sharded_worker(rank, world, port, q):
    import oracle as O
    from fp4_block_scaled_quantizer_b200 import sharded, workloads as W

    try:
        _init(rank, world, port)
        rows, cols = 60, 256
        x = W.bf16_bits(W.random_bf16((rows, cols), seed=3, outlier_frac=0.02))
        seg = [0, 10, 10, 45, 60]
        b, e = sharded.shard_rows(rows, world, rank)
        xs = x[b:e]
        seg_s = sharded.shard_segments(seg, b, e)

        def fake_amax(xt, so):
            a, _ = O.segment_amax(xt.numpy().view(np.uint16), so)
            return torch.from_numpy(a.copy())

        def fake_capture(xt, seg_off=None, guidance=True, amax_in=None):
            st = np.array([O.nvfp4_tensor_scale(float(v)) for v in amax_in.numpy()], np.float32)
            return O.quantize(xt.numpy().view(np.uint16), O.NVFP4, O.RTN, seg_off=seg_off, bits=guidance, s_t=st)

        sharded._ops["segment_amax"] = fake_amax
        sharded._ops["quantize_capture"] = fake_capture
        r = sharded.sharded_capture(torch.from_numpy(xs.view(np.int16).copy()), seg_off=seg_s)
        full = O.quantize(x, O.NVFP4, O.RTN, seg_off=seg, bits=True)
        ok = (np.array_equal(r["codes"], full["codes"][b * cols // 2:e * cols // 2])
              and np.array_equal(r["scales"], full["scales"][b * cols // 16:e * cols // 16])
              and np.array_equal(r["bits"], full["bits"][b * cols // 8:e * cols // 8])
              and np.array_equal(r["s_t"], full["s_t"]))
        q.put((rank, bool(ok)))
    except Exception as ex:  # report instead of hanging the peer
        q.put((rank, repr(ex)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _timing_worker(rank, world, port, q):
    import bench

    try:
        _init(rank, world, port)
        ms = bench.max_over_ranks(10.0 + 5.0 * rank, world, "cpu")
        q.put((rank, ms))
    except Exception as ex:
        q.put((rank, repr(ex)))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
    return out


def test_sharded_capture_equals_unsharded():
    """Two ranks, rows split, ragged segments (one empty, one spanning both
    shards): after the all-reduce MAX each rank's capture equals its rows of
    the whole-tensor capture, s_t included."""
    out = _run(_sharded_worker)
    assert out == {0: True, 1: True}, out


def test_bench_time_is_max_over_ranks():
    out = _run(_timing_worker)
    assert out == {0: 15.0, 1: 15.0}, out


def test_shard_helpers():
    from fp4_block_scaled_quantizer_b200 import sharded

    spans = [sharded.shard_rows(10, 3, r) for r in range(3)]
    assert spans == [(0, 4), (4, 7), (7, 10)]
    assert sharded.shard_segments([0, 2, 2, 6, 10], 4, 7) == [0, 0, 0, 2, 3]
