"""Host-side logic of the multi-GPU run (bench.py under torch.distributed), on CPU with two
gloo ranks: the path shards by lanes with no data exchange, so what N > 1 adds is a batch of
its own per rank, a max-over-ranks device time and one printing rank."""
import os
import socket
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import datetime

    import torch.distributed as dist

    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        res = {}
        # every rank sees the slowest rank's time
        res["max"] = bench.max_over_ranks(1.5 + rank, world, "cpu")
        w = bench.workload_for_rank("int4_2b", rank)
        res["shape"] = (w.d, w.H, w.hd, w.B, tuple(w.ctx), tuple(w.loops))
        res["seed"] = w.seed
        res["row0"] = float(w.h_rows(w.n_pre, 0, 0, 1)[0, 0])
        res["rate"] = bench.whole_job_rate(w.cached_positions_per_step(), 10, res["max"], world)

        # the reference arm does its work on rank 0 only: another rank returns at once
        class Args:
            workload, steps, warmup = "tiny_fp16", 1, 0
        if rank != 0:
            import io
            import contextlib
            buf = io.StringIO()
            with contextlib.redirect_stdout(buf):
                bench.run_reference(Args, rank, world)
            res["ref_out"] = buf.getvalue()
        dist.barrier()
        out.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0]["max"] == got[1]["max"] == 2.5
    assert got[0]["shape"] == got[1]["shape"]                     # same batch shape on every rank
    assert got[0]["seed"] != got[1]["seed"] and got[0]["row0"] != got[1]["row0"]  # independent data
    ranks_rate = got[0]["rate"]
    import bench
    w = bench.workload_for_rank("int4_2b", 0)
    assert ranks_rate == pytest.approx(2 * 10 * w.cached_positions_per_step() / 2.5e-3)
    assert got[1]["ref_out"] == ""
