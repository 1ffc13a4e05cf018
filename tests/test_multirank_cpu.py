"""The multi-rank host logic of bench.py on CPU: two `gloo` ranks.

bench.py runs one replica of the whole hot path per GPU (the path has no
exchange step, so there is no data-path collective).  What spans ranks is host
logic only: each rank draws its own sequence, the ranks meet at barriers
around the timed region, the job's time is the maximum over ranks, and the
reported rate counts the units every rank processed.  These tests run that
logic in two spawned processes over the gloo backend.
"""

import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    from hierarchical_routed_sparse_hga_b200 import synth
    r, wsz, local = bench.dist_env()
    dist.init_process_group("gloo", rank=r, world_size=wsz,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w0 = synth.workloads()["qwen3_fwdbwd_16k"]
        w = bench.rank_workload(w0, r)
        bench.barrier(wsz)
        # a rank-dependent "elapsed time": the job's time is the slowest rank's
        ms = 10.0 + 5.0 * r
        ms_max = bench.max_over_ranks(ms, wsz)
        bench.barrier(wsz)
        rate = bench.job_throughput(1000.0, 4, wsz, ms_max)
        out[r] = (r, wsz, local, w.seed, w.ctx_len, w.seg_len, ms_max, rate)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_share_timing_and_count_all_units():
    import torch.multiprocessing as mp
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    with ctx.Manager() as mgr:
        out = mgr.dict()
        procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(120)
        codes = [p.exitcode for p in procs]
        for p in procs:
            if p.is_alive():
                p.kill()
        assert codes == [0, 0], codes
        res = dict(out)
    assert sorted(res) == [0, 1]
    (r0, w0, l0, seed0, ctx0, seg0, max0, rate0) = res[0]
    (r1, w1, l1, seed1, ctx1, seg1, max1, rate1) = res[1]
    assert (w0, w1, l0, l1) == (2, 2, 0, 1)
    # every rank: same shapes, its own sequence
    assert (ctx0, seg0) == (ctx1, seg1) and seed0 != seed1
    # the max over ranks is the slowest rank's time, seen identically by all
    assert max0 == max1 == 15.0
    # both ranks' units over the slowest time: 2 x 1000 x 4 / 15 ms
    assert rate0 == rate1 == pytest.approx(2 * 1000 * 4 / 0.015)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5
    bench.barrier(1)  # no process group: a no-op
    assert bench.job_throughput(2048, 30, 1, 60.0) == pytest.approx(2048 * 30 / 0.06)


def test_reference_arm_runs_on_rank_zero_only(capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload = "qwen3_fwdbwd_16k"
        steps = 1
        warmup = 3

    bench.run_reference(Args(), rank=1, world=2)   # returns at once, no work, no output
    assert capsys.readouterr().out == ""
