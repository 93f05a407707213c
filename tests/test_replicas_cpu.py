"""Host logic of the multi-GPU bench path (replicas, no data-path collective), on CPU with gloo ranks.

Each rank runs its own replica on its own requests; the ranks only combine the timing: the job's
throughput is the tokens all ranks decoded divided by the slowest rank's time.
"""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import focus_synth as fs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = [12.5, 20.0, 7.0][rank]
        decoded = [32, 30, 31][rank]
        mx, tot = bench.reduce_over_ranks(elapsed, decoded, world, torch.device("cpu"))
        seed = bench.rank_seed(fs.SEEDS["tiny"], rank)
        case = fs.make_case("tiny", seed=seed)
        q.put((rank, mx, tot, bench.whole_job_rate(tot, mx), seed,
               tuple(case.batch["prefix_len"].tolist()), tuple(case.batch["block_tokens"].shape)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_replicas_combine_max_time_and_total_tokens(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want_max = max([12.5, 20.0, 7.0][:world])
    want_tot = sum([32, 30, 31][:world])
    for rank, mx, tot, rate, seed, plen, shape in res:
        assert mx == want_max and tot == want_tot
        assert rate == pytest.approx(want_tot / (want_max / 1e3))
    # every rank draws its own requests of the same shape
    assert len({r[4] for r in res}) == world
    assert len({r[6] for r in res}) == 1


def test_single_rank_needs_no_process_group():
    mx, tot = bench.reduce_over_ranks(3.0, 8, 1, torch.device("cpu"))
    assert (mx, tot) == (3.0, 8.0)
    assert bench.whole_job_rate(tot, mx) == pytest.approx(8 / 3e-3)
