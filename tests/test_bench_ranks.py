"""The bench's multi-rank plumbing on the CPU: two gloo ranks (the N > 1 path
shards with no data-path collective; the only collectives are the barrier and
the max-over-ranks reduction of the timings)."""
import os
import socket

import pytest
import torch.multiprocessing as mp

import bench


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=__import__("datetime").timedelta(seconds=60))
    try:
        # rank r measured (10 + r, 4 + 2 r, 6 - r) ms: the job time is the max per entry
        mine = [10.0 + rank, 4.0 + 2.0 * rank, 6.0 - rank]
        dist.barrier()
        got = bench.reduce_max(mine, world, dist, "cpu")
        q.put((rank, got, bench.job_gbps(1_000_000, world, got[0])))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max_and_count_all_bytes():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = [q.get(timeout=120) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, gbps in results:
        assert got == [11.0, 6.0, 6.0]                   # max over the two ranks, per entry
        assert gbps == pytest.approx(2 * 1e6 / 11.0 / 1e6)  # bytes of both ranks / slowest time


def test_single_rank_is_a_no_op():
    assert bench.reduce_max([3.0, 1.5], 1, None, "cpu") == [3.0, 1.5]
    assert bench.job_gbps(2e9, 1, 4.0) == pytest.approx(500.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    # ranks other than 0 leave the reference arm at once, without work
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")

    class Args:
        steps, warmup, gpus = 1, 0, 2

    assert bench.run_reference(Args()) == 0


def test_smem_ceiling_arithmetic():
    # 32 x 10^9 symbols in 1 s at ~7.5 wavefronts per warp-symbol on 148 SMs at
    # 1965 MHz: ~7.5e9 wavefronts/s against 290.8e9
    got = bench.smem_ceiling(32_000_000_000, 1000.0, 1965.0, 148)
    wf = bench.DECODE_SMEM_WAVEFRONTS_PER_WARP_SYMBOL
    assert 7.4 < wf < 7.6
    assert got["bound"] == "smem" and got["peak"] == round(148 * 1965e6 / 1e9, 1)
    assert abs(got["achieved"] - wf) < 0.06
    assert abs(got["frac"] - wf / 290.82) < 1e-3
    assert bench.smem_ceiling(1, 1.0, None, 148) is None
