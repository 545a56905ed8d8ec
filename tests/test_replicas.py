"""Multi-process (gloo, world size 2, CPU) tests of the host logic that
bench.py uses on N GPUs: per-rank workloads and max-over-ranks timing."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from sparse_attention_fp4_kv_b200 import replicas, synth
        w = synth.WORKLOADS["decoder_stack20_b4_ctx1m"]
        rw = replicas.rank_workload(w, rank, world)
        times = [10.0 + rank, 3.0 - rank]          # rank-dependent timings (ms)
        worst = replicas.slowest(times)
        rate = replicas.aggregate_rate(rw.n_layers, world, worst[0])
        q.put((rank, rw.seed, rw.B, rw.ctx, worst, rate))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_by_seed_and_time_by_the_slowest():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (r0, seed0, b0, c0, worst0, rate0), (r1, seed1, b1, c1, worst1, rate1) = res
    assert seed0 != seed1 and (b0, c0) == (b1, c1)     # own sequences, same shapes
    assert worst0 == worst1 == [11.0, 3.0]             # max over ranks, element-wise
    assert rate0 == rate1 == pytest.approx(2 * 20 / 11e-3)


def test_single_process_is_a_no_op():
    from sparse_attention_fp4_kv_b200 import replicas, synth
    w = synth.WORKLOADS["decoder_stack20_b4_ctx1m"]
    assert replicas.rank_workload(w, 0, 1) is w
    assert replicas.slowest([1.5, 2.5]) == [1.5, 2.5]
    assert replicas.aggregate_rate(20, 1, 2.0) == pytest.approx(10000.0)
