"""Multi-process (gloo, world size 2, CPU) tests of the host logic that
bench.py uses on N GPUs: per-rank workloads and max-over-ranks timing; and the
bench's clock record."""
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


def test_clock_summary_of_sampled_lines():
    """The bench's clock record: median SM clock under load, the max clock and
    every throttle reason reported active (from nvidia-smi CSV lines)."""
    import importlib.util
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    spec = importlib.util.spec_from_file_location("bench_mod", os.path.join(root, "bench.py"))
    bench = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(bench)
    lines = "\n".join([
        "0, 1965, 1965, 812.4, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "0, 1920, 1965, 998.1, 0x0000000000000004, Not Active, Not Active, Not Active, Active",
        "0, 1965, 1965, 905.0, 0x0000000000000000, Not Active, Not Active, Not Active, Not Active",
        "garbage line",
        "0, [N/A], 1965, 0, 0x0, Not Active, Not Active, Not Active, Not Active",
    ])
    c = bench.summarize_clocks(lines)
    assert c == {"sm_mhz": 1965.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}
    hot = "0, 1400, 1965, 1000, 0x48, Active, Active, Not Active, Not Active"
    assert bench.summarize_clocks(hot)["reasons"] == ["hw_slowdown", "hw_thermal_slowdown"]
    assert bench.summarize_clocks("")["samples"] == 0
    # the sampler's stop(): ends the sampling process, reads and removes its file
    import tempfile

    class _Proc:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    cs = bench.ClockSampler.__new__(bench.ClockSampler)
    cs.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
    cs.file.write(lines + "\n")
    cs.proc = _Proc()
    name = cs.file.name
    assert cs.stop() == c and not os.path.exists(name)


def test_reference_arm_runs_on_host_inputs_without_the_cuda_library():
    """bench.py --impl reference draws its inputs with the seeded generators on
    the host and runs only the oracle: libcsa2 is never imported or loaded."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    code = ("import sys, json; sys.argv = ['bench.py', '--impl', 'reference', '--workload', "
            "'full_b1_ctx4k', '--steps', '3', '--warmup', '3']; sys.path.insert(0, %r); import bench; "
            "bench.main(); maps = open('/proc/self/maps').read(); "
            "print(json.dumps({'binding': 'sparse_attention_fp4_kv_b200.binding' in sys.modules, "
            "'libcsa2': 'libcsa2.so' in maps, 'omp': 'libcsa2_oracle_omp.so' in maps}))" % root)
    r = subprocess.run([sys.executable, "-c", code], cwd=root, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    line, loaded = lines[0], lines[-1]
    assert loaded == {"binding": False, "libcsa2": False, "omp": True}
    assert line["impl"] == "reference" and line["steps"] == 3 and line["warmup"] == 3
    assert line["config"]["workload"] == "full_b1_ctx4k" and line["unit"] == "layer-steps/s"
    assert line["cpu_baseline"]["cores"] >= 1 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["value"] > 0
    # a 4K-context step is short enough that every step covers the whole batch
    assert "1 of 1 sequences per step" in line["cpu_baseline"]["sample"]
