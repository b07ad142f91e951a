"""Host logic of bench.py that runs without a GPU: the multi-rank timing reduction
(max over ranks) and barrier on world_size-2 gloo process groups, the byte model,
and the clock-sample parser."""
import os
import socket
import subprocess
import sys
import textwrap

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_max_over_ranks_with_two_gloo_ranks(tmp_path):
    script = tmp_path / "ranks.py"
    script.write_text(textwrap.dedent(f"""
        import os, sys
        sys.path.insert(0, {ROOT!r})
        import bench
        world, rank, local = bench.dist_setup()
        assert world == 2
        bench.barrier(world)
        m = bench.max_over_ranks(10.0 + 5.0 * rank, world)
        assert m == 15.0, m
        print(f"rank {{rank}} ok {{m}}")
        import torch.distributed as dist
        dist.destroy_process_group()
    """))
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE="2", MASTER_ADDR="127.0.0.1",
                   MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.STDOUT, text=True))
    outs = [p.communicate(timeout=120)[0] for p in procs]
    for r, (p, o) in enumerate(zip(procs, outs)):
        assert p.returncode == 0, o
        assert f"rank {r} ok 15.0" in o


def test_single_rank_reduction_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_step_bytes_grows_with_instances_and_views():
    sys.path.insert(0, ROOT)
    import bench
    one = bench.step_bytes(1_000_000, 3, [(10_000_000, 900_000, 2)], 8160, 1920 * 1080)
    two = bench.step_bytes(1_000_000, 3, [(10_000_000, 900_000, 2)] * 2, 8160, 1920 * 1080)
    more_k = bench.step_bytes(1_000_000, 3, [(20_000_000, 900_000, 2)], 8160, 1920 * 1080)
    assert 0 < one < two < 2 * one and more_k > one


def test_clock_parser(tmp_path):
    sys.path.insert(0, ROOT)
    import bench
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    f = open(tmp_path / "c.csv", "w+")
    f.write("0, 1965, 1965, 700.1, 0x0, Not Active, Not Active, Not Active, Not Active\n"
            "0, 1800, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n"
            "0, 1900, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
    f.flush()
    c.f = f
    c.p = None
    r = bench.ClockSampler.stop(c)
    assert r["reasons"] == ["nvidia-smi unavailable"]

    class P:
        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0
    c.p = P()
    r = bench.ClockSampler.stop(c)
    assert r["sm_mhz"] == 1900.0 and r["sm_max_mhz"] == 1965.0 and r["reasons"] == ["sw_power_cap"]
    assert r["samples"] == 3


def test_raster_roofline_counts_the_method_work():
    """achieved = (14 per traversed pair + 46 per blended pair) / time against the measured
    float32 peak; the special-function rate counts ex2 + rcp per evaluated pair."""
    sys.path.insert(0, ROOT)
    import bench
    work = {"traversed_pairs": 1e9, "fwd_evaluated_pairs": 2e9, "fwd_blended_pairs": 4e8,
            "bwd_evaluated_pairs": 1.5e9, "bwd_gradient_pairs": 4e8}
    alu = {"fp32_tflops": 70.0, "ex2_tops": 4.0, "source": "test"}
    r = bench.raster_roofline("raster_bwd", 2.0, work, alu)
    assert r["bound"] == "alu" and r["unit"] == "TFLOP/s" and r["peak"] == 70.0
    assert abs(r["achieved"] - (14 * 1e9 + 46 * 4e8) / 2e-3 / 1e12) < 1e-9
    assert abs(r["frac"] - r["achieved"] / 70.0) < 1e-12
    assert abs(r["sfu"]["achieved_tops"] - 2 * 1.5e9 / 2e-3 / 1e12) < 1e-9
    f = bench.raster_roofline("raster_fwd", 1.0, work, alu)
    assert abs(f["achieved"] - (14 * 1e9 + 8 * 4e8) / 1e-3 / 1e12) < 1e-9
    assert abs(f["sfu"]["achieved_tops"] - 2e9 / 1e-3 / 1e12) < 1e-9
    # with the counted forward's fifth counter the forward charges the pairs its
    # per-pixel loop visits (up to each pixel's stop); the reverse pass keeps sum(n_contrib)
    work["fwd_visited_pairs"] = 1.25e9
    f = bench.raster_roofline("raster_fwd", 1.0, work, alu)
    assert abs(f["achieved"] - (14 * 1.25e9 + 8 * 4e8) / 1e-3 / 1e12) < 1e-9
    assert abs(f["evaluated_over_visited"] - 2e9 / 1.25e9) < 1e-12
    r = bench.raster_roofline("raster_bwd", 2.0, work, alu)
    assert abs(r["achieved"] - (14 * 1e9 + 46 * 4e8) / 2e-3 / 1e12) < 1e-9


def test_cpu_baseline_times_all_cores_and_one_thread():
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    wl = bench.make_workload("tiny")
    before = oracle.set_threads(0)
    cb = bench.cpu_baseline(bench.cpu_oracle_sample, wl, 0.25, "iterations/s")
    assert oracle.set_threads(0) == before          # the thread count is restored
    assert cb["kind"] == "oracle" and cb["cores"] == before and cb["host_cpu_count"] == os.cpu_count()
    assert cb["single_thread"]["cores"] == 1 and cb["value"] > 0 and cb["single_thread"]["value"] > 0
