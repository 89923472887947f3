"""The replica path of bench.py on CPU: two gloo ranks reduce their timings to
the max over ranks, whole-job throughput counts every rank's tokens, and the
reference arm runs on rank 0 only."""
import os
import socket
import subprocess
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_q):
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", init_method=f"tcp://127.0.0.1:{port}", rank=rank,
                            world_size=world)
    try:
        ms, e2e, kms = bench.reduce_max_over_ranks([1.0 + rank, 10.0 * rank, 3.0], world, "cpu")
        out_q.put((rank, ms, e2e, kms))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get() for _ in range(world))
    for rank, ms, e2e, kms in got:
        assert (ms, e2e, kms) == (2.0, 10.0, 3.0), rank


def test_job_throughput_counts_every_replica():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max_over_ranks([1.5, 2.5], 1, "cpu") == [1.5, 2.5]
    assert bench.job_tokens_per_s(1, 512, 1000.0) == pytest.approx(512.0)
    assert bench.job_tokens_per_s(4, 512, 1000.0) == pytest.approx(2048.0)


def test_reference_arm_runs_on_rank_zero_only():
    env = dict(os.environ, RANK="1", LOCAL_RANK="1", WORLD_SIZE="2")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "1", "--warmup", "3"], env=env, capture_output=True,
                         text=True, timeout=600)
    assert res.returncode == 0 and res.stdout.strip() == ""


def test_traffic_is_scaled_only_for_the_captured_kernel_and_workload():
    sys.path.insert(0, ROOT)
    import bench
    import json
    with open(bench.TRAFFIC_FILE) as f:
        rec = json.load(f)
    current = bench.kernel_sources_digest(rec["files"]) == rec["kernel_sources_sha256"]
    t, src = bench.dram_traffic(1e9, int(rec["workload"]))
    if current:
        assert t == pytest.approx(rec["ratio"] * 1e9) and src == rec["capture"]
    else:
        assert t is None and "kernel changed" in src
    other = (int(rec["workload"]) + 1) % 5
    t, src = bench.dram_traffic(1e9, other)
    assert t is None


def test_reference_arm_line_keeps_the_contract():
    """The reference arm (the oracle on the host cores) prints one JSON line
    with the keys of the bench contract, the same metric, unit and config as
    the GPU arm, and its own cpu_baseline and e2e objects."""
    import json
    sys.path.insert(0, ROOT)
    import bench
    import synth
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "LOCAL_RANK", "WORLD_SIZE")}
    res = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--steps", "2", "--warmup", "3", "--cpu-seconds", "1"], env=env,
                         capture_output=True, text=True, timeout=900)
    assert res.returncode == 0, res.stderr[-2000:]
    line = json.loads(res.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "impl", "cpu_baseline", "e2e"):
        assert key in line, key
    w = synth.WORKLOADS[1]
    assert line["impl"] == "reference" and line["metric"] == bench.METRIC
    assert line["unit"] == "tokens/s" and line["higher_is_better"] is True
    assert line["n_gpus"] == 1 and line["warmup"] == 3 and 1 <= line["steps"] <= 2
    assert line["config"] == bench.run_config(w, w.prompt_len, 2, 1, "dependency",
                                              synth.streamed_weight_bytes(w.model))
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["value"] == line["value"] > 0
    assert cb["unit"] == line["unit"] and cb["sample"]
    assert cb["prefill_s"] > 0 and cb["cpu"] and cb["host_cpus"] >= 1
    assert cb["cores"] == 1     # single-threaded, as the CPU baseline is planned
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"],
                           "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_algorithmic_bytes_agree_between_bench_and_the_counter_case():
    """bench.py and the counter-capture case count the same bytes for the same
    steps: every weight once per step (from the generator's tensor table), the
    K/V of positions 0..p read and position p written."""
    sys.path.insert(0, ROOT)
    import dataclasses
    import bench
    import synth
    from decode_persistent_monokernel_b200 import profile_case
    for wid in (0, 1, 4):
        w = synth.WORKLOADS[wid]
        m = dataclasses.replace(w.model, n_layers=3)
        P, steps = w.prompt_len, 5
        kvpp = 2 * m.n_layers * m.n_kv_heads * m.head_dim * 2
        # the counter case times the launch after a warm-up launch of `steps`
        got = bench.workload_bytes(m, P + steps, steps, synth.streamed_weight_bytes(m), kvpp)
        assert got == profile_case.algorithmic_bytes(m, P, steps), wid


def test_sampling_option_reaches_the_config():
    """`--sample T,K,P` is parsed into (temperature, top-k, top-p) and named in
    the bench line's config; greedy runs carry no sampling key."""
    import bench
    import synth
    w = synth.WORKLOADS[1]
    assert bench.parse_sample(None) is None and bench.parse_sample("") is None
    smp = bench.parse_sample("0.8,40,0.9")
    assert smp == (0.8, 40, 0.9) and isinstance(smp[1], int)
    cfg = bench.run_config(w, 128, 512, 1, "dependency", 4.4e9, smp)
    assert cfg["sampling"] == {"temperature": 0.8, "top_k": 40, "top_p": 0.9,
                               "uniforms": "seeded, one per step"}
    assert "sampling" not in bench.run_config(w, 128, 512, 1, "dependency", 4.4e9)
    with pytest.raises(ValueError):
        bench.parse_sample("0.8,40")
