#!/usr/bin/env python
"""Batch-1 decode benchmark of the persistent decode kernel.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kie|reference]

One "step" is one decode token: one pass of the whole decode path (every
layer, LM head, greedy argmax, token feedback).  The timed region is one
kie_decode(K) call -- a single persistent launch that runs K steps -- after
an untimed prefill of the workload's prompt and W untimed warm-up steps.

Default workload: the 2.3B-class dense decoder (34 layers, d 2048, 16x128
query heads / 8 KV heads, F 8192, V 32768, fp16 weights and KV cache), prompt
128 -> decode 512, seeded synthetic weights and prompt.  Every step streams
4.41 GB of weights, far more than the 126 MB L2, so no L2 flush is needed
between steps.

Multi-GPU: the path is one request's serial decode chain, so it does not
shard; N GPUs run N independent replicas (one request each) and `value` is
the sum of their tokens/s, timed as the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-1 decode tokens/s/request on 1 B200; % of HBM roofline (bytes/token)"
FALLBACK_HBM_GBS = 6650.0


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=512, help="timed decode steps (tokens)")
    ap.add_argument("--warmup", type=int, default=3, help="untimed decode steps before timing")
    ap.add_argument("--impl", choices=["kie", "reference"], default="kie")
    ap.add_argument("--workload", type=int, default=1, help="workload id (see synth/configs.py)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="bounded CPU work for the oracle baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sync", choices=["dependency", "grid"], default="dependency",
                    help="how SMs wait for one another: per-dependency counters (default) or "
                         "a grid-wide barrier at every dependency point (ablation)")
    ap.add_argument("--sum", choices=["fp32_atomic", "exact"], default=None,
                    help="how the O / down projections are added over SMs (default: the "
                         "library's default mode)")
    ap.add_argument("--sample", metavar="T,K,P", default=None,
                    help="decode by sampling (kie_decode_sample) with temperature T, top-k K "
                         "and top-p P, one seeded uniform per step, instead of greedy")
    ap.add_argument("--profile", action="store_true",
                    help="run the profiling build (libkie_prof.so) and report where each "
                         "SM's time goes; its timings are not the benchmark value")
    return ap.parse_args()


PROF_NAMES = ["total", "wait_other_sms", "gemv", "wait_tiles", "attention", "staging_norm",
              "stage_barrier", "lm_head", "producer_ring_full", "producer_total"]


def profile_summary(prof, steps, mhz):
    """Per-step microseconds per activity: mean and max over SMs."""
    import numpy as np
    cyc = prof.astype(np.float64)
    us = cyc / (mhz * 1e6) * 1e6 / steps
    out = {}
    for i, name in enumerate(PROF_NAMES):
        out[name] = {"mean_us": round(float(us[:, i].mean()), 2),
                     "max_us": round(float(us[:, i].max()), 2)}
    tot = us[:, 0].mean()
    out["sync_share"] = round(float(us[:, 1].mean() / tot), 4) if tot > 0 else None
    out["dependency_waits_per_step"] = round(float(prof[:, 11].mean() / steps), 1)
    stages = ["qkv", "o", "gate_up", "down", "mix", "lm_head"]
    out["gemv_by_stage_us"] = {n: round(float(us[:, 12 + i].mean()), 1) for i, n in enumerate(stages)}
    # dependency counters in the kernel's order: after O (grid), after down
    # (grid), lane-mix flush, token, q/k/v of the KV group, attention partials
    gates = ["o_done_grid", "down_done_grid", "mix_flush", "token", "qkv_group", "attn_group"]
    out["wait_by_counter_us"] = {n: round(float(us[:, 18 + i].mean()), 1) for i, n in enumerate(gates)}
    out["wait_by_counter_min_us"] = {n: round(float(us[:, 18 + i].min()), 1) for i, n in enumerate(gates)}
    out["tile_wait_per_warp_us"] = {n: round(float(us[:, 24 + i].mean()), 1)
                                     for i, n in enumerate(["mean", "max", "min"])}
    out["tiles_per_step"] = round(float(prof[:, 10].mean() / steps), 1)
    out["clock_mhz_used"] = mhz
    return out


TRAFFIC_FILE = os.path.join(os.path.dirname(os.path.abspath(__file__)), "profiles",
                            "monokernel_traffic.json")


def kernel_sources_digest(files):
    import hashlib
    h = hashlib.sha256()
    root = os.path.dirname(os.path.abspath(__file__))
    for f in files:
        with open(os.path.join(root, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def dram_traffic(algorithmic_bytes, workload):
    """DRAM bytes of the timed launch, from the last hardware-counter capture of
    the decode kernel: that capture's DRAM bytes / algorithmic bytes, times this
    launch's algorithmic bytes (the traffic scales with the bytes streamed).
    None when there is no capture, the capture ran another workload's model
    (other stage shapes, another K/V share), or the kernel sources changed
    since."""
    try:
        with open(TRAFFIC_FILE) as f:
            rec = json.load(f)
        if kernel_sources_digest(rec["files"]) != rec["kernel_sources_sha256"]:
            return None, "kernel changed since the last counter capture"
        if int(rec["workload"]) != workload:
            return None, f"the counter capture covers workload {rec['workload']}'s layer shapes only"
        return rec["ratio"] * algorithmic_bytes, rec["capture"]
    except (OSError, KeyError, ValueError):
        return None, "no counter capture recorded"


def prompt_gemm_flops(m, P):
    """Algorithmic tensor-core work of the prompt pass over P tokens: 2 flops
    per weight element per prompt row in the q/k/v, O, gate/up and down
    projections of every layer, and the LM head for the last row (the
    operand parts the pass splits activations into are not counted)."""
    d, dh, F = m.d_model, m.head_dim, m.ffn_dim
    per_layer = ((m.n_heads + 2 * m.n_kv_heads) * dh * d + d * m.n_heads * dh + 3 * F * d)
    return 2.0 * P * m.n_layers * per_layer + 2.0 * m.vocab * d


def peak_tensor():
    """Measured dense bf16 tensor throughput (TFLOP/s, burst) of this machine's
    B200s; fp16 has the same nominal rate."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


def peak_hbm():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period: float = 0.02):
        self.index, self.period = index, period
        self.samples, self.reasons = [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._t = None

    def __enter__(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
            return self
        self._t = threading.Thread(target=self._run, daemon=True)
        self._t.start()
        return self

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def workload_bytes(m, P, K, weight_bytes_per_step, kv_bytes_per_position):
    """Algorithmic bytes of K decode steps after a P-token prompt: every weight
    once per step, K and V of all positions 0..p read at step p, and position
    p's K and V written."""
    kv_positions = sum(P + k + 1 for k in range(K))
    return K * weight_bytes_per_step + (kv_positions + K) * kv_bytes_per_position


def oracle_decode_rate(w, bits, seconds, warmup=0, max_steps=None, threads=1):
    """Greedy decode tokens/s of the float64 oracle on this host (bounded
    sample), with its BLAS limited to `threads` threads (None: the library's
    default, all cores).  Returns (rate, steps, seconds, threads used,
    prompt seconds)."""
    import contextlib
    from oracle import Oracle
    try:
        from threadpoolctl import threadpool_info, threadpool_limits
        limit = threadpool_limits(limits=threads) if threads else contextlib.nullcontext()
    except Exception:
        threadpool_info = None
        limit = contextlib.nullcontext()
    m = w.model
    import synth
    prompt = synth.prompt(w)
    with limit:
        try:
            cores = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
        except Exception:
            cores = threads or os.cpu_count()
        orc = Oracle(m, bits, w.prompt_len + 4096, cache_f64=True)
        t_pre = time.perf_counter()
        orc.prefill(prompt)
        prefill_s = time.perf_counter() - t_pre
        if warmup:
            orc.decode(warmup)
        n, t0 = 0, time.perf_counter()
        while True:
            orc.decode(1)
            n += 1
            el = time.perf_counter() - t0
            if el >= seconds or (max_steps and n >= max_steps):
                break
    return n / el, n, el, cores, prefill_s


def host_cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_baseline_obj(rate, n, el, cores, prefill_s, P):
    """The `cpu_baseline` object: the float64 oracle's greedy decode rate on
    this host (a bounded sample, BLAS on `cores` threads), with its untimed
    prompt's time beside it."""
    return {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} greedy decode steps of the float64 numpy oracle after the "
                      f"{P}-token prompt ({el:.1f} s, {cores} thread{'s' if cores != 1 else ''})",
            "prefill_s": prefill_s, "cpu": host_cpu_model(), "host_cpus": os.cpu_count()}


def run_config(w, P, K, world, sync, weight_bytes_per_step, sample=None):
    """The `config` object of the bench line, the same for both arms."""
    cfg = {"workload": w.name, "prompt": P, "decode_steps": K, "batch": 1,
           "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
           "sync": sync,
           "l2": "inputs larger than L2: %.2f GB of weights streamed per step"
                 % (weight_bytes_per_step / 1e9)}
    if sample is not None:
        cfg["sampling"] = {"temperature": sample[0], "top_k": sample[1], "top_p": sample[2],
                           "uniforms": "seeded, one per step"}
    return cfg


def parse_sample(text):
    """(temperature, top_k, top_p) from "T,K,P", or None."""
    if not text:
        return None
    t, k, p = text.split(",")
    return float(t), int(k), float(p)


def reduce_max_over_ranks(values, world, device):
    """Max over ranks of per-rank timings (a job takes as long as its slowest
    rank); identity for one rank."""
    if world == 1:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_tokens_per_s(world, steps, ms):
    """Whole-job throughput: every rank decodes `steps` tokens of its own
    request (replicas), in the max-over-ranks device time `ms`."""
    return world * steps / (ms * 1e-3)


def main():
    args = parse()
    import numpy as np
    import torch

    import synth
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    w = synth.WORKLOADS[args.workload]
    m = w.model
    P, K, W = w.prompt_len, args.steps, max(3, args.warmup)
    smp = parse_sample(args.sample)

    if args.impl == "reference":
        # the oracle as it stands, on this host's cores, rank 0 only
        if rank != 0:
            return
        bits = synth.generate_weights(m, w.weight_seed)
        budget = max(5.0, min(120.0, args.cpu_seconds * 4))
        # single-threaded, as the CPU baseline is planned (one core)
        rate, n, el, cores, prefill_s = oracle_decode_rate(w, bits, budget, warmup=W,
                                                           max_steps=K, threads=1)
        line = {"metric": METRIC, "value": rate, "unit": "tokens/s", "n_gpus": world, "steps": n,
                "warmup": W, "ms_per_step": 1e3 / rate, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
                "impl": "reference",
                "config": run_config(w, P, K, world, args.sync, synth.streamed_weight_bytes(m)),
                "cpu_baseline": cpu_baseline_obj(rate, n, el, cores, prefill_s, P),
                "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line))
        return

    import decode_persistent_monokernel_b200 as kie
    kie.load(kie.PROF_LIB_PATH if args.profile else kie.LIB_PATH)
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)
    max_seq = P + max(K, W) + 8
    wdev = torch.from_numpy(bits.view(np.int16)).cuda()
    stream = torch.cuda.current_stream()
    dec = kie.Decoder(kie.make_desc(m, max_seq), wdev, stream=stream)
    if args.sync == "grid":
        dec.kie_set_sync_mode(kie.KIE_SYNC_GRID)
    if args.sum is not None:
        dec.kie_set_sum_mode(kie.KIE_SUM_EXACT if args.sum == "exact"
                             else kie.KIE_SUM_FP32_ATOMIC)
    del wdev
    torch.cuda.empty_cache()
    st = dec.kie_get_stats()

    # greedy, or sampling with uniforms drawn before any timed region
    urng = np.random.default_rng(2024)
    u_warm = urng.random(W).astype(np.float32)
    u_timed = urng.random(K).astype(np.float32)

    def decode(n, u):
        if smp is None:
            return dec.kie_decode(n)
        return dec.kie_decode_sample(n, smp[0], smp[1], smp[2], u)

    # warm-up: prompt + W steps, untimed
    dec.kie_prefill(prompt)
    decode(W, u_warm)
    # timed: K steps from the workload's own starting point (position P)
    dec.kie_prefill(prompt)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ev0.record(stream)
        toks = decode(K, u_timed)
        ev1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms = ev0.elapsed_time(ev1)
    kernel_ms = dec.kie_get_stats().last_kernel_ms
    # the prompt pass, timed on the device by the library (the prompt of the
    # timed run above)
    pf_ms = dec.kie_get_stats().last_prefill_ms
    pf_mode = "tensor-core GEMM pass" if st.prefill_mode == kie.KIE_PREFILL_GEMM else \
        "persistent kernel, one position per step"
    # end to end through the C ABI with host buffers: the prompt goes in from
    # host memory (timed on its own), then the decode call, whose wall time
    # includes the launch, the device-to-host copy of the K tokens and status,
    # and the synchronisation
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    dec.kie_prefill(prompt)
    prefill_s = time.perf_counter() - t0
    barrier()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    toks2 = decode(K, u_timed)
    e2e_s = time.perf_counter() - t0
    barrier()
    # With fp32 atomic O/down sums the last bits of the logits vary between
    # runs, so a free-running greedy decode may take a different token at a
    # near tie; with exact sums the two runs are identical.  Report how
    # long they agree.
    diff = np.nonzero(toks != toks2)[0]
    repro_prefix = int(diff[0]) if diff.size else int(K)

    ms, e2e_s, kernel_ms, prefill_s = reduce_max_over_ranks([ms, e2e_s, kernel_ms, prefill_s],
                                                            world, "cuda")

    total_bytes = workload_bytes(m, P, K, st.weight_bytes_per_step, st.kv_bytes_per_position)
    peak, peak_kind = peak_hbm()
    traffic, traffic_src = dram_traffic(total_bytes, args.workload)
    # the same device time as `value` (stream events around the decode call);
    # the launches alone (the library's own events) give frac_kernel_only
    achieved = total_bytes / (ms * 1e-3) / 1e9
    achieved_kernel = total_bytes / (kernel_ms * 1e-3) / 1e9
    value = job_tokens_per_s(world, K, ms)
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
        "warmup": W, "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32 (fp16 weights/KV)" if m.dtype == "f16"
        else "f32 (bf16 weights/KV)", "data": "synthetic (seeded weights and prompt)",
        "config": run_config(w, P, K, world, args.sync, st.weight_bytes_per_step, smp),
        "us_per_token": 1e3 * ms / K,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "frac_of_8TBps_nominal": achieved / 8000.0,
                     "frac_kernel_only": achieved_kernel / peak,
                     "bytes_per_step": total_bytes / K, "traffic": traffic,
                     "traffic_source": traffic_src, "kernel_ms": kernel_ms},
        "clocks": clk.summary(),
        "gpu_launches": 1,
        "repeat_agreement": {"tokens_equal_prefix": repro_prefix, "of": K},
        "sum_mode": args.sum or "library default",
        "e2e": {"value": job_tokens_per_s(world, K, e2e_s * 1e3), "unit": "tokens/s",
                "what": "decode tokens / wall time of one kie_decode(K) call into a host "
                        "array (launch, K steps, token and status copies, synchronisation)"
                        + ("; kie_decode_sample with the K uniforms copied in" if smp else ""),
                "h2d_bytes_per_step": 4 if smp else 0, "d2h_bytes_per_step": (4 * K + 4) / K,
                "prefill_wall_s": prefill_s, "prefill_tokens": P},
        "kernel": {"ctas": st.n_ctas, "threads": st.threads_per_cta, "ring_slots": st.ring_slots,
                   "smem_bytes": st.smem_bytes},
    }
    tpeak, tpeak_kind = peak_tensor()
    gflop = prompt_gemm_flops(m, P) / 1e9
    line["prefill"] = {"tokens": P, "mode": pf_mode, "device_ms": pf_ms,
                       "tokens_per_s": P / (pf_ms * 1e-3) if pf_ms > 0 else None,
                       "gemm_gflop": gflop,
                       "gemm_tflops": gflop / pf_ms if pf_ms > 0 else None,
                       "tensor_peak_tflops": tpeak, "peak_kind": tpeak_kind,
                       "frac_of_tensor_peak": gflop / pf_ms / tpeak if pf_ms > 0 else None}
    if args.profile:
        mhz = line["clocks"]["sm_mhz"] or 1965
        line["profile"] = profile_summary(dec.kie_get_profile(), K, mhz)
        line["profile_build"] = "libkie_prof.so (activity counters on): not the benchmark value"
    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.profile:
        dec.kie_destroy()
        # the oracle on one core (the planned baseline), then on all cores beside it
        rate, n, el, cores, pre_s = oracle_decode_rate(w, bits, args.cpu_seconds, threads=1)
        line["cpu_baseline"] = cpu_baseline_obj(rate, n, el, cores, pre_s, P)
        rate, n, el, cores, pre_s = oracle_decode_rate(w, bits, args.cpu_seconds / 2, threads=None)
        line["cpu_baseline"]["all_cores"] = cpu_baseline_obj(rate, n, el, cores, pre_s, P)
    if rank == 0:
        print(json.dumps(line))
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
