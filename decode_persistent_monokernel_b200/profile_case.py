"""A short decode run for hardware-counter captures.

A profiler replays each captured kernel launch dozens of times and saves and
restores device memory around the replays, so a capture wants a small case:
a workload's layer shapes with fewer layers and a few decode steps, still far
larger than the L2 cache so that DRAM counters mean what they do at full size.

    python -m decode_persistent_monokernel_b200.profile_case --workload 1 --layers 4 --steps 4

The weights are the seeded synthetic ones for the reduced shape; one kie_decode
launch of ``--steps`` tokens follows an untimed prefill and one warm-up launch.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import os
import sys


KERNEL_FILES = ["decode_persistent_monokernel_b200/csrc/monokernel.cu",
                "decode_persistent_monokernel_b200/csrc/kie_internal.h"]


def algorithmic_bytes(m, P, steps):
    """Bytes the first timed launch must move: every weight once per step, the
    K/V of positions 0..p read and position p written, at p = P + steps ..
    P + 2 * steps - 1 (after the prefill and the warm-up launch)."""
    import synth
    d = m.d_model
    weights = (synth.total_elements(m) - m.vocab * d + d) * 2
    kv_pos = 2 * m.n_layers * m.n_kv_heads * m.head_dim * 2
    reads = sum(p + 1 for p in range(P + steps, P + 2 * steps)) * kv_pos
    return steps * weights + reads + steps * kv_pos


def record_traffic(report, args):
    """Writes profiles/monokernel_traffic.json from an ncu report of this case:
    DRAM bytes over algorithmic bytes, tagged with the kernel sources' digest."""
    import csv
    import io
    import subprocess
    import synth
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import bench
    out = subprocess.check_output(["ncu", "-i", report, "--page", "raw", "--csv",
                                   "--print-units", "base"], text=True)
    rows = list(csv.reader(io.StringIO(out)))
    rec = dict(zip(rows[0], rows[2]))
    dram = float(rec["dram__bytes_read.sum"]) + float(rec["dram__bytes_write.sum"])
    w = synth.WORKLOADS[args.workload]
    m = dataclasses.replace(w.model, n_layers=args.layers)
    alg = algorithmic_bytes(m, args.prompt or w.prompt_len, args.steps)
    data = {"files": KERNEL_FILES, "kernel_sources_sha256": bench.kernel_sources_digest(KERNEL_FILES),
            "capture": f"ncu --set full of profile_case --workload {args.workload} --layers "
                       f"{args.layers} --steps {args.steps}; traffic scaled by algorithmic bytes",
            "workload": args.workload,
            "dram_bytes": dram, "algorithmic_bytes": alg, "ratio": dram / alg,
            "gpu_time_ns": float(rec["gpu__time_duration.sum"])}
    with open(os.path.join(root, "profiles", "monokernel_traffic.json"), "w") as f:
        json.dump(data, f, indent=1)
        f.write("\n")
    print(json.dumps(data))


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--steps", type=int, default=4)
    ap.add_argument("--prompt", type=int, default=0, help="prompt length (0: the workload's)")
    ap.add_argument("--launches", type=int, default=1, help="timed kie_decode launches")
    ap.add_argument("--prefill-only", action="store_true",
                    help="run only the prompt (twice: a warm-up and the captured one)")
    ap.add_argument("--record-traffic", metavar="NCU_REPORT",
                    help="no GPU run: record DRAM traffic / algorithmic bytes from a report of "
                         "this case (read with ncu -i) for bench.py")
    args = ap.parse_args(argv)
    if args.record_traffic:
        record_traffic(args.record_traffic, args)
        return

    import numpy as np
    import torch

    import synth
    import decode_persistent_monokernel_b200 as kie

    kie.load()
    w = synth.WORKLOADS[args.workload]
    m = dataclasses.replace(w.model, n_layers=args.layers)
    P = args.prompt or w.prompt_len
    bits = synth.generate_weights(m, w.weight_seed)
    prompt = synth.prompt(w)[:P] if P <= w.prompt_len else \
        np.resize(synth.prompt(w), P).astype(np.int32)
    dev = torch.from_numpy(bits.view(np.int16)).cuda()
    dec = kie.Decoder(kie.make_desc(m, P + args.steps * (args.launches + 1) + 8), dev)
    del dev
    torch.cuda.synchronize()
    if args.prefill_only:
        for _ in range(2):
            dec.kie_prefill(prompt)
        st = dec.kie_get_stats()
        print(json.dumps({"workload": w.name, "layers": m.n_layers, "prompt": P,
                          "prefill_mode": st.prefill_mode, "prefill_ms": st.last_prefill_ms}))
        dec.kie_destroy()
        return
    dec.kie_prefill(prompt)
    dec.kie_decode(args.steps)                 # warm-up launch
    ms = []
    for _ in range(args.launches):
        dec.kie_decode(args.steps)
        ms.append(dec.kie_get_stats().last_kernel_ms)
    st = dec.kie_get_stats()
    print(json.dumps({"workload": w.name, "layers": m.n_layers, "steps": args.steps,
                      "prompt": P, "kernel_ms": ms,
                      "weight_bytes_per_step": st.weight_bytes_per_step,
                      "kv_bytes_per_position": st.kv_bytes_per_position,
                      "pos_after": st.pos}))
    dec.kie_destroy()


if __name__ == "__main__":
    main()
