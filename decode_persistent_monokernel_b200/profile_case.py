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


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--workload", type=int, default=1)
    ap.add_argument("--layers", type=int, default=4)
    ap.add_argument("--steps", type=int, default=4)
    ap.add_argument("--prompt", type=int, default=0, help="prompt length (0: the workload's)")
    ap.add_argument("--launches", type=int, default=1, help="timed kie_decode launches")
    args = ap.parse_args(argv)

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
