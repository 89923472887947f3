"""Writes synth_checksums.json: FNV-1a 64 of the generated weight bytes and
prompts of the small workloads.  Calls only the input generator (synth)."""
import json
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
import synth  # noqa: E402

out = {}
for cid in (0, 2):
    w = synth.WORKLOADS[cid]
    bits = synth.generate_weights(w.model, w.weight_seed)
    out[str(cid)] = {"weights_fnv1a64": hex(synth.fnv1a64(bits)),
                     "prompt_fnv1a64": hex(synth.fnv1a64(synth.prompt(w))),
                     "elements": int(bits.size)}
path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "synth_checksums.json")
with open(path, "w") as f:
    json.dump(out, f, indent=1)
print(out)
