"""Write tests/golden/tiny_layer.json from the oracle alone.

The pages print no tensor values for this layer, so this fixture is a
regression pin: it freezes the oracle's output on one tiny seeded case
(hidden 64, 4 query / 2 KV heads, head_dim 16, 5 image tokens, 3 cached keys,
LoRA rank 2, alpha 4, two branches). The independent pins live in
tests/test_oracle_pins.py. Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import mot_attn_oracle as O  # noqa: E402
from mot_flow_matching_b200 import synth  # noqa: E402

SEED = 777


def compute():
    wl = synth.tiny_workload()
    t64 = O.to_f64(synth.make_inputs(wl, SEED, with_dy=True))
    dims = O.dims_of(wl)
    s = wl.lora_alpha / wl.lora_rank
    y = O.layer_forward(t64, dims, s)["y"]
    g = O.layer_backward(t64, dims, s, t64["dy"])
    return {"seed": SEED, "y": y.tolist(), "dx": g["dx"].tolist(),
            "dA_q": g["dA_q"].tolist(), "dB_o": g["dB_o"].tolist()}


if __name__ == "__main__":
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_layer.json")
    with open(out, "w") as f:
        json.dump(compute(), f)
    print("wrote", out)
