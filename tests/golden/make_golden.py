"""Write tests/golden/tiny_layer.json and tiny_mlp.json from the oracles alone.

The pages print no tensor values for this layer, so this fixture is a
regression pin: it freezes the oracle's output on one tiny seeded case
(hidden 64, 4 query / 2 KV heads, head_dim 16, 5 image tokens, 3 cached keys,
LoRA rank 2, alpha 4, two branches), and likewise the gen-tower MLP oracle's
on one tiny case (hidden 16, intermediate 24, 6 tokens, rank 2, alpha 4). The
independent pins live in tests/test_oracle_pins.py and
tests/test_mlp_oracle_pins.py. Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from oracle import mot_attn_oracle as O  # noqa: E402
from oracle import mot_mlp_oracle as MO  # noqa: E402
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


MLP_SEED = 778


def compute_mlp():
    t64 = O.to_f64(synth.make_mlp_inputs(6, 16, 24, 2, MLP_SEED, with_dy=True))
    s = 4.0 / 2
    y = MO.mlp_forward(t64["x"], t64, s)["y"]
    g = MO.mlp_backward(t64["x"], t64, s, t64["dy"])
    return {"seed": MLP_SEED, "y": y.tolist(), "dx": g["dx"].tolist(), "dA_up": g["dA_up"].tolist(),
            "dB_down": g["dB_down"].tolist()}


if __name__ == "__main__":
    here = os.path.dirname(os.path.abspath(__file__))
    for name, fn in (("tiny_layer.json", compute), ("tiny_mlp.json", compute_mlp)):
        out = os.path.join(here, name)
        with open(out, "w") as f:
            json.dump(fn(), f)
        print("wrote", out)
