"""Shared helpers of the GPU parity tests: run the CUDA layer through the C
ABI on seeded synth inputs and compare with the oracle on the same inputs."""
from __future__ import annotations

import numpy as np
import torch

from mot_flow_matching_b200 import build as build_mod
from mot_flow_matching_b200.layer import MotAttnLayer
from oracle import mot_attn_oracle as O

# parity bar on the f32 output: max |err| <= 1e-2 RMS(ref), mean |err| <= 2e-3 RMS(ref)
MAX_TOL = 1e-2
MEAN_TOL = 2e-3

_built = False


def ensure_built():
    global _built
    if not _built:
        build_mod.build()
        _built = True


def to_dev(t, dev="cuda"):
    return {k: (v.to(dev) if k != "prefix_len" else v) for k, v in t.items()}


def weights_of(td):
    return {k: td[k] for k in ("w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm", "a_q", "a_k", "a_v", "a_o",
                               "b_q", "b_k", "b_v", "b_o") if k in td}


def make_layer(wl, td, max_batch=None, max_img=None, max_prefix=None, backward=False):
    ensure_built()
    d = wl.dims
    return MotAttnLayer(weights_of(td), lora_rank=wl.lora_rank if "a_q" in td else 0,
                        lora_alpha=wl.lora_alpha, max_batch=max_batch or wl.batch,
                        max_img_tokens=max_img or wl.img_tokens, max_prefix=max_prefix if max_prefix is not None
                        else wl.prefix, enable_backward=backward, hidden=d.hidden, n_q_heads=d.n_q_heads,
                        n_kv_heads=d.n_kv_heads, head_dim=d.head_dim, rms_eps=d.rms_eps, rope_theta=d.rope_theta)


def run_forward(layer, td, saved=False, prefix_len=None):
    x = td["x"]
    B, N, d = x.shape
    P = td["k_cache"].shape[2]
    pl = [int(v) for v in (prefix_len if prefix_len is not None else td["prefix_len"])]
    y = torch.empty_like(x)
    y32 = torch.empty(B, N, d, dtype=torch.float32, device=x.device)
    sv = layer.new_saved(B, N, P) if saved else None
    layer.forward(x, td["k_cache"], td["v_cache"], pl, y=y, y_f32=y32, saved=sv)
    torch.cuda.synchronize()
    status = layer.device_status()
    return y, y32, sv, status


def parity_stats(got: np.ndarray, ref: np.ndarray):
    err = np.abs(np.asarray(got, dtype=np.float64) - ref)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(err.max()) / rms, float(err.mean()) / rms


def assert_parity(got, ref, what="", max_tol=MAX_TOL, mean_tol=MEAN_TOL):
    mx, mean = parity_stats(got, ref)
    assert mx <= max_tol and mean <= mean_tol, f"{what}: max {mx:.3e} mean {mean:.3e} (x RMS)"
    return mx, mean


def bf16_is_rne_of_f32(y_bf16: torch.Tensor, y32: torch.Tensor) -> bool:
    return torch.equal(y32.to(torch.bfloat16).view(torch.int16), y_bf16.view(torch.int16))


def oracle_forward(wl, t_cpu, rows=None, keep=False, prefix_len=None):
    t64 = O.to_f64(t_cpu)
    if prefix_len is not None:
        t64["prefix_len"] = np.asarray(prefix_len)
    s = wl.lora_alpha / wl.lora_rank if wl.lora_rank else 0.0
    return O.layer_forward(t64, O.dims_of(wl), s, query_rows=rows, keep=keep)


def sample_rows(n, count, seed):
    g = np.random.default_rng(seed)
    rows = np.sort(g.choice(n, size=min(count, n), replace=False))
    # always include the first and last token (tile edges)
    return np.unique(np.concatenate([rows, [0, n - 1]]))
