#!/usr/bin/env python
"""Throughput of the gen-tower attention layer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one forward call of the layer (LoRA-down, QKV projection + LoRA up +
QK-RMSNorm + RoPE, attention over [prefix cache ; self], LoRA-down o, O
projection + LoRA up) on the 2048^2 text-to-image CFG workload: B = 2
branches x N = 4096 image tokens (64 x 64 grid of 32-px patches), P = 400
cached prefix keys, LoRA rank 32, hidden 4096, 32 / 8 heads, head_dim 128.
Inputs are seeded synthetic tensors (mot_flow_matching_b200.synth), resident
in HBM before timing; L2 is flushed (256 MiB write) before every timed step.
Rank 0 prints one JSON line. Under torchrun every rank runs its own
independent layer call (CFG branches / samples shard with no exchange), so
scaling is weak and value = tokens of all ranks / max-over-ranks time.

--impl reference times the CPU oracle (fp64 numpy) on the same workload, on a
bounded sample of query rows per step, on rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "gen-tower attn-layer image tokens/s at 1024²/2048²; % of BF16 tensor peak"
UNIT = "image tokens/s"
WORKLOAD_INDEX = 2          # 2048^2 text-to-image CFG layer call
ALSO_INDEX = 1              # 1024^2 CFG, reported beside it
EDIT_INDEX = 3              # 2048^2 dual-CFG edit, merged LoRA, reported beside it
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) from
# one ncu capture of the 2048^2 CFG workload, keyed by the sha256 of the
# kernel's source file at capture time: a changed kernel reports null.
TRAFFIC = {
    "attn_fwd": {"sha256": "f35c17d939924ee887ac497ea302c33107340a8f3b9650d1cb8c6f22c4442d80",
                 "bytes": 105389568 + 32933376},
    "qkv_gemm": {"sha256": "0d41e561dca3ab88617e17057778f06f2ba99e11707cd22bdf0b5b1c8b2cb2a0",
                 "bytes": 234373120 + 84449536},
}
KERNEL_SOURCES = {"attn_fwd": "attn_fwd.cuh", "qkv_gemm": "gemm.cuh", "o_gemm": "gemm.cuh"}


def kernel_traffic(stage):
    import hashlib
    src = KERNEL_SOURCES.get(stage)
    entry = TRAFFIC.get(stage)
    if not src or not entry:
        return None
    path = os.path.join(ROOT, "mot_flow_matching_b200", "csrc", src)
    with open(path, "rb") as f:
        sha = hashlib.sha256(f.read()).hexdigest()
    return entry["bytes"] if sha == entry["sha256"] else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def stage_work(wl, stage):
    """Algorithmic (flops, bytes) of one launch of a stage."""
    d = wl.dims
    B, N, P, r = wl.batch, wl.img_tokens, wl.prefix, (0 if wl.merged else wl.lora_rank)
    M, dh, Hq, Hkv, hid = B * N, d.head_dim, d.n_q_heads, d.n_kv_heads, d.hidden
    qkv = (Hq + 2 * Hkv) * dh
    L = P + N
    if stage == "qkv_gemm":
        return 2.0 * M * hid * qkv + 2.0 * M * r * qkv, 2.0 * (M * hid + qkv * hid + M * qkv)
    if stage == "attn_fwd":
        return 4.0 * B * Hq * N * L * dh, 2.0 * (B * Hq * N * dh + 2 * B * Hkv * L * dh + M * Hq * dh)
    if stage == "o_gemm":
        return 2.0 * M * Hq * dh * hid + 2.0 * M * r * hid, 2.0 * (M * Hq * dh + hid * Hq * dh + M * hid) + 4.0 * M * hid
    if stage == "lora_down_qkv":
        return 2.0 * M * hid * 3 * r, 2.0 * (M * hid + 3 * r * hid + M * 3 * r)
    if stage == "lora_down_o":
        return 2.0 * M * Hq * dh * r, 2.0 * (M * Hq * dh + r * Hq * dh + M * r)
    if stage == "build_kv":
        # cache prefix rows in (bf16) and out (f16), zero tail rows out, LoRA f16 copies in and out
        tail = (-(P + N)) % 128
        lora = 2.0 * 2 * r * (Hq * dh + hid + qkv)
        return 0.0, 2.0 * 2 * B * Hkv * P * dh * 2 + 2.0 * 2 * B * Hkv * tail * dh + lora
    if stage == "cvt_lora_o":
        return 0.0, 2.0 * 2 * r * (Hq * dh + hid + qkv)
    # backward (LoRA training): base, gains and cache frozen
    if stage == "bwd_do_gemm":
        return 2.0 * M * hid * Hq * dh + 2.0 * M * r * Hq * dh, 2.0 * (M * hid + hid * Hq * dh + 2 * M * Hq * dh)
    if stage in ("bwd_g_o", "bwd_db_o"):
        return 2.0 * M * hid * r, 2.0 * (M * hid + M * r)
    if stage == "bwd_da_o":
        return 2.0 * M * Hq * dh * r, 2.0 * (M * Hq * dh + M * r)
    if stage == "attn_bwd":
        # S, dP and dQ over all L keys; dK and dV over the N self keys (the
        # dk/dv CTAs recompute S^T and dP^T on top: not counted)
        return (6.0 * B * Hq * N * L * dh + 4.0 * B * Hq * N * N * dh,
                2.0 * (2 * B * Hq * N * dh + 2 * B * Hkv * L * dh + M * qkv))
    if stage in ("bwd_g_qkv", "bwd_db_qkv"):
        return 2.0 * M * qkv * r / 3.0, 2.0 * (M * qkv + M * r) / 3.0
    if stage == "bwd_da_qkv":
        return 2.0 * M * hid * r, 2.0 * (M * hid + M * r)
    if stage == "bwd_dx_gemm":
        return 2.0 * M * qkv * hid + 2.0 * M * 3 * r * hid, 2.0 * (M * qkv + qkv * hid + M * hid) + 4.0 * M * hid
    if stage == "bwd_cvt_lora":
        return 0.0, 2.0 * 2 * r * qkv
    return 0.0, 0.0


class ClockSampler:
    """SM clock and throttle reasons of this process's GPU, sampled every
    10 ms through NVML from a background thread while the timed region runs."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown", 0x4: "sw_power_cap"}

    def __init__(self, device_index):
        self.dev = device_index
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = None
        self._thread = None

    def _handle(self, nvml):
        import torch
        try:
            p = torch.cuda.get_device_properties(self.dev)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            return nvml.nvmlDeviceGetHandleByPciBusId(bus.encode())
        except Exception:
            return nvml.nvmlDeviceGetHandleByIndex(self.dev)

    def start(self):
        import threading
        try:
            import pynvml as nvml
            nvml.nvmlInit()
            h = self._handle(nvml)
            self.max_mhz = float(nvml.nvmlDeviceGetMaxClockInfo(h, nvml.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: report that, do not guess
            self.reasons.add(f"nvml unavailable: {type(e).__name__}")
            return
        self._stop = threading.Event()

        def loop():
            while not self._stop.is_set():
                try:
                    self.samples.append(float(nvml.nvmlDeviceGetClockInfo(h, nvml.NVML_CLOCK_SM)))
                    bits = nvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                    for bit, name in self.REASONS.items():
                        if bits & bit:
                            self.reasons.add(name)
                except Exception:
                    pass
                self._stop.wait(0.01)

        self._thread = threading.Thread(target=loop, daemon=True)
        self._thread.start()

    def stop(self):
        if self._thread is not None:
            self._stop.set()
            self._thread.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


def oracle_sample(wl, inputs_cpu, rows_per_branch, seed=0):
    """One oracle forward restricted to `rows_per_branch` query rows per branch."""
    import numpy as np
    from oracle import mot_attn_oracle as O
    t64 = O.to_f64(inputs_cpu)
    g = np.random.default_rng(seed)
    rows = [np.sort(g.choice(wl.img_tokens, rows_per_branch, replace=False)) for _ in range(wl.batch)]
    s = wl.lora_alpha / wl.lora_rank if wl.lora_rank else 0.0
    t0 = time.perf_counter()
    O.layer_forward(t64, O.dims_of(wl), s, query_rows=rows)
    return time.perf_counter() - t0


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((i.get("num_threads", 1) for i in info), default=os.cpu_count())
    except Exception:
        return os.cpu_count()


def run_reference(args):
    from mot_flow_matching_b200 import dp
    world, rank, _ = dp.world_info()
    if rank != 0:
        return 0
    from mot_flow_matching_b200 import synth
    wl = synth.WORKLOADS[WORKLOAD_INDEX]
    inputs = synth.workload_inputs(WORKLOAD_INDEX)
    rows = args.ref_rows
    for _ in range(args.warmup):
        oracle_sample(wl, inputs, rows)
    times = [oracle_sample(wl, inputs, rows, seed=i + 1) for i in range(args.steps)]
    t = sum(times) / len(times)
    value = wl.batch * rows / t
    sample = (f"{rows} of {wl.img_tokens} query rows per branch, all {wl.img_tokens} keys/values projected, "
              f"one oracle forward per step")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "img_tokens": wl.img_tokens, "prefix": wl.prefix,
                   "lora_rank": wl.lora_rank, "parallelism": "none (CPU oracle, rank 0)"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line), flush=True)
    return 0


def run_once_mlp(args):
    """Two warm MLP calls (forward, or forward + backward with --train) of
    an MLP workload (the target of ncu captures)."""
    import torch
    from mot_flow_matching_b200 import synth
    from mot_flow_matching_b200.mlp import MotMlp
    wl = synth.MLP_WORKLOADS[args.workload]
    t = synth.mlp_workload_inputs(args.workload, with_dy=args.train)
    td = {k: v.cuda() for k, v in t.items()}
    w = {k: td[k] for k in td if k.startswith(("w_", "a_", "b_"))}
    m = MotMlp(w, lora_rank=wl.lora_rank, lora_alpha=wl.lora_alpha, max_tokens=wl.tokens,
               enable_backward=args.train, hidden=wl.hidden, intermediate=wl.inter)
    sv = m.new_saved(wl.tokens) if args.train else None
    names = ("gate", "up", "down")
    d_a = [torch.zeros(td["a_" + n].shape, device="cuda") for n in names] if args.train else None
    d_b = [torch.zeros(td["b_" + n].shape, device="cuda") for n in names] if args.train else None
    for _ in range(2):
        y = m.forward(td["x"], saved=sv)
        if args.train:
            m.backward(td["dy"], td["x"], sv, d_a=d_a, d_b=d_b)
    torch.cuda.synchronize()
    status = m.device_status()
    m.close()
    print(json.dumps({"once": wl.name, "train": bool(args.train), "status": status,
                      "y_abs_mean": float(y.float().abs().mean())}))
    return 0 if status == 0 else 1


def run_once_moe(args):
    """Two warm calls of the A3B mixture-of-experts MLP over the 8192 image
    tokens of a 2048^2 CFG call (the target of ncu captures)."""
    import torch
    from mot_flow_matching_b200 import synth
    from mot_flow_matching_b200.moe import MotMoe
    dev = torch.device("cuda", 0)
    T, d, E, K, I = 8192, synth.MOE_HIDDEN, synth.MOE_EXPERTS, synth.MOE_TOP_K, synth.MOE_INTER
    draw = lambda shape, std, seed: synth.draw_device(shape, std, 0.0, seed, dev)
    w = {"w_router": draw((E, d), 0.02, 980_001), "w_gate": draw((E, I, d), 0.02, 980_002),
         "w_up": draw((E, I, d), 0.02, 980_003), "w_down": draw((E, d, I), 0.02, 980_004)}
    x = draw((T, d), 1.0, 980_005)
    moe = MotMoe(w, top_k=K, max_tokens=T)
    for _ in range(2):
        y = moe.forward(x)
    torch.cuda.synchronize()
    status = moe.device_status()
    moe.close()
    print(json.dumps({"once": "moe_a3b_8192_tokens", "status": status, "y_abs_mean": float(y.float().abs().mean())}))
    return 0 if status == 0 else 1


def run_once(args):
    """One warm forward of a workload (the target of ncu captures)."""
    import torch
    from mot_flow_matching_b200 import build as build_mod
    from mot_flow_matching_b200 import synth
    from mot_flow_matching_b200.layer import MotAttnLayer
    build_mod.build()
    if args.mlp:
        return run_once_mlp(args)
    if args.moe:
        return run_once_moe(args)
    wl = synth.WORKLOADS[args.workload]
    t = synth.workload_inputs(args.workload)
    td = {k: (v.cuda() if k != "prefix_len" else v) for k, v in t.items()}
    wts = {k: td[k] for k in ("w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm", "a_q", "a_k", "a_v", "a_o",
                              "b_q", "b_k", "b_v", "b_o") if k in td}
    layer = MotAttnLayer(wts, lora_rank=wl.lora_rank, lora_alpha=wl.lora_alpha, max_batch=wl.batch,
                         max_img_tokens=wl.img_tokens, max_prefix=wl.prefix)
    pl = [int(v) for v in td["prefix_len"]]
    if args.train:
        # forward keeping activations + backward, twice (the second is the one to capture)
        layer.close()
        layer = MotAttnLayer(wts, lora_rank=wl.lora_rank, lora_alpha=wl.lora_alpha, max_batch=wl.batch,
                             max_img_tokens=wl.img_tokens, max_prefix=wl.prefix, enable_backward=True)
        sv = layer.new_saved(wl.batch, wl.img_tokens, wl.prefix)
        names = ("q", "k", "v", "o")
        d_a = [torch.zeros(td["a_" + n].shape, device="cuda") for n in names] if wl.lora_rank else None
        d_b = [torch.zeros(td["b_" + n].shape, device="cuda") for n in names] if wl.lora_rank else None
        dy = td.get("dy", torch.randn_like(td["x"]))
        for _ in range(2):
            y = layer.forward(td["x"], td["k_cache"], td["v_cache"], pl, saved=sv)
            dx = layer.backward(dy, td["x"], td["k_cache"], td["v_cache"], pl, sv, d_a=d_a, d_b=d_b)
    else:
        for _ in range(2):
            y = layer.forward(td["x"], td["k_cache"], td["v_cache"], pl)
    torch.cuda.synchronize()
    status = layer.device_status()
    layer.close()
    print(json.dumps({"once": wl.name, "train": bool(args.train), "status": status,
                      "y_abs_mean": float(y.float().abs().mean())}))
    return 0 if status == 0 else 1


TRAIN_INDEX = 4  # 2048^2 LoRA training layer call: B = 1, N = 4096, P = 400, r = 32


def train_steps(bundle, dev, flush, stream, args, world):
    """Forward (activations kept) + backward of the training workload; each
    timed separately with CUDA events, per-launch times from the library."""
    import torch
    from mot_flow_matching_b200 import dp
    from mot_flow_matching_b200.layer import mot_dev_profile, mot_dev_stage_timeline, mot_dev_stage_times
    wl, td, layer = bundle
    pl = [int(v) for v in td["prefix_len"]]
    x, kc, vc, dy = td["x"], td["k_cache"], td["v_cache"], td["dy"]
    y = torch.empty_like(x)
    dx = torch.empty_like(x)
    sv = layer.new_saved(wl.batch, wl.img_tokens, wl.prefix, dev)
    ws = layer.workspace(wl.batch, wl.img_tokens, wl.prefix, dev)
    names = ("q", "k", "v", "o")
    d_a = [torch.zeros(td["a_" + n].shape, device=dev) for n in names]
    d_b = [torch.zeros(td["b_" + n].shape, device=dev) for n in names]

    def step():
        layer.forward(x, kc, vc, pl, y=y, saved=sv, workspace=ws)
        layer.backward(dy, x, kc, vc, pl, sv, dx=dx, d_a=d_a, d_b=d_b, accumulate=True, workspace=ws)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    dp.barrier(world)
    fwd_ms, bwd_ms, stages, launches = [], [], {}, 0
    for _ in range(args.steps):
        flush.zero_()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
        # forward and backward issued back to back, as a training loop does:
        # nothing on the host waits for the GPU between them
        e[0].record(stream)
        layer.forward(x, kc, vc, pl, y=y, saved=sv, workspace=ws)
        e[1].record(stream)
        launches += layer.last_launch_count()
        layer.backward(dy, x, kc, vc, pl, sv, dx=dx, d_a=d_a, d_b=d_b, accumulate=True, workspace=ws)
        e[2].record(stream)
        launches += layer.last_launch_count()
        e[2].synchronize()
        fwd_ms.append(e[0].elapsed_time(e[1]))
        bwd_ms.append(e[1].elapsed_time(e[2]))
    # per-launch times from separate untimed passes (the profiling events sit
    # between launches; reading them inside a timed step would also stall the
    # host between the two calls)
    mot_dev_profile(layer.handle, True)
    for _ in range(args.steps):
        flush.zero_()
        layer.forward(x, kc, vc, pl, y=y, saved=sv, workspace=ws)
        for name, ms in mot_dev_stage_times(layer.handle):
            stages.setdefault(name, []).append(ms)
        layer.backward(dy, x, kc, vc, pl, sv, dx=dx, d_a=d_a, d_b=d_b, accumulate=True, workspace=ws)
        for name, ms in mot_dev_stage_times(layer.handle):
            stages.setdefault(name, []).append(ms)
        # the backward's launches on one clock (main and side stream), last pass
        timeline = [[n, round(a, 4), round(b, 4)] for n, a, b in mot_dev_stage_timeline(layer.handle)]
    mot_dev_profile(layer.handle, False)
    assert layer.device_status() == 0
    layer.close()
    f = dp.max_over_ranks(statistics.mean(fwd_ms), world, dev)
    b = dp.max_over_ranks(statistics.mean(bwd_ms), world, dev)
    fwd_flops = sum(stage_work(wl, n)[0] for n in ("lora_down_qkv", "qkv_gemm", "attn_fwd", "lora_down_o", "o_gemm"))
    bwd_flops = sum(stage_work(wl, n)[0] * (3 if n in ("bwd_g_qkv", "bwd_db_qkv", "bwd_da_qkv") else 1)
                    for n in stages if n.startswith(("bwd_", "attn_bwd")))
    peaks, _ = load_peaks()
    per = {}
    for n, v in stages.items():
        mult = 3 if n in ("bwd_g_qkv", "bwd_db_qkv", "bwd_da_qkv") else 1
        ms = sum(v) / args.steps  # per step (the q/k/v stages launch three times)
        fl = stage_work(wl, n)[0] * mult
        per[n] = {"ms": ms, "tflops": fl / (ms / 1e3) / 1e12 if fl else None}
    return {"workload": wl.name, "fwd_ms": f, "bwd_ms": b, "tokens_per_s": world * wl.batch * wl.img_tokens / ((f + b) / 1e3),
            "fwd_tflops": fwd_flops / (f / 1e3) / 1e12, "bwd_tflops": bwd_flops / (b / 1e3) / 1e12,
            "bwd_pct_of_bf16_peak": 100.0 * bwd_flops / (b / 1e3) / 1e12 / peaks["bf16_tflops"],
            "bwd_algorithmic_gflop": bwd_flops / 1e9, "gpu_launches": launches * world, "stages": per,
            "bwd_timeline_ms": timeline}


MLP_INDEX = 2        # the MLP over the 2048^2 CFG call's 8192 tokens
MLP_TRAIN_INDEX = 4  # the MLP training step over 4096 tokens


def mlp_flops(wl):
    """Algorithmic FLOPs of one MLP forward (gate/up, down, LoRA down and up)."""
    T, d, I, r = wl.tokens, wl.hidden, wl.inter, wl.lora_rank
    return 6.0 * T * d * I + 2.0 * T * r * (2 * d + 2 * I + I + d)


def mlp_steps(dev, flush, stream, args, world):
    """The SwiGLU MLP: forward over the 2048^2 CFG tokens, forward + backward
    over the training tokens; CUDA events on the launching stream, L2 flushed
    before every step; per-launch times from separate passes."""
    import torch
    from mot_flow_matching_b200 import dp, synth
    from mot_flow_matching_b200.mlp import MotMlp, mot_dev_mlp_profile, mot_dev_mlp_stage_times
    peaks, _ = load_peaks()
    out = {}
    for key, idx in (("forward", MLP_INDEX), ("train", MLP_TRAIN_INDEX)):
        wl = synth.MLP_WORKLOADS[idx]
        t = synth.mlp_workload_inputs(idx)
        td = {k: v.to(dev) for k, v in t.items()}
        w = {k: td[k] for k in td if k.startswith(("w_", "a_", "b_"))}
        m = MotMlp(w, lora_rank=wl.lora_rank, lora_alpha=wl.lora_alpha, max_tokens=wl.tokens,
                   enable_backward=wl.train, hidden=wl.hidden, intermediate=wl.inter)
        x = td["x"]
        y = torch.empty_like(x)
        ws = m.workspace(wl.tokens, dev)
        train = wl.train
        sv = m.new_saved(wl.tokens, dev) if train else None
        names = ("gate", "up", "down")
        d_a = [torch.zeros(td["a_" + n].shape, device=dev) for n in names] if train else None
        d_b = [torch.zeros(td["b_" + n].shape, device=dev) for n in names] if train else None
        dx = torch.empty_like(x)

        def step(ev=None):
            if ev:
                ev[0].record(stream)
            m.forward(x, y=y, saved=sv, workspace=ws)
            if ev:
                ev[1].record(stream)
            if train:
                m.backward(td["dy"], x, sv, dx=dx, d_a=d_a, d_b=d_b, accumulate=True, workspace=ws)
                if ev:
                    ev[2].record(stream)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        dp.barrier(world)
        steps = max(3, args.steps // 2)
        f_ms, b_ms = [], []
        clk = ClockSampler(dev.index if dev.index is not None else 0)
        clk.start()
        for _ in range(steps):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            step(ev)
            ev[2 if train else 1].synchronize()
            f_ms.append(ev[0].elapsed_time(ev[1]))
            if train:
                b_ms.append(ev[1].elapsed_time(ev[2]))
        clocks = clk.stop()
        stages = {}
        mot_dev_mlp_profile(m.handle, True)
        for _ in range(steps):
            flush.zero_()
            m.forward(x, y=y, saved=sv, workspace=ws)
            for n, v in mot_dev_mlp_stage_times(m.handle):
                stages.setdefault(n, []).append(v)
            if train:
                m.backward(td["dy"], x, sv, dx=dx, d_a=d_a, d_b=d_b, accumulate=True, workspace=ws)
                for n, v in mot_dev_mlp_stage_times(m.handle):
                    stages.setdefault(n, []).append(v)
        mot_dev_mlp_profile(m.handle, False)
        assert m.device_status() == 0
        m.close()
        f = dp.max_over_ranks(statistics.mean(f_ms), world, dev)
        fl = mlp_flops(wl)
        rec = {"workload": wl.name, "tokens": wl.tokens, "intermediate": wl.inter, "lora_rank": wl.lora_rank,
               "fwd_ms": f, "fwd_tflops": fl / (f / 1e3) / 1e12,
               "fwd_frac_of_bf16_peak": fl / (f / 1e3) / 1e12 / peaks["bf16_tflops"],
               "tokens_per_s": world * wl.tokens / (f / 1e3),
               "stages_ms": {n: sum(v) / steps for n, v in stages.items()}, "clocks": clocks}
        if train:
            b = dp.max_over_ranks(statistics.mean(b_ms), world, dev)
            bfl = 6.0 * wl.tokens * wl.hidden * wl.inter + 2.0 * wl.tokens * wl.lora_rank * 4 * (wl.hidden + wl.inter)
            rec.update({"bwd_ms": b, "bwd_tflops": bfl / (b / 1e3) / 1e12,
                        "bwd_frac_of_bf16_peak": bfl / (b / 1e3) / 1e12 / peaks["bf16_tflops"]})
        out[key] = rec
    return out


STEP_LAYERS = 42  # decoder layers of the gen tower ("SenseNova-U1" DiffSynth-Studio docs, architecture note)


def denoise_step_bench(dev, flush, stream, args, world):
    """One gen-tower denoise step over all 42 layers (attention + MLP, LoRA
    rank 32 on both) for the 2048^2 CFG call (B = 2, N = 4096, P = 400),
    weights drawn on the device per layer; plus the prefix-tower layer that
    builds one layer's cache for two 400-token prompts. CUDA events, L2
    flushed before every step."""
    import torch
    from mot_flow_matching_b200 import dp, synth
    from mot_flow_matching_b200.layer import MotAttnLayer
    from mot_flow_matching_b200.mlp import MotMlp
    from mot_flow_matching_b200.step import MotStep
    wl = synth.WORKLOADS[WORKLOAD_INDEX]
    d, r, I, C = wl.dims.hidden, wl.lora_rank, synth.MLP_INTER, 3 * 32 * 32
    qd, kvd = wl.dims.n_q_heads * wl.dims.head_dim, wl.dims.n_kv_heads * wl.dims.head_dim
    B, N, P = wl.batch, wl.img_tokens, wl.prefix
    draw = lambda shape, std, mean, seed: synth.draw_device(shape, std, mean, seed, dev)
    attn, mlps, keep = [], [], []
    for l in range(STEP_LAYERS):
        sd = 900_000 + 100 * l
        a = {"w_q": draw((qd, d), 0.02, 0.0, sd + 1), "w_k": draw((kvd, d), 0.02, 0.0, sd + 2),
             "w_v": draw((kvd, d), 0.02, 0.0, sd + 3), "w_o": draw((d, qd), 0.02, 0.0, sd + 4),
             "q_norm": draw((128,), 0.1, 1.0, sd + 5), "k_norm": draw((128,), 0.1, 1.0, sd + 6)}
        for i, (n, shape) in enumerate({"a_q": (r, d), "a_k": (r, d), "a_v": (r, d), "a_o": (r, qd), "b_q": (qd, r),
                                        "b_k": (kvd, r), "b_v": (kvd, r), "b_o": (d, r)}.items()):
            a[n] = draw(shape, 1 / 16 if n.startswith("a_") else 0.01, 0.0, sd + 10 + i)
        m = {"w_gate": draw((I, d), 0.02, 0.0, sd + 30), "w_up": draw((I, d), 0.02, 0.0, sd + 31),
             "w_down": draw((d, I), 0.02, 0.0, sd + 32)}
        for i, (n, shape) in enumerate({"a_gate": (r, d), "a_up": (r, d), "a_down": (r, I), "b_gate": (I, r),
                                        "b_up": (I, r), "b_down": (d, r)}.items()):
            m[n] = draw(shape, 1 / 16 if n.startswith("a_") else 0.01, 0.0, sd + 40 + i)
        cache = (draw((B, wl.dims.n_kv_heads, P, 128), 1.0, 0.0, sd + 60),
                 draw((B, wl.dims.n_kv_heads, P, 128), 1.0, 0.0, sd + 61))
        norms = (draw((d,), 0.1, 1.0, sd + 70), draw((d,), 0.1, 1.0, sd + 71))
        attn.append(MotAttnLayer(a, lora_rank=r, lora_alpha=wl.lora_alpha, max_batch=B, max_img_tokens=N,
                                 max_prefix=P))
        mlps.append(MotMlp(m, lora_rank=r, lora_alpha=wl.lora_alpha, max_tokens=B * N, intermediate=I))
        keep.append((a, m, cache, norms))
    w_in, norm_out, w_out = draw((d, C), 0.02, 0.0, 990_001), draw((d,), 0.1, 1.0, 990_002), draw((C, d), 0.02, 0.0,
                                                                                                   990_003)
    step = MotStep(attn, mlps, [k[3][0] for k in keep], [k[3][1] for k in keep], w_in, norm_out, w_out)
    z = torch.randn(N, C, generator=torch.Generator(device=dev).manual_seed(990_004), device=dev)
    zn = torch.empty_like(z)
    kc, vc = [k[2][0] for k in keep], [k[2][1] for k in keep]
    pl = [P] * B
    ws = step.workspace(B, N, P, dev)
    for _ in range(2):
        step.forward(z, kc, vc, pl, 0.6, 0.55, z_next=zn, workspace=ws)
    torch.cuda.synchronize(dev)
    dp.barrier(world)
    steps = 3
    ms = []
    clk = ClockSampler(dev.index if dev.index is not None else 0)
    clk.start()
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        step.forward(z, kc, vc, pl, 0.6, 0.55, z_next=zn, workspace=ws)
        e1.record(stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    clocks = clk.stop()
    for a in attn:
        assert a.device_status() == 0
    for m in mlps:
        assert m.device_status() == 0
    t = dp.max_over_ranks(statistics.mean(ms), world, dev)
    peaks, _ = load_peaks()
    layer_fl = sum(stage_work(wl, n)[0] for n in ("lora_down_qkv", "qkv_gemm", "attn_fwd", "lora_down_o", "o_gemm"))
    fl = STEP_LAYERS * (layer_fl + mlp_flops(synth.MLP_WORKLOADS[MLP_INDEX])) + 2.0 * N * C * d + 2.0 * B * N * C * d
    out = {"workload": f"denoise_step_2048sq_cfg2_{STEP_LAYERS}layers", "layers": STEP_LAYERS, "batch": B,
           "img_tokens": N, "prefix": P, "lora_rank": r, "ms_per_step": t, "image_tokens_per_s": world * B * N / (t / 1e3),
           "tflops": fl / (t / 1e3) / 1e12, "frac_of_bf16_peak": fl / (t / 1e3) / 1e12 / peaks["bf16_tflops"],
           # each step keeps the GPU busy for ~0.15 s: the power-capped
           # sustained peak is the denominator that applies
           "frac_of_bf16_sustained": fl / (t / 1e3) / 1e12 / peaks["bf16_tflops_sustained"],
           "algorithmic_tflop": fl / 1e12, "clocks": clocks}
    if clocks.get("sm_mhz") and clocks.get("sm_max_mhz"):
        out["ms_per_step_at_max_clock"] = t * clocks["sm_mhz"] / clocks["sm_max_mhz"]
    step.close()
    # the prefix-tower layer that builds a layer's cache: two 400-token prompts
    a0 = keep[0][0]
    base = {k: v for k, v in a0.items() if not k.startswith(("a_", "b_"))}
    player = MotAttnLayer(base, max_batch=B, max_img_tokens=P, max_prefix=0)
    xp = draw((B, P, d), 1.0, 0.0, 990_010)
    for _ in range(3):
        player.prefix_forward(xp, [P] * B)
    torch.cuda.synchronize(dev)
    pms = []
    for _ in range(5):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        player.prefix_forward(xp, [P] * B)
        e1.record(stream)
        e1.synchronize()
        pms.append(e0.elapsed_time(e1))
    assert player.device_status() == 0
    player.close()
    pt = dp.max_over_ranks(statistics.mean(pms), world, dev)
    pfl = 2.0 * B * P * d * (qd + 2 * kvd) + 2.0 * B * wl.dims.n_q_heads * P * (P + 1) * 128 + 2.0 * B * P * qd * d
    out["prefix_layer"] = {"batch": B, "prompt_tokens": P, "ms": pt, "tflops": pfl / (pt / 1e3) / 1e12}
    for a in attn:
        a.close()
    for m in mlps:
        m.close()
    return out


def moe_bench(dev, flush, stream, args, world):
    """The A3B gen tower's mixture-of-experts MLP (hidden 2048, 32 experts,
    top 8, width 768) over the 8192 image tokens of a 2048^2 CFG call;
    weights and tokens drawn on the device; CUDA events, L2 flushed."""
    import torch
    from mot_flow_matching_b200 import dp, synth
    from mot_flow_matching_b200.moe import MotMoe
    T, d, E, K, I = 8192, synth.MOE_HIDDEN, synth.MOE_EXPERTS, synth.MOE_TOP_K, synth.MOE_INTER
    draw = lambda shape, std, seed: synth.draw_device(shape, std, 0.0, seed, dev)
    w = {"w_router": draw((E, d), 0.02, 980_001), "w_gate": draw((E, I, d), 0.02, 980_002),
         "w_up": draw((E, I, d), 0.02, 980_003), "w_down": draw((E, d, I), 0.02, 980_004)}
    x = draw((T, d), 1.0, 980_005)
    moe = MotMoe(w, top_k=K, max_tokens=T)
    y = torch.empty_like(x)
    ws = moe.workspace(T, dev)
    for _ in range(args.warmup):
        moe.forward(x, y=y, workspace=ws)
    torch.cuda.synchronize(dev)
    dp.barrier(world)
    ms = []
    clk = ClockSampler(dev.index if dev.index is not None else 0)
    clk.start()
    for _ in range(max(3, args.steps // 2)):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        moe.forward(x, y=y, workspace=ws)
        e1.record(stream)
        e1.synchronize()
        ms.append(e0.elapsed_time(e1))
    clocks = clk.stop()
    assert moe.device_status() == 0
    moe.close()
    t = dp.max_over_ranks(statistics.mean(ms), world, dev)
    fl = 6.0 * T * K * d * I + 2.0 * T * d * E
    peaks, _ = load_peaks()
    return {"workload": "moe_a3b_2048sq_cfg2_tokens", "tokens": T, "hidden": d, "experts": E, "top_k": K,
            "intermediate": I, "ms": t, "tokens_per_s": world * T / (t / 1e3), "tflops": fl / (t / 1e3) / 1e12,
            "frac_of_bf16_peak": fl / (t / 1e3) / 1e12 / peaks["bf16_tflops"], "clocks": clocks}


def sustained_steps(bundle, dev, stream, args, world, local):
    """Back-to-back forwards of one workload for at least args.sustained_s
    seconds under one pair of CUDA events, SM clock sampled throughout;
    reported against the sustained bf16 peak and normalised by the clock."""
    import torch
    from mot_flow_matching_b200 import dp
    wl, _, td, layer = bundle
    x, kc, vc = td["x"], td["k_cache"], td["v_cache"]
    pl = [int(v) for v in td["prefix_len"]]
    y = torch.empty_like(x)
    ws = layer.workspace(wl.batch, wl.img_tokens, wl.prefix, dev)
    for _ in range(args.warmup):
        layer.forward(x, kc, vc, pl, y=y, workspace=ws)
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(20):
        layer.forward(x, kc, vc, pl, y=y, workspace=ws)
    e1.record(stream)
    e1.synchronize()
    n = max(20, int(args.sustained_s * 1e3 / (e0.elapsed_time(e1) / 20)))
    dp.barrier(world)
    clocks = ClockSampler(local)
    clocks.start()
    e0.record(stream)
    for _ in range(n):
        layer.forward(x, kc, vc, pl, y=y, workspace=ws)
    e1.record(stream)
    e1.synchronize()
    clk = clocks.stop()
    total = dp.max_over_ranks(e0.elapsed_time(e1), world, dev)
    layer.close()
    peaks, kind = load_peaks()
    fl = sum(stage_work(wl, s)[0] for s in ("lora_down_qkv", "qkv_gemm", "attn_fwd", "lora_down_o", "o_gemm"))
    ms = total / n
    tf = fl / (ms / 1e3) / 1e12
    out = {"workload": wl.name, "steps": n, "seconds": total / 1e3, "ms_per_step": ms, "tflops": tf,
           "peak": peaks["bf16_tflops_sustained"], "frac": tf / peaks["bf16_tflops_sustained"],
           "peak_source": f"{kind} (sustained)", "clocks": clk,
           "value": dp.aggregate_rate(wl.batch * wl.img_tokens, n, total, world)}
    if clk.get("sm_mhz") and clk.get("sm_max_mhz"):
        # the same time at the maximum SM clock, if the layer scaled with it
        out["ms_per_step_at_max_clock"] = ms * clk["sm_mhz"] / clk["sm_max_mhz"]
    return out


def run_ours(args):
    import torch
    from mot_flow_matching_b200 import build as build_mod
    from mot_flow_matching_b200 import synth
    from mot_flow_matching_b200.layer import MotAttnLayer, mot_dev_profile, mot_dev_stage_times

    from mot_flow_matching_b200 import dp
    world, rank, local = dp.world_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dp.init_group(world, "nccl", dev)
    if rank == 0:
        build_mod.build()
    dp.barrier(world)

    # each rank: its own data shard (x, cache, dy), replicated weights
    def make(index):
        wl = synth.WORKLOADS[index]
        t = synth.workload_inputs(index, shard=rank)
        td = {k: (v.to(dev) if k != "prefix_len" else v) for k, v in t.items()}
        wts = {k: td[k] for k in ("w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm", "a_q", "a_k", "a_v", "a_o",
                                  "b_q", "b_k", "b_v", "b_o") if k in td}
        layer = MotAttnLayer(wts, lora_rank=wl.lora_rank, lora_alpha=wl.lora_alpha, max_batch=wl.batch,
                             max_img_tokens=wl.img_tokens, max_prefix=wl.prefix)
        return wl, t, td, layer

    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def make_train():
        wl = synth.WORKLOADS[TRAIN_INDEX]
        t = synth.workload_inputs(TRAIN_INDEX, shard=rank)
        td = {k: (v.to(dev) if k != "prefix_len" else v) for k, v in t.items()}
        wts = {k: td[k] for k in ("w_q", "w_k", "w_v", "w_o", "q_norm", "k_norm", "a_q", "a_k", "a_v", "a_o",
                                  "b_q", "b_k", "b_v", "b_o") if k in td}
        layer = MotAttnLayer(wts, lora_rank=wl.lora_rank, lora_alpha=wl.lora_alpha, max_batch=wl.batch,
                             max_img_tokens=wl.img_tokens, max_prefix=wl.prefix, enable_backward=True)
        return wl, td, layer

    def device_steps(wl, td, layer, steps, warmup, profile):
        x, kc, vc = td["x"], td["k_cache"], td["v_cache"]
        pl = [int(v) for v in td["prefix_len"]]
        y = torch.empty_like(x)
        ws = layer.workspace(wl.batch, wl.img_tokens, wl.prefix, dev)
        for _ in range(warmup):
            layer.forward(x, kc, vc, pl, y=y, workspace=ws)
        torch.cuda.synchronize(dev)
        dp.barrier(world)
        torch.cuda.synchronize(dev)
        step_ms, stages = [], {}
        launches = 0
        for _ in range(steps):
            flush.zero_()
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            layer.forward(x, kc, vc, pl, y=y, workspace=ws)
            e1.record(stream)
            launches += layer.last_launch_count()
            e1.synchronize()
            step_ms.append(e0.elapsed_time(e1))
        torch.cuda.synchronize(dev)
        if profile:
            # per-launch times from separate passes: the library's profiling
            # events sit between launches and would keep consecutive kernels
            # from overlapping their prologues (programmatic launch)
            mot_dev_profile(layer.handle, True)
            for _ in range(steps):
                flush.zero_()
                layer.forward(x, kc, vc, pl, y=y, workspace=ws)
                for name, ms in mot_dev_stage_times(layer.handle):
                    stages.setdefault(name, []).append(ms)
            mot_dev_profile(layer.handle, False)
            torch.cuda.synchronize(dev)
        return step_ms, stages, launches

    wl, t_cpu, td, layer = make(WORKLOAD_INDEX)
    clocks = ClockSampler(local)
    clocks.start()
    step_ms, stages, launches = device_steps(wl, td, layer, args.steps, args.warmup, True)
    clk = clocks.stop()
    total_ms = dp.max_over_ranks(sum(step_ms), world, dev)
    ms_per_step = total_ms / args.steps
    tokens = wl.batch * wl.img_tokens
    value = dp.aggregate_rate(tokens, args.steps, total_ms, world)

    # unflushed: the same K steps back to back with no L2 flush between them
    # (weights and cache may stay in the 126 MB L2, which a 42-layer model
    # would not allow: context beside the flushed headline)
    def unflushed_ms(k):
        x_u, kc_u, vc_u = td["x"], td["k_cache"], td["v_cache"]
        pl_u = [int(v) for v in td["prefix_len"]]
        y_u = torch.empty_like(x_u)
        ws_u = layer.workspace(wl.batch, wl.img_tokens, wl.prefix, dev)
        for _ in range(3):
            layer.forward(x_u, kc_u, vc_u, pl_u, y=y_u, workspace=ws_u)
        torch.cuda.synchronize(dev)
        dp.barrier(world)
        torch.cuda.synchronize(dev)
        u0, u1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        uclk = ClockSampler(local)
        uclk.start()
        u0.record(stream)
        for _ in range(k):
            layer.forward(x_u, kc_u, vc_u, pl_u, y=y_u, workspace=ws_u)
        u1.record(stream)
        u1.synchronize()
        return dp.max_over_ranks(u0.elapsed_time(u1) / k, world, dev), uclk.stop()

    unflushed, unflushed_clocks = unflushed_ms(args.steps)

    # end to end through the public call with host buffers. Every step copies
    # its inputs (x and the prefix cache) in from pinned host memory and its
    # output y back. Headline: the host-buffer C-ABI call over all K steps
    # (mot_attn_forward_host: two device staging slots, the copy-in of step
    # i+1 and the copy-out of step i-1 overlap the layer of step i);
    # serial_value: the same steps with each one's copies and layer in turn.
    x_h = td["x"].cpu().pin_memory()
    kc_h = td["k_cache"].cpu().pin_memory()
    vc_h = td["v_cache"].cpu().pin_memory()
    y_h = torch.empty_like(x_h).pin_memory()
    pl = [int(v) for v in td["prefix_len"]]
    ws = layer.workspace(wl.batch, wl.img_tokens, wl.prefix, dev)
    staging = layer.host_staging(wl.batch, wl.img_tokens, wl.prefix, dev)

    def host_steps(k):
        layer.forward_host([x_h] * k, [kc_h] * k, [vc_h] * k, pl, [y_h] * k, staging=staging, workspace=ws)

    host_steps(max(3, args.warmup))
    torch.cuda.synchronize(dev)
    dp.barrier(world)
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    host_steps(args.steps)
    e1.record(stream)
    e1.synchronize()
    e2e_ms = dp.max_over_ranks(e0.elapsed_time(e1), world, dev)
    e2e_value = dp.aggregate_rate(tokens, args.steps, e2e_ms, world)
    assert layer.device_status() == 0

    x_d, kc_d, vc_d = torch.empty_like(td["x"]), torch.empty_like(td["k_cache"]), torch.empty_like(td["v_cache"])
    y_d = torch.empty_like(td["x"])

    def e2e_step():
        x_d.copy_(x_h, non_blocking=True)
        kc_d.copy_(kc_h, non_blocking=True)
        vc_d.copy_(vc_h, non_blocking=True)
        layer.forward(x_d, kc_d, vc_d, pl, y=y_d, workspace=ws)
        y_h.copy_(y_d, non_blocking=True)

    for _ in range(max(3, args.warmup)):
        e2e_step()
    torch.cuda.synchronize(dev)
    dp.barrier(world)
    serial_ms = 0.0
    for _ in range(args.steps):
        flush.zero_()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        e2e_step()
        e1.record(stream)
        e1.synchronize()
        serial_ms += e0.elapsed_time(e1)
    serial_ms = dp.max_over_ranks(serial_ms, world, dev)
    serial_value = dp.aggregate_rate(tokens, args.steps, serial_ms, world)
    h2d = (x_h.numel() + kc_h.numel() + vc_h.numel()) * 2
    d2h = y_h.numel() * 2

    # LoRA training step at 2048^2 (forward keeping activations + backward)
    train = None
    if not args.skip_train:
        train = train_steps(make_train(), dev, flush, stream, args, world)

    # 1024^2 CFG beside it (same protocol, fewer steps)
    also = None
    if not args.skip_also:
        wl1, _, td1, layer1 = make(ALSO_INDEX)
        ms1, st1, _ = device_steps(wl1, td1, layer1, max(3, args.steps // 2), args.warmup, True)
        max1 = dp.max_over_ranks(sum(ms1), world, dev)
        fl1 = sum(stage_work(wl1, n)[0] for n in st1)
        also = {"workload": wl1.name, "value": dp.aggregate_rate(wl1.batch * wl1.img_tokens, len(ms1), max1, world),
                "ms_per_step": max1 / len(ms1), "tflops": fl1 / (max1 / len(ms1) / 1e3) / 1e12,
                "stages_ms": {n: sum(v) / len(ms1) for n, v in st1.items()}}
        layer1.close()
        # the edit workload: adapters baked into the base (merge at load), then rank-0 calls
        wl3, _, td3, layer3 = make(EDIT_INDEX)
        merged = {n: torch.empty_like(td3["w_" + n]) for n in ("q", "k", "v", "o")}
        # the one-off merge at load, timed on its own (flushed L2)
        torch.cuda.synchronize(dev)
        flush.zero_()
        em0, em1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        em0.record(stream)
        layer3.merge_lora(merged["q"], merged["k"], merged["v"], merged["o"])
        em1.record(stream)
        em1.synchronize()
        merge_ms = em0.elapsed_time(em1)
        ms3, _, _ = device_steps(wl3, td3, layer3, max(3, args.steps // 2), args.warmup, False)
        max3 = dp.max_over_ranks(sum(ms3), world, dev)
        fl3 = 4.0 * wl3.batch * wl3.dims.n_q_heads * wl3.img_tokens * (wl3.prefix + wl3.img_tokens) * wl3.dims.head_dim
        fl3 += 2.0 * wl3.batch * wl3.img_tokens * wl3.dims.hidden * (
            (wl3.dims.n_q_heads + 2 * wl3.dims.n_kv_heads) * wl3.dims.head_dim + wl3.dims.n_q_heads * wl3.dims.head_dim)
        also = [also, {"workload": wl3.name, "value": dp.aggregate_rate(wl3.batch * wl3.img_tokens, len(ms3), max3, world),
                       "ms_per_step": max3 / len(ms3), "tflops": fl3 / (max3 / len(ms3) / 1e3) / 1e12,
                       "merge_lora_ms": merge_ms}]
        layer3.close()
        # the 512^2 single-branch workload (the smallest; latency-bound)
        wl0, _, td0, layer0 = make(0)
        ms0, st0, _ = device_steps(wl0, td0, layer0, max(3, args.steps // 2), args.warmup, True)
        max0 = dp.max_over_ranks(sum(ms0), world, dev)
        fl0 = sum(stage_work(wl0, n)[0] for n in st0)
        also.insert(0, {"workload": wl0.name, "value": dp.aggregate_rate(wl0.batch * wl0.img_tokens, len(ms0), max0, world),
                        "ms_per_step": max0 / len(ms0), "tflops": fl0 / (max0 / len(ms0) / 1e3) / 1e12,
                        "attn_ms": sum(st0.get("attn_fwd", [0.0])) / len(ms0)})
        layer0.close()

    # the gen-tower SwiGLU MLP on the same token counts
    mlp = None
    if not args.skip_mlp:
        mlp = mlp_steps(dev, flush, stream, args, world)

    # the A3B tower's mixture-of-experts MLP
    moe = None
    if not args.skip_mlp:
        moe = moe_bench(dev, flush, stream, args, world)

    # one full denoise step (42 layers) and the prefix-tower layer
    denoise = None
    if not args.skip_step:
        denoise = denoise_step_bench(dev, flush, stream, args, world)

    # sustained: back-to-back 2048^2 CFG forwards for >= 2 s, clocks sampled
    sustained = None
    if args.sustained_s > 0:
        sustained = sustained_steps(make(WORKLOAD_INDEX), dev, stream, args, world, local)

    if rank == 0:
        peaks, peak_kind = load_peaks()
        total_flops = sum(stage_work(wl, s)[0] for s in stages)
        stage_summary = {}
        for name, v in stages.items():
            fl, by = stage_work(wl, name)
            avg = sum(v) / args.steps  # per step (a stage may launch more than once per step)
            stage_summary[name] = {"ms": avg, "share": sum(v) / sum(sum(x) for x in stages.values()),
                                   "tflops": fl / (avg / 1e3) / 1e12 if fl else None,
                                   "gbs": by / (avg / 1e3) / 1e9}
        top = max(stages, key=lambda n: sum(stages[n]))
        fl, by = stage_work(wl, top)
        avg_top = sum(stages[top]) / args.steps
        if fl > 0:
            achieved, peak, unit, bound = fl / (avg_top / 1e3) / 1e12, peaks["bf16_tflops"], "TFLOP/s", "tensor"
        else:
            achieved, peak, unit, bound = by / (avg_top / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s", "hbm"
        traffic = kernel_traffic(top)
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            rows = args.cpu_rows
            tcpu = oracle_sample(wl, t_cpu, rows)
            cpu = {"value": wl.batch * rows / tcpu, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                   "sample": f"one oracle forward over {rows} of {wl.img_tokens} query rows per branch "
                             f"({wl.batch} branches; K/V of all tokens projected), {tcpu:.1f} s"}
        layer_tflops = total_flops / (ms_per_step / 1e3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16+f16 (f32 accumulate)", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.batch, "img_tokens": wl.img_tokens,
                       "prefix": wl.prefix, "lora_rank": wl.lora_rank, "hidden": wl.dims.hidden,
                       "heads": [wl.dims.n_q_heads, wl.dims.n_kv_heads], "head_dim": wl.dims.head_dim,
                       "parallelism": f"independent layer call per GPU x{world}",
                       "l2": "flushed (256 MiB write) before every timed step; e2e: not flushed, each "
                             "step's inputs arrive by DMA from host memory into one of two 137 MB staging slots"},
            "layer_tflops": layer_tflops,
            "pct_of_bf16_peak": 100.0 * layer_tflops / peaks["bf16_tflops"],
            "roofline": {"bound": bound, "kernel": top, "achieved": achieved, "peak": peak, "unit": unit,
                         "frac": achieved / peak, "traffic": traffic,
                         "peak_source": f"{peak_kind} (burst)"},
            "stages": stage_summary,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "call": "mot_attn_forward_host (pinned host buffers, two device staging slots; copy-in of "
                            "step i+1 and copy-out of step i-1 overlap the layer of step i)",
                    "serial_value": serial_value},
            "gpu_launches": launches * world,
            "clocks": clk,
            "also": also,
            "train": train,
            "mlp": mlp,
            "denoise_step": denoise,
            "moe": moe,
            "sustained": sustained,
            "unflushed": {"ms_per_step": unflushed, "value": dp.aggregate_rate(tokens, 1, unflushed, world),
                          "note": "same steps back to back, L2 not flushed", "clocks": unflushed_clocks},
        }
        print(json.dumps(line), flush=True)
    layer.close()
    dp.finish(world)
    return 0


def run_rank_check(args):
    """The rank plumbing of run_ours on CPU (gloo): group, per-rank data
    shards, barrier, max over ranks of each rank's time and the whole-job
    rate; rank 0 prints one JSON line. For the multi-process CPU tests."""
    import torch
    from mot_flow_matching_b200 import dp, synth
    world, rank, local = dp.world_info()
    dp.init_group(world, "gloo", timeout_s=60)
    wl = synth.tiny_workload()
    t = synth.make_inputs(wl, 77, shard=rank)
    dp.barrier(world)
    t0 = time.perf_counter()
    ref = sum(float(v.float().sum()) for k, v in t.items() if k != "prefix_len")
    ms = (time.perf_counter() - t0) * 1e3 + 1.0
    total = dp.max_over_ranks(ms * args.steps, world)
    sums = torch.tensor([ref], dtype=torch.float64)
    gathered = [torch.zeros_like(sums) for _ in range(world)]
    if world > 1:
        torch.distributed.all_gather(gathered, sums)
    else:
        gathered = [sums]
    if rank == 0:
        print(json.dumps({"check": "ranks", "n_gpus": world, "local_rank": local, "steps": args.steps,
                          "value": dp.aggregate_rate(wl.batch * wl.img_tokens, args.steps, total, world),
                          "shard_sums": [float(g[0]) for g in gathered]}), flush=True)
    dp.finish(world)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--skip-also", action="store_true")
    ap.add_argument("--skip-train", action="store_true")
    ap.add_argument("--skip-mlp", action="store_true")
    ap.add_argument("--skip-step", action="store_true", help="skip the 42-layer denoise step and the prefix layer")
    ap.add_argument("--sustained-s", type=float, default=2.0,
                    help="seconds of back-to-back forwards for the sustained figure (0: skip)")
    ap.add_argument("--cpu-rows", type=int, default=512)
    ap.add_argument("--ref-rows", type=int, default=128)
    ap.add_argument("--once", action="store_true", help="one warm forward, no timing (ncu target)")
    ap.add_argument("--workload", type=int, default=WORKLOAD_INDEX)
    ap.add_argument("--train", action="store_true", help="with --once: forward keeping activations + backward")
    ap.add_argument("--mlp", action="store_true", help="with --once: the gen-tower MLP instead of the attention")
    ap.add_argument("--moe", action="store_true", help="with --once: the A3B mixture-of-experts MLP")
    ap.add_argument("--check-ranks", action="store_true",
                    help="CPU check of the rank plumbing (gloo): spawn/launcher handling, shards, max over ranks")
    args = ap.parse_args()
    if args.once:
        return run_once(args)
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    # --gpus N means N ranks, one per GPU: as launched by torchrun (whose
    # WORLD_SIZE must then be N), or started here when no launcher did
    from mot_flow_matching_b200 import dp
    try:
        how = dp.check_world(args.gpus)
    except ValueError as e:
        print(f"bench.py: {e}", file=sys.stderr)
        return 2
    if how == "spawn":
        return dp.spawn_local_ranks(args.gpus, [sys.executable, os.path.abspath(__file__)] + sys.argv[1:])
    if args.check_ranks:
        return run_rank_check(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
