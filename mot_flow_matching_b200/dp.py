"""Data-parallel plumbing for the layer: one process per GPU.

The layer partitions without exchange: every rank runs its own layer calls
(a shard of the CFG samples or of the training micro-batches) against
replicated weights, so nothing crosses ranks on the data path ("SenseNova-U1"
vLLM-Omni recipe, CFG-parallel: branches are gathered only once per denoise
step, outside the layer). Ranks meet only at barriers and at the final
max-over-ranks of their device time; whole-job throughput is the units all
ranks processed over that slowest time (weak scaling).

Host-side only: the reductions run through whatever process group is
initialised (NCCL on GPUs, gloo in the CPU tests).
"""
import datetime
import os
import socket
import subprocess
from typing import Mapping, Optional, Sequence, Tuple


def world_info(env: Optional[Mapping[str, str]] = None) -> Tuple[int, int, int]:
    """(world size, global rank, local rank) from the launcher's environment."""
    env = os.environ if env is None else env
    world = int(env.get("WORLD_SIZE", "1"))
    rank = int(env.get("RANK", "0"))
    local = int(env.get("LOCAL_RANK", str(rank)))
    if world < 1 or not 0 <= rank < world or local < 0:
        raise ValueError(f"inconsistent launcher environment: WORLD_SIZE={world} RANK={rank} LOCAL_RANK={local}")
    return world, rank, local


def init_group(world: int, backend: str, device=None, timeout_s: float = 120.0) -> None:
    """Join the process group when there is more than one rank. A short
    timeout makes ranks that wait for a missing peer end with an error."""
    if world <= 1:
        return
    import torch.distributed as dist
    kwargs = {"timeout": datetime.timedelta(seconds=timeout_s)}
    if backend == "nccl" and device is not None:
        kwargs["device_id"] = device
    dist.init_process_group(backend, **kwargs)


def barrier(world: int) -> None:
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest `value` over all ranks (every rank gets it)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device if device is not None else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(units_per_rank_per_step: float, steps: int, max_ms: float, world: int) -> float:
    """Whole-job units per second: every rank processed `units_per_rank_per_step`
    units in each of `steps` steps; the job took the slowest rank's `max_ms`."""
    if max_ms <= 0.0:
        raise ValueError("max_ms must be positive")
    return world * units_per_rank_per_step * steps / (max_ms / 1e3)


def finish(world: int) -> None:
    """Last barrier, then leave the process group."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()


def free_port() -> int:
    """A TCP port on 127.0.0.1 that nothing listens on right now."""
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as sock:
        sock.bind(("127.0.0.1", 0))
        return sock.getsockname()[1]


def check_world(requested: int, env: Optional[Mapping[str, str]] = None) -> str:
    """How a command asked for `requested` ranks (one per GPU) should run:
    "run" when it is already one of the launcher's ranks and the launcher's
    world size is the request (or one rank was asked for without a
    launcher), "spawn" when no launcher started it and it must start the
    ranks itself. A launcher world size that differs from the request is an
    error (the job would report a GPU count it did not use)."""
    env = os.environ if env is None else env
    if requested < 1:
        raise ValueError(f"rank count must be >= 1, got {requested}")
    if "WORLD_SIZE" not in env:
        return "spawn" if requested > 1 else "run"
    world, _, _ = world_info(env)
    if world != requested:
        raise ValueError(f"launched with WORLD_SIZE={world} but {requested} ranks were requested")
    return "run"


def spawn_local_ranks(nprocs: int, argv: Sequence[str], master_port: Optional[int] = None,
                      extra_env: Optional[Mapping[str, str]] = None) -> int:
    """Run `argv` as ranks 0..nprocs-1 of one job on this node (rank i on
    local GPU i), the way a launcher would: each child gets RANK, LOCAL_RANK,
    WORLD_SIZE and a MASTER_ADDR/MASTER_PORT on 127.0.0.1, inherits stdout
    and stderr, and is waited for. Returns the first non-zero exit code (0
    when every rank succeeded)."""
    port = master_port or free_port()
    procs = []
    for rank in range(nprocs):
        env = dict(os.environ)
        env.update({"RANK": str(rank), "LOCAL_RANK": str(rank), "WORLD_SIZE": str(nprocs),
                    "LOCAL_WORLD_SIZE": str(nprocs), "MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
        if extra_env:
            env.update(extra_env)
        procs.append(subprocess.Popen(list(argv), env=env))
    codes = [p.wait() for p in procs]
    return next((c for c in codes if c != 0), 0)
