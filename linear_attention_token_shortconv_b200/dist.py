"""Rank plumbing for data-parallel runs of the GDN token mixer: one process per
GPU, each solving its own independent problem.

(Sequence, head) chains of the gated delta rule share nothing, so N ranks run N
independent problems with no collective on the data path (weak scaling).  The
only collectives are the barriers around a timed region and the max-over-ranks
reduction of its duration; every rank takes them in the same order.
"""
from __future__ import annotations

import os
import socket
import subprocess
import sys
from datetime import timedelta

import torch
import torch.distributed as dist

SEED_STRIDE = 1000   # rank r draws its problem with seed base + SEED_STRIDE * r


def env_ranks() -> tuple[int, int, int]:
    """(world size, global rank, local rank) from the launcher's environment."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def free_port() -> int:
    """A TCP port on 127.0.0.1 that is free right now (for a rendezvous)."""
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def launch(n: int, script: str, argv: list, env: dict | None = None) -> int:
    """Runs `python script *argv` as n ranks on this node, one process per rank,
    under torch.distributed.run with the rendezvous on 127.0.0.1 and a free port;
    every rank finds RANK, LOCAL_RANK, WORLD_SIZE and MASTER_* in its
    environment.  Returns the launcher's exit code (non-zero if any rank failed)."""
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr", "127.0.0.1", f"--master-port={free_port()}", script, *argv]
    full_env = dict(os.environ)
    for k in ("RANK", "LOCAL_RANK", "WORLD_SIZE", "MASTER_ADDR", "MASTER_PORT"):
        full_env.pop(k, None)
    full_env.update(env or {})
    return subprocess.run(cmd, env=full_env).returncode


def group_size() -> int:
    """World size of the joined process group (1 when no group was joined)."""
    return dist.get_world_size() if dist.is_available() and dist.is_initialized() else 1


def setup(backend: str = "nccl", timeout_s: float = 300.0) -> tuple[int, int, int]:
    """Joins the process group when more than one rank runs; with NCCL the rank
    is bound to GPU LOCAL_RANK first."""
    world, rank, local = env_ranks()
    if world > 1:
        kw = {}
        if backend == "nccl":
            torch.cuda.set_device(local)
            kw["device_id"] = torch.device("cuda", local)
        dist.init_process_group(backend, timeout=timedelta(seconds=timeout_s), **kw)
    return world, rank, local


def barrier(world: int) -> None:
    if world > 1:
        dist.barrier()


def max_over_ranks(x: float, world: int, device: torch.device | str = "cuda") -> float:
    """The largest of every rank's x (a duration: the job ends with its slowest rank)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def shard_seed(base: int, rank: int) -> int:
    """Seed of rank `rank`'s problem: distinct per rank, rank 0 keeps the base."""
    return base + SEED_STRIDE * rank


def job_throughput(world: int, units_per_rank: float, ms_per_step: float) -> float:
    """Whole-job units per second: every rank's units over the slowest rank's time."""
    return world * units_per_rank / (ms_per_step * 1e-3)
