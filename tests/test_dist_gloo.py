"""The N > 1 host path on CPU: two ranks over gloo run the same rank plumbing
(`dist.setup`, barriers, max over ranks, per-rank problem seeds, whole-job
throughput) that bench.py uses over NCCL, each on its own independent problem."""
import json
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp

from linear_attention_token_shortconv_b200 import dist as rankio
from linear_attention_token_shortconv_b200.workloads import PRETRAIN, make_prefill_inputs, scaled

WORLD = 2
SMALL = scaled(PRETRAIN, lengths=(48, 17), H=2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(WORLD),
                      RANK=str(rank), LOCAL_RANK=str(rank))
    world, r, local = rankio.setup("gloo", timeout_s=60)
    assert (world, r, local) == (WORLD, rank, rank)
    inp = make_prefill_inputs(SMALL, "cpu", seed=rankio.shard_seed(SMALL.seed, rank))
    digest = float(inp["q"].float().sum() + inp["a_logit"].float().sum())
    digests = [None] * world
    torch.distributed.all_gather_object(digests, digest)
    rankio.barrier(world)
    # a rank-dependent "duration": the job's is the slowest rank's
    ms = rankio.max_over_ranks(1.5 + rank, world, "cpu")
    rankio.barrier(world)
    value = rankio.job_throughput(world, SMALL.total_tokens, ms)
    with open(os.path.join(outdir, f"rank{rank}.json"), "w") as f:
        json.dump({"digests": digests, "ms": ms, "value": value}, f)
    torch.distributed.destroy_process_group()


def test_two_ranks_gloo(tmp_path):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, port, str(tmp_path))) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WORLD)]
    # every rank saw the same collective results
    assert res[0] == res[1]
    d = res[0]["digests"]
    # each rank solves its own problem; rank 0's is the single-GPU problem
    assert d[0] != d[1]
    single = make_prefill_inputs(SMALL, "cpu")
    assert d[0] == float(single["q"].float().sum() + single["a_logit"].float().sum())
    assert res[0]["ms"] == 2.5
    assert res[0]["value"] == pytest.approx(WORLD * SMALL.total_tokens / 2.5e-3)


def test_single_rank_helpers_are_local():
    assert rankio.max_over_ranks(3.25, 1) == 3.25
    rankio.barrier(1)
    assert rankio.shard_seed(7, 0) == 7 and rankio.shard_seed(7, 3) == 7 + 3 * rankio.SEED_STRIDE
    assert rankio.job_throughput(1, 1000, 2.0) == pytest.approx(5e5)


def test_launcher_starts_one_process_per_rank(tmp_path):
    """dist.launch (what `bench.py --gpus N` runs when no launcher started it)
    starts N processes that join one process group with distinct ranks."""
    probe = os.path.join(os.path.dirname(os.path.abspath(__file__)), "rank_probe.py")
    rc = rankio.launch(WORLD, probe, [str(tmp_path)])
    assert rc == 0
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(WORLD)]
    for r in res:
        assert r["world"] == WORLD and r["group"] == WORLD
        assert sorted(tuple(x) for x in r["seen"]) == [(0, 0), (1, 1)]
