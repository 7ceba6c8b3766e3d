"""Context parallelism for one long sequence, in fp64 on the CPU: the exchange step
that would let several GPUs share one sequence, pinned against the token-by-token
oracle, once in one process and once over two and three gloo ranks.

The erase-then-write update (write-up of "On the Design of Qwen3.8-Next
Architecture", 模块 A, 递归状态) is affine in the state:
S_t = A_t S_{t-1} + B_t with A_t = alpha_t (I - beta_t k_t k_t^T) and
B_t = beta_t k_t v_t^T. A segment of tokens therefore maps its start state to its
end state by S -> M S + N:
- M = prod A_t: the segment run from S = I with v = 0;
- N: the segment run from S = 0.
Each rank reduces its segment to (M, N); the ranks all-gather the maps, and rank
r composes those of ranks < r into its start state; then it recomputes its
segment's outputs from that state. One exchange of d_k (d_k + d_v) floats per
head and rank, whatever the segment length.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle


def _sequence(T, dk, dv, seed):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, dk)); q /= np.linalg.norm(q, axis=1, keepdims=True)
    k = rng.standard_normal((T, dk)); k /= np.linalg.norm(k, axis=1, keepdims=True)
    v = rng.standard_normal((T, dv))
    alpha = np.exp(-rng.uniform(0.01, 0.1) * np.logaddexp(0, rng.standard_normal(T) - 2))   # long memory
    beta = 1 / (1 + np.exp(-rng.standard_normal(T)))
    S0 = 0.14 * rng.standard_normal((dk, dv))
    return q, k, v, alpha, beta, S0


def segment_map(q, k, v, alpha, beta):
    """(M [dk, dk], N [dk, dv]) with end state = M S + N for any start state S."""
    dk = k.shape[1]
    _, M = oracle.delta_rule(q, k, np.zeros((q.shape[0], dk)), alpha, beta, np.eye(dk))
    _, N = oracle.delta_rule(q, k, v, alpha, beta, np.zeros((dk, v.shape[1])))
    return M, N


def start_state(maps, r, S0):
    """The state entering segment r: the maps of segments 0 .. r-1 applied to S0."""
    S = S0
    for M, N in maps[:r]:
        S = M @ S + N
    return S


def _bounds(T, P):
    return [(T * p) // P for p in range(P + 1)]


@pytest.mark.parametrize("P", [1, 2, 5])
def test_segment_maps_compose_to_the_sequence(P):
    T, dk, dv = 97, 12, 7
    q, k, v, alpha, beta, S0 = _sequence(T, dk, dv, 40 + P)
    y_ref, S_ref = oracle.delta_rule(q, k, v, alpha, beta, S0)
    b = _bounds(T, P)
    maps = [segment_map(q[b[p]:b[p + 1]], k[b[p]:b[p + 1]], v[b[p]:b[p + 1]], alpha[b[p]:b[p + 1]],
                        beta[b[p]:b[p + 1]]) for p in range(P)]
    ys = []
    for p in range(P):
        sl = slice(b[p], b[p + 1])
        y, _ = oracle.delta_rule(q[sl], k[sl], v[sl], alpha[sl], beta[sl], start_state(maps, p, S0))
        ys.append(y)
    S_end = start_state(maps, P, S0)
    np.testing.assert_allclose(np.concatenate(ys), y_ref, rtol=0, atol=1e-12 * np.abs(y_ref).max())
    np.testing.assert_allclose(S_end, S_ref, rtol=0, atol=1e-12 * np.abs(S_ref).max())


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


T_CP, DK, DV, SEED = 120, 8, 5, 77


def _rank_main(rank, world, port, outdir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank))
    torch.distributed.init_process_group("gloo", timeout=__import__("datetime").timedelta(seconds=60))
    q, k, v, alpha, beta, S0 = _sequence(T_CP, DK, DV, SEED)
    b = _bounds(T_CP, world)
    sl = slice(b[rank], b[rank + 1])
    M, N = segment_map(q[sl], k[sl], v[sl], alpha[sl], beta[sl])
    mine = torch.from_numpy(np.concatenate([M, N], axis=1))          # the one exchange: [dk, dk + dv]
    got = [torch.empty_like(mine) for _ in range(world)]
    torch.distributed.all_gather(got, mine)
    maps = [(g[:, :DK].numpy(), g[:, DK:].numpy()) for g in got]
    y, _ = oracle.delta_rule(q[sl], k[sl], v[sl], alpha[sl], beta[sl], start_state(maps, rank, S0))
    np.save(os.path.join(outdir, f"y{rank}.npy"), y)
    if rank == world - 1:
        np.save(os.path.join(outdir, "S_end.npy"), start_state(maps, world, S0))
    torch.distributed.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_over_gloo(tmp_path, world):
    ctx = mp.get_context("spawn")
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, str(tmp_path))) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    q, k, v, alpha, beta, S0 = _sequence(T_CP, DK, DV, SEED)
    y_ref, S_ref = oracle.delta_rule(q, k, v, alpha, beta, S0)
    y = np.concatenate([np.load(tmp_path / f"y{r}.npy") for r in range(world)])
    np.testing.assert_allclose(y, y_ref, rtol=0, atol=1e-12 * np.abs(y_ref).max())
    np.testing.assert_allclose(np.load(tmp_path / "S_end.npy"), S_ref, rtol=0, atol=1e-12 * np.abs(S_ref).max())
