"""GPU QSA indexer vs the fp64 oracle.

Scores: normwise over the complete blocks.  Selection: the block indices are
decided by the scores, which the kernel forms from fp16-rounded rotated rows
(fp32 accumulation) and the oracle in fp64, so a block whose oracle score lies
within twice the row's largest score difference (kernel vs oracle) of the row's
threshold (the K_B-th largest oracle score) may go either way; every other
block must agree exactly, and the kernel's set must be a valid selection: K_B
distinct complete blocks (or all of them when fewer), ascending, padded with -1.  With all queries zero every score is 0 and
the tie rule alone decides: the result must be bit-exact.
"""
from dataclasses import replace

import numpy as np
import pytest
import torch

from harness import normwise
from linear_attention_token_shortconv_b200 import gdn
from linear_attention_token_shortconv_b200.workloads import QSA, make_qsa_inputs
from oracle import qsa as oq

pytestmark = pytest.mark.gpu

TOL_SCORE = 2e-3   # normwise; fp16 rows (2^-11 relative) summed over 128 dims and 4 heads

CASES = [
    ("B2-n300-K64", replace(QSA, B=2, n=300, budget=64)),            # ragged tiles, radix path
    ("n1030-K2048", replace(QSA, n=1030, budget=2048)),              # fewer complete blocks than K_B
    ("n4101-K512", replace(QSA, n=4101, budget=512, seed=7)),        # several block tiles, n % 4 = 1
]


def _oracle_row_check(I_row, sel_row, n_valid, KB, tol_abs):
    """The kernel's selection for one row against the oracle scores of that row."""
    m = min(KB, n_valid)
    chosen = sel_row[:m]
    assert np.all(sel_row[m:] == -1)
    assert np.all(np.diff(chosen) > 0) and (m == 0 or (chosen[0] >= 0 and chosen[-1] < n_valid))
    if n_valid <= KB:
        assert chosen.tolist() == list(range(n_valid))
        return 0
    valid = I_row[:n_valid]
    order = sorted(range(n_valid), key=lambda b: (-valid[b], b))
    want = np.sort(order[:KB])
    T = valid[order[KB - 1]]
    diff = np.setxor1d(want, chosen)
    near = np.abs(valid[diff] - T) <= tol_abs
    assert np.all(near), (diff[~near], valid[diff[~near]], T)
    return len(diff)


@pytest.mark.parametrize("name,cfg", CASES, ids=[c[0] for c in CASES])
def test_qsa_matches_oracle(cuda_device, name, cfg):
    inp = make_qsa_inputs(cfg, "cpu")
    dev = {key: val.to(cuda_device) for key, val in inp.items()}
    sel, sc = gdn.qsa_indexer(dev["q"], dev["k"], dev["w_q"], dev["w_k"], budget=cfg.budget, want_scores=True)
    torch.cuda.synchronize()
    sel, sc = sel.cpu().numpy(), sc.cpu().numpy()
    KB, nb = cfg.budget // 4, cfg.n // 4
    worst, n_near = 0.0, 0
    for s in range(cfg.B):
        q = inp["q"][s].float().numpy()
        k = inp["k"][s].float().numpy()
        I = oq.scores(q, k, inp["w_q"].numpy(), inp["w_k"].numpy())
        valid = np.isfinite(I)
        err = normwise(sc[s][valid], I[valid])
        worst = max(worst, err)
        for i in range(cfg.n):
            nv = (i + 1) // 4
            tol_abs = 2 * np.abs(sc[s, i, :nv] - I[i, :nv]).max() if nv else 0.0
            n_near += _oracle_row_check(I[i], sel[s, i], nv, KB, tol_abs)
    print(f"{name}: score error {worst:.1e}, near-tie swaps {n_near}")
    assert worst <= TOL_SCORE


def test_qsa_ties_are_bit_exact(cuda_device):
    """All queries zero: every complete block scores 0; the smallest indices win."""
    cfg = replace(QSA, B=1, n=700, budget=32)
    inp = make_qsa_inputs(cfg, "cpu")
    q = torch.zeros_like(inp["q"]).to(cuda_device)
    sel, _ = gdn.qsa_indexer(q, inp["k"].to(cuda_device), inp["w_q"].to(cuda_device), inp["w_k"].to(cuda_device),
                             budget=cfg.budget)
    torch.cuda.synchronize()
    want, _ = oq.indexer(np.zeros((cfg.n, 4, 128)), inp["k"][0].float().numpy(), inp["w_q"].numpy(),
                         inp["w_k"].numpy(), K=cfg.budget)
    np.testing.assert_array_equal(sel[0].cpu().numpy(), want)


def test_qsa_equal_positive_scores(cuda_device):
    """Keys that live in the unrotated dims 64..127 only and are the same for every
    token: every block's pooled, rotated key is the same vector, so all complete
    blocks of a row score the same positive value (bit-identical products).  More
    equal keys than the threshold bucket's candidate list holds: the kernel's
    fallback path; the smallest blocks win, as in the oracle."""
    cfg = replace(QSA, B=1, n=900, budget=64)
    inp = make_qsa_inputs(cfg, "cpu")
    k = torch.zeros_like(inp["k"])
    k[..., 64:] = inp["k"][0, 0, 64:].abs() + 0.5      # one positive key for every token
    q = inp["q"].clone()
    q[..., 64:] = q[..., 64:].abs()                       # positive products in every head
    sel, sc = gdn.qsa_indexer(q.to(cuda_device), k.to(cuda_device), inp["w_q"].to(cuda_device),
                              inp["w_k"].to(cuda_device), budget=cfg.budget, want_scores=True)
    torch.cuda.synchronize()
    sc = sc[0].cpu().numpy()
    last = cfg.n - 1
    assert (sc[last, :(last + 1) // 4] > 0).all() and np.unique(sc[last, :(last + 1) // 4]).size == 1
    want, _ = oq.indexer(q[0].float().numpy(), k[0].float().numpy(), inp["w_q"].numpy(), inp["w_k"].numpy(),
                         K=cfg.budget)
    np.testing.assert_array_equal(sel[0].cpu().numpy(), want)


def test_qsa_full_size_sampled_rows(cuda_device):
    """The bench workload (n = 32768, K = 2048): sampled rows against the oracle."""
    cfg = QSA
    inp = make_qsa_inputs(cfg, "cpu")
    dev = {key: val.to(cuda_device) for key, val in inp.items()}
    sel, sc = gdn.qsa_indexer(dev["q"], dev["k"], dev["w_q"], dev["w_k"], budget=cfg.budget, want_scores=True)
    torch.cuda.synchronize()
    q = inp["q"][0].float().numpy()
    kb = oq.keys(inp["k"][0].float().numpy(), inp["w_k"].numpy())
    rows = [0, 3, 4, 2047, 2051, 4100, 9999, 20000, 32766, 32767]
    KB = cfg.budget // 4
    for i in rows:
        qi = oq.prope(oq.rmsnorm(q[i], inp["w_q"].numpy()), np.full(4, i))
        n_valid = (i + 1) // 4
        I_row = np.maximum(qi @ kb[:n_valid].T, 0.0).sum(axis=0) if n_valid else np.zeros(0)
        got = sc[0, i, :n_valid].cpu().numpy()
        if n_valid:
            assert normwise(got, I_row) <= TOL_SCORE, i
        tol_abs = 2 * np.abs(got - I_row).max() if n_valid else 0.0
        _oracle_row_check(I_row, sel[0, i].cpu().numpy(), n_valid, KB, tol_abs)


def test_qsa_deterministic(cuda_device):
    cfg = CASES[0][1]
    inp = make_qsa_inputs(cfg, cuda_device)
    a, _ = gdn.qsa_indexer(inp["q"], inp["k"], inp["w_q"], inp["w_k"], budget=cfg.budget)
    b, _ = gdn.qsa_indexer(inp["q"], inp["k"], inp["w_q"], inp["w_k"], budget=cfg.budget)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_qsa_rows_past_the_shared_memory_cap(cuda_device):
    """n = 49,203: rows with more than 12,288 complete blocks keep their keys in the
    score row instead of shared memory (and 12,287 blocks: the last row in shared
    memory); sampled rows against the oracle."""
    cfg = replace(QSA, n=49203, budget=2048, seed=11)
    inp = make_qsa_inputs(cfg, "cpu")
    dev = {key: val.to(cuda_device) for key, val in inp.items()}
    sel, sc = gdn.qsa_indexer(dev["q"], dev["k"], dev["w_q"], dev["w_k"], budget=cfg.budget, want_scores=True)
    torch.cuda.synchronize()
    rows = [49150, 49155, 49170, 49202]
    assert (49150 + 1) // 4 <= 12288 < (49155 + 1) // 4
    sel_rows = sel[0, rows].cpu().numpy()
    sc_rows = sc[0, rows].cpu().numpy()
    del sel, sc
    q = inp["q"][0].float().numpy()
    kb = oq.keys(inp["k"][0].float().numpy(), inp["w_k"].numpy())
    KB = cfg.budget // 4
    for r, i in enumerate(rows):
        qi = oq.prope(oq.rmsnorm(q[i], inp["w_q"].numpy()), np.full(4, i))
        n_valid = (i + 1) // 4
        I_row = np.maximum(qi @ kb[:n_valid].T, 0.0).sum(axis=0)
        got = sc_rows[r, :n_valid]
        assert normwise(got, I_row) <= TOL_SCORE, i
        _oracle_row_check(I_row, sel_rows[r], n_valid, KB, 2 * np.abs(got - I_row).max())
