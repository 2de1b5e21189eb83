"""On-device quantile mapping (ace_tau_quantile) against the oracle's
definition of the threshold ([ACE] "Efficiency Results", Table 6): tau is
the (n+1)-th smallest non-top-1 score, bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads

pytestmark = pytest.mark.gpu


def _gpu_tau(pool, n_skip):
    from token_dynamic_expert_b200 import ace
    sc = torch.from_numpy(np.ascontiguousarray(pool, dtype=np.float32)).cuda()
    tau = torch.full((1,), float("nan"), dtype=torch.float32, device="cuda")
    ws = ace.alloc_workspace(ace.ace_tau_workspace_size())
    ws.fill_(0xAB)  # contents need no initialisation
    ace.ace_tau_quantile(sc, n_skip, tau, ws)
    torch.cuda.synchronize()
    return float(tau.item())


def _same(a, b):
    """Equal as fp32 values (-0 and +0 are the same threshold: c < tau
    decides identically)."""
    if math.isinf(a) or math.isinf(b):
        return a == b
    return np.float32(a) == np.float32(b)


@pytest.mark.parametrize("n_tok,k", [(1, 2), (37, 8), (4096, 8), (1000, 16), (5000, 3)])
def test_random_pools_every_budget_edge(n_tok, k):
    rng = np.random.default_rng(n_tok * 31 + k)
    pool = rng.random((n_tok, k), dtype=np.float32) * 0.5
    N = n_tok * (k - 1)
    for n in sorted({-3, 0, 1, N // 3, N // 2, N - 1, N, N + 5}):
        got = _gpu_tau(pool, n)
        ref = oracle.tau_quantile(pool.astype(np.float64), n)
        assert _same(got, ref), (n, got, ref)
        if 0 <= n < N and np.unique(pool[:, 1:]).size == N:   # no ties: exactly n below tau
            assert int((pool[:, 1:] < np.float32(got)).sum()) == n


def test_ties_negative_and_huge_values():
    rng = np.random.default_rng(7)
    vals = np.array([-3.0, -0.0, 0.0, 1e-30, 0.25, 0.25, 0.25, 1e30, -1e30], np.float32)
    pool = rng.choice(vals, size=(300, 8)).astype(np.float32)
    N = 300 * 7
    for n in range(0, N + 1, 97):
        assert _same(_gpu_tau(pool, n), oracle.tau_quantile(pool.astype(np.float64), n)), n


def test_top1_column_is_never_a_candidate():
    pool = np.full((64, 4), 0.5, np.float32)
    pool[:, 0] = -1.0  # smaller than every candidate, but top-1
    assert _gpu_tau(pool, 0) == 0.5
    pool1 = np.ones((10, 1), np.float32)   # k = 1: no candidates at all
    assert math.isinf(_gpu_tau(pool1, 0))


def test_pool_of_forward_scores_matches_the_oracle_quantile():
    """The decode threshold recipe: a 4096-token pool of one layer's scores
    from ace_moe_scores, tau for 60% of all slots."""
    from token_dynamic_expert_b200 import ace
    w = workloads.WORKLOADS["decode_bs8"]
    layer = workloads.make_layer(w, seed=3, device="cuda")
    u = workloads.make_tokens(w, T=w.pool, token_seed=4000, device="cuda")
    amax = torch.linspace(0.5, 1.5, w.E, device="cuda")
    c = ace.make_layer(layer["gamma"], layer["wr"], layer["wg"], layer["wu"], layer["wd"], w.k,
                       amax=amax, router_bias=layer["bias"])
    ws = ace.alloc_workspace(ace.ace_workspace_size(c, w.pool))
    score = torch.empty(w.pool, w.k, dtype=torch.float32, device="cuda")
    ace.ace_moe_scores(c, u, score, ws)
    n = oracle.n_skip_for(w.pool, w.k, w.skip)
    got = _gpu_tau(score.cpu().numpy(), n)
    ref = oracle.tau_quantile(score.cpu().numpy().astype(np.float64), n)
    assert _same(got, ref)
