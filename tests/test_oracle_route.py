"""Pins of the oracle's route (softmax + top-k): hand-worked cases, brute force
over every k-subset on tiny inputs, torch.topk on tie-free rows, and
torch.softmax in float64 for the weights."""
import itertools

import numpy as np
import pytest
import torch

from conftest import load_golden
from harness import inputs


def test_route_hand_cases(oracle_mod):
    for c in load_golden("route_hand.json")["cases"]:
        logits = np.array([c["logits"]], np.float32)
        idx, w = oracle_mod.route(logits, c["k"])
        assert idx[0].tolist() == c["topk_idx"], c["name"]
        if "topk_w" in c:
            assert w[0].tolist() == c["topk_w"], c["name"]
            _, wr = oracle_mod.route(logits, c["k"], renormalize=True)
            assert wr[0].tolist() == c["topk_w_renormalized"], c["name"]


def _brute_force_set(row, k):
    """The k-subset with the largest logit sum; among equal sums the one whose
    sorted index list is lexicographically smallest."""
    best, best_key = None, None
    for sub in itertools.combinations(range(len(row)), k):
        s = sum(float(row[e]) for e in sub)
        key = (-s, sub)
        if best_key is None or key < best_key:
            best, best_key = sub, key
    return set(best)


@pytest.mark.parametrize("E,k,levels", [(5, 2, 3), (6, 3, 2), (7, 1, 4), (6, 6, 2), (8, 4, 3)])
def test_route_brute_force_subsets_with_ties(oracle_mod, E, k, levels):
    logits, _ = inputs.make_random_case(40, 8, E, k, seed=100 + E * 10 + k, tie_levels=levels)
    logits = logits.numpy()
    idx, _ = oracle_mod.route(logits, k)
    for g in range(logits.shape[0]):
        assert set(idx[g].tolist()) == _brute_force_set(logits[g], k)
        # order: non-increasing logits, ascending index among equal logits
        vals = logits[g][idx[g]]
        for a, b, ia, ib in zip(vals, vals[1:], idx[g], idx[g][1:]):
            assert a > b or (a == b and ia < ib)


@pytest.mark.parametrize("E,k", [(8, 2), (64, 8), (256, 8), (384, 8)])
def test_route_matches_torch_topk_and_softmax(oracle_mod, E, k):
    logits, _ = inputs.make_random_case(64, 8, E, k, seed=E + k)
    idx, w = oracle_mod.route(logits.numpy(), k)
    # tie-free rows: torch.topk gives the same indices in descending order
    ti = torch.topk(logits, k, dim=1, largest=True, sorted=True).indices.numpy()
    assert np.array_equal(idx, ti)
    p = torch.softmax(logits.double(), dim=1)
    want = torch.gather(p, 1, torch.from_numpy(idx).long()).numpy()
    # oracle = binary64 value rounded once to binary32: within one binary32 ulp
    ulp = np.spacing(want.astype(np.float32))
    assert np.all(np.abs(w.astype(np.float64) - want) <= ulp)
    # renormalised: softmax over the chosen logits only
    _, wr = oracle_mod.route(logits.numpy(), k, renormalize=True)
    chosen = torch.gather(logits.double(), 1, torch.from_numpy(idx).long())
    want_r = torch.softmax(chosen, dim=1).numpy()
    assert np.all(np.abs(wr.astype(np.float64) - want_r) <= np.spacing(want_r.astype(np.float32)))
    assert np.allclose(wr.astype(np.float64).sum(1), 1.0, atol=k * 2 ** -23)


def test_route_weights_sum_to_one_over_all_experts(oracle_mod):
    logits, _ = inputs.make_random_case(16, 8, 12, 12, seed=5)
    _, w = oracle_mod.route(logits.numpy(), 12)   # k = E: every probability
    assert np.allclose(w.astype(np.float64).sum(1), 1.0, atol=12 * 2 ** -24)
    assert np.all(np.diff(w, axis=1) <= 0)        # weights descend along j


def test_route_zipf_bias_makes_expert0_hottest():
    cfg = inputs.CONFIGS["kimi"]
    b = inputs.zipf_bias(cfg.E, cfg.zipf).double()
    assert abs(torch.logsumexp(b, 0).item()) < 1e-6
    assert torch.all(b[1:] < b[:-1])
