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


# ------------------------------------------------ shared experts and replicas

def test_route_ex_hand_case(oracle_mod):
    fx = load_golden("route_ex_hand.json")
    logits = np.array(fx["logits"], np.float32)
    idx, w, st = oracle_mod.route_ex(logits, fx["k"], fx["n_shared"], fx["shared_weight"],
                                     fx["replica_offsets"], fx["replica_ids"], fx["E_phys"],
                                     fx["T_r"])
    assert st == oracle_mod.OK
    assert idx.tolist() == fx["topk_idx"]
    assert w[:, fx["k"]:].ravel().tolist() == fx["shared_w"]
    # the routed weights are those of the plain route
    _, w_plain = oracle_mod.route(logits, fx["k"])
    assert np.array_equal(w[:, :fx["k"]], w_plain)


def test_route_ex_workload_invariants(oracle_mod):
    cfg = inputs.CONFIGS["dsv3_shared"]
    logits = inputs.make_logits(cfg).numpy()
    offs, ids = inputs.expert_placement(cfg)
    idx, w, st = oracle_mod.route_ex(logits, cfg.k, cfg.n_shared, 1.0, offs, ids, cfg.E_phys,
                                     cfg.T_r)
    assert st == oracle_mod.OK and idx.shape == (cfg.T, cfg.k_total)
    plain_idx, plain_w = oracle_mod.route(logits, cfg.k)
    L, per = cfg.E // cfg.R, cfg.E // cfg.R + cfg.n_shared
    # routed slots: the plain top-k mapped to their physical ids, same weights
    assert np.array_equal(idx[:, :cfg.k], (plain_idx // L) * per + plain_idx % L)
    assert np.array_equal(w[:, :cfg.k], plain_w)
    # shared slot: weight 1, the replica on the token's own logical rank
    ranks = np.arange(cfg.T) // cfg.T_r
    assert np.array_equal(idx[:, cfg.k], ranks * per + L)
    assert np.all(w[:, cfg.k] == 1.0)
    # every rank now receives exactly its own T_r shared slots
    lay = oracle_mod.layout(idx, cfg.E_phys, cfg.R)
    shared_rows = lay["expert_counts"].reshape(cfg.R, per)[:, L]
    assert np.all(shared_rows == cfg.T_r)


def test_route_ex_multi_replica_choice_and_bad_table(oracle_mod):
    logits, _ = inputs.make_random_case(24, 8, 6, 2, seed=31)
    # expert 0 has 3 replicas (ids 6, 7, 8), the others one each (ids 0..5)
    offs = np.array([0, 3, 4, 5, 6, 7, 8], np.int32)
    ids = np.array([6, 7, 8, 1, 2, 3, 4, 5], np.int32)
    idx, _, st = oracle_mod.route_ex(logits.numpy(), 2, 0, 1.0, offs, ids, 9, 4)
    assert st == oracle_mod.OK
    plain, _ = oracle_mod.route(logits.numpy(), 2)
    for g in range(24):
        for j in range(2):
            if plain[g, j] == 0:
                assert idx[g, j] == [6, 7, 8][(g // 4) % 3]
            else:
                assert idx[g, j] == plain[g, j]
    bad = ids.copy()
    bad[4] = 99                        # expert 2's only replica is out of range
    idx_b, _, st_b = oracle_mod.route_ex(logits.numpy(), 2, 0, 1.0, offs, bad, 9, 4)
    assert st_b == oracle_mod.ERR_INVALID
    assert np.all(idx_b[plain == 2] == -1) and np.all(idx_b[plain != 2] == idx[plain != 2])


def test_route_ex_several_shared_experts_and_their_weight(oracle_mod):
    """Shared experts E, E+1, ... follow the routed slots in that order, each
    with the given shared weight; without a replica table every logical id is
    its own physical id."""
    logits, _ = inputs.make_random_case(20, 8, 10, 3, seed=41)
    idx, w, st = oracle_mod.route_ex(logits.numpy(), 3, 2, 0.25, E_phys=12)
    assert st == oracle_mod.OK and idx.shape == (20, 5)
    plain_idx, plain_w = oracle_mod.route(logits.numpy(), 3)
    assert np.array_equal(idx[:, :3], plain_idx) and np.array_equal(w[:, :3], plain_w)
    assert np.all(idx[:, 3] == 10) and np.all(idx[:, 4] == 11)
    assert np.all(w[:, 3:] == np.float32(0.25))
