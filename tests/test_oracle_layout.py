"""Pins of the oracle's layout: hand-worked cases, a brute-force counting
restatement of every slot on tiny inputs, and the invariants the pages fix
(counts sum to T*k, every slot lands once, per-expert regions are contiguous
and grouped by logical rank, the per-rank receive bound)."""
import numpy as np
import pytest

from conftest import load_golden
from harness import inputs


@pytest.mark.parametrize("case", load_golden("layout_hand.json")["cases"], ids=lambda c: c["name"])
def test_layout_hand_cases(oracle_mod, case):
    idx = np.array(case["topk_idx"], np.int32)
    out = oracle_mod.layout(idx, case["E"], case["R"], case["capacity"], case["rows"])
    assert out["status"] == case["status"]
    for key in ["expert_counts", "expert_src_counts", "rank_counts", "expert_offsets",
                "dispatch_pos", "recv_src"]:
        assert out[key].tolist() == case[key], key


def _random_idx(T, E, k, seed, skew=0.0, masked=0.0):
    rng = np.random.default_rng(seed)
    idx = np.empty((T, k), np.int32)
    p = None
    if skew:
        p = (np.arange(1, E + 1) ** -skew)
        p /= p.sum()
    for g in range(T):
        idx[g] = rng.choice(E, size=k, replace=False, p=p)
    if masked:
        idx[rng.random((T, k)) < masked] = -1
    return idx


def _brute(idx, E, capacity):
    """Restate each slot by counting: its position inside expert e is the
    number of earlier slots (smaller flat index) routed to e; the packed base
    of e is the number of slots routed to experts below e."""
    flat = idx.ravel()
    valid = (flat >= 0) & (flat < E)
    pos = np.full(flat.shape, -1, np.int64)
    for i, e in enumerate(flat):
        if not valid[i]:
            continue
        p = int(np.sum(flat[:i] == e))
        if capacity:
            pos[i] = e * capacity + p if p < capacity else -1
        else:
            pos[i] = int(np.sum(valid & (flat < e))) + p
    return pos.reshape(idx.shape)


@pytest.mark.parametrize("T,E,k,R,cap,masked", [
    (6, 4, 2, 2, 0, 0.0), (9, 6, 3, 3, 0, 0.2), (8, 5, 1, 1, 0, 0.0),
    (10, 4, 2, 2, 3, 0.0), (12, 8, 4, 4, 5, 0.1), (4, 3, 3, 1, 0, 0.0)])
def test_layout_brute_force_tiny(oracle_mod, T, E, k, R, cap, masked):
    idx = _random_idx(T, E, k, seed=T * 100 + E, masked=masked)
    rows = T * k if cap == 0 else E * cap
    out = oracle_mod.layout(idx, E, R, cap, rows)
    assert np.array_equal(out["dispatch_pos"], _brute(idx, E, cap))
    flat = idx.ravel()
    assert out["expert_counts"].tolist() == [int(np.sum(flat == e)) for e in range(E)]


def _check_invariants(idx, out, E, R, cap):
    T, k = idx.shape
    L = E // R
    Tr = T // R
    counts = out["expert_counts"]
    pos = out["dispatch_pos"].ravel()
    src = out["recv_src"]
    off = out["expert_offsets"]
    valid = idx.ravel() >= 0
    # counts sum to the number of routed slots (T*k when nothing is masked)
    assert counts.sum() == valid.sum()
    assert np.array_equal(out["expert_src_counts"].sum(1), counts)
    assert np.array_equal(out["rank_counts"], counts.reshape(R, L).sum(1))
    # source-rank counts equal a direct tally of each rank's tokens
    for r in range(R):
        part = idx[r * Tr:(r + 1) * Tr].ravel()
        assert np.array_equal(out["expert_src_counts"][:, r],
                              [int(np.sum(part == e)) for e in range(E)])
    # each expert receives at most T rows; each rank at most T*min(k, L)
    assert counts.max(initial=0) <= T
    assert out["rank_counts"].max(initial=0) <= T * min(k, L)
    # every kept slot lands exactly once and the inverse map points back
    kept = np.nonzero(pos >= 0)[0]
    assert len(np.unique(pos[kept])) == len(kept)
    assert np.array_equal(src[pos[kept]], kept)
    assert np.sum(src >= 0) == len(kept)
    # contiguous expert regions, rows ascending in flat index (g then j)
    for e in range(E):
        rows_e = np.sort(pos[(idx.ravel() == e) & (pos >= 0)])
        n = len(rows_e)
        assert np.array_equal(rows_e, off[e] + np.arange(n))
        assert np.all(np.diff(src[rows_e]) > 0)
        if cap:
            assert off[e] == e * cap and n == min(counts[e], cap)
    if not cap:
        assert np.array_equal(off, np.concatenate([[0], np.cumsum(counts)]))
        # rank r's region is experts [r*L, (r+1)*L): laid out by logical rank
        assert np.array_equal(off[(np.arange(R) + 1) * L] - off[np.arange(R) * L],
                              out["rank_counts"])


@pytest.mark.parametrize("name", ["tiny", "mixtral", "dsv3", "kimi"])
def test_layout_invariants_on_workload_routing(oracle_mod, name):
    cfg = inputs.CONFIGS[name]
    idx, _ = oracle_mod.route(inputs.make_logits(cfg).numpy(), cfg.k)
    out = oracle_mod.layout(idx, cfg.E, cfg.R)
    assert out["status"] == oracle_mod.OK
    _check_invariants(idx, out, cfg.E, cfg.R, 0)


@pytest.mark.parametrize("cap_frac", [1.0, 0.5])
def test_layout_padded_invariants_and_capacity(oracle_mod, cap_frac):
    T, E, k, R = 512, 16, 4, 4
    idx = _random_idx(T, E, k, seed=11, skew=1.2)
    packed = oracle_mod.layout(idx, E, R)
    cap = max(1, int(packed["expert_counts"].max() * cap_frac))
    out = oracle_mod.layout(idx, E, R, cap)
    want_status = oracle_mod.OK if cap_frac == 1.0 else oracle_mod.ERR_CAPACITY
    assert out["status"] == want_status
    _check_invariants(idx, out, E, R, cap)
    # with cap = max count nothing is dropped
    if cap_frac == 1.0:
        assert np.all(out["dispatch_pos"] >= 0)


def test_layout_masked_slots_and_empty(oracle_mod):
    idx = _random_idx(64, 8, 3, seed=12, masked=0.3)
    out = oracle_mod.layout(idx, 8, 4)
    _check_invariants(idx, out, 8, 4, 0)
    empty = oracle_mod.layout(np.zeros((0, 2), np.int32), 8, 2)
    assert empty["status"] == oracle_mod.OK
    assert empty["expert_counts"].tolist() == [0] * 8
    assert empty["expert_offsets"].tolist() == [0] * 9


# ------------------------------------------------- two-phase (private regions)

@pytest.mark.parametrize("case", load_golden("private_layout_hand.json")["cases"],
                         ids=lambda c: f"max_m{c['max_m']}")
def test_private_layout_hand_cases(oracle_mod, case):
    fx = load_golden("private_layout_hand.json")
    idx = np.array(fx["topk_idx"], np.int32)
    pos, base, src, st = oracle_mod.private_layout(idx, fx["E"], fx["R"], case["max_m"])
    assert st == case["status"]
    assert pos.tolist() == case["private_pos"]
    assert base.tolist() == fx["region_base"]
    kept = pos.ravel() >= 0
    assert np.array_equal(src[pos.ravel()[kept]], np.nonzero(kept)[0])
    assert np.sum(src >= 0) == kept.sum()


@pytest.mark.parametrize("name", ["tiny", "dsv3", "kimi"])
def test_private_layout_reproduces_packed_rows(oracle_mod, name):
    """region_base[e][r] + (position in the private region) is the slot's
    packed row: compacting the private regions gives the direct layout."""
    cfg = inputs.CONFIGS[name]
    idx, _ = oracle_mod.route(inputs.make_logits(cfg).numpy(), cfg.k)
    packed = oracle_mod.layout(idx, cfg.E, cfg.R)
    pos, base, src, st = oracle_mod.private_layout(idx, cfg.E, cfg.R, cfg.T_r)
    assert st == oracle_mod.OK
    max_m = cfg.T_r
    region = pos // max_m
    p = pos - region * max_m
    assert np.array_equal(base.ravel()[region] + p, packed["dispatch_pos"])
    # regions are (expert, source rank) pairs
    ranks = (np.arange(cfg.T) // cfg.T_r)[:, None]
    assert np.array_equal(region, idx * cfg.R + ranks)
