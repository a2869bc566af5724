"""Parity of the fused route -> layout -> dispatch entry points
(moe_route_dispatch_fp8 / _bf16, one cooperative launch) with the oracle, and
bit-identity with the separate entry points, on the seeded workloads at full
size and on edge shapes: every grid geometry branch (more chunks than CTAs,
more experts than CTAs, one token per chunk, E = 1024), padded layouts with
drops, T = 0, repeated calls on one workspace (the grid barrier must leave
itself ready) and CUDA-graph replay on new inputs."""
import numpy as np
import pytest
import torch

import oracle
from harness import inputs
from gpu_util import gpu_bits, route_w_tol, to_dev, workload

pytestmark = pytest.mark.gpu

LAYOUT_KEYS = ["expert_counts", "expert_src_counts", "rank_counts", "expert_offsets",
               "dispatch_pos", "recv_src"]
PLAIN = ["tiny", "mixtral", "dsv3", "kimi", "prefill"]
GUARD = 3


@pytest.fixture(scope="module")
def moe():
    import combine_moe_route_08_b200 as m
    assert torch.cuda.is_available()
    return m


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _out_buffers(T, E, k, R, H, rows, fp8):
    """Output dict for the fused call, receive rows inside guard rows filled
    with a canary pattern."""
    dev = "cuda"
    out = dict(
        topk_idx=torch.full((T, k), -5, dtype=torch.int32, device=dev),
        topk_w=torch.full((T, k), -5.0, dtype=torch.float32, device=dev),
        expert_counts=torch.full((E,), -5, dtype=torch.int32, device=dev),
        expert_src_counts=torch.full((E, R), -5, dtype=torch.int32, device=dev),
        rank_counts=torch.full((R,), -5, dtype=torch.int32, device=dev),
        expert_offsets=torch.full((E + 1,), -5, dtype=torch.int32, device=dev),
        dispatch_pos=torch.full((T, k), -5, dtype=torch.int32, device=dev),
        recv_src=torch.full((max(rows, 1),), -5, dtype=torch.int32, device=dev),
    )
    n = rows + 2 * GUARD
    if fp8:
        qbuf = torch.full((n, H), 0xA5, dtype=torch.uint8, device=dev)
        sbuf = torch.full((n, H // 128), -1.0, dtype=torch.float32, device=dev)
        out["recv_q"], out["recv_scale"] = qbuf[GUARD:GUARD + rows], sbuf[GUARD:GUARD + rows]
        guards = [(qbuf, 0xA5), (sbuf, -1.0)]
    else:
        xbuf = torch.full((n, H), -7.0, dtype=torch.bfloat16, device=dev)
        out["recv_x"] = xbuf[GUARD:GUARD + rows]
        guards = [(xbuf, -7.0)]
    return out, guards


def _check_guards(guards, rows):
    for buf, fill in guards:
        assert torch.all(buf[:GUARD] == fill) and torch.all(buf[GUARD + rows:] == fill)


def _fused(moe, logits, x, k, R, cap, rows, fp8, renormalize=False, ws=None, st=None):
    T, E = logits.shape
    out, guards = _out_buffers(T, E, k, R, x.shape[1], rows, fp8)
    f = moe.moe_route_dispatch_fp8 if fp8 else moe.moe_route_dispatch_bf16
    f(logits, x, k, R, capacity=cap, rows=rows, renormalize=renormalize, out=out, workspace=ws,
      dev_status=st)
    torch.cuda.synchronize()
    _check_guards(guards, rows)
    return out


def _separate(moe, logits, x, k, R, cap, rows, fp8, renormalize=False):
    """The same step through the separate entry points."""
    E = logits.shape[1]
    idx, w = moe.moe_route_topk(logits, k, renormalize=renormalize)
    return _separate_from(moe, idx, w, x, E, R, cap, rows, fp8)


def _separate_from(moe, idx, w, x, E, R, cap, rows, fp8):
    """Layout and dispatch of a given route through the separate entry points."""
    lay = moe.moe_dispatch_layout(idx, E, R, capacity=cap, rows=rows)
    got = dict(topk_idx=idx, topk_w=w, **{key: lay[key] for key in LAYOUT_KEYS})
    if fp8:
        got["recv_q"], got["recv_scale"] = moe.moe_dispatch_fp8(x, lay["dispatch_pos"], rows)
    else:
        got["recv_x"] = moe.moe_dispatch_bf16(x, lay["dispatch_pos"], rows)
    torch.cuda.synchronize()
    return got


def _assert_same_as_separate(fused, sep, fp8, where):
    filled = sep["recv_src"] >= 0
    for key in ["topk_idx", "topk_w", *LAYOUT_KEYS]:
        a, b = fused[key], sep[key]
        assert torch.equal(a.view(torch.int32), b.view(torch.int32)), f"{where}: {key}"
    if fp8:
        assert torch.equal(fused["recv_q"][filled], sep["recv_q"][filled]), where
        assert torch.equal(fused["recv_scale"][filled].view(torch.int32),
                           sep["recv_scale"][filled].view(torch.int32)), where
    else:
        assert torch.equal(fused["recv_x"][filled].view(torch.int16),
                           sep["recv_x"][filled].view(torch.int16)), where


def _assert_unfilled_untouched(fused, fp8):
    empty = fused["recv_src"] < 0
    if not bool(empty.any()):
        return
    if fp8:
        assert torch.all(fused["recv_q"][empty] == 0xA5)
        assert torch.all(fused["recv_scale"][empty] == -1.0)
    else:
        assert torch.all(fused["recv_x"][empty] == -7.0)


# ---------------------------------------------------------- seeded workloads

@pytest.mark.parametrize("name", PLAIN)
def test_fused_parity_on_workloads(moe, name):
    """Indices and layout bit-exact against the oracle, weights within the
    route's bound, rows bit-exact against the oracle's dispatch (prefill: a
    sample of tokens quantised one by one), and every output bit-identical to
    the separate entry points."""
    wl = workload(name)
    cfg = wl["cfg"]
    fp8 = cfg.dispatch == "fp8"
    logits, x = to_dev(wl["logits"]), to_dev(wl["x"])
    st = _status()
    got = _fused(moe, logits, x, cfg.k, cfg.R, wl["cap"], wl["rows"], fp8, st=st)
    assert st.item() == 0
    assert np.array_equal(got["topk_idx"].cpu().numpy(), wl["idx"])
    w = got["topk_w"].cpu().numpy()
    assert np.all(np.abs(w.astype(np.float64) - wl["w"]) <= route_w_tol(wl["w"]))
    for key in LAYOUT_KEYS:
        assert np.array_equal(got[key].cpu().numpy(),
                              wl["layout"][key].reshape(got[key].shape)), key
    pos_o = wl["layout"]["dispatch_pos"]
    filled = wl["layout"]["recv_src"] >= 0
    if not fp8:
        want = oracle.dispatch_bf16(wl["x_bits"], pos_o, wl["rows"])
        assert np.array_equal(gpu_bits(got["recv_x"])[filled], want[filled])
    elif name != "prefill":
        qo, so = oracle.dispatch_fp8(wl["x_bits"], pos_o, wl["rows"])
        assert np.array_equal(got["recv_q"].cpu().numpy()[filled], qo[filled])
        assert np.array_equal(got["recv_scale"].cpu().numpy()[filled].view(np.uint32),
                              so[filled].view(np.uint32))
    else:
        rng = np.random.default_rng(3)
        tokens = np.unique(np.concatenate([[0, cfg.T - 1, cfg.T_r - 1, cfg.T_r],
                                           rng.choice(cfg.T, 300, replace=False)]))
        tokens = tokens.astype(np.int32)
        qt, st_ = oracle.quantize_tokens(wl["x_bits"], tokens)
        rows_t = torch.from_numpy(pos_o[tokens].ravel().astype(np.int64)).cuda()
        gq = got["recv_q"].index_select(0, rows_t).cpu().numpy().reshape(len(tokens), cfg.k, -1)
        gs = got["recv_scale"].index_select(0, rows_t).cpu().numpy().reshape(len(tokens), cfg.k, -1)
        assert np.array_equal(gq, np.repeat(qt[:, None], cfg.k, 1))
        assert np.array_equal(gs.view(np.uint32), np.repeat(st_[:, None], cfg.k, 1).view(np.uint32))
    _assert_unfilled_untouched(got, fp8)
    sep = _separate(moe, logits, x, cfg.k, cfg.R, wl["cap"], wl["rows"], fp8)
    _assert_same_as_separate(got, sep, fp8, name)


@pytest.mark.parametrize("name", ["dsv3", "mixtral"])
def test_fused_renormalized_route(moe, name):
    wl = workload(name)
    cfg = wl["cfg"]
    fp8 = cfg.dispatch == "fp8"
    logits, x = to_dev(wl["logits"]), to_dev(wl["x"])
    got = _fused(moe, logits, x, cfg.k, cfg.R, 0, cfg.T * cfg.k, fp8, renormalize=True)
    idx_o, w_o = oracle.route(wl["logits"].numpy(), cfg.k, renormalize=True)
    assert np.array_equal(got["topk_idx"].cpu().numpy(), idx_o)
    w = got["topk_w"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(w - w_o) <= route_w_tol(w_o))
    sep = _separate(moe, logits, x, cfg.k, cfg.R, 0, cfg.T * cfg.k, fp8, renormalize=True)
    _assert_same_as_separate(got, sep, fp8, name)


def test_fused_padded_overflow_drops_and_reports(moe):
    wl = workload("kimi")   # skewed: expert 0 is far above the mean
    cfg = wl["cfg"]
    cap = max(1, int(wl["layout"]["expert_counts"].max()) // 2)
    rows = cfg.E * cap + 37
    want = oracle.layout(wl["idx"], cfg.E, cfg.R, cap, rows)
    assert want["status"] == oracle.ERR_CAPACITY
    st = _status()
    logits, x = to_dev(wl["logits"]), to_dev(wl["x"])
    got = _fused(moe, logits, x, cfg.k, cfg.R, cap, rows, True, st=st)
    assert st.item() == moe.MOE_ERR_CAPACITY
    for key in LAYOUT_KEYS:
        assert np.array_equal(got[key].cpu().numpy(), want[key].reshape(got[key].shape)), key
    _assert_unfilled_untouched(got, True)
    sep = _separate(moe, logits, x, cfg.k, cfg.R, cap, rows, True)
    _assert_same_as_separate(got, sep, True, "overflow")


# ------------------------------------------------------------ edge shapes

EDGE = [
    # (T, H, E, k, R, cap, fp8, tie_levels)
    (64, 256, 8, 2, 2, 0, False, 0),          # tiny-like, bf16
    (48, 128, 32, 4, 16, 0, True, 0),         # 3 tokens per rank
    (96, 128, 96, 3, 96, 0, True, 0),         # R = E: one expert per rank, T_r = 1
    (1536, 128, 1024, 32, 4, 0, True, 0),     # E = 1024 (32 logits per lane), k = 32
    (2048, 256, 37, 5, 1, 0, False, 0),       # E not a multiple of 32, one rank
    (16384, 128, 64, 1, 2, 0, True, 0),       # k = 1, many chunks per rank
    (163840, 128, 16, 8, 1, 0, True, 0),      # chunk size capped by slots (4096 / k)
    (640, 128, 320, 6, 320, 0, False, 0),     # more ranks than resident CTAs may hold
    (512, 256, 64, 4, 8, 24, True, 0),        # padded with drops
    (256, 128, 24, 3, 4, 0, True, 3),         # heavy logit ties
    (512, 128, 256, 8, 8, 0, True, 1),        # every logit equal: order by expert id alone
    (64, 16384, 16, 4, 2, 0, True, 0),        # wide rows, FP8
    (64, 10248, 16, 4, 2, 0, False, 0),       # wide rows, bf16, H not a multiple of 128
]


@pytest.mark.parametrize("case", EDGE, ids=lambda c: "T{}_H{}_E{}_k{}_R{}_cap{}_{}".format(
    c[0], c[1], c[2], c[3], c[4], c[5], "fp8" if c[6] else "bf16"))
def test_fused_edge_shapes(moe, case):
    T, H, E, k, R, cap, fp8, ties = case
    logits, x = inputs.make_random_case(T, H, E, k, seed=T + E + k, tie_levels=ties)
    idx_o, _ = oracle.route(logits.numpy(), k)
    lay_o = oracle.layout(idx_o, E, R, cap)
    rows = lay_o["recv_src"].shape[0]
    st = _status()
    got = _fused(moe, to_dev(logits), to_dev(x), k, R, cap, rows, fp8, st=st)
    want_st = moe.MOE_ERR_CAPACITY if lay_o["status"] == oracle.ERR_CAPACITY else 0
    assert st.item() == want_st
    assert np.array_equal(got["topk_idx"].cpu().numpy(), idx_o)
    for key in LAYOUT_KEYS:
        assert np.array_equal(got[key].cpu().numpy(), lay_o[key].reshape(got[key].shape)), key
    filled = lay_o["recv_src"] >= 0
    xb = inputs.bf16_bits(x)
    if fp8:
        qo, so = oracle.dispatch_fp8(xb, lay_o["dispatch_pos"], rows)
        assert np.array_equal(got["recv_q"].cpu().numpy()[filled], qo[filled])
        assert np.array_equal(got["recv_scale"].cpu().numpy()[filled].view(np.uint32),
                              so[filled].view(np.uint32))
    else:
        want = oracle.dispatch_bf16(xb, lay_o["dispatch_pos"], rows)
        assert np.array_equal(gpu_bits(got["recv_x"])[filled], want[filled])
    _assert_unfilled_untouched(got, fp8)


def test_fused_empty_batch(moe):
    """T = 0 still writes the layout: zero counts and offsets, every row -1."""
    E, k, R, rows = 16, 2, 4, 10
    logits = torch.zeros(0, E, dtype=torch.float32, device="cuda")
    x = torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda")
    st = _status()
    got = _fused(moe, logits, x, k, R, 0, rows, True, st=st)
    assert st.item() == 0
    assert torch.all(got["expert_counts"] == 0) and torch.all(got["expert_offsets"] == 0)
    assert torch.all(got["expert_src_counts"] == 0) and torch.all(got["rank_counts"] == 0)
    assert torch.all(got["recv_src"] == -1)


def test_fused_repeated_calls_on_one_workspace(moe):
    """Many calls on one workspace, alternating workloads (so the chunk
    geometry changes between calls): each must match its first result, so the
    grid barrier leaves its counter ready every time."""
    ws = moe.Workspace(torch.device("cuda", 0))
    cases = []
    for name in ["dsv3", "mixtral"]:
        wl = workload(name)
        cfg = wl["cfg"]
        cases.append((to_dev(wl["logits"]), to_dev(wl["x"]), cfg, wl["rows"],
                      cfg.dispatch == "fp8"))
    first = []
    for it in range(6):
        logits, x, cfg, rows, fp8 = cases[it % 2]
        st = _status()
        got = _fused(moe, logits, x, cfg.k, cfg.R, 0, rows, fp8, ws=ws, st=st)
        assert st.item() == 0
        key = "recv_q" if fp8 else "recv_x"
        snap = {kk: got[kk].clone() for kk in ["dispatch_pos", "topk_w", key]}
        if it < 2:
            first.append(snap)
        else:
            ref = first[it % 2]
            for kk in snap:
                assert torch.equal(snap[kk].view(torch.uint8), ref[kk].view(torch.uint8)), kk


def test_fused_in_a_cuda_graph_replayed_on_new_inputs(moe):
    """The fused launch plus combine captured in a CUDA graph and replayed
    on new inputs copied into the captured buffers: each replay equals the
    eager calls bit for bit."""
    wl = workload("dsv3")
    cfg = wl["cfg"]
    T, H, E, k, R = cfg.T, cfg.H, cfg.E, cfg.k, cfg.R
    rows = wl["rows"]
    logits = to_dev(wl["logits"])
    x = to_dev(wl["x"])
    y = inputs.make_row_bank(H, seed=7, n=512).cuda().index_select(
        0, inputs.bank_rows_map(rows, 512).cuda())
    ws = moe.Workspace(torch.device("cuda", 0))
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        res = moe.moe_route_dispatch_fp8(logits, x, k, R, workspace=ws)
        out = moe.moe_combine_bf16(y, res["dispatch_pos"], res["topk_w"])
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        moe.moe_route_dispatch_fp8(logits, x, k, R, out=res, workspace=ws, stream=s)
        moe.moe_combine_bf16(y, res["dispatch_pos"], res["topk_w"], out=out, stream=s)
    for seed in (11, 12):
        gen = torch.Generator().manual_seed(seed)
        new_logits = torch.randn(T, E, generator=gen)
        new_x = torch.randn(T, H, generator=gen).to(torch.bfloat16)
        logits.copy_(new_logits)
        x.copy_(new_x)
        with torch.cuda.stream(s):
            g.replay()
        s.synchronize()
        replayed = {kk: res[kk].clone() for kk in ["topk_idx", "dispatch_pos", "recv_q",
                                                   "recv_scale"]}
        out_r = out.clone()
        eager = _separate(moe, logits, x, k, R, 0, rows, True)
        out_e = moe.moe_combine_bf16(y, eager["dispatch_pos"], eager["topk_w"])
        torch.cuda.synchronize()
        for kk in replayed:
            assert torch.equal(replayed[kk].view(torch.uint8), eager[kk].view(torch.uint8)), kk
        assert torch.equal(out_r.view(torch.int16), out_e.view(torch.int16))
        # and against the oracle's indices for the new logits
        idx_o, _ = oracle.route(new_logits.numpy(), k)
        assert np.array_equal(replayed["topk_idx"].cpu().numpy(), idx_o)


def test_fused_wait_gives_up_and_reports_timeout(moe):
    """A barrier that can never open (its arrival count preset far from the
    grid size, as after a corrupted workspace): every wait ends after its
    time limit, the kernel returns MOE_ERR_TIMEOUT through dev_status, and the
    context stays usable: the next call on a zeroed workspace is correct."""
    wl = workload("mixtral")
    cfg = wl["cfg"]
    logits, x = to_dev(wl["logits"]), to_dev(wl["x"])
    ws = moe.Workspace(torch.device("cuda", 0))
    nbytes = moe.moe_route_dispatch_workspace_bytes(cfg.T, cfg.k, cfg.E, cfg.R)
    buf = ws.get(nbytes)
    buf[:8].view(torch.int64).fill_(1 << 30)   # arrivals = 2^30: no CTA is ever the last
    st = _status()
    moe.moe_route_dispatch_bf16(logits, x, cfg.k, cfg.R, workspace=ws, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_ERR_TIMEOUT
    buf.zero_()
    st2 = _status()
    got = _fused(moe, logits, x, cfg.k, cfg.R, 0, wl["rows"], False, ws=ws, st=st2)
    assert st2.item() == 0
    assert np.array_equal(got["dispatch_pos"].cpu().numpy(), wl["layout"]["dispatch_pos"])


def _random_shapes(n, seed):
    """Seeded random (T, H, E, k, R, cap, fp8) with T % R == 0, E % R == 0."""
    rng = np.random.default_rng(seed)
    shapes = []
    while len(shapes) < n:
        E = int(rng.choice([4, 8, 16, 24, 37, 64, 96, 128, 256, 320, 384, 512, 1000, 1024]))
        divs = [r for r in range(1, E + 1) if E % r == 0]
        R = int(rng.choice(divs))
        k = int(rng.integers(1, min(E, 32) + 1))
        Tr = int(rng.choice([1, 2, 3, 7, 16, 33, 128, 400]))
        T = Tr * R
        if T * k > 400000 or T > 40000:
            continue
        fp8 = bool(rng.integers(0, 2))
        H = int(rng.choice([128, 256, 512])) if fp8 else int(rng.choice([64, 136, 256]))
        cap = 0 if rng.random() < 0.6 else int(rng.integers(1, max(2, T * k // E + 3)))
        shapes.append((T, H, E, k, R, cap, fp8))
    return shapes


@pytest.mark.parametrize("case", _random_shapes(24, 2026),
                         ids=lambda c: "T{}_H{}_E{}_k{}_R{}_cap{}_{}".format(
                             c[0], c[1], c[2], c[3], c[4], c[5], "fp8" if c[6] else "bf16"))
def test_fused_random_shapes_match_separate_and_oracle(moe, case):
    T, H, E, k, R, cap, fp8 = case
    logits, x = inputs.make_random_case(T, H, E, k, seed=T * 7 + E + k)
    idx_o, _ = oracle.route(logits.numpy(), k)
    lay_o = oracle.layout(idx_o, E, R, cap)
    rows = lay_o["recv_src"].shape[0]
    st = _status()
    lg, xd = to_dev(logits), to_dev(x)
    got = _fused(moe, lg, xd, k, R, cap, rows, fp8, st=st)
    want_st = moe.MOE_ERR_CAPACITY if lay_o["status"] == oracle.ERR_CAPACITY else 0
    assert st.item() == want_st
    assert np.array_equal(got["topk_idx"].cpu().numpy(), idx_o)
    for key in LAYOUT_KEYS:
        assert np.array_equal(got[key].cpu().numpy(), lay_o[key].reshape(got[key].shape)), key
    sep = _separate(moe, lg, xd, k, R, cap, rows, fp8)
    _assert_same_as_separate(got, sep, fp8, str(case))
    _assert_unfilled_untouched(got, fp8)


# ------------------------------------------- shared experts and replicas

def _fused_ex(moe, logits, x, k, R, ex, cap, rows, fp8, renormalize=False, st=None):
    T = logits.shape[0]
    out, guards = _out_buffers(T, ex["E_phys"], k + ex["n_shared"], R, x.shape[1], rows, fp8)
    f = moe.moe_route_dispatch_ex_fp8 if fp8 else moe.moe_route_dispatch_ex_bf16
    f(logits, x, k, R, n_shared=ex["n_shared"], shared_weight=ex["shared_weight"],
      replica_offsets=ex["offs"], replica_ids=ex["ids"], E_phys=ex["E_phys"], capacity=cap,
      rows=rows, renormalize=renormalize, out=out, dev_status=st)
    torch.cuda.synchronize()
    _check_guards(guards, rows)
    return out


def _separate_ex(moe, logits, x, k, R, ex, cap, rows, fp8, renormalize=False):
    """moe_route_topk_ex with T / R tokens per source rank, then the
    separate layout and dispatch over E_phys experts."""
    T = logits.shape[0]
    idx, w = moe.moe_route_topk_ex(logits, k, ex["n_shared"], ex["shared_weight"], ex["offs"],
                                   ex["ids"], ex["E_phys"], max(1, T // R),
                                   renormalize=renormalize)
    return _separate_from(moe, idx, w, x, ex["E_phys"], R, cap, rows, fp8)


def _np(t):
    return None if t is None else t.cpu().numpy()


def _check_ex_against_oracle(got, logits, x, k, R, ex, cap, rows, fp8, renormalize, st,
                             moe, where):
    T = logits.shape[0]
    idx_o, w_o, st_o = oracle.route_ex(logits.numpy(), k, ex["n_shared"], ex["shared_weight"],
                                       _np(ex["offs"]), _np(ex["ids"]), ex["E_phys"],
                                       max(1, T // R), renormalize=renormalize)
    lay_o = oracle.layout(idx_o, ex["E_phys"], R, cap, rows)
    want_st = 0
    if st_o != oracle.OK:
        want_st = moe.MOE_ERR_INVALID_ARG
    elif lay_o["status"] == oracle.ERR_CAPACITY:
        want_st = moe.MOE_ERR_CAPACITY
    assert st.item() == want_st, where
    assert np.array_equal(got["topk_idx"].cpu().numpy(), idx_o), where
    gw = got["topk_w"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(gw - w_o) <= route_w_tol(w_o)), where
    for key in LAYOUT_KEYS:
        assert np.array_equal(got[key].cpu().numpy(),
                              lay_o[key].reshape(got[key].shape)), f"{where}: {key}"
    filled = lay_o["recv_src"] >= 0
    x_bits = inputs.bf16_bits(x)
    if fp8:
        qo, so = oracle.dispatch_fp8(x_bits, lay_o["dispatch_pos"], rows)
        assert np.array_equal(got["recv_q"].cpu().numpy()[filled], qo[filled]), where
        assert np.array_equal(got["recv_scale"].cpu().numpy()[filled].view(np.uint32),
                              so[filled].view(np.uint32)), where
    else:
        want = oracle.dispatch_bf16(x_bits, lay_o["dispatch_pos"], rows)
        assert np.array_equal(gpu_bits(got["recv_x"])[filled], want[filled]), where


def test_fused_ex_on_shared_expert_workload(moe):
    """The DeepSeek-V3-like workload with a shared expert replicated on every
    rank: route (routed + shared slots, physical ids), layout over E_phys and
    FP8 rows against the oracle, and bit-identical to the separate calls."""
    wl = workload("dsv3_shared")
    cfg = wl["cfg"]
    fp8 = cfg.dispatch == "fp8"
    offs, ids = wl["placement"]
    ex = dict(n_shared=cfg.n_shared, shared_weight=1.0, offs=to_dev(offs), ids=to_dev(ids),
              E_phys=cfg.E_phys)
    logits, x = to_dev(wl["logits"]), to_dev(wl["x"])
    st = _status()
    got = _fused_ex(moe, logits, x, cfg.k, cfg.R, ex, wl["cap"], wl["rows"], fp8, st=st)
    assert st.item() == 0
    assert np.array_equal(got["topk_idx"].cpu().numpy(), wl["idx"])
    w = got["topk_w"].cpu().numpy().astype(np.float64)
    assert np.all(np.abs(w - wl["w"]) <= route_w_tol(wl["w"]))
    for key in LAYOUT_KEYS:
        assert np.array_equal(got[key].cpu().numpy(),
                              wl["layout"][key].reshape(got[key].shape)), key
    filled = wl["layout"]["recv_src"] >= 0
    qo, so = oracle.dispatch_fp8(wl["x_bits"], wl["layout"]["dispatch_pos"], wl["rows"])
    assert np.array_equal(got["recv_q"].cpu().numpy()[filled], qo[filled])
    assert np.array_equal(got["recv_scale"].cpu().numpy()[filled].view(np.uint32),
                          so[filled].view(np.uint32))
    _assert_unfilled_untouched(got, fp8)
    sep = _separate_ex(moe, logits, x, cfg.k, cfg.R, ex, wl["cap"], wl["rows"], fp8)
    _assert_same_as_separate(got, sep, fp8, "dsv3_shared")


def _random_ex_cases(n, seed):
    """Seeded random shapes with random replica tables: each logical expert
    (routed and shared) gets 1-3 replicas drawn from E_phys physical ids (a
    multiple of R, some ids unused, some shared between logical experts)."""
    rng = np.random.default_rng(seed)
    cases = []
    while len(cases) < n:
        E = int(rng.choice([4, 8, 16, 40, 64, 256, 384]))
        n_shared = int(rng.integers(0, 3))
        k = int(rng.integers(1, min(E, 32 - n_shared) + 1))
        R = int(rng.choice([1, 2, 4, 8]))
        n_log = E + n_shared
        E_phys = min(1024, -(-(n_log + int(rng.integers(0, n_log + 1))) // R) * R)
        if k + n_shared > E_phys or E_phys > 1024:
            continue
        Tr = int(rng.choice([1, 3, 16, 50, 256]))
        T = Tr * R
        reps = rng.integers(1, 4, size=n_log)
        offs = np.concatenate([[0], np.cumsum(reps)]).astype(np.int32)
        ids = rng.integers(0, E_phys, size=int(offs[-1])).astype(np.int32)
        fp8 = bool(rng.integers(0, 2))
        H = int(rng.choice([128, 256])) if fp8 else int(rng.choice([64, 136]))
        cap = 0 if rng.random() < 0.6 else int(rng.integers(1, max(2, T * (k + n_shared) // E_phys + 3)))
        sw = float(rng.choice([1.0, 0.5, 0.8125]))
        renorm = bool(rng.integers(0, 2))
        cases.append((T, H, E, k, R, n_shared, E_phys, offs, ids, cap, fp8, sw, renorm))
    return cases


_EX_CASES = _random_ex_cases(12, 77)


@pytest.mark.parametrize("i", range(len(_EX_CASES)),
                         ids=lambda i: "T{}_E{}_k{}+{}_Ep{}_R{}_cap{}_{}".format(
                             _EX_CASES[i][0], _EX_CASES[i][2], _EX_CASES[i][3], _EX_CASES[i][5],
                             _EX_CASES[i][6], _EX_CASES[i][4], _EX_CASES[i][9],
                             "fp8" if _EX_CASES[i][10] else "bf16"))
def test_fused_ex_random_replica_tables(moe, i):
    T, H, E, k, R, n_shared, E_phys, offs, ids, cap, fp8, sw, renorm = _EX_CASES[i]
    logits, x = inputs.make_random_case(T, H, E, k, seed=500 + i)
    ex = dict(n_shared=n_shared, shared_weight=sw, offs=to_dev(torch.from_numpy(offs)),
              ids=to_dev(torch.from_numpy(ids)), E_phys=E_phys)
    idx_o, _, _ = oracle.route_ex(logits.numpy(), k, n_shared, sw, offs, ids, E_phys, T // R)
    rows = oracle.layout(idx_o, E_phys, R, cap)["recv_src"].shape[0]
    lg, xd = to_dev(logits), to_dev(x)
    st = _status()
    got = _fused_ex(moe, lg, xd, k, R, ex, cap, rows, fp8, renormalize=renorm, st=st)
    _check_ex_against_oracle(got, logits, x, k, R, ex, cap, rows, fp8, renorm, st, moe,
                             str(_EX_CASES[i][:7]))
    _assert_unfilled_untouched(got, fp8)
    sep = _separate_ex(moe, lg, xd, k, R, ex, cap, rows, fp8, renormalize=renorm)
    _assert_same_as_separate(got, sep, fp8, str(_EX_CASES[i][:7]))


def test_fused_ex_without_table_and_bad_table(moe):
    """No replica table: logical ids are the physical ones.  Then a table
    entry past E_phys: that slot gets -1 and no row, MOE_ERR_INVALID_ARG is
    reported, and everything else matches the oracle."""
    T, H, E, k, R = 96, 256, 16, 3, 4
    logits, x = inputs.make_random_case(T, H, E, k, seed=41)
    lg, xd = to_dev(logits), to_dev(x)
    ex = dict(n_shared=2, shared_weight=0.75, offs=None, ids=None, E_phys=20)
    st = _status()
    got = _fused_ex(moe, lg, xd, k, R, ex, 0, T * 5, True, st=st)
    _check_ex_against_oracle(got, logits, x, k, R, ex, 0, T * 5, True, False, st, moe, "no table")
    sep = _separate_ex(moe, lg, xd, k, R, ex, 0, T * 5, True)
    _assert_same_as_separate(got, sep, True, "no table")

    offs, ids = [0], []
    for l in range(E + 2):
        ids += [l] if l != 5 else [5, 18, 19]
        offs.append(len(ids))
    offs, ids = np.array(offs, np.int32), np.array(ids, np.int32)
    bad = ids.copy()
    bad[offs[7]] = 24                                # expert 7's replica: one past E_phys
    ex = dict(n_shared=2, shared_weight=0.75, offs=to_dev(torch.from_numpy(offs)),
              ids=to_dev(torch.from_numpy(bad)), E_phys=24)
    st = _status()
    got = _fused_ex(moe, lg, xd, k, R, ex, 0, T * 5, False, st=st)
    assert bool((got["topk_idx"] == -1).any())
    _check_ex_against_oracle(got, logits, x, k, R, ex, 0, T * 5, False, False, st, moe,
                             "bad table")
