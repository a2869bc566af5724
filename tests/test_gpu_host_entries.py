"""The host-buffer entry points, through the C ABI: router logits and hidden
states copied in from host memory, the combined tokens copied out to host
memory, on the caller's stream.  Compared with the oracle (indices, every
layout output, bf16 rows, e4m3 codes and fp32 scales bit-exact; combine
within one bf16 ulp and bit-identical) and with the device-pointer entry
points (router weights bit-identical), with page-locked and pageable host
memory, the separate kernels and the single fused launch, inside a CUDA
graph, and at T = 0."""
import numpy as np
import pytest
import torch

import oracle
from harness import inputs
from gpu_util import check_combine, gpu_bits, stand_in_y_cpu, to_dev, workload

pytestmark = pytest.mark.gpu

LAYOUT_KEYS = ["expert_counts", "expert_src_counts", "rank_counts", "expert_offsets",
               "dispatch_pos", "recv_src"]


@pytest.fixture(scope="module")
def moe():
    import combine_moe_route_08_b200 as m
    assert torch.cuda.is_available()
    return m


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _host(t: torch.Tensor, pinned: bool) -> torch.Tensor:
    t = t.contiguous()
    return t.pin_memory() if pinned else t.clone()


def _route_dispatch_host(moe, wl, pinned, fused, **kw):
    cfg = wl["cfg"]
    f = (moe.moe_route_dispatch_fp8_host if cfg.dispatch == "fp8"
         else moe.moe_route_dispatch_bf16_host)
    return f(_host(wl["logits"], pinned), _host(wl["x"], pinned), cfg.k, cfg.R,
             capacity=wl["cap"], rows=wl["rows"], fused=fused, **kw)


def _check_dispatch(moe, wl, res, where):
    cfg = wl["cfg"]
    lay = wl["layout"]
    assert np.array_equal(res["topk_idx"].cpu().numpy(), wl["idx"]), where
    for key in LAYOUT_KEYS:
        got = res[key].cpu().numpy()
        assert np.array_equal(got, lay[key].reshape(got.shape)), f"{where}: {key}"
    # the weights: the same kernels as the device-pointer route, bit for bit
    _, w_dev = moe.moe_route_topk(to_dev(wl["logits"].numpy()), cfg.k)
    assert torch.equal(res["topk_w"].view(torch.int32), w_dev.view(torch.int32)), where
    filled = lay["recv_src"] >= 0
    pos = lay["dispatch_pos"]
    if cfg.dispatch == "fp8":
        want_q, want_s = oracle.dispatch_fp8(wl["x_bits"], pos, wl["rows"])
        assert np.array_equal(res["recv_q"].cpu().numpy()[filled], want_q[filled]), where
        assert np.array_equal(res["recv_scale"].cpu().numpy()[filled].view(np.uint32),
                              want_s[filled].view(np.uint32)), where
    else:
        want = oracle.dispatch_bf16(wl["x_bits"], pos, wl["rows"])
        assert np.array_equal(gpu_bits(res["recv_x"])[filled], want[filled]), where


@pytest.mark.parametrize("name,pinned,fused", [
    ("tiny", True, False), ("mixtral", False, False), ("dsv3", True, False),
    ("kimi", True, False), ("prefill_r2", True, False), ("dsv3", True, True),
    ("mixtral", True, True), ("tiny", False, True)])
def test_route_dispatch_host_parity(moe, name, pinned, fused):
    wl = workload(name)
    st = _status()
    res = _route_dispatch_host(moe, wl, pinned, fused, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(res["logits"].cpu(), wl["logits"])          # the staged inputs
    assert torch.equal(res["x"].cpu().view(torch.int16), wl["x"].view(torch.int16))
    _check_dispatch(moe, wl, res, f"{name} pinned={pinned} fused={fused}")


@pytest.mark.parametrize("name,pinned", [("tiny", True), ("mixtral", False), ("dsv3", True)])
def test_combine_bf16_host_parity(moe, name, pinned):
    wl = workload(name)
    cfg = wl["cfg"]
    pos = wl["layout"]["dispatch_pos"]
    if cfg.dispatch == "fp8":
        q, s = oracle.dispatch_fp8(wl["x_bits"], pos, wl["rows"])
        y_bits = stand_in_y_cpu(wl, recv_q=q, recv_scale=s)
    else:
        y_bits = stand_in_y_cpu(wl, recv_bits=oracle.dispatch_bf16(wl["x_bits"], pos, wl["rows"]))
    acc, out_o = oracle.combine(y_bits, pos, wl["w"])
    out_host = _host(torch.zeros(cfg.T, cfg.H, dtype=torch.bfloat16), pinned)
    st = _status()
    got = moe.moe_combine_bf16_host(to_dev(inputs.bits_to_bf16(y_bits)), to_dev(pos),
                                    to_dev(wl["w"]), out_host=out_host, dev_status=st)
    torch.cuda.synchronize()
    assert got.data_ptr() == out_host.data_ptr() and not got.is_cuda
    assert st.item() == 0
    assert check_combine(gpu_bits(got), acc, out_o, name) == 1.0


@pytest.mark.parametrize("pinned", [True, False])
def test_combine_fp8_host_parity(moe, pinned):
    wl = workload("dsv3")
    cfg = wl["cfg"]
    pos = wl["layout"]["dispatch_pos"]
    q, s = oracle.dispatch_fp8(wl["x_bits"], pos, wl["rows"])
    acc, out_o = oracle.combine_fp8(q, s, pos, wl["w"])
    out_host = _host(torch.zeros(cfg.T, cfg.H, dtype=torch.bfloat16), pinned)
    st = _status()
    got = moe.moe_combine_fp8_host(to_dev(q), to_dev(s), to_dev(pos), to_dev(wl["w"]),
                                   out_host=out_host, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert check_combine(gpu_bits(got), acc, out_o, "dsv3 fp8") == 1.0


def test_host_step_in_a_cuda_graph(moe):
    """A whole step (host inputs in, host result out) captured once and
    replayed: page-locked buffers, new host contents on every replay."""
    wl = workload("tiny")
    cfg = wl["cfg"]
    logits_h = _host(wl["logits"], True)
    x_h = _host(wl["x"], True)
    out_h = _host(torch.zeros(cfg.T, cfg.H, dtype=torch.bfloat16), True)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        res = moe.moe_route_dispatch_bf16_host(logits_h, x_h, cfg.k, cfg.R, capacity=wl["cap"],
                                               rows=wl["rows"])
        out_d = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
        moe.moe_combine_bf16_host(res["recv_x"], res["dispatch_pos"], res["topk_w"],
                                  out_host=out_h, out=out_d)
    s.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        moe.moe_route_dispatch_bf16_host(logits_h, x_h, cfg.k, cfg.R, capacity=wl["cap"],
                                         rows=wl["rows"], out=res)
        moe.moe_combine_bf16_host(res["recv_x"], res["dispatch_pos"], res["topk_w"],
                                  out_host=out_h, out=out_d)
    for seed in (3, 4):
        logits = torch.randn(cfg.T, cfg.E, generator=torch.Generator().manual_seed(seed))
        x = torch.randn(cfg.T, cfg.H, generator=torch.Generator().manual_seed(seed + 10))
        x = x.to(torch.bfloat16)
        logits_h.copy_(logits)
        x_h.copy_(x)
        out_h.zero_()
        g.replay()
        s.synchronize()
        idx, w = oracle.route(logits.numpy(), cfg.k)
        lay = oracle.layout(idx, cfg.E, cfg.R, wl["cap"], wl["rows"]) if wl["cap"] else \
            oracle.layout(idx, cfg.E, cfg.R)
        assert np.array_equal(res["topk_idx"].cpu().numpy(), idx)
        x_bits = inputs.bf16_bits(x)
        recv = oracle.dispatch_bf16(x_bits, lay["dispatch_pos"], wl["rows"])
        acc, out_o = oracle.combine(recv, lay["dispatch_pos"], res["topk_w"].cpu().numpy())
        assert check_combine(gpu_bits(out_h), acc, out_o, f"graph seed {seed}") == 1.0
    del g


def test_host_entries_with_no_tokens(moe):
    """T = 0: nothing is copied; the layout still writes zero counts; the
    combine enqueues nothing."""
    E, R, k, H = 16, 4, 2, 256
    logits = torch.zeros(0, E, dtype=torch.float32)
    x = torch.zeros(0, H, dtype=torch.bfloat16)
    res = moe.moe_route_dispatch_fp8_host(logits, x, k, R, rows=0)
    torch.cuda.synchronize()
    assert int(res["expert_counts"].sum()) == 0 and int(res["rank_counts"].sum()) == 0
    assert int(res["expert_offsets"].abs().sum()) == 0
    y = torch.zeros(1, H, dtype=torch.bfloat16, device="cuda")
    out_h = moe.moe_combine_bf16_host(y, torch.zeros(0, k, dtype=torch.int32, device="cuda"),
                                      torch.zeros(0, k, dtype=torch.float32, device="cuda"))
    torch.cuda.synchronize()
    assert out_h.shape == (0, H)


@pytest.mark.parametrize("T,E,k,R,H,cap,fused", [
    (7, 8, 2, 1, 256, 0, False),
    (257, 384, 8, 1, 7168, 0, False),      # ragged against a chunk
    (520, 1024, 32, 8, 128, 0, False),     # maximum E and k
    (1200, 24, 6, 3, 512, 120, False),     # padded with drops
    (96, 16, 4, 2, 16384, 0, False),       # wide rows
    (1024, 64, 8, 8, 128, 0, False),       # single-launch layout
    (1200, 24, 6, 3, 512, 120, True),      # the single fused launch, padded with drops
    (300, 16, 16, 2, 128, 0, True),
])
def test_host_entries_equal_device_entries_on_edge_shapes(moe, T, E, k, R, H, cap, fused):
    """Every output of the host-buffer entry points (FP8 and bf16 dispatch,
    both combines) equals the device-pointer entry points' bit for bit,
    status codes included (a capacity drop is reported the same way)."""
    logits, x = inputs.make_random_case(T, H, E, k, seed=7 * T + E + k + H)
    rows = T * k if cap == 0 else E * cap
    dev = torch.device("cuda")
    for fp8 in ([True, False] if H % 128 == 0 else [False]):
        st_d, st_h = _status(), _status()
        if fused:
            f = moe.moe_route_dispatch_fp8 if fp8 else moe.moe_route_dispatch_bf16
            want = f(logits.to(dev), x.to(dev), k, R, capacity=cap, rows=rows, dev_status=st_d)
        else:
            idx, w = moe.moe_route_topk(logits.to(dev), k)
            want = moe.moe_dispatch_layout(idx, E, R, capacity=cap, rows=rows, dev_status=st_d)
            want["topk_idx"], want["topk_w"] = idx, w
            if fp8:
                want["recv_q"], want["recv_scale"] = moe.moe_dispatch_fp8(
                    x.to(dev), want["dispatch_pos"], rows, dev_status=st_d)
            else:
                want["recv_x"] = moe.moe_dispatch_bf16(x.to(dev), want["dispatch_pos"], rows,
                                                       dev_status=st_d)
        f = moe.moe_route_dispatch_fp8_host if fp8 else moe.moe_route_dispatch_bf16_host
        got = f(_host(logits, True), _host(x, True), k, R, capacity=cap, rows=rows, fused=fused,
                dev_status=st_h)
        torch.cuda.synchronize()
        assert st_h.item() == st_d.item()
        filled = want["recv_src"][:rows] >= 0
        for key in ["topk_idx", "topk_w"] + LAYOUT_KEYS:
            a, b = got[key], want[key]
            if key == "recv_src":
                a, b = a[:rows], b[:rows]
            assert torch.equal(a.view(torch.int32), b.view(torch.int32)), (key, fp8)
        for key in (["recv_q", "recv_scale"] if fp8 else ["recv_x"]):
            a, b = got[key][:rows][filled], want[key][:rows][filled]
            assert torch.equal(a.contiguous().view(torch.uint8), b.contiguous().view(torch.uint8)), key
        # combine of the dispatched rows (an identity expert), back to host memory
        if fp8:
            out_d = moe.moe_combine_fp8(want["recv_q"], want["recv_scale"], want["dispatch_pos"],
                                        want["topk_w"])
            out_h = moe.moe_combine_fp8_host(got["recv_q"], got["recv_scale"], got["dispatch_pos"],
                                             got["topk_w"])
        else:
            out_d = moe.moe_combine_bf16(want["recv_x"], want["dispatch_pos"], want["topk_w"])
            out_h = moe.moe_combine_bf16_host(got["recv_x"], got["dispatch_pos"], got["topk_w"])
        torch.cuda.synchronize()
        assert torch.equal(out_h.view(torch.int16), out_d.cpu().view(torch.int16)), fp8
