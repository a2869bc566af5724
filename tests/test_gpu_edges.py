"""Edge cases of the CUDA path against the oracle: empty and ragged inputs,
maximum sizes (E = 1024, k = 32), masked and invalid expert ids, capacity
overflow, out-of-range rows, extreme fp8 inputs, workspace reuse,
determinism, and the e4m3 converter on every binary32 bit pattern."""
import concurrent.futures as cf
import os

import numpy as np
import pytest
import torch

import oracle
from harness import inputs
from gpu_util import bf16_to_f64, check_combine, gpu_bits, route_w_tol, to_dev

pytestmark = pytest.mark.gpu

LAYOUT_KEYS = ["expert_counts", "expert_src_counts", "rank_counts", "expert_offsets",
               "dispatch_pos", "recv_src"]


@pytest.fixture(scope="module")
def moe():
    import combine_moe_route_08_b200 as m
    return m


def _status():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def _full_path_vs_oracle(moe, logits, x, E, k, R, cap=0, fp8=True, idx_override=None):
    """Every stage on the GPU against the oracle on the same inputs (with FP8
    dispatch, also the FP8-payload combine of the dispatched rows)."""
    T, H = x.shape
    idx_o, w_o = oracle.route(logits.numpy(), k)
    if T:
        idx, w = moe.moe_route_topk(to_dev(logits), k)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), idx_o)
        assert np.all(np.abs(w.cpu().numpy().astype(np.float64) - w_o) <= route_w_tol(w_o))
    if idx_override is not None:
        idx_o = idx_override
    lay_o = oracle.layout(idx_o, E, R, cap)
    rows = lay_o["recv_src"].shape[0]
    st = _status()
    lay = moe.moe_dispatch_layout(to_dev(idx_o.reshape(T, k)), E, R, capacity=cap, rows=rows,
                                  dev_status=st)
    torch.cuda.synchronize()
    for key in LAYOUT_KEYS:
        assert np.array_equal(lay[key].cpu().numpy(), lay_o[key].reshape(lay[key].shape)), key
    want_status = {oracle.OK: 0, oracle.ERR_CAPACITY: moe.MOE_ERR_CAPACITY,
                   oracle.ERR_INVALID: moe.MOE_ERR_INVALID_ARG}[lay_o["status"]]
    assert st.item() == want_status
    pos_o = lay_o["dispatch_pos"]
    filled = lay_o["recv_src"] >= 0
    xb = inputs.bf16_bits(x)
    if fp8:
        q, s = moe.moe_dispatch_fp8(to_dev(x), lay["dispatch_pos"], rows)
        qo, so = oracle.dispatch_fp8(xb, pos_o, rows)
        torch.cuda.synchronize()
        assert np.array_equal(q.cpu().numpy()[filled], qo[filled])
        assert np.array_equal(s.cpu().numpy()[filled].view(np.uint32), so[filled].view(np.uint32))
        if T:  # the FP8-payload combine on the dispatched rows themselves
            acc8, out8_o = oracle.combine_fp8(qo, so, pos_o, w_o)
            out8 = moe.moe_combine_fp8(q, s, lay["dispatch_pos"], to_dev(w_o))
            torch.cuda.synchronize()
            assert check_combine(gpu_bits(out8), acc8, out8_o, "edge fp8") == 1.0
    else:
        r = moe.moe_dispatch_bf16(to_dev(x), lay["dispatch_pos"], rows)
        ro = oracle.dispatch_bf16(xb, pos_o, rows)
        torch.cuda.synchronize()
        assert np.array_equal(gpu_bits(r)[filled], ro[filled])
    y = inputs.make_random_rows(rows, H, seed=T * 31 + E)
    acc, out_o = oracle.combine(inputs.bf16_bits(y), pos_o, w_o)
    out = moe.moe_combine_bf16(to_dev(y), lay["dispatch_pos"], to_dev(w_o))
    torch.cuda.synchronize()
    if T:
        assert check_combine(gpu_bits(out), acc, out_o, "edge") == 1.0


@pytest.mark.parametrize("T,E,k,R,H,cap", [
    (1, 4, 1, 1, 128, 0),
    (7, 8, 2, 1, 256, 0),
    (33, 64, 8, 1, 384, 0),
    (257, 384, 8, 1, 7168, 0),       # ragged against the 256-token chunk
    (300, 16, 16, 2, 128, 0),        # k = E
    (300, 16, 16, 2, 128, 300),      # k = E, padded, cap = T
    (520, 1024, 32, 8, 128, 0),      # maximum E and k
    (4096 + 44, 32, 4, 4, 256, 0),   # several chunks per rank, ragged
    (1200, 24, 6, 3, 512, 120),      # padded with drops
    (96, 16, 4, 2, 16384, 0),        # wide rows: several passes per CTA in every kernel
    (64, 32, 8, 4, 12416, 0),        # wide and not a multiple of the CTA's span
    (512, 1024, 16, 64, 128, 0),     # single-launch layout: 8 ranks per CTA, E at maximum
    (2048, 64, 4, 16, 128, 100),     # single-launch layout, padded with drops
    (960, 96, 8, 24, 128, 0),        # single-launch layout: 3 ranks per CTA, 10 warps each
    (1024, 64, 8, 8, 128, 0),        # single-launch layout: one 1024-slot rank per CTA
])
def test_random_shapes_all_stages(moe, T, E, k, R, H, cap):
    logits, x = inputs.make_random_case(T, H, E, k, seed=T + E + k + H)
    _full_path_vs_oracle(moe, logits, x, E, k, R, cap=cap, fp8=(H % 128 == 0))
    _full_path_vs_oracle(moe, logits, x, E, k, R, cap=cap, fp8=False)


def test_ties_in_logits(moe):
    logits, x = inputs.make_random_case(200, 256, 64, 8, seed=3, tie_levels=3)
    _full_path_vs_oracle(moe, logits, x, 64, 8, 4)


@pytest.mark.parametrize("E,k", [(1024, 32), (256, 8), (37, 5), (8, 8), (64, 1)])
def test_route_all_equal_logits_and_signed_zeros(moe, E, k):
    """Every logit +0.0 or -0.0 (equal keys everywhere): the top-k is experts
    0..k-1 in order and every weight is 1/E (1/k renormalised), the case
    where each lane's best and second-best keys tie and the selection order
    rests entirely on the expert index."""
    T = 70
    rng = np.random.default_rng(E + k)
    logits = np.where(rng.random((T, E)) < 0.5, np.float32(-0.0), np.float32(0.0)).astype(np.float32)
    for renorm in (False, True):
        idx_o, w_o = oracle.route(logits, k, renormalize=renorm)
        assert np.array_equal(idx_o, np.tile(np.arange(k, dtype=np.int32), (T, 1)))
        idx, w = moe.moe_route_topk(to_dev(torch.from_numpy(logits)), k, renormalize=renorm)
        torch.cuda.synchronize()
        assert np.array_equal(idx.cpu().numpy(), idx_o)
        gw = w.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(gw - w_o) <= route_w_tol(w_o))


def test_masked_and_invalid_ids(moe):
    T, E, k, R, H = 96, 16, 4, 4, 256
    logits, x = inputs.make_random_case(T, H, E, k, seed=21)
    idx, _ = oracle.route(logits.numpy(), k)
    rng = np.random.default_rng(4)
    idx[rng.random(idx.shape) < 0.2] = -1
    _full_path_vs_oracle(moe, logits, x, E, k, R, idx_override=idx.copy())
    idx[3, 1] = E + 5
    idx[7, 0] = -9
    _full_path_vs_oracle(moe, logits, x, E, k, R, idx_override=idx.copy())


def test_empty_token_set(moe):
    E, k, R, H = 8, 2, 2, 256
    for cap in [0, 3]:
        rows = 0 if cap == 0 else E * cap + 2
        idx = torch.empty(0, k, dtype=torch.int32, device="cuda")
        lay = moe.moe_dispatch_layout(idx, E, R, capacity=cap, rows=rows)
        torch.cuda.synchronize()
        assert lay["expert_counts"].sum().item() == 0
        assert lay["expert_src_counts"].sum().item() == 0
        assert lay["rank_counts"].sum().item() == 0
        assert lay["expert_offsets"].cpu().tolist() == [e * cap for e in range(E + 1)]
        if rows:
            assert torch.all(lay["recv_src"][:rows] == -1)
    x = torch.empty(0, H, dtype=torch.bfloat16, device="cuda")
    pos = torch.empty(0, k, dtype=torch.int32, device="cuda")
    moe.moe_dispatch_bf16(x, pos, 0, recv_x=torch.empty(1, H, dtype=torch.bfloat16, device="cuda"))
    moe.moe_dispatch_fp8(x, pos, 0, recv_q=torch.empty(1, H, dtype=torch.uint8, device="cuda"),
                         recv_scale=torch.empty(1, 2, device="cuda"))
    moe.moe_combine_bf16(torch.empty(1, H, dtype=torch.bfloat16, device="cuda"), pos,
                         torch.empty(0, k, device="cuda"))
    moe.moe_route_topk(torch.empty(0, E, device="cuda"), k)
    torch.cuda.synchronize()


def test_out_of_range_rows_are_skipped_and_reported(moe):
    T, H, k, rows = 16, 256, 2, 32
    x = inputs.make_random_rows(T, H, seed=5)
    pos = np.arange(T * k, dtype=np.int32).reshape(T, k)
    pos[2, 1] = rows          # one past the end
    pos[5, 0] = -3            # below -1
    pos[9, 1] = 1 << 30       # far away
    guard = 4
    buf = torch.zeros(rows + guard, H, dtype=torch.bfloat16, device="cuda")
    st = _status()
    moe.moe_dispatch_bf16(to_dev(x), to_dev(pos), rows, recv_x=buf[:rows], dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == moe.MOE_ERR_INVALID_ARG
    assert torch.all(buf[rows:] == 0)
    clean = pos.copy()
    clean[clean >= rows] = -1
    clean[clean < -1] = -1
    want = oracle.dispatch_bf16(inputs.bf16_bits(x), clean, rows)
    got = gpu_bits(buf[:rows])
    rows_ok = sorted(set(clean[clean >= 0].tolist()))
    assert np.array_equal(got[rows_ok], want[rows_ok])
    for fn in ("fp8", "combine"):
        st = _status()
        if fn == "fp8":
            qb = torch.zeros(rows + guard, H, dtype=torch.uint8, device="cuda")
            moe.moe_dispatch_fp8(to_dev(x), to_dev(pos), rows, recv_q=qb[:rows],
                                 recv_scale=torch.zeros(rows, H // 128, device="cuda"), dev_status=st)
            torch.cuda.synchronize()
            assert torch.all(qb[rows:] == 0)
        else:
            w = np.ones((T, k), np.float32)
            out = moe.moe_combine_bf16(buf[:rows], to_dev(pos), to_dev(w), dev_status=st)
            y = gpu_bits(buf[:rows])
            acc, out_o = oracle.combine(y, clean, w)
            torch.cuda.synchronize()
            check_combine(gpu_bits(out), acc, out_o, "bad rows")
        assert st.item() == moe.MOE_ERR_INVALID_ARG


def test_fp8_extreme_values(moe):
    """All-zero blocks, signed zeros, bf16 subnormals, the largest bf16
    magnitudes and single spikes, quantised exactly like the oracle."""
    H, T = 1024, 12
    x = torch.zeros(T, H, dtype=torch.float32)
    x[1] = -0.0
    x[2] = torch.linspace(-1e-38, 1e-38, H)                 # bf16 subnormals
    x[3] = 3.0e38
    x[3, ::3] = -3.3e38
    x[4, 5] = 1.0                                            # one spike per row
    x[5] = torch.randn(H) * 1e-30
    x[6] = torch.randn(H) * 1e30
    x[7, :128] = 448.0
    x[8] = torch.arange(H, dtype=torch.float32) - 500
    x[9:] = torch.randn(T - 9, H)
    xb = x.to(torch.bfloat16)
    pos = np.arange(T * 2, dtype=np.int32).reshape(T, 2)
    q, s = moe.moe_dispatch_fp8(to_dev(xb), to_dev(pos), T * 2)
    qo, so = oracle.dispatch_fp8(inputs.bf16_bits(xb), pos, T * 2)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))


def test_fp8_nan_and_infinite_inputs(moe):
    """NaN and infinite inputs, which the pages do not discuss, follow the
    definition literally on both sides: a NaN never raises the block's amax
    and quantises to the NaN code 0x7F; an infinity makes s infinite, so
    finite values give signed zeros and the infinity gives NaN (inf / inf).
    Codes and scales equal the oracle's bit for bit."""
    H, T = 512, 6
    x = torch.randn(T, H, generator=torch.Generator().manual_seed(8), dtype=torch.float32)
    x[0, 3] = float("nan")                      # one NaN in a block
    x[1, :128] = float("nan")                   # an all-NaN block: amax 0, s = 1
    x[2, 7] = float("inf")
    x[3, 200] = float("-inf")
    x[4, 130] = float("inf")
    x[4, 131] = float("-inf")
    x[4, 300] = float("nan")
    xb = x.to(torch.bfloat16)
    pos = np.arange(T * 2, dtype=np.int32).reshape(T, 2)
    q, s = moe.moe_dispatch_fp8(to_dev(xb), to_dev(pos), T * 2)
    qo, so = oracle.dispatch_fp8(inputs.bf16_bits(xb), pos, T * 2)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), qo)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), so.view(np.uint32))
    # token g fills rows 2g and 2g + 1
    assert qo[0, 3] == 0x7F                                   # the NaN element
    assert np.all(qo[2, :128] == 0x7F) and so[2, 0] == 1.0    # all-NaN block: s = 1
    assert qo[4, 7] == 0x7F and np.isinf(so[4, 0])            # inf / inf, s infinite
    assert np.all(qo[4, :128][np.arange(128) != 7] & 0x7F == 0)  # finite / inf: signed zeros


def _same_up_to_nan_payload(got_bits, acc, want_bits, where):
    """Outputs whose oracle sum is NaN must be NaN (payload and sign are not
    part of the contract), infinite sums the same infinity, every other
    output within 1 bf16 ulp and bit-identical."""
    nan = np.isnan(acc)
    inf = np.isinf(acc)
    got_f = bf16_to_f64(got_bits)
    assert np.all(np.isnan(got_f[nan])), where
    assert not np.any(np.isnan(got_f[~nan])), where
    assert np.array_equal(got_bits[inf], want_bits[inf]), where      # signed infinities
    keep = ~(nan | inf)
    assert check_combine(got_bits[keep], acc[keep], want_bits[keep], where) == 1.0


def test_combine_nan_and_infinite_rows(moe):
    """bf16 rows holding NaN, +inf and -inf (a token summing +inf and -inf
    gets NaN), and FP8 rows holding the NaN code: NaN where the oracle's sum
    is NaN, infinities where it is infinite, everything else bit-identical."""
    T, k, H = 16, 4, 256
    rows = T * k
    rng = np.random.default_rng(21)
    y = torch.randn(rows, H, generator=torch.Generator().manual_seed(9), dtype=torch.float32)
    y[1, 0] = float("nan")
    y[5, 10] = float("inf")
    y[6, 10] = float("-inf")                    # rows 5 and 6 belong to token 1
    y[9, 20] = float("inf")
    yb = y.to(torch.bfloat16)
    pos = np.arange(rows, dtype=np.int32).reshape(T, k)
    w = rng.random((T, k)).astype(np.float32)
    acc, out_o = oracle.combine(inputs.bf16_bits(yb), pos, w)
    out = moe.moe_combine_bf16(to_dev(yb), to_dev(pos), to_dev(w))
    torch.cuda.synchronize()
    _same_up_to_nan_payload(gpu_bits(out), acc, out_o, "bf16 rows")
    assert np.isnan(acc[1, 10]) and np.isinf(acc[2, 20])
    # the same rows as E4M3 + scales (each row quantised on its own)
    qo, so = oracle.dispatch_fp8(inputs.bf16_bits(yb), np.arange(rows, dtype=np.int32)[:, None], rows)
    qo[3, 40] = 0x7F
    qo[12, 41] = 0xFF
    acc8, out8_o = oracle.combine_fp8(qo, so, pos, w)
    out8 = moe.moe_combine_fp8(to_dev(qo), to_dev(so), to_dev(pos), to_dev(w))
    torch.cuda.synchronize()
    _same_up_to_nan_payload(gpu_bits(out8), acc8, out8_o, "fp8 rows")
    assert np.isnan(acc8[0, 40]) and np.isnan(acc8[3, 41])


def test_workspace_reuse_and_determinism(moe):
    ws = moe.Workspace("cuda")
    cfgs = [(4096, 256, 8, 32), (64, 8, 2, 2), (32768, 256, 8, 8), (4096, 256, 8, 32)]
    first = {}
    for T, E, k, R in cfgs:
        logits, _ = inputs.make_random_case(T, 8, E, k, seed=T + E)
        idx_o, _ = oracle.route(logits.numpy(), k)
        want = oracle.layout(idx_o, E, R)
        idx = to_dev(idx_o)
        for rep in range(2):
            lay = moe.moe_dispatch_layout(idx, E, R, workspace=ws)
            torch.cuda.synchronize()
            for key in LAYOUT_KEYS:
                assert np.array_equal(lay[key].cpu().numpy(), want[key].reshape(lay[key].shape))
        first.setdefault((T, E), lay["dispatch_pos"].clone())


def _mismatch_range(args):
    first_bits, codes = args
    return oracle.e4m3_count_mismatch(first_bits, codes)


def test_e4m3_converter_every_binary32_pattern(moe):
    """The dispatch kernel's converter on all 2^32 bit patterns against the
    oracle's encoder (written from the OCP OFP8 definition)."""
    oracle.build()
    chunk = 1 << 28
    workers = max(1, min(16, os.cpu_count() or 1))
    bad_total = 0
    with cf.ThreadPoolExecutor(workers) as pool:   # ctypes calls release the GIL
        for start in range(0, 1 << 32, chunk):
            bits = torch.arange(start, start + chunk, dtype=torch.int64, device="cuda")
            v = bits.to(torch.int32).view(torch.float32) if start < (1 << 31) else \
                (bits - (1 << 32)).to(torch.int32).view(torch.float32)
            codes = moe.moe_quantize_e4m3(v).cpu().numpy()
            del bits, v
            part = chunk // workers
            jobs = [(start + i * part, codes[i * part:(i + 1) * part if i < workers - 1 else chunk])
                    for i in range(workers)]
            for n_bad, first_bad in pool.map(_mismatch_range, jobs):
                bad_total += n_bad
    assert bad_total == 0


def test_layout_large_token_count_many_chunks(moe):
    """1M slots (131072 tokens x 8) over 8 logical ranks: 16 chunks per rank,
    128 chunks in all; packed and padded layouts bit-exact."""
    T, E, k, R = 131072, 256, 8, 8
    rng = np.random.default_rng(17)
    idx = np.argsort(rng.random((T, E), dtype=np.float32), axis=1)[:, :k].astype(np.int32)
    want = oracle.layout(idx, E, R)
    st = _status()
    lay = moe.moe_dispatch_layout(to_dev(idx), E, R, dev_status=st)
    torch.cuda.synchronize()
    for key in LAYOUT_KEYS:
        assert np.array_equal(lay[key].cpu().numpy(), want[key].reshape(lay[key].shape)), key
    cap = int(want["expert_counts"].max()) - 7          # a few drops in the hottest experts
    want_p = oracle.layout(idx, E, R, cap)
    lay_p = moe.moe_dispatch_layout(to_dev(idx), E, R, capacity=cap, rows=E * cap, dev_status=st)
    torch.cuda.synchronize()
    for key in LAYOUT_KEYS:
        assert np.array_equal(lay_p[key].cpu().numpy(), want_p[key].reshape(lay_p[key].shape)), key
    assert st.item() == moe.MOE_ERR_CAPACITY


def test_layout_launch_count(moe):
    """Small layouts (T * k <= 8192, one chunk per rank) take the
    single-launch cluster layout; the decode and prefill workloads the
    histogram + placement pair."""
    assert moe.moe_dispatch_layout_launches(512, 2, 8, 8) == 1          # mixtral
    assert moe.moe_dispatch_layout_launches(64, 2, 8, 2) == 1           # tiny
    assert moe.moe_dispatch_layout_launches(1024, 8, 64, 8) == 1        # 8192 slots
    assert moe.moe_dispatch_layout_launches(1032, 8, 64, 8) == 2        # 8256 slots
    assert moe.moe_dispatch_layout_launches(4096, 8, 256, 32) == 2      # dsv3
    assert moe.moe_dispatch_layout_launches(6144, 8, 384, 48) == 2      # kimi
    assert moe.moe_dispatch_layout_launches(32768, 8, 256, 8) == 2      # prefill
    assert moe.moe_dispatch_layout_launches(4096, 8, 256, 3) == 0       # R does not divide E


def test_all_slots_masked(moe):
    """Every slot empty (-1): nothing counted, nothing dispatched, combine
    writes zeros."""
    T, E, k, R, H = 64, 8, 2, 2, 256
    idx = np.full((T, k), -1, np.int32)
    st = _status()
    lay = moe.moe_dispatch_layout(to_dev(idx), E, R, dev_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert lay["expert_counts"].sum().item() == 0
    assert torch.all(lay["dispatch_pos"] == -1) and torch.all(lay["recv_src"] == -1)
    x = inputs.make_random_rows(T, H, seed=3)
    recv = torch.full((T * k, H), 5.0, dtype=torch.bfloat16, device="cuda")
    moe.moe_dispatch_bf16(to_dev(x), lay["dispatch_pos"], T * k, recv_x=recv)
    out = moe.moe_combine_bf16(recv, lay["dispatch_pos"], torch.ones(T, k, device="cuda"))
    torch.cuda.synchronize()
    assert torch.all(recv == 5.0)
    assert torch.all(out == 0)


def test_route_ex_replicas_and_bad_table(moe):
    """Extended route against the oracle: an expert with three replicas
    chosen by source rank, two shared experts, renormalised routed weights,
    then a table entry out of range (slot -1, reported)."""
    T, E, k, Tr = 96, 16, 3, 8
    logits, _ = inputs.make_random_case(T, 8, E, k, seed=41)
    n_shared = 2
    # logical 0..15 routed, 16..17 shared; physical ids 0..21
    offs = [0]
    ids = []
    for l in range(E + n_shared):
        reps = [l] if l != 5 else [5, 18, 19]
        if l >= E:
            reps = [l, l + 4]                      # shared: 16 -> {16, 20}, 17 -> {17, 21}
        ids += reps
        offs.append(len(ids))
    offs = np.array(offs, np.int32)
    ids = np.array(ids, np.int32)
    for renorm in (False, True):
        want_i, want_w, st_o = oracle.route_ex(logits.numpy(), k, n_shared, 0.75, offs, ids, 22, Tr,
                                               renormalize=renorm)
        assert st_o == oracle.OK
        st = _status()
        got_i, got_w = moe.moe_route_topk_ex(to_dev(logits), k, n_shared, 0.75, to_dev(offs),
                                             to_dev(ids), 22, Tr, renormalize=renorm, dev_status=st)
        torch.cuda.synchronize()
        assert np.array_equal(got_i.cpu().numpy(), want_i)
        gw = got_w.cpu().numpy().astype(np.float64)
        assert np.all(np.abs(gw - want_w) <= route_w_tol(want_w))
        assert st.item() == 0
    bad = ids.copy()
    bad[offs[7]] = 22                               # expert 7's replica: one past E_phys
    want_i, _, st_o = oracle.route_ex(logits.numpy(), k, n_shared, 0.75, offs, bad, 22, Tr)
    st = _status()
    got_i, _ = moe.moe_route_topk_ex(to_dev(logits), k, n_shared, 0.75, to_dev(offs), to_dev(bad),
                                     22, Tr, dev_status=st)
    torch.cuda.synchronize()
    assert st_o == oracle.ERR_INVALID and st.item() == moe.MOE_ERR_INVALID_ARG
    assert np.array_equal(got_i.cpu().numpy(), want_i)


def _two_phase_shapes(n, seed):
    """Seeded random (T, H, E, k, R, max_m, fp8) for the two-phase path."""
    rng = np.random.default_rng(seed)
    out = []
    while len(out) < n:
        E = int(rng.choice([4, 8, 16, 37, 64, 128, 256, 384]))
        R = int(rng.choice([r for r in range(1, E + 1) if E % r == 0 and r <= 64]))
        k = int(rng.integers(1, min(E, 12) + 1))
        Tr = int(rng.choice([1, 2, 5, 16, 64, 130]))
        T = Tr * R
        if T * k > 200000 or E * R * Tr * 256 > 2 ** 31:
            continue
        max_m = int(rng.choice([1, 2, max(1, Tr // 2), Tr]))
        fp8 = bool(rng.integers(0, 2))
        H = int(rng.choice([128, 256])) if fp8 else int(rng.choice([8, 64, 136]))
        out.append((T, H, E, k, R, max_m, fp8))
    return out


@pytest.mark.parametrize("case", _two_phase_shapes(16, 77),
                         ids=lambda c: "T{}_H{}_E{}_k{}_R{}_m{}_{}".format(
                             c[0], c[1], c[2], c[3], c[4], c[5], "fp8" if c[6] else "bf16"))
def test_two_phase_random_shapes(moe, case):
    """Private layout against the oracle (drops when max_m < the largest
    per-(expert, rank) count); send + compact equals the direct dispatch on
    the rows that were kept."""
    T, H, E, k, R, max_m, fp8 = case
    logits, x = inputs.make_random_case(T, H, E, k, seed=T + E * 3 + k)
    idx_o, _ = oracle.route(logits.numpy(), k)
    ppos_o, base_o, _, st_o = oracle.private_layout(idx_o, E, R, max_m)
    st = _status()
    lay = moe.moe_dispatch_layout_private(to_dev(idx_o), E, R, max_m, dev_status=st)
    torch.cuda.synchronize()
    want_st = moe.MOE_ERR_CAPACITY if st_o == oracle.ERR_CAPACITY else 0
    assert st.item() == want_st
    assert np.array_equal(lay["private_pos"].cpu().numpy(), ppos_o)
    packed = oracle.layout(idx_o, E, R)
    want_pos = np.where(ppos_o >= 0, packed["dispatch_pos"], -1)
    assert np.array_equal(lay["dispatch_pos"].cpu().numpy(), want_pos)
    prows, rows = lay["private_rows"], T * k
    xd = to_dev(x)
    st2 = _status()
    if fp8:
        pq, ps = moe.moe_dispatch_fp8(xd, lay["private_pos"], prows, dev_status=st2)
        q, s = moe.moe_compact_fp8(pq, ps, lay["private_pos"], lay["dispatch_pos"], rows,
                                   dev_status=st2)
        q_ref, s_ref = moe.moe_dispatch_fp8(xd, lay["dispatch_pos"], rows)
        torch.cuda.synchronize()
        kept = torch.from_numpy(np.nonzero(lay["recv_src"].cpu().numpy() >= 0)[0]).cuda()
        assert torch.equal(q.index_select(0, kept), q_ref.index_select(0, kept))
        assert torch.equal(s.index_select(0, kept), s_ref.index_select(0, kept))
    else:
        px = moe.moe_dispatch_bf16(xd, lay["private_pos"], prows, dev_status=st2)
        rx = moe.moe_compact_bf16(px, lay["private_pos"], lay["dispatch_pos"], rows,
                                  dev_status=st2)
        rx_ref = moe.moe_dispatch_bf16(xd, lay["dispatch_pos"], rows)
        torch.cuda.synchronize()
        kept = torch.from_numpy(np.nonzero(lay["recv_src"].cpu().numpy() >= 0)[0]).cuda()
        assert torch.equal(rx.index_select(0, kept).view(torch.int16),
                           rx_ref.index_select(0, kept).view(torch.int16))
    assert st2.item() == 0
