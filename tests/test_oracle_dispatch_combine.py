"""Pins of the oracle's dispatch (bf16 copy, fp8 1x128 quantisation) and
combine (router-weighted sum): hand-worked fixtures, the quantisation error
bound of E4M3, sign symmetry, Higham's bound for recursive summation against
a binary64 recomputation, and the dispatch -> identity expert -> combine
invariant (the weight-scaled input)."""
import numpy as np
import pytest
import torch

from conftest import load_golden
from harness import inputs

U = 2.0 ** -24  # binary32 unit roundoff


def _bits(t):
    return inputs.bf16_bits(t)


def _f(bits):
    return inputs.bits_to_bf16(bits).float().numpy()


# ----------------------------------------------------------------- dispatch

def test_dispatch_bf16_copies_rows_and_leaves_others(oracle_mod):
    cfg = inputs.CONFIGS["tiny"]
    idx, _ = oracle_mod.route(inputs.make_logits(cfg).numpy(), cfg.k)
    lay = oracle_mod.layout(idx, cfg.E, cfg.R)
    x = _bits(inputs.make_x(cfg))
    rows = cfg.T * cfg.k + 3                      # 3 spare rows: canaries
    canary = np.full((rows, cfg.H), 0xBEEF, np.uint16)
    out = oracle_mod.dispatch_bf16(x, lay["dispatch_pos"], rows, canary.copy())
    for g in range(cfg.T):
        for j in range(cfg.k):
            assert np.array_equal(out[lay["dispatch_pos"][g, j]], x[g])
    assert np.all(out[cfg.T * cfg.k:] == 0xBEEF)


def test_fp8_block_hand_example(oracle_mod):
    fx = load_golden("fp8_block_hand.json")
    b0 = torch.tensor([i / 127 for i in range(128)], dtype=torch.float64).to(torch.bfloat16)
    x = torch.cat([b0, -b0, torch.zeros(128, dtype=torch.bfloat16)]).reshape(1, fx["H"])
    q, s = oracle_mod.quantize_tokens(_bits(x), [0])
    inv448 = np.float32(1.0 / 448.0)            # nearest binary32 to 1/448
    assert s[0].tolist() == [inv448, inv448, 1.0]
    blocks = {"b0": 0, "b1": 1, "b2": 2}
    for b, i, code in fx["expect"]["codes"]:
        assert q[0, blocks[b] * 128 + i] == int(code, 16), (b, i)


def test_fp8_exact_tie_pins_true_division(oracle_mod):
    tb = load_golden("fp8_block_hand.json")["tie_block"]
    x = torch.zeros(1, 128, dtype=torch.float64)
    x[0, :2] = torch.tensor(tb["x"], dtype=torch.float64)
    q, s = oracle_mod.quantize_tokens(_bits(x.to(torch.bfloat16)), [0])
    assert s[0, 0] == np.float32(tb["scale"])
    assert [int(c) for c in q[0, :3]] == [int(c, 16) for c in tb["codes"]]


def test_fp8_properties_on_workload_rows(oracle_mod):
    cfg = inputs.CONFIGS["dsv3"]
    x = inputs.make_x(cfg)[:64]
    q, s = oracle_mod.quantize_tokens(_bits(x), np.arange(64))
    S = cfg.H // 128
    mag = q & 0x7F
    assert np.all(mag.reshape(64, S, 128).max(2) == 0x7E)   # amax maps to 448
    assert np.all(s > 0)
    # |dequant - x| <= max(2^-4 |x|, s 2^-10) (half an E4M3 ulp), plus the
    # binary32 roundings of x/s and of the dequantising product
    xf = x.float().numpy().reshape(64, S, 128)
    deq = (oracle_mod.e4m3_decode(q).reshape(64, S, 128).astype(np.float64)
           * s.reshape(64, S, 1))
    bound = np.maximum(2.0 ** -4 * np.abs(xf), s.reshape(64, S, 1) * 2.0 ** -10) * (1 + 4 * U)
    assert np.all(np.abs(deq - xf) <= bound)
    # sign symmetry: -x gives the same scales and codes with the sign flipped
    qn, sn = oracle_mod.quantize_tokens(_bits(-x), np.arange(64))
    assert np.array_equal(sn, s)
    assert np.array_equal(qn, q ^ 0x80)


def test_fp8_nan_and_infinity_follow_the_definition(oracle_mod):
    """The literal reading for inputs the pages do not discuss: the block
    amax is a maximum a NaN never raises, s = amax / 448 (1 for amax 0), and
    each code is e4m3(x / s) with NaN -> 0x7F.  So a NaN element gives 0x7F
    and leaves its neighbours' codes as without it, an all-NaN block has s = 1,
    and an infinity makes s infinite: finite elements become signed zeros and
    the infinity itself NaN (inf / inf)."""
    H = 256
    base = torch.linspace(-3.0, 3.0, H)
    x = torch.stack([base, base, base, base]).to(torch.float32)
    x[1, 5] = float("nan")
    x[2, :128] = float("nan")
    x[3, 9] = float("-inf")
    xb = _bits(x.to(torch.bfloat16))
    q, s = oracle_mod.dispatch_fp8(xb, np.arange(4, dtype=np.int32)[:, None], 4)
    assert q[1, 5] == 0x7F
    keep = np.arange(H) != 5
    assert np.array_equal(q[1][keep], q[0][keep]) and np.array_equal(s[1], s[0])
    assert np.all(q[2, :128] == 0x7F) and s[2, 0] == 1.0
    assert np.array_equal(q[2, 128:], q[0, 128:]) and s[2, 1] == s[0, 1]
    assert np.isinf(s[3, 0]) and s[3, 0] > 0 and q[3, 9] == 0x7F
    signs = np.signbit(base[:128].numpy())
    others = np.arange(128) != 9
    assert np.array_equal(q[3, :128][others], np.where(signs, 0x80, 0x00)[others].astype(np.uint8))


def test_fp8_dispatch_writes_each_token_to_its_k_rows(oracle_mod):
    cfg = inputs.CONFIGS["dsv3"]
    T = 96
    logits = inputs.make_logits(cfg)[:T].numpy()
    idx, _ = oracle_mod.route(logits, cfg.k)
    lay = oracle_mod.layout(idx, cfg.E, 1)
    x = _bits(inputs.make_x(cfg)[:T])
    q, s = oracle_mod.dispatch_fp8(x, lay["dispatch_pos"], T * cfg.k)
    qt, st = oracle_mod.quantize_tokens(x, np.arange(T))
    for g in range(T):
        for j in range(cfg.k):
            r = lay["dispatch_pos"][g, j]
            assert np.array_equal(q[r], qt[g]) and np.array_equal(s[r], st[g])


# ------------------------------------------------------------------ combine

@pytest.mark.parametrize("case", load_golden("combine_hand.json")["cases"], ids=lambda c: c["name"])
def test_combine_hand_cases(oracle_mod, case):
    y = _bits(torch.tensor(case["y"], dtype=torch.float64).to(torch.bfloat16))
    pos = np.array(case["dispatch_pos"], np.int32)
    w = np.array(case["topk_w"], np.float32)
    acc, out = oracle_mod.combine(y, pos, w)
    assert acc[0].tolist() == case["acc"]
    assert np.array_equal(out[0], oracle_mod.float_to_bf16_bits(acc[0]))


@pytest.mark.parametrize("k", [1, 2, 8, 16])
def test_combine_higham_bound_vs_binary64(oracle_mod, k):
    """|acc - exact| <= gamma_k * sum_j |w_j y_j|, gamma_k = k u / (1 - k u)
    (recursive summation of k rounded products)."""
    T, H, rows = 64, 256, 64 * k
    rng = np.random.default_rng(k)
    pos = rng.permutation(rows).astype(np.int32).reshape(T, k)
    w = rng.random((T, k)).astype(np.float32)
    y = _bits(inputs.make_random_rows(rows, H, seed=k))
    acc, out = oracle_mod.combine(y, pos, w)
    yf = _f(y).astype(np.float64)
    terms = w.astype(np.float64)[:, :, None] * yf[pos]          # [T][k][H]
    exact = terms.sum(1)
    gamma = k * U / (1 - k * U)
    assert np.all(np.abs(acc - exact) <= gamma * np.abs(terms).sum(1))
    # k = 1 with w = 1 is an exact copy
    if k == 1:
        acc1, out1 = oracle_mod.combine(y, pos, np.ones((T, 1), np.float32))
        assert np.array_equal(out1, y[pos[:, 0]])


def test_combine_token_subset_matches_full(oracle_mod):
    T, H, k = 40, 128, 4
    rng = np.random.default_rng(3)
    pos = rng.permutation(T * k).astype(np.int32).reshape(T, k)
    pos[5, 2] = -1
    w = rng.random((T, k)).astype(np.float32)
    y = _bits(inputs.make_random_rows(T * k, H, seed=4))
    acc, out = oracle_mod.combine(y, pos, w)
    sub = np.array([39, 5, 0, 17], np.int32)
    acc_s, out_s = oracle_mod.combine(y, pos, w, tokens=sub)
    assert np.array_equal(acc_s, acc[sub]) and np.array_equal(out_s, out[sub])


@pytest.mark.parametrize("renormalize", [False, True])
def test_dispatch_identity_combine_returns_weight_scaled_input(oracle_mod, renormalize):
    """dispatch (bf16) -> identity expert -> combine gives bf16(x * sum_j w_j)
    up to the summation bound; renormalised weights give back x within one
    bf16 ulp plus that bound."""
    cfg = inputs.CONFIGS["mixtral"]
    logits = inputs.make_logits(cfg).numpy()
    idx, w = oracle_mod.route(logits, cfg.k, renormalize=renormalize)
    lay = oracle_mod.layout(idx, cfg.E, cfg.R)
    x = _bits(inputs.make_x(cfg))
    recv = oracle_mod.dispatch_bf16(x, lay["dispatch_pos"], cfg.T * cfg.k)
    acc, out = oracle_mod.combine(recv, lay["dispatch_pos"], w)
    xf = _f(x).astype(np.float64)
    wsum = w.astype(np.float64).sum(1, keepdims=True)
    target = xf * wsum
    gamma = cfg.k * U / (1 - cfg.k * U)
    assert np.all(np.abs(acc - target) <= gamma * np.abs(target) + 1e-45)
    if renormalize:
        outf = _f(out).astype(np.float64)
        ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(xf), 2.0 ** -126))) - 7)
        assert np.all(np.abs(outf - xf) <= ulp + cfg.k * 2 ** -23 * np.abs(xf))


# ------------------------------------------------------- combine, FP8 payload

def _fp8_case_arrays(case):
    H, rows = case["H"], case["rows"]
    yq = np.zeros((rows, H), np.uint8)
    for r, cols in case["codes"].items():
        for h, code in cols.items():
            yq[int(r), int(h)] = code
    ys = np.array(case["scales"], np.float32)
    pos = np.array(case["dispatch_pos"], np.int32)
    w = np.array(case["topk_w"], np.float32)
    return yq, ys, pos, w


@pytest.mark.parametrize("case", load_golden("combine_fp8_hand.json")["cases"],
                         ids=lambda c: c["name"][:24])
def test_combine_fp8_hand_cases(oracle_mod, case):
    yq, ys, pos, w = _fp8_case_arrays(case)
    acc, out = oracle_mod.combine_fp8(yq, ys, pos, w)
    want = np.zeros(case["H"], np.float32)
    for h, v in case["expect_acc"].items():
        want[int(h)] = v
    assert np.array_equal(acc[0], want)
    if "wrong_order_acc" in case:
        assert acc[0][0] != np.float32(case["wrong_order_acc"])
    assert np.array_equal(out[0], oracle_mod.float_to_bf16_bits(want))


def test_combine_fp8_power_of_two_scales_equal_bf16_combine(oracle_mod):
    """With power-of-two scales decode(q) * s is exact and representable in
    bf16, so the FP8-payload combine must equal the pinned bf16 combine of the
    restored rows, bit for bit."""
    rng = np.random.default_rng(21)
    T, k, H, rows = 24, 4, 256, 70
    yq = rng.integers(0, 256, (rows, H)).astype(np.uint8)
    yq[(yq & 0x7F) == 0x7F] = 0x11                   # no NaN codes
    ys = (2.0 ** rng.integers(-8, 8, (rows, H // 128))).astype(np.float32)
    pos = rng.integers(-1, rows, (T, k)).astype(np.int32)
    w = rng.random((T, k)).astype(np.float32)
    restored = oracle_mod.e4m3_decode(yq) * np.repeat(ys, 128, axis=1)
    y_bits = oracle_mod.float_to_bf16_bits(restored)
    assert np.array_equal(_f(y_bits), restored)   # exact in bf16
    acc8, out8 = oracle_mod.combine_fp8(yq, ys, pos, w)
    acc16, out16 = oracle_mod.combine(y_bits, pos, w)
    assert np.array_equal(acc8, acc16) and np.array_equal(out8, out16)


def test_combine_fp8_of_dispatched_tokens_is_weighted_input(oracle_mod):
    """dispatch (fp8) -> identity expert -> FP8-payload combine returns
    sum_j w_j * x within the E4M3 error (half an ulp: 2^-4 relative above the
    subnormal range, s * 2^-10 below) plus the binary32 rounding of k terms."""
    T, H, k, E = 40, 256, 3, 8
    logits, x = inputs.make_random_case(T, H, E, k, seed=23)
    idx, w = oracle_mod.route(logits.numpy(), k)
    lay = oracle_mod.layout(idx, E, 2)
    xb = inputs.bf16_bits(x)
    q, s = oracle_mod.dispatch_fp8(xb, lay["dispatch_pos"], T * k)
    acc, _ = oracle_mod.combine_fp8(q, s, lay["dispatch_pos"], w)
    xf = x.float().numpy().astype(np.float64)
    wsum = w.astype(np.float64).sum(1, keepdims=True)
    scale_tok = np.repeat(oracle_mod.quantize_tokens(xb, np.arange(T, dtype=np.int32))[1], 128, 1)
    bound = wsum * (2.0 ** -4 * np.abs(xf) + scale_tok * 2.0 ** -10) * (1 + 2 ** -20) \
        + 2 * k * 2.0 ** -24 * wsum * (np.abs(xf) * (1 + 2 ** -4) + scale_tok)
    assert np.all(np.abs(acc - wsum * xf) <= bound)
