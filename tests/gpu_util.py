"""Helpers shared by the GPU tests: cached seeded inputs and oracle results
per workload, tolerance checks.  Everything the oracle sees comes from the
harness generators (CPU), never from the CUDA path."""
from __future__ import annotations

import functools

import numpy as np
import torch

import oracle
from harness import experts, inputs

U = 2.0 ** -24


def to_dev(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def ulp_bf16(a: np.ndarray) -> np.ndarray:
    """Spacing of bf16 at |a|: 2^(max(floor(log2|a|), -126) - 7)."""
    a = np.abs(a.astype(np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return 2.0 ** (np.maximum(e, -126) - 7)


def ulp_f32(a: np.ndarray) -> np.ndarray:
    return np.spacing(np.abs(a.astype(np.float32))).astype(np.float64)


def route_w_tol(w_oracle: np.ndarray) -> np.ndarray:
    """Bound on |w_gpu - w_oracle| for the router weights.  The kernel's
    softmax is within 7u of the exact probability p (u = 2^-24): each term
    exp(l - m) within 5u (an exact split of l - m, expf within 2 ulp = 4u,
    one rounding), their binary64 sum rounded once to binary32 (u), one IEEE
    division (u); the oracle rounds a binary64 value once (within u).  Hence
    8u * p, plus the spacing of fp32 subnormals."""
    return 8 * 2.0 ** -24 * np.abs(w_oracle.astype(np.float64)) * (1 + 2.0 ** -20) + 2.0 ** -149


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return inputs.bits_to_bf16(bits).float().numpy().astype(np.float64)


def gpu_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 CUDA tensor -> numpy uint16 bit patterns."""
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@functools.lru_cache(maxsize=5)
def workload(name: str):
    """Seeded inputs of a workload and the oracle's route and layout on them.
    Workloads with shared experts route through the extended route (physical
    expert ids over cfg.E_phys experts, cfg.k_total slots per token)."""
    cfg = inputs.CONFIGS[name]
    logits = inputs.make_logits(cfg)
    x = inputs.make_x(cfg)
    placement = None
    if cfg.n_shared:
        placement = inputs.expert_placement(cfg)
        idx, w, st = oracle.route_ex(logits.numpy(), cfg.k, cfg.n_shared, 1.0, *placement,
                                     cfg.E_phys, cfg.T_r)
        assert st == oracle.OK
    else:
        idx, w = oracle.route(logits.numpy(), cfg.k)
    E_lay = cfg.E_phys if cfg.n_shared else cfg.E
    packed = oracle.layout(idx, E_lay, cfg.R)
    cap = int(packed["expert_counts"].max()) if cfg.layout == "padded" else 0
    lay = oracle.layout(idx, E_lay, cfg.R, cap) if cap else packed
    return dict(cfg=cfg, logits=logits, x=x, x_bits=inputs.bf16_bits(x), idx=idx, w=w,
                layout=lay, cap=cap, rows=int(lay["recv_src"].shape[0]), E_lay=E_lay,
                k=idx.shape[1], placement=placement)


def gpu_route(moe, wl, renormalize=False):
    """The GPU route of a workload (the extended one when it has shared experts)."""
    cfg = wl["cfg"]
    logits = to_dev(wl["logits"])
    if not cfg.n_shared:
        return moe.moe_route_topk(logits, cfg.k, renormalize=renormalize)
    offs, ids = wl["placement"]
    return moe.moe_route_topk_ex(logits, cfg.k, cfg.n_shared, 1.0, to_dev(offs), to_dev(ids),
                                 cfg.E_phys, cfg.T_r, renormalize=renormalize)


def stand_in_y_cpu(wl, recv_bits=None, recv_q=None, recv_scale=None):
    """The workload's stand-in expert applied on the CPU to oracle outputs."""
    cfg = wl["cfg"]
    if cfg.expert == "identity":
        return recv_bits
    if cfg.expert == "affine":
        noise = inputs.make_expert_noise(cfg, recv_bits.shape[0])
        return inputs.bf16_bits(experts.affine(inputs.bits_to_bf16(recv_bits), noise))
    y = experts.dequantise(torch.from_numpy(recv_q), torch.from_numpy(recv_scale))
    return inputs.bf16_bits(y)


def check_combine(out_bits: np.ndarray, acc: np.ndarray, oracle_out_bits: np.ndarray, where: str):
    """The contract: |out - acc| <= 1 bf16 ulp of the oracle's fp32 sum.
    Returns the fraction of outputs bit-identical to the oracle's bf16."""
    out = bf16_to_f64(out_bits)
    err = np.abs(out - acc.astype(np.float64))
    bad = err > ulp_bf16(acc)
    assert not bad.any(), f"{where}: {int(bad.sum())} outputs beyond 1 bf16 ulp, max err {err.max()}"
    return float(np.mean(out_bits == oracle_out_bits))
