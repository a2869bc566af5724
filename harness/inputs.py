"""Seeded synthetic inputs for the five workloads of the MoE dispatch/combine
path.  This module holds none of the method's arithmetic: it only draws
random numbers (CPU torch generators) and names the shapes.  Both the oracle
side and the CUDA side of every test, and bench.py, take their inputs from
here, so the two see the same bytes.

Workloads (the pages' decode and prefill settings: hidden 7168, block-scaled
fp8 dispatch, bf16 combine, batch 128 per rank for decode and 4096 for
prefill -- "Enabling trillion-parameter models on AWS EFA", section
"Dağıtım/Birleştirme Gecikmesi"; Mixtral 8x7B and DeepSeek as named in
"Efficient and portable mixture-of-experts communication", "Introdução"):

==========  ====  ===  =====  ===  =  ========  =======  ===============
name        T_r   R    H      E    k  dispatch  layout   stand-in expert
==========  ====  ===  =====  ===  =  ========  =======  ===============
tiny        32    2    256    8    2  bf16      packed   identity
mixtral     64    8    4096   8    2  bf16      packed   0.5*x + N(0,.01)
dsv3        128   32   7168   256  8  fp8       packed   dequantise
kimi        128   48   7168   384  8  fp8       packed   dequantise
prefill     4096  8    7168   256  8  fp8       padded   dequantise
==========  ====  ===  =====  ===  =  ========  =======  ===============

Two more: dsv3_shared (dsv3 with one shared expert routed as a ninth slot,
seed 1005) and prefill_r2 (prefill on 2 of its logical ranks, seed 1006, for
profiler captures that must stay small).

Recipe: config i (0..4 in the order above) uses seed_i = 1000 + i and three
independent CPU generators seeded seed_i*10 + s: s = 0 router logits
N(0, 1) fp32 [T][E]; s = 1 hidden states N(0, 1) drawn in fp32 and rounded
to bf16 [T][H]; s = 2 expert-side draws (the Mixtral-like noise, or random
expert outputs).  The Kimi-like config adds a Zipf(s = 1.2) bias per expert to
every token's logits: bias_e = ln((e+1)^-1.2 / sum_e' (e'+1)^-1.2), computed in
float64, rounded to fp32 and added in fp32, so expert 0 is the hottest.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    index: int          # position in the workload list; fixes the seed
    T_r: int            # tokens per logical source rank
    R: int              # logical expert-parallel ranks
    H: int              # hidden size
    E: int              # experts
    k: int              # experts per token
    dispatch: str       # "bf16" or "fp8"
    layout: str         # "packed" or "padded"
    expert: str         # stand-in expert: "identity", "affine", "dequant"
    zipf: float = 0.0   # Zipf exponent of the per-expert logit bias (0: none)
    n_shared: int = 0   # shared experts every token selects (one replica per rank)

    @property
    def T(self) -> int:
        return self.T_r * self.R

    @property
    def L(self) -> int:
        return self.E // self.R

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def k_total(self) -> int:
        """Experts each token selects: the k routed ones and the shared ones."""
        return self.k + self.n_shared

    @property
    def E_phys(self) -> int:
        """Physical experts: each rank hosts its E/R routed experts and one
        replica of every shared expert."""
        return self.E + self.n_shared * self.R

    def describe(self) -> str:
        shared = (f" + {self.n_shared} shared (replicated per rank, {self.E_phys} physical experts)"
                  if self.n_shared else "")
        return (f"{self.name}: T={self.T} ({self.T_r}x{self.R} ranks), H={self.H}, "
                f"E={self.E}, k={self.k}{shared}, {self.dispatch} dispatch, {self.layout} layout")


CONFIGS = {
    c.name: c
    for c in [
        Config("tiny", 0, 32, 2, 256, 8, 2, "bf16", "packed", "identity"),
        Config("mixtral", 1, 64, 8, 4096, 8, 2, "bf16", "packed", "affine"),
        Config("dsv3", 2, 128, 32, 7168, 256, 8, "fp8", "packed", "dequant"),
        Config("kimi", 3, 128, 48, 7168, 384, 8, "fp8", "packed", "dequant", zipf=1.2),
        Config("prefill", 4, 4096, 8, 7168, 256, 8, "fp8", "padded", "dequant"),
        # beyond the five: DeepSeek-V3-like decode where the shared expert is
        # routed too (9 experts per token, 8 routed + 1 shared per rank)
        Config("dsv3_shared", 5, 128, 32, 7168, 256, 8, "fp8", "packed", "dequant", n_shared=1),
        # the prefill workload on 2 of its 8 logical ranks (same per-rank
        # shape, a quarter of the tokens): small enough for full per-kernel
        # profiler captures (about 2 GB on the device), still larger than L2
        Config("prefill_r2", 6, 4096, 2, 7168, 256, 8, "fp8", "padded", "dequant"),
    ]
}


def expert_placement(cfg: Config):
    """Replica table of a config with shared experts: rank r hosts physical
    experts [r*(L+S), (r+1)*(L+S)): its L = E/R routed experts, then one
    replica of each of the S shared experts.  Returns (replica_offsets
    [E+S+1], replica_ids) as int32 numpy arrays; routed expert e has one
    replica, shared expert s has R (token of rank r uses the one on rank r)."""
    import numpy as np
    L, S, R = cfg.E // cfg.R, cfg.n_shared, cfg.R
    per = L + S
    ids, offs = [], [0]
    for e in range(cfg.E):
        ids.append((e // L) * per + e % L)
        offs.append(len(ids))
    for s_ in range(S):
        ids += [r * per + L + s_ for r in range(R)]
        offs.append(len(ids))
    return np.array(offs, np.int32), np.array(ids, np.int32)


def generator(seed: int, stream: int) -> torch.Generator:
    return torch.Generator().manual_seed(seed * 10 + stream)


def zipf_bias(E: int, s: float) -> torch.Tensor:
    """Per-expert log-probability bias of a Zipf(s) law over experts 0..E-1."""
    w = [(e + 1) ** (-s) for e in range(E)]
    z = math.fsum(w)
    return torch.tensor([math.log(v / z) for v in w], dtype=torch.float64).to(torch.float32)


def make_logits(cfg: Config) -> torch.Tensor:
    """Router logits, fp32 [T][E], on the CPU."""
    logits = torch.randn(cfg.T, cfg.E, generator=generator(cfg.seed, 0), dtype=torch.float32)
    if cfg.zipf:
        logits = logits + zipf_bias(cfg.E, cfg.zipf)
    return logits


def make_x(cfg: Config) -> torch.Tensor:
    """Token hidden states, bf16 [T][H], on the CPU."""
    x = torch.randn(cfg.T, cfg.H, generator=generator(cfg.seed, 1), dtype=torch.float32)
    return x.to(torch.bfloat16)


def make_expert_noise(cfg: Config, rows: int) -> torch.Tensor:
    """The Mixtral-like stand-in expert's additive noise, N(0, 0.01) fp32."""
    n = torch.randn(rows, cfg.H, generator=generator(cfg.seed, 2), dtype=torch.float32)
    return n * 0.01


def make_random_rows(rows: int, H: int, seed: int) -> torch.Tensor:
    """Random bf16 rows N(0, 1) [rows][H] (stand-in expert outputs)."""
    y = torch.randn(rows, H, generator=torch.Generator().manual_seed(seed), dtype=torch.float32)
    return y.to(torch.bfloat16)


def make_row_bank(H: int, seed: int, n: int = 4096) -> torch.Tensor:
    """A bank of n random bf16 rows N(0, 1); large synthetic row sets (expert
    outputs of the prefill workload) are drawn from it by bank_rows_map."""
    return make_random_rows(n, H, seed)


def bank_rows_map(rows: int, n: int = 4096) -> torch.Tensor:
    """Row r of a bank-drawn set is bank row (r * 7919) mod n (int64)."""
    return (torch.arange(rows, dtype=torch.int64) * 7919) % n


def make_random_case(T: int, H: int, E: int, k: int, seed: int, tie_levels: int = 0):
    """A small random case: (logits fp32 [T][E], x bf16 [T][H]).  With
    ``tie_levels`` > 0 the logits are integers in [0, tie_levels) so that ties
    are frequent."""
    g = torch.Generator().manual_seed(seed)
    if tie_levels > 0:
        logits = torch.randint(0, tie_levels, (T, E), generator=g).to(torch.float32)
    else:
        logits = torch.randn(T, E, generator=g, dtype=torch.float32)
    x = torch.randn(T, H, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return logits, x


def bf16_bits(t: torch.Tensor):
    """The uint16 bit patterns of a bf16 tensor, as a numpy array."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view("uint16")


def bits_to_bf16(a) -> torch.Tensor:
    import numpy as np
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16)).view(torch.bfloat16)
