"""Stand-in experts for the harness.

The grouped GEMM that multiplies each expert's tokens by its weights sits
between dispatch and combine ("Enabling trillion-parameter models on AWS EFA",
"EFA Üzerinden MoE All-to-All"); it needs trained weights and is not part of
the path built here.  These torch functions stand in for it so that combine
has expert outputs to gather.  They run on whatever device their inputs are
on, outside every timed region.
"""
from __future__ import annotations

import torch


def identity(recv_x: torch.Tensor) -> torch.Tensor:
    """tiny: the expert returns its input."""
    return recv_x


def affine(recv_x: torch.Tensor, noise: torch.Tensor) -> torch.Tensor:
    """Mixtral-like: y = bf16(0.5 * x + n), n ~ N(0, 0.01) drawn per element."""
    return (recv_x.float() * 0.5 + noise.to(recv_x.device)).to(torch.bfloat16)


def dequantise(recv_q: torch.Tensor, recv_scale: torch.Tensor) -> torch.Tensor:
    """FP8 configs: y = bf16(e4m3(q) * s), s the row's 1x128 block scale."""
    v = recv_q.view(torch.float8_e4m3fn).float()
    s = recv_scale.repeat_interleave(128, dim=1)
    return (v * s).to(torch.bfloat16)
