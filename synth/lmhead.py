"""Seeded synthetic inputs of the LM-head step: decoder hidden states and an
LM-head weight, both bf16.

Input generator only (shared by the tests, the benchmark and the smoke
check); it holds none of the sampler's arithmetic.  Every value is a small
integer over 8 (exact in bf16), so every product is a multiple of 1/64 and
every logit z = h . w_v is an integer over 64 of magnitude at most d / 16:
the fp32 contraction is exact under any summation order, and the logits the
tensor cores form equal the float64 ones bit for bit.

Recipe (d = hidden size, codes uniform in {-2, ..., 2}):
  weight  W[v, k] = c / 8, one code per element, seed `seed`;
  hidden  h[row, k] = c / 8 at step s; a row is confident when its fixed
          uniform u_row < f(s) = f0 + (1 - f0) s / (N - 1), and then a fixed
          random subset of min(1, 384 / d) of its coordinates copies the codes
          of its target row W[t_row] (logit boost about 12 at d = 2560);
          elsewhere the codes are fresh each step.
"""
from __future__ import annotations

import torch

CODE_LO, CODE_HI = -2, 2


def _gen(seed: int, tag: int, s: int = 0) -> torch.Generator:
    return torch.Generator().manual_seed((seed * 1000003 + tag * 7919 + s * 104729) % (2**63))


def weight_codes(V: int, d: int, seed: int) -> torch.Tensor:
    """int8 [V, d] codes of the LM-head weight."""
    g = _gen(seed, 1)
    return torch.randint(CODE_LO, CODE_HI + 1, (V, d), generator=g, dtype=torch.int8)


def to_bf16(codes: torch.Tensor, chunk: int = 1 << 24) -> torch.Tensor:
    """codes / 8 as bf16 (exact), converted in chunks."""
    out = torch.empty(codes.shape, dtype=torch.bfloat16)
    flat_in, flat_out = codes.reshape(-1), out.reshape(-1)
    for i in range(0, flat_in.numel(), chunk):
        flat_out[i:i + chunk] = (flat_in[i:i + chunk].to(torch.float32) / 8.0).to(torch.bfloat16)
    return out


def targets(rows: int, V: int, seed: int) -> torch.Tensor:
    return torch.randint(0, V, (rows,), generator=_gen(seed, 2), dtype=torch.int64)


def hidden_codes(wcodes: torch.Tensor, B: int, L: int, s: int, num_steps: int, seed: int,
                 f0: float = 0.05) -> torch.Tensor:
    """int8 [B * L, d] codes of the hidden states at step s."""
    V, d = wcodes.shape
    rows = B * L
    u = torch.rand((rows,), generator=_gen(seed, 3), dtype=torch.float64)
    f = f0 + (1.0 - f0) * (s / max(1, num_steps - 1))
    conf = u < f
    share = min(1.0, 384.0 / d)
    keep = torch.rand((rows, d), generator=_gen(seed, 4), dtype=torch.float64) < share
    codes = torch.randint(CODE_LO, CODE_HI + 1, (rows, d), generator=_gen(seed, 5, s + 1),
                          dtype=torch.int8)
    t = targets(rows, V, seed)
    aligned = wcodes[t]
    mask = keep & conf[:, None]
    codes[mask] = aligned[mask]
    return codes
