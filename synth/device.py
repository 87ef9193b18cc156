"""Seeded generators that draw directly on the GPU (torch), for benchmark inputs too large
to draw on the host in reasonable time.  Same processes as ``synth.gen`` (i.i.d. N(0, 1);
AR(1) along the sequence with x_0 = e_0, x_t = rho x_{t-1} + sqrt(1 - rho^2) e_t), from
torch's device generator instead of NumPy's PCG64, so the values differ from
``synth.gen``'s for the same seed.  Random draws and their layout only: nothing of the
method's arithmetic.
"""
from __future__ import annotations

import math

import torch

_BLK = 64   # rows per block of the blocked AR(1) scan


def generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def normal_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


class AR1:
    """AR(1) along axis -2 of [lead, L, D] float32 tensors, produced piece by piece (the
    filter state carried across pieces).  Within a 64-row block the response to the
    block's innovations is one matmul with the lower-triangular matrix
    T[i, j] = b rho^(i - j) (b = sqrt(1 - rho^2)); the state entering each block adds
    rho^(i + 1) x_prev, carried block to block."""

    def __init__(self, lead: tuple, D: int, rho: float, gen: torch.Generator, device):
        self.lead, self.D, self.rho, self.gen, self.dev = tuple(lead), D, rho, gen, device
        self.b = math.sqrt(1.0 - rho * rho)
        i = torch.arange(_BLK, device=device, dtype=torch.float64)
        e = (i[:, None] - i[None, :])
        T = torch.where(e >= 0, self.b * rho ** e.clamp(min=0), torch.zeros_like(e))
        self.T = T.to(torch.float32)                               # [BLK, BLK]
        self.decay = (rho ** (i + 1)).to(torch.float32)            # [BLK]
        self.state = None                                          # [*lead, D]

    def next(self, n: int) -> torch.Tensor:
        """The next n rows (n a multiple of 64): float32 [*lead, n, D]."""
        assert n % _BLK == 0
        e = torch.randn(*self.lead, n, self.D, generator=self.gen, device=self.dev)
        if self.rho == 0.0:
            return e
        if self.state is None:
            e[..., 0, :] /= self.b                                 # x_0 = e_0
        nb = n // _BLK
        eb = e.view(*self.lead, nb, _BLK, self.D)
        y = torch.matmul(self.T, eb)                               # zero-state responses
        last = y[..., _BLK - 1, :]                                 # [*lead, nb, D]
        carry = torch.empty_like(last)
        s = self.state if self.state is not None else torch.zeros_like(last[..., 0, :])
        r64 = float(self.rho ** _BLK)
        for m in range(nb):                                        # state entering block m
            carry[..., m, :] = s
            s = last[..., m, :] + r64 * s
        self.state = s
        y += self.decay[:, None] * carry.unsqueeze(-2)
        return y.view(*self.lead, n, self.D)
