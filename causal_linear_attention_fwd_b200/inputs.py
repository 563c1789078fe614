"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and nothing else: it holds none of the
attention arithmetic, so the CUDA path and the fp64 oracle can both be fed
from it without sharing any of the method.

Recipe (the same for every workload):
  * one torch generator per tensor, seeded with ``seed * 16 + tensor_id``
    (q=0, k=1, v=2, dO=3, kv0=4; decode steps use ``seed * 16 + 5`` and draw
    q, k, v for each step in that order);
  * q, k ~ N(0,1)/sqrt(d); v, dO ~ N(0,1); decode kv0 ~ 0.01 * N(0,1) (fp32);
  * values are drawn in fp32 and rounded once to the I/O dtype;
  * large tensors are filled in fixed-size slabs, in order, from the one
    generator, so the result does not depend on memory limits;
  * per-head decay lambda_h = 1 - 2^-(5 + 8h/H), h = 0..H-1, evaluated in fp64
    and rounded once to fp32 (both sides receive the rounded value).
"""
from __future__ import annotations

import math

import torch

TENSOR_ID = {"q": 0, "k": 1, "v": 2, "dO": 3, "kv0": 4, "decode": 5}
_SLAB = 1 << 26  # elements per fill step


def _gen(device, seed: int, tid: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 16 + int(tid))
    return g


def randn(shape, *, dtype, device, seed: int, tid: int, scale: float = 1.0,
          out: torch.Tensor | None = None) -> torch.Tensor:
    """N(0,1)*scale drawn in fp32 slab by slab, rounded once to ``dtype``."""
    device = torch.device(device)
    if out is None:
        out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    g = _gen(device, seed, tid)
    for i in range(0, n, _SLAB):
        m = min(_SLAB, n - i)
        x = torch.randn(m, generator=g, dtype=torch.float32, device=device)
        if scale != 1.0:
            x.mul_(scale)
        flat[i:i + m].copy_(x)
    return out


def decay_lambdas(H: int, device="cpu") -> torch.Tensor:
    """lambda_h = 1 - 2^-(5 + 8h/H) in fp64, rounded once to fp32."""
    vals = [1.0 - 2.0 ** (-(5.0 + 8.0 * h / H)) for h in range(H)]
    return torch.tensor(vals, dtype=torch.float64).to(torch.float32).to(device)


def fixed_lambdas(vals, device="cpu") -> torch.Tensor:
    return torch.tensor(list(vals), dtype=torch.float64).to(torch.float32).to(device)


def make_inputs(B: int, H: int, L: int, d: int, e: int, *, dtype=torch.bfloat16,
                device="cpu", seed: int = 0, with_dO: bool = True,
                with_kv0: bool = False) -> dict:
    """q,k [B,H,L,d]; v (and dO) [B,H,L,e]; optional kv0 [B,H,d,e] fp32."""
    out = {
        "q": randn((B, H, L, d), dtype=dtype, device=device, seed=seed,
                   tid=TENSOR_ID["q"], scale=1.0 / math.sqrt(d)),
        "k": randn((B, H, L, d), dtype=dtype, device=device, seed=seed,
                   tid=TENSOR_ID["k"], scale=1.0 / math.sqrt(d)),
        "v": randn((B, H, L, e), dtype=dtype, device=device, seed=seed,
                   tid=TENSOR_ID["v"]),
    }
    if with_dO:
        out["dO"] = randn((B, H, L, e), dtype=dtype, device=device, seed=seed,
                          tid=TENSOR_ID["dO"])
    if with_kv0:
        out["kv0"] = randn((B, H, d, e), dtype=torch.float32, device=device,
                           seed=seed, tid=TENSOR_ID["kv0"], scale=0.01)
    return out


class DecodeStream:
    """Per-step decode tokens q,k [B,H,d], v [B,H,e] from one generator."""

    def __init__(self, B, H, d, e, *, dtype=torch.bfloat16, device="cpu",
                 seed: int = 0):
        self.B, self.H, self.d, self.e = B, H, d, e
        self.dtype, self.device = dtype, torch.device(device)
        self.g = _gen(self.device, seed, TENSOR_ID["decode"])
        self.sd = 1.0 / math.sqrt(d)

    def next(self):
        B, H, d, e = self.B, self.H, self.d, self.e
        q = (torch.randn((B, H, d), generator=self.g, device=self.device) * self.sd)
        k = (torch.randn((B, H, d), generator=self.g, device=self.device) * self.sd)
        v = torch.randn((B, H, e), generator=self.g, device=self.device)
        return q.to(self.dtype), k.to(self.dtype), v.to(self.dtype)


def decode_state0(B, H, d, e, *, device="cpu", seed: int = 0) -> torch.Tensor:
    """Initial decode state kv0 ~ 0.01 * N(0,1), fp32 [B,H,d,e]."""
    return randn((B, H, d, e), dtype=torch.float32, device=device, seed=seed,
                 tid=TENSOR_ID["kv0"], scale=0.01)


def varlen_lengths(total: int, seed: int = 0, lo: int = 64, hi: int = 8192) -> list:
    """Document lengths of a packed training batch: log-uniform in [lo, hi]
    rows, drawn from a seeded numpy generator until `total` rows are filled
    (the last one cut to fit)."""
    import numpy as np
    rng = np.random.default_rng(seed)
    lens = []
    while sum(lens) < total:
        n = int(round(float(np.exp(rng.uniform(np.log(lo), np.log(hi))))))
        lens.append(min(n, total - sum(lens)))
    return lens
