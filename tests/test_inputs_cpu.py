"""The seeded input recipe (CPU): the same seed gives the same tensors bit for
bit, each tensor has its own stream, the scales and decays are the stated
ones, and the packed-batch lengths fill the batch within their bounds."""
import math

import numpy as np
import torch

from causal_linear_attention_fwd_b200 import inputs


def test_same_seed_same_tensors_and_streams_differ():
    a = inputs.make_inputs(2, 3, 50, 64, 32, dtype=torch.bfloat16, seed=5, with_kv0=True)
    b = inputs.make_inputs(2, 3, 50, 64, 32, dtype=torch.bfloat16, seed=5, with_kv0=True)
    c = inputs.make_inputs(2, 3, 50, 64, 32, dtype=torch.bfloat16, seed=6, with_kv0=True)
    for n in a:
        assert torch.equal(a[n], b[n]), n
        assert not torch.equal(a[n], c[n]), n
    # q and k share a shape and a scale but come from different streams
    assert not torch.equal(a["q"], a["k"])
    # with_dO / with_kv0 do not shift the other tensors' streams
    d = inputs.make_inputs(2, 3, 50, 64, 32, dtype=torch.bfloat16, seed=5, with_dO=False)
    for n in ("q", "k", "v"):
        assert torch.equal(a[n], d[n]), n


def test_scales_and_rounding():
    d = 128
    x = inputs.make_inputs(1, 4, 4096, d, d, dtype=torch.float32, seed=0, with_kv0=True)
    for n, sd in (("q", 1 / math.sqrt(d)), ("k", 1 / math.sqrt(d)), ("v", 1.0), ("dO", 1.0),
                  ("kv0", 0.01)):
        t = x[n].double()
        assert abs(t.mean().item()) < 5 * sd / math.sqrt(t.numel()), n
        assert abs(t.std().item() / sd - 1) < 0.01, n
    # bf16 inputs are the fp32 draw rounded once
    y = inputs.make_inputs(1, 4, 4096, d, d, dtype=torch.bfloat16, seed=0)
    for n in ("q", "v"):
        assert torch.equal(y[n], x[n].to(torch.bfloat16)), n


def test_decay_lambdas():
    for H in (2, 16, 32, 64):
        lam = inputs.decay_lambdas(H)
        assert lam.dtype == torch.float32 and lam.shape == (H,)
        assert lam[0].item() == 1 - 2.0 ** -5          # exact in fp32
        want = np.array([1 - 2.0 ** -(5 + 8 * h / H) for h in range(H)], np.float64)
        assert np.array_equal(lam.numpy(), want.astype(np.float32))   # one rounding
        assert (np.diff(lam.numpy()) > 0).all() and lam[-1].item() < 1.0


def test_varlen_lengths():
    for seed in range(5):
        lens = inputs.varlen_lengths(65536, seed=seed)
        assert sum(lens) == 65536
        assert all(64 <= n <= 8192 for n in lens[:-1]) and 1 <= lens[-1] <= 8192
        assert lens == inputs.varlen_lengths(65536, seed=seed)


def test_decode_stream_is_seeded():
    a = inputs.DecodeStream(2, 3, 64, 32, seed=1)
    b = inputs.DecodeStream(2, 3, 64, 32, seed=1)
    for _ in range(3):
        for x, y in zip(a.next(), b.next()):
            assert torch.equal(x, y)
    q, k, v = a.next()
    assert q.shape == (2, 3, 64) and v.shape == (2, 3, 32) and q.dtype == torch.bfloat16
