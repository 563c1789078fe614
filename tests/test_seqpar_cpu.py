"""Sequence parallelism's exchange on CPU: two or three gloo ranks each hold one shard
of a sequence and run seqpar.forward / seqpar.backward with the library calls
replaced by plain fp64 stand-ins (the oracle and the definitions of the shard
summaries); the shards' slices must reassemble the oracle's result for the
whole sequence.  This checks the rank order of the all-gather and the
prefix indexing; the library's own shard calls are checked on the GPU."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from causal_linear_attention_fwd_b200 import inputs, seqpar

B, H, LS, D, E = 1, 2, 37, 6, 5
LAM = (0.93, 1.0)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _full_inputs(world):
    x = inputs.make_inputs(B, H, world * LS, D, E, dtype=torch.float32, seed=3, with_kv0=True)
    return {n: t.double() for n, t in x.items()}


class OracleOps:
    """fp64 stand-ins for the library calls seqpar makes."""
    orc = None

    @staticmethod
    def shard_state(a, b, lam, reverse=False):
        A, Bm, lh = a.numpy(), b.numpy(), lam.numpy()
        L = A.shape[2]
        out = np.zeros((A.shape[0], A.shape[1], A.shape[3], Bm.shape[3]))
        for i in range(A.shape[0]):
            for h in range(A.shape[1]):
                w = np.power(lh[h], np.arange(L) if reverse else L - 1 - np.arange(L))
                out[i, h] = (A[i, h] * w[:, None]).T @ Bm[i, h]
        return torch.from_numpy(out)

    @staticmethod
    def state_prefix(delta, lam, L, kv0=None, reverse=False):
        dl, lh = delta.numpy(), lam.numpy()
        R = dl.shape[0]
        out = np.zeros_like(dl)
        f = np.power(lh, L)[None, :, None, None]
        if not reverse:
            out[0] = kv0.numpy() if kv0 is not None else 0.0
            for r in range(1, R):
                out[r] = f * out[r - 1] + dl[r - 1]
        else:
            for r in range(R - 2, -1, -1):
                out[r] = f * out[r + 1] + dl[r + 1]
        return torch.from_numpy(out)

    @classmethod
    def forward(cls, q, k, v, lam, kv0, want_state=False):
        o, st = cls.orc.forward(q.numpy(), k.numpy(), v.numpy(), lam.numpy(), kv0.numpy(),
                                want_state=True)
        return (torch.from_numpy(o), torch.from_numpy(st)) if want_state else torch.from_numpy(o)

    @classmethod
    def backward_shard(cls, q, k, v, lam, dO, kv0, dend, want_dkv0=False):
        g = cls.orc.backward(q.numpy(), k.numpy(), v.numpy(), lam.numpy(), dO.numpy(),
                             kv0.numpy(), dstate_end=dend.numpy())
        g = tuple(torch.from_numpy(a) for a in g)
        return g if want_dkv0 else g[:3]


def _rank_main(rank, world, port, out):
    import oracle
    OracleOps.orc = oracle.load()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = _full_inputs(world)
        sl = {n: t[:, :, rank * LS:(rank + 1) * LS].contiguous()
              for n, t in x.items() if n != "kv0"}
        lam = torch.tensor(LAM, dtype=torch.float64)
        o, st = seqpar.forward(sl["q"], sl["k"], sl["v"], lam, x["kv0"], want_state=True,
                               ops=OracleOps)
        dq, dk, dv, dkv0 = seqpar.backward(sl["q"], sl["k"], sl["v"], lam, sl["dO"], x["kv0"],
                                           want_dkv0=True, ops=OracleOps)
        out[rank] = tuple(t.numpy() for t in (o, st, dq, dk, dv, dkv0))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_ranks_reassemble_the_whole_sequence(orc, world):
    """Three ranks give the middle rank a predecessor and a successor and the
    end ranks a summary two shards away, which two ranks cannot show."""
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    x = _full_inputs(world)
    lam = np.array(LAM)
    o, st = orc.forward(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), lam,
                        x["kv0"].numpy(), want_state=True)
    g = orc.backward(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(), lam, x["dO"].numpy(),
                     x["kv0"].numpy())
    cat = lambda i: np.concatenate([res[r][i] for r in range(world)], axis=2)
    np.testing.assert_allclose(cat(0), o, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(res[world - 1][1], st, rtol=1e-12, atol=1e-12)  # final state
    for i, ref in zip((2, 3, 4), g[:3]):
        np.testing.assert_allclose(cat(i), ref, rtol=1e-11, atol=1e-11)
    np.testing.assert_allclose(res[0][5], g[3], rtol=1e-11, atol=1e-11)  # dkv0 on rank 0
