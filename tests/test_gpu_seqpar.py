"""GPU parity of the sequence-sharding calls: R shards of one sequence run
one after another on this GPU (the exchange done by stacking the shards'
summaries, as the all-gather would) reassemble the oracle's result for the
whole sequence; seqpar over a one-rank NCCL group equals the plain calls."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist

import causal_linear_attention_fwd_b200 as la2
from causal_linear_attention_fwd_b200 import inputs, seqpar
from gpu_util import check, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
PATHS = {"simt": 1, "tc": 2}


@pytest.mark.parametrize("split", [0, 3])
@pytest.mark.parametrize("path,dtype,de", [("tc", torch.bfloat16, (128, 128)),
                                           ("simt", torch.float32, (64, 64))])
def test_shards_reassemble_the_sequence(orc, path, dtype, de, split):
    d, e = de
    R, B, H, LS = 3, 2, 2, 333
    x = inputs.make_inputs(B, H, R * LS, d, e, dtype=dtype, device=DEV, seed=7 + split,
                           with_kv0=True)
    lam = inputs.fixed_lambdas((0.97, 0.9999), DEV)
    sh = lambda t, r: t[:, :, r * LS:(r + 1) * LS].contiguous()
    old_p = la2.set_option(la2.LA2_OPT_PATH, PATHS[path])
    old_s = la2.set_option(la2.LA2_OPT_SPLIT, split)
    try:
        fwd_d = torch.stack([la2.shard_state(sh(x["k"], r), sh(x["v"], r), lam) for r in range(R)])
        rev_d = torch.stack([la2.shard_state(sh(x["q"], r), sh(x["dO"], r), lam, reverse=True)
                             for r in range(R)])
        entry = la2.state_prefix(fwd_d, lam, LS, x["kv0"])
        end = la2.state_prefix(rev_d, lam, LS, reverse=True)
        outs, grads = [], []
        for r in range(R):
            outs.append(la2.forward(sh(x["q"], r), sh(x["k"], r), sh(x["v"], r), lam,
                                    entry[r].contiguous(), want_state=True))
            grads.append(la2.backward_shard(sh(x["q"], r), sh(x["k"], r), sh(x["v"], r), lam,
                                            sh(x["dO"], r), entry[r].contiguous(),
                                            end[r].contiguous(), want_dkv0=True))
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_PATH, old_p)
        la2.set_option(la2.LA2_OPT_SPLIT, old_s)
    assert la2.last_device_error() == 0
    h = {n: host(t) for n, t in x.items()}
    lam_h = lam.double().cpu().numpy()
    o_ref, st_ref = orc.forward(h["q"], h["k"], h["v"], lam_h, h["kv0"], want_state=True)
    g_ref = orc.backward(h["q"], h["k"], h["v"], lam_h, h["dO"], h["kv0"])
    tag = f"{path} S={split}"
    check(f"{tag} o", torch.cat([o for o, _ in outs], 2), o_ref, dtype)
    check(f"{tag} final state", outs[-1][1], st_ref, dtype)
    for i, name in enumerate(("dq", "dk", "dv")):
        check(f"{tag} {name}", torch.cat([g[i] for g in grads], 2), g_ref[i], dtype)
    check(f"{tag} dkv0", grads[0][3], g_ref[3], dtype)
    # the summaries themselves against their definitions (fp64 on the host)
    for r in range(R):
        q_, k_, v_, g_ = (h[n][:, :, r * LS:(r + 1) * LS] for n in ("q", "k", "v", "dO"))
        t = np.arange(LS)
        for hh in range(H):
            wf = np.power(lam_h[hh], LS - 1 - t)[:, None]
            wr = np.power(lam_h[hh], t)[:, None]
            for b in range(B):
                check(f"{tag} forward delta r={r}", fwd_d[r, b, hh],
                      (k_[b, hh] * wf).T @ v_[b, hh], dtype)
                check(f"{tag} reverse delta r={r}", rev_d[r, b, hh],
                      (q_[b, hh] * wr).T @ g_[b, hh], dtype)


def test_seqpar_one_rank_equals_plain_calls():
    """With one rank the entry state is kv0 and the end state zero."""
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        x = inputs.make_inputs(1, 4, 1500, 128, 128, dtype=torch.bfloat16, device=DEV, seed=8,
                               with_kv0=True)
        lam = inputs.decay_lambdas(4, DEV)
        o, st = seqpar.forward(x["q"], x["k"], x["v"], lam, x["kv0"], want_state=True)
        g = seqpar.backward(x["q"], x["k"], x["v"], lam, x["dO"], x["kv0"], want_dkv0=True)
        o_ref, st_ref = la2.forward(x["q"], x["k"], x["v"], lam, x["kv0"], want_state=True)
        g_ref = la2.backward(x["q"], x["k"], x["v"], lam, x["dO"], x["kv0"], want_dkv0=True)
        torch.cuda.synchronize()
        for a, b in zip((o, st) + tuple(g), (o_ref, st_ref) + tuple(g_ref)):
            check("seqpar vs plain", a, host(b), torch.bfloat16)
    finally:
        dist.destroy_process_group()
