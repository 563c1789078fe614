"""GPU parity of the state-pool serving calls against the oracle: multi-token
decode through a slot table (with inactive requests), prefill straight into
the pool, and a chunked continuation that reads and writes the same slots
(also with the sequence split across CTAs)."""
import numpy as np
import pytest
import torch

import causal_linear_attention_fwd_b200 as la2
from causal_linear_attention_fwd_b200 import inputs
from gpu_util import check, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
PATHS = {"simt": 1, "tc": 2}
CASES = [("tc", torch.bfloat16, (128, 128)), ("simt", torch.float32, (64, 64))]


def tokens(B, H, T, d, e, dtype, seed):
    """T decode tokens per request, [B,H,T,d|e], from the seeded decode stream."""
    gen = inputs.DecodeStream(B, H, d, e, dtype=dtype, device=DEV, seed=seed)
    steps = [gen.next() for _ in range(T)]
    return tuple(torch.stack([s[i] for s in steps], dim=2).contiguous() for i in range(3))


@pytest.mark.parametrize("block_from", [0, 1, 100000])
@pytest.mark.parametrize("T", [1, 3, 8, 9, 16, 17, 40, 128, 129])
@pytest.mark.parametrize("dtype,de", [(torch.bfloat16, (128, 128)), (torch.float32, (64, 64))])
def test_decode_tokens_matches_oracle(orc, T, dtype, de, block_from):
    """block_from: 0 = the library's crossover (token by token up to 16 tokens,
    the decode-unit kernel from 17), 1 = the tensor-core block form for every
    T (up to 128 tokens the decode-unit kernel, beyond it one chunk-schedule
    CTA per request; bf16 128 x 128 only), 100000 = the token-by-token kernel
    for every T (tokens staged 8 at a time, groups of 4 and a ragged last
    group)."""
    d, e = de
    B, H, P = 6, 3, 10
    slots_h = [7, -1, 2, 9, 0, 4]
    pool = inputs.decode_state0(P, H, d, e, device=DEV, seed=4)
    pool0 = pool.clone()
    slots = torch.tensor(slots_h, dtype=torch.int32, device=DEV)
    lam = inputs.fixed_lambdas((1.0, 0.99, 0.5), DEV)
    q, k, v = tokens(B, H, T, d, e, dtype, seed=T)
    o = torch.full((B, H, T, e), 7.0, dtype=dtype, device=DEV)
    old = la2.set_option(la2.LA2_OPT_DECODE_BLOCK_TOKENS, block_from)
    try:
        la2.decode_tokens(q, k, v, lam, pool, slots, out=o)
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_DECODE_BLOCK_TOKENS, old)
    assert la2.last_device_error() == 0
    lam_h = lam.double().cpu().numpy()
    for b, s in enumerate(slots_h):
        if s < 0:
            assert bool((o[b] == 7.0).all())  # inactive: outputs untouched
            continue
        kv = pool0[s:s + 1].double().cpu().numpy().copy()
        ref = np.stack([orc.decode_step(host(q[b:b + 1, :, t]), host(k[b:b + 1, :, t]),
                                        host(v[b:b + 1, :, t]), lam_h, kv)[0]
                        for t in range(T)], axis=1)
        check(f"decode T={T} req {b} o", o[b], ref, dtype)
        check(f"decode T={T} req {b} state", pool[s], kv[0], dtype)
    untouched = [i for i in range(P) if i not in slots_h]
    assert torch.equal(pool[untouched], pool0[untouched])


@pytest.mark.parametrize("split", [1, 3])
@pytest.mark.parametrize("path,dtype,de", CASES)
def test_prefill_decode_continue_matches_forward(orc, path, dtype, de, split):
    """prefill (L1 rows) into fresh slots, decode T tokens, continue with L2
    rows in place: every output equals the oracle's forward over the
    concatenated sequence, and the slot holds its final state."""
    d, e = de
    B, H, P, L1, T, L2 = 4, 2, 6, 300, 5, 200
    slots_h = [3, 0, 5, 1]
    slots = torch.tensor(slots_h, dtype=torch.int32, device=DEV)
    lam = inputs.decay_lambdas(H, DEV)
    x = inputs.make_inputs(B, H, L1 + T + L2, d, e, dtype=dtype, device=DEV, seed=split,
                           with_dO=False)
    pool = torch.full((P, H, d, e), 3.0, dtype=torch.float32, device=DEV)  # stale contents
    cut = lambda t, a, b: t[:, :, a:b].contiguous()
    old_p = la2.set_option(la2.LA2_OPT_PATH, PATHS[path])
    old_s = la2.set_option(la2.LA2_OPT_SPLIT, split)
    try:
        o1 = la2.forward_pool(cut(x["q"], 0, L1), cut(x["k"], 0, L1), cut(x["v"], 0, L1), lam,
                              pool, slots)
        o2 = la2.decode_tokens(cut(x["q"], L1, L1 + T), cut(x["k"], L1, L1 + T),
                               cut(x["v"], L1, L1 + T), lam, pool, slots)
        n = L1 + T
        o3 = la2.forward_pool(cut(x["q"], n, n + L2), cut(x["k"], n, n + L2),
                              cut(x["v"], n, n + L2), lam, pool, slots, continue_state=True)
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_PATH, old_p)
        la2.set_option(la2.LA2_OPT_SPLIT, old_s)
    assert la2.last_device_error() == 0
    o_ref, st_ref = orc.forward(host(x["q"]), host(x["k"]), host(x["v"]),
                                lam.double().cpu().numpy(), None, want_state=True)
    got = torch.cat([o1, o2, o3], dim=2)
    check(f"{path} S={split} o", got, o_ref, dtype)
    check(f"{path} S={split} final states", pool[slots_h], st_ref, dtype)
    assert bool((pool[[2, 4]] == 3.0).all())  # slots no request uses


def test_pool_slot_past_end_reported():
    """A slot >= pool_size: that request is skipped, the device error word
    reports LA2_ERR_INVALID, nothing faults."""
    B, H, P = 2, 2, 3
    pool = torch.zeros((P, H, 128, 128), dtype=torch.float32, device=DEV)
    slots = torch.tensor([1, 3], dtype=torch.int32, device=DEV)
    lam = inputs.decay_lambdas(H, DEV)
    q, k, v = tokens(B, H, 2, 128, 128, torch.bfloat16, seed=1)
    la2.last_device_error()
    la2.decode_tokens(q, k, v, lam, pool, slots)
    torch.cuda.synchronize()
    assert la2.last_device_error() == 1
    # the same through the decode-unit kernel (20 tokens per request); the
    # valid request's state still advances
    before = pool[1].clone()
    q20, k20, v20 = tokens(B, H, 20, 128, 128, torch.bfloat16, seed=3)
    la2.decode_tokens(q20, k20, v20, lam, pool, slots)
    torch.cuda.synchronize()
    assert la2.last_device_error() == 1
    assert not torch.equal(pool[1], before)
    x = inputs.make_inputs(B, H, 200, 128, 128, dtype=torch.bfloat16, device=DEV, seed=2,
                           with_dO=False)
    la2.forward_pool(x["q"], x["k"], x["v"], lam, pool, slots)
    torch.cuda.synchronize()
    assert la2.last_device_error() == 1
    assert la2.last_device_error() == 0


@pytest.mark.parametrize("T", [4, 64])
def test_decode_tokens_bench_batch_sampled(orc, T):
    """Multi-token decode on the batch the bench times (256 requests x H 64,
    d = e = 128, bf16 tokens, fp32 state of 1 GiB): two calls of T tokens,
    token by token at T = 4 and through the tensor-core block path at T = 64;
    sampled requests against the oracle's decode steps."""
    B, H, d, e = 256, 64, 128, 128
    kv = inputs.decode_state0(B, H, d, e, device=DEV, seed=0)
    kv0 = kv[[0, 77, 255]].double().cpu().numpy()
    lam = inputs.decay_lambdas(H, DEV)
    calls = [tokens(B, H, T, d, e, torch.bfloat16, seed=10 + c) for c in range(2)]
    outs = [la2.decode_tokens(q, k, v, lam, kv) for q, k, v in calls]
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    lam_h = lam.double().cpu().numpy()
    for i, b in enumerate((0, 77, 255)):
        st = kv0[i:i + 1].copy()
        for c, (q, k, v) in enumerate(calls):
            ref = np.stack([orc.decode_step(host(q[b:b + 1, :, t]), host(k[b:b + 1, :, t]),
                                            host(v[b:b + 1, :, t]), lam_h, st)[0]
                            for t in range(T)], axis=1)
            check(f"T={T} call {c} request {b} o", outs[c][b], ref, torch.bfloat16)
        check(f"T={T} request {b} state", kv[b], st[0], torch.bfloat16)


@pytest.mark.parametrize("T", [5, 64])
def test_decode_units_many_per_cta(orc, T):
    """The decode-unit kernel with several (request, head) units per CTA and
    ranges that cross a head: 300 requests x 3 heads (900 units), a slot
    table with inactive requests and a permuted pool; every request against
    the oracle's decode steps, inactive outputs and unused slots untouched."""
    d = e = 128
    B, H, P = 300, 3, 320
    rng = np.random.default_rng(T)
    perm = rng.permutation(P)[:B]
    slots_h = [int(s) if rng.random() > 0.1 else -1 for s in perm]
    pool = inputs.decode_state0(P, H, d, e, device=DEV, seed=5)
    pool0 = pool.clone()
    slots = torch.tensor(slots_h, dtype=torch.int32, device=DEV)
    lam = inputs.decay_lambdas(H, DEV)
    q, k, v = tokens(B, H, T, d, e, torch.bfloat16, seed=100 + T)
    o = torch.full((B, H, T, e), 7.0, dtype=torch.bfloat16, device=DEV)
    old = la2.set_option(la2.LA2_OPT_DECODE_BLOCK_TOKENS, 1)
    try:
        la2.decode_tokens(q, k, v, lam, pool, slots, out=o)
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_DECODE_BLOCK_TOKENS, old)
    assert la2.last_device_error() == 0
    lam_h = lam.double().cpu().numpy()
    qh, kh, vh = host(q), host(k), host(v)
    p0 = pool0.double().cpu().numpy()
    got_o, got_p = o.float().cpu().numpy(), pool.cpu().numpy()
    for b, s in enumerate(slots_h):
        if s < 0:
            assert bool((o[b] == 7.0).all())
            continue
        kv = p0[s:s + 1].copy()
        ref = np.stack([orc.decode_step(qh[b:b + 1, :, t], kh[b:b + 1, :, t], vh[b:b + 1, :, t],
                                        lam_h, kv)[0] for t in range(T)], axis=1)
        check(f"T={T} request {b} o", got_o[b], ref, torch.bfloat16)
        check(f"T={T} request {b} state", got_p[s], kv[0], torch.bfloat16)
    untouched = sorted(set(range(P)) - {s for s in slots_h if s >= 0})
    assert torch.equal(pool[untouched], pool0[untouched])


def test_decode_tokens_many_heads_fall_back(orc):
    """2 requests x 160 heads (320 units over at most one CTA per SM would
    give a CTA more than two heads): the call falls back to one CTA per
    (request, head), against the oracle."""
    B, H, T, d, e = 2, 160, 40, 128, 128
    pool = inputs.decode_state0(B, H, d, e, device=DEV, seed=6)
    pool0 = pool.double().cpu().numpy()
    lam = inputs.decay_lambdas(H, DEV)
    q, k, v = tokens(B, H, T, d, e, torch.bfloat16, seed=7)
    o = la2.decode_tokens(q, k, v, lam, pool)
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    lam_h = lam.double().cpu().numpy()
    for b in range(B):
        kv = pool0[b:b + 1].copy()
        ref = np.stack([orc.decode_step(host(q[b:b + 1, :, t]), host(k[b:b + 1, :, t]),
                                        host(v[b:b + 1, :, t]), lam_h, kv)[0]
                        for t in range(T)], axis=1)
        check(f"request {b} o", o[b], ref, torch.bfloat16)
        check(f"request {b} state", pool[b], kv[0], torch.bfloat16)


@pytest.mark.parametrize("case", range(12))
def test_decode_units_agree_with_token_kernel(case):
    """Seeded random shapes (B up to 300, H up to 20, T up to 128, slot tables
    with inactive requests): the decode-unit kernel and the token-by-token
    kernel, two independent paths, give the same outputs and states to the
    bf16 tolerance."""
    rng = np.random.default_rng(1000 + case)
    B, H, T = int(rng.integers(1, 301)), int(rng.integers(1, 21)), int(rng.integers(1, 129))
    P = B + int(rng.integers(0, 8))
    perm = rng.permutation(P)[:B]
    slots_h = [int(s) if rng.random() > 0.15 else -1 for s in perm]
    slots = torch.tensor(slots_h, dtype=torch.int32, device=DEV)
    lam = inputs.decay_lambdas(H, DEV)
    q, k, v = tokens(B, H, T, 128, 128, torch.bfloat16, seed=2000 + case)
    pool0 = inputs.decode_state0(P, H, 128, 128, device=DEV, seed=case)
    res = {}
    for name, frm in (("units", 1), ("token", 100000)):
        pool = pool0.clone()
        o = torch.full((B, H, T, 128), 7.0, dtype=torch.bfloat16, device=DEV)
        old = la2.set_option(la2.LA2_OPT_DECODE_BLOCK_TOKENS, frm)
        try:
            la2.decode_tokens(q, k, v, lam, pool, slots, out=o)
            torch.cuda.synchronize()
        finally:
            la2.set_option(la2.LA2_OPT_DECODE_BLOCK_TOKENS, old)
        assert la2.last_device_error() == 0
        res[name] = (o, pool)
    tag = f"B={B} H={H} T={T}"
    check(f"{tag} o", res["units"][0], host(res["token"][0]), torch.bfloat16)
    check(f"{tag} pool", res["units"][1], host(res["token"][1]), torch.bfloat16)
    assert torch.equal(res["units"][0][[b for b, s in enumerate(slots_h) if s < 0]],
                       res["token"][0][[b for b, s in enumerate(slots_h) if s < 0]])
