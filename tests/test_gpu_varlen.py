"""GPU parity of the packed variable-length entry points against the oracle.

Each sequence of a packed batch is an independent problem with its own state,
so the reference is the oracle run on each sequence's rows alone (B = 1), its
initial state the sequence's slice of kv0.  The lengths mix empty, single-row,
block-sized, ragged and multi-block sequences; every sequence but the last is
followed by another one's rows, which its last block reads and must ignore."""
import numpy as np
import pytest
import torch

import causal_linear_attention_fwd_b200 as la2
from causal_linear_attention_fwd_b200 import inputs
from gpu_util import check, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
PATHS = {"simt": 1, "tc": 2}
LENS = [300, 0, 1, 127, 128, 129, 1000, 5, 256]


def packed_inputs(lens, H, d, e, dtype, seed):
    T = sum(lens)
    N = len(lens)
    x = inputs.make_inputs(1, H, T, d, e, dtype=dtype, device=DEV, seed=seed)
    x = {n: t[0] for n, t in x.items()}  # [H, T, .]
    kv0 = inputs.make_inputs(N, H, 1, d, e, dtype=dtype, device=DEV, seed=seed + 1,
                             with_dO=False, with_kv0=True)["kv0"]
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int64, device=DEV)
    return x, kv0, cu


def reference(orc, x, kv0, cu, lam):
    """Per-sequence oracle results scattered back to the packed layout."""
    H, T, d = x["q"].shape
    e = x["v"].shape[-1]
    N = cu.numel() - 1
    h = {n: host(t) for n, t in x.items()}
    lam_h = lam.double().cpu().numpy()
    s0 = kv0.double().cpu().numpy()
    o = np.zeros((H, T, e)); dq = np.zeros((H, T, d)); dk = np.zeros((H, T, d))
    dv = np.zeros((H, T, e))
    st = np.zeros((N, H, d, e)); dkv0 = np.zeros((N, H, d, e))
    offs = cu.cpu().numpy()
    for n in range(N):
        a, b = int(offs[n]), int(offs[n + 1])
        if a == b:
            st[n] = s0[n]
            continue
        sl = {k: v[None, :, a:b] for k, v in h.items()}
        on, sn = orc.forward(sl["q"], sl["k"], sl["v"], lam_h, s0[n:n + 1], want_state=True)
        g = orc.backward(sl["q"], sl["k"], sl["v"], lam_h, sl["dO"], s0[n:n + 1])
        o[:, a:b] = on[0]
        st[n] = sn[0]
        dq[:, a:b], dk[:, a:b], dv[:, a:b] = g[0][0], g[1][0], g[2][0]
        dkv0[n] = g[3][0]
    return o, st, dq, dk, dv, dkv0


@pytest.mark.parametrize("path,dtype,de", [("tc", torch.bfloat16, (128, 128)),
                                           ("simt", torch.float32, (64, 64)),
                                           ("simt", torch.bfloat16, (64, 128))])
def test_varlen_matches_oracle(orc, path, dtype, de):
    d, e = de
    H = 3
    x, kv0, cu = packed_inputs(LENS, H, d, e, dtype, seed=5)
    lam = inputs.fixed_lambdas((1.0, 0.97, 0.0), DEV)
    old = la2.set_option(la2.LA2_OPT_PATH, PATHS[path])
    try:
        o, st = la2.forward_varlen(x["q"], x["k"], x["v"], lam, cu, kv0, want_state=True)
        dq, dk, dv, dkv0 = la2.backward_varlen(x["q"], x["k"], x["v"], lam, cu, x["dO"], kv0,
                                               want_dkv0=True)
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_PATH, old)
    assert la2.last_device_error() == 0
    ref = reference(orc, x, kv0, cu, lam)
    for name, got, r in zip(("o", "kv_out", "dq", "dk", "dv", "dkv0"),
                            (o, st, dq, dk, dv, dkv0), ref):
        check(f"varlen {path} {name}", got, r, dtype)


def test_varlen_equals_batched_call():
    """Equal-length sequences packed give what the [B,H,L,d] call gives for
    the same rows (the tensor-core path in both)."""
    Bn, H, L = 3, 2, 700
    x = inputs.make_inputs(Bn, H, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=9,
                           with_kv0=True)
    lam = inputs.decay_lambdas(H, DEV)
    o_b, st_b = la2.forward(x["q"], x["k"], x["v"], lam, x["kv0"], want_state=True)
    pack = {n: x[n].permute(1, 0, 2, 3).reshape(H, Bn * L, -1).contiguous()
            for n in ("q", "k", "v")}
    cu = torch.arange(0, (Bn + 1) * L, L, dtype=torch.int64, device=DEV)
    o_v, st_v = la2.forward_varlen(pack["q"], pack["k"], pack["v"], lam, cu, x["kv0"],
                                   want_state=True)
    torch.cuda.synchronize()
    o_v = o_v.reshape(H, Bn, L, -1).permute(1, 0, 2, 3)
    # the batched call may split each sequence into chunks (another
    # summation order), so the two agree to the parity tolerance
    check("packed vs batched o", o_v, host(o_b), torch.bfloat16)
    check("packed vs batched state", st_v, host(st_b), torch.bfloat16)


def test_varlen_bad_offsets_reported():
    """Offsets outside [0, T] or decreasing: that sequence is treated as
    empty and the device error word reports LA2_ERR_INVALID; nothing faults."""
    H, T = 2, 600
    x = inputs.make_inputs(1, H, T, 128, 128, dtype=torch.bfloat16, device=DEV, seed=3)
    lam = inputs.decay_lambdas(H, DEV)
    la2.last_device_error()  # clear
    for bad in ([0, 400, 200, 600], [0, 300, 900]):
        cu = torch.tensor(bad, dtype=torch.int64, device=DEV)
        la2.forward_varlen(x["q"][0], x["k"][0], x["v"][0], lam, cu)
        torch.cuda.synchronize()
        assert la2.last_device_error() == 1  # LA2_ERR_INVALID
    assert la2.last_device_error() == 0


def test_varlen_bench_batch_sampled(orc):
    """The packed batch the bench times (35 sequences of 64..8,082 rows,
    65,536 rows per head, H = 32, bf16, seed 0), forward and backward in one
    launch each; sampled (sequence, head) pairs -- the longest, the shortest,
    the first and the last sequence, heads 0, 17 and 31 -- against the oracle
    on that sequence's rows alone."""
    H, T = 32, 65536
    lens = inputs.varlen_lengths(T, seed=0)
    offs = np.concatenate([[0], np.cumsum(lens)])
    cu = torch.tensor(offs, dtype=torch.int64, device=DEV)
    x = inputs.make_inputs(1, H, T, 128, 128, dtype=torch.bfloat16, device=DEV, seed=0)
    x = {n: t[0] for n, t in x.items()}
    lam = inputs.decay_lambdas(H, DEV)
    o = la2.forward_varlen(x["q"], x["k"], x["v"], lam, cu)
    dq, dk, dv = la2.backward_varlen(x["q"], x["k"], x["v"], lam, cu, x["dO"])
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    lam_h = lam.double().cpu().numpy()
    seqs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 0, len(lens) - 1})
    for n in seqs:
        a, b = int(offs[n]), int(offs[n + 1])
        for hh in (0, 17, 31):
            sl = {k: host(t[hh:hh + 1, a:b])[None] for k, t in x.items()}
            o_ref = orc.forward(sl["q"], sl["k"], sl["v"], lam_h[hh:hh + 1])
            g = orc.backward(sl["q"], sl["k"], sl["v"], lam_h[hh:hh + 1], sl["dO"])
            tag = f"seq {n} ({b - a} rows) head {hh}"
            check(f"{tag} o", o[hh, a:b], o_ref[0, 0], torch.bfloat16)
            for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), g[:3]):
                check(f"{tag} {name}", got[hh, a:b], ref[0, 0], torch.bfloat16)


def _varlen_all(x, kv0, cu, lam, order):
    """Every output of a packed forward + backward with the given CTA order
    option; outputs pre-filled with NaN, so a (sequence, head) that no CTA
    served would show."""
    H, T, d = x["q"].shape
    e = x["v"].shape[-1]
    N = cu.numel() - 1
    nan = lambda *s: torch.full(s, float("nan"), dtype=x["q"].dtype, device=DEV)
    o = nan(H, T, e)
    outs = (nan(H, T, d), nan(H, T, d), nan(H, T, e))
    old = la2.set_option(la2.LA2_OPT_VARLEN_ORDER, order)
    try:
        _, st = la2.forward_varlen(x["q"], x["k"], x["v"], lam, cu, kv0, want_state=True, out=o)
        g = la2.backward_varlen(x["q"], x["k"], x["v"], lam, cu, x["dO"], kv0, want_dkv0=True,
                                outs=outs)
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_VARLEN_ORDER, old)
    assert la2.last_device_error() == 0
    assert N > 0
    return (o, st) + tuple(g)


def test_varlen_longest_first_is_a_reordering():
    """Longest-first CTA order (the default for <= 64 sequences; lengths with
    ties, an empty and a one-row sequence) serves every (sequence, head) once
    with the same arithmetic: results bitwise equal to the given order's."""
    lens = [300, 0, 1, 1000, 128, 1000, 5, 256, 129, 300, 2000, 7]
    x, kv0, cu = packed_inputs(lens, 4, 128, 128, torch.bfloat16, seed=11)
    lam = inputs.decay_lambdas(4, DEV)
    a = _varlen_all(x, kv0, cu, lam, 0)
    b = _varlen_all(x, kv0, cu, lam, 1)
    for name, u, w in zip(("o", "kv_out", "dq", "dk", "dv", "dkv0"), a, b):
        assert not torch.isnan(u).any(), name
        assert torch.equal(u, w), name


def test_varlen_many_sequences_matches_oracle(orc):
    """70 sequences (above the longest-first limit: the given order), lengths
    0..400 rows, against the oracle per sequence."""
    lens = [int(v) for v in np.random.default_rng(70).integers(0, 400, size=70)]
    x, kv0, cu = packed_inputs(lens, 2, 128, 128, torch.bfloat16, seed=12)
    lam = inputs.decay_lambdas(2, DEV)
    got = _varlen_all(x, kv0, cu, lam, 0)
    ref = reference(orc, x, kv0, cu, lam)
    for name, u, r in zip(("o", "kv_out", "dq", "dk", "dv", "dkv0"), got, ref):
        check(f"70 sequences {name}", u, r, torch.bfloat16)


@pytest.mark.parametrize("case", range(8))
def test_varlen_random_batches_agree_with_per_document_calls(case):
    """Seeded random packed batches (1..80 documents of 0..700 rows, 1..6
    heads, both CTA orders by the document count) against the library's
    batched calls on each document alone, forward and backward, with the
    documents' own initial states."""
    rng = np.random.default_rng(500 + case)
    N, H = int(rng.integers(1, 81)), int(rng.integers(1, 7))
    lens = [int(x) for x in rng.integers(0, 701, size=N)]
    if sum(lens) == 0:
        lens[0] = 1
    x, kv0, cu = packed_inputs(lens, H, 128, 128, torch.bfloat16, seed=600 + case)
    lam = inputs.decay_lambdas(H, DEV)
    got = _varlen_all(x, kv0, cu, lam, 0)
    offs = cu.cpu().numpy()
    for n in range(N):
        a, b = int(offs[n]), int(offs[n + 1])
        if a == b:
            continue
        sl = {k: t[None, :, a:b].contiguous() for k, t in x.items()}
        s0 = kv0[n:n + 1].contiguous()
        o, st = la2.forward(sl["q"], sl["k"], sl["v"], lam, s0, want_state=True)
        dq, dk, dv, dkv0 = la2.backward(sl["q"], sl["k"], sl["v"], lam, sl["dO"], s0,
                                        want_dkv0=True)
        tag = f"case {case} doc {n} ({b - a} rows, N={N}, H={H})"
        for name, u, r in (("o", got[0][:, a:b], o[0]), ("dq", got[2][:, a:b], dq[0]),
                           ("dk", got[3][:, a:b], dk[0]), ("dv", got[4][:, a:b], dv[0]),
                           ("kv_out", got[1][n], st[0]), ("dkv0", got[5][n], dkv0[0])):
            check(f"{tag} {name}", u, host(r), torch.bfloat16)


@pytest.mark.parametrize("order", [0, 1])
def test_varlen_paired_reverse_matches_two_passes(order):
    """The packed backward's dV and dK from the paired launch equal the two
    separate passes' bitwise (both CTA orders; an empty, a one-row and a
    ragged sequence included)."""
    lens = [300, 0, 1, 1000, 129, 2000, 7]
    x, kv0, cu = packed_inputs(lens, 4, 128, 128, torch.bfloat16, seed=17)
    lam = inputs.decay_lambdas(4, DEV)
    res = {}
    for form in (0, 1):
        old = la2.set_option(la2.LA2_OPT_BWD_FORM, form)
        try:
            res[form] = _varlen_all(x, kv0, cu, lam, order)
        finally:
            la2.set_option(la2.LA2_OPT_BWD_FORM, old)
    for a, b in zip(res[0], res[1]):
        assert torch.equal(a, b)
