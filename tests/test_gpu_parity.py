"""GPU parity: the CUDA path through the C ABI against the fp64 oracle on the
same seeded inputs, element by element, at the parity bar of gpu_util.TOL.

Small cases span several blocks and chunks with ragged tails; the full-size
workloads are checked on sampled heads / states that the oracle computes in
full, plus properties that hold at any size (adjoint identities)."""
import contextlib

import numpy as np
import pytest
import torch

import causal_linear_attention_fwd_b200 as la2
from causal_linear_attention_fwd_b200 import inputs
from gpu_util import check, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
PATHS = {"simt": 1, "tc": 2}


@contextlib.contextmanager
def options(path=None, split=None, variant=None):
    old_p = la2.set_option(la2.LA2_OPT_PATH, PATHS[path]) if path else None
    old_s = la2.set_option(la2.LA2_OPT_SPLIT, split) if split is not None else None
    old_v = la2.set_option(la2.LA2_OPT_VARIANT, variant) if variant is not None else None
    try:
        yield
    finally:
        if path:
            la2.set_option(la2.LA2_OPT_PATH, old_p)
        if split is not None:
            la2.set_option(la2.LA2_OPT_SPLIT, old_s)
        if variant is not None:
            la2.set_option(la2.LA2_OPT_VARIANT, old_v)


def run_fwd_bwd(x, lam, kv0=None):
    """forward (with final state) + backward (with dkv0); None if the forced
    path does not cover this shape."""
    try:
        o, st = la2.forward(x["q"], x["k"], x["v"], lam, kv0, want_state=True)
        dq, dk, dv, dkv0 = la2.backward(x["q"], x["k"], x["v"], lam, x["dO"], kv0,
                                        want_dkv0=True)
    except la2.LA2Error as err:
        if err.code == 2:  # LA2_ERR_UNSUPPORTED
            return None
        raise
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    return o, st, dq, dk, dv, dkv0


def oracle_all(orc, x, lam, kv0=None):
    h = {n: host(t) for n, t in x.items()}
    lam_h = lam.double().cpu().numpy()
    s0 = None if kv0 is None else kv0.double().cpu().numpy()
    o, st = orc.forward(h["q"], h["k"], h["v"], lam_h, s0, want_state=True)
    g = orc.backward(h["q"], h["k"], h["v"], lam_h, h["dO"], s0)
    return (o, st) + tuple(g)


NAMES = ("o", "kv_out", "dq", "dk", "dv", "dkv0")


def compare(got, ref, dtype, tag):
    for name, a, r in zip(NAMES, got, ref):
        check(f"{tag} {name}", a, r, dtype)


# ------------------------------------------------------------------ fp32 PR1
def test_pr1_fp32(orc):
    """B=1, H=2, L=256, d=e=64, fp32, lambda = (1.0, 0.99), seed 0."""
    x = inputs.make_inputs(1, 2, 256, 64, 64, dtype=torch.float32, device=DEV, seed=0)
    lam = inputs.fixed_lambdas((1.0, 0.99), DEV)
    got = run_fwd_bwd(x, lam)
    compare(got, oracle_all(orc, x, lam), torch.float32, "pr1")


@pytest.mark.parametrize("split", [1, 3])
def test_fp32_with_state(orc, split):
    x = inputs.make_inputs(2, 3, 300, 64, 128, dtype=torch.float32, device=DEV, seed=3,
                           with_kv0=True)
    lam = inputs.fixed_lambdas((1.0, 0.9, 0.0), DEV)
    with options(split=split):
        got = run_fwd_bwd(x, lam, x["kv0"])
    compare(got, oracle_all(orc, x, lam, x["kv0"]), torch.float32, f"fp32 S={split}")


# --------------------------------------------------------- small bf16 shapes
@pytest.mark.parametrize("path", ["simt", "tc"])
@pytest.mark.parametrize("L", [1, 127, 128, 257, 1000])
@pytest.mark.parametrize("de", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_bf16_small(orc, path, L, de):
    d, e = de
    x = inputs.make_inputs(2, 3, L, d, e, dtype=torch.bfloat16, device=DEV, seed=L + d,
                           with_kv0=True)
    lam = inputs.fixed_lambdas((1.0, 0.97, 0.0), DEV)
    with options(path=path):
        got = run_fwd_bwd(x, lam, x["kv0"])
    if got is None:
        pytest.skip(f"{path} path does not cover d={d}, e={e}")
    compare(got, oracle_all(orc, x, lam, x["kv0"]), torch.bfloat16, f"{path} L={L} d={d} e={e}")


@pytest.mark.parametrize("path", ["simt", "tc"])
@pytest.mark.parametrize("split", [1, 2, 3, 7])
def test_forced_split(orc, path, split):
    """Chunk split (pre-pass + scan) gives the oracle's result for any S,
    with a ragged last chunk and a ragged last block."""
    x = inputs.make_inputs(1, 4, 1000, 128, 128, dtype=torch.bfloat16, device=DEV, seed=11,
                           with_kv0=True)
    lam = inputs.decay_lambdas(4, DEV)
    with options(path=path, split=split):
        got = run_fwd_bwd(x, lam, x["kv0"])
    if got is None:
        pytest.skip(f"{path} path unavailable")
    compare(got, oracle_all(orc, x, lam, x["kv0"]), torch.bfloat16, f"{path} S={split}")


@pytest.mark.parametrize("split", [1, 3])
@pytest.mark.parametrize("L", [129, 1000])
def test_tc_decay_range(orc, L, split):
    """Heads across the range of lambda, from fast decay (lambda^128 far
    below fp32's normal range) to none, agree with the oracle on the
    tensor-core path (ragged block, forced chunk split, initial state and
    dkv0)."""
    x = inputs.make_inputs(2, 6, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=L + split,
                           with_kv0=True)
    lam = inputs.fixed_lambdas((0.3, 0.8, 0.81, 0.9, 0.999, 1.0), DEV)
    with options(path="tc", split=split):
        got = run_fwd_bwd(x, lam, x["kv0"])
    compare(got, oracle_all(orc, x, lam, x["kv0"]), torch.bfloat16, f"decay range L={L} S={split}")


@pytest.mark.parametrize("split", [1, 3])
@pytest.mark.parametrize("L", [200, 1000])
def test_tc_phase_serial_variant(orc, L, split):
    """The simpler phase-serial form of the tensor-core kernel (kept for
    comparison) gives the oracle's result too."""
    x = inputs.make_inputs(2, 2, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=L,
                           with_kv0=True)
    lam = inputs.fixed_lambdas((0.9, 1.0), DEV)
    with options(path="tc", split=split, variant=1):
        got = run_fwd_bwd(x, lam, x["kv0"])
    compare(got, oracle_all(orc, x, lam, x["kv0"]), torch.bfloat16, f"v1 L={L} S={split}")


@pytest.mark.parametrize("de", [(128, 128), (64, 128), (64, 64)])
@pytest.mark.parametrize("path", ["simt", "tc"])
def test_backward_reuses_forward_states(orc, path, de):
    """A training step that hands the forward's workspace to the backward
    (LA2_BWD_REUSE_FORWARD_STATES) gives the same gradients as a backward
    that recomputes the chunk states, and the oracle's (with 64-column heads
    the tensor-core workspace also holds the padded states after the chunk
    states)."""
    B, H, L = 1, 3, 1000
    d, e = de
    x = inputs.make_inputs(B, H, L, d, e, dtype=torch.bfloat16, device=DEV, seed=13,
                           with_kv0=True)
    lam = inputs.fixed_lambdas((1.0, 0.95, 0.5), DEV)
    with options(path=path, split=4):
        n = la2.workspace_size(la2.LA2_OP_BACKWARD, B, H, L, d, e, torch.bfloat16)
        assert n > 0
        ws = torch.empty(n, dtype=torch.uint8, device=DEV)
        o = la2.forward(x["q"], x["k"], x["v"], lam, x["kv0"], workspace=ws)
        got = la2.backward(x["q"], x["k"], x["v"], lam, x["dO"], x["kv0"], want_dkv0=True,
                           workspace=ws, reuse_forward_states=True)
        ref = la2.backward(x["q"], x["k"], x["v"], lam, x["dO"], x["kv0"], want_dkv0=True)
        torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
    want = oracle_all(orc, x, lam, x["kv0"])
    for name, a, r in zip(("dq", "dk", "dv", "dkv0"), got, want[2:]):
        check(f"reuse {path} {name}", a, r, torch.bfloat16)
    check(f"reuse {path} o", o, want[0], torch.bfloat16)


def test_split_invariance_gpu():
    """Different splits agree with each other (same kernels, other chunking)."""
    x = inputs.make_inputs(2, 2, 2048, 128, 128, dtype=torch.bfloat16, device=DEV, seed=5)
    lam = inputs.decay_lambdas(2, DEV)
    res = []
    for s in (1, 4, 16):
        with options(split=s):
            res.append(run_fwd_bwd(x, lam))
    for other in res[1:]:
        for name, a, b in zip(NAMES, other, res[0]):
            check(f"split {name}", a, host(b), torch.bfloat16)


def test_empty_and_degenerate(orc):
    lam = inputs.fixed_lambdas((0.5, 1.0), DEV)
    kv0 = inputs.randn((1, 2, 128, 128), dtype=torch.float32, device=DEV, seed=9, tid=4)
    e0 = torch.empty((1, 2, 0, 128), dtype=torch.bfloat16, device=DEV)
    o, st = la2.forward(e0, e0, e0, lam, kv0, want_state=True)
    dq, dk, dv, dkv0 = la2.backward(e0, e0, e0, lam, e0, kv0, want_dkv0=True)
    torch.cuda.synchronize()
    assert o.numel() == 0 and torch.equal(st, kv0)
    assert torch.count_nonzero(dkv0) == 0


def test_head_and_batch_independence():
    """Changing one (b,h) problem leaves every other output untouched."""
    x = inputs.make_inputs(2, 3, 300, 128, 128, dtype=torch.bfloat16, device=DEV, seed=21)
    lam = inputs.decay_lambdas(3, DEV)
    base = run_fwd_bwd(x, lam)
    y = {n: t.clone() for n, t in x.items()}
    y["v"][1, 2] *= -3
    y["q"][1, 2] *= 2
    pert = run_fwd_bwd(y, lam)
    for name, a, b in zip(NAMES, base, pert):
        a = a.view(6, *a.shape[2:])
        b = b.view(6, *b.shape[2:])
        assert torch.equal(a[:5], b[:5]), name


# ------------------------------------------------------ workload: 2 (B4 H16)
def test_b4_h16_l2048(orc):
    """B=4, H=16, L=2048, d=e=128, bf16, decay lambda_h, fwd+bwd, full check."""
    x = inputs.make_inputs(4, 16, 2048, 128, 128, dtype=torch.bfloat16, device=DEV, seed=0)
    lam = inputs.decay_lambdas(16, DEV)
    got = run_fwd_bwd(x, lam)
    compare(got, oracle_all(orc, x, lam), torch.bfloat16, "B4H16L2048")


# ------------------------------------------- workload: length sweep (H=32)
SWEEP = [(16, 4096), (8, 8192), (4, 16384), (2, 32768), (1, 65536)]


@pytest.fixture(scope="module")
def sweep_buffers():
    n = 65536 * 32
    x = inputs.make_inputs(1, 32, 65536, 128, 128, dtype=torch.bfloat16, device=DEV, seed=0)
    return x, n


def sweep_picks(Bn, H=32, n=8):
    """n distinct (b, h) sequences of a [Bn, H] sweep point: the first and
    the last, middle heads of the middle batch row, and others spread over
    the rows and heads."""
    cand = [(0, 0), (Bn - 1, H - 1), (Bn // 2, H // 2), (Bn // 2, 0), (0, H - 1),
            ((Bn - 1) // 3, 21 % H), ((2 * Bn) // 3, 10 % H), (Bn - 1, 0),
            (Bn // 2, 5), (Bn // 2, 26), (0, 13), (Bn - 1, 18)]
    out = []
    for p in cand:
        if p not in out:
            out.append(p)
    return out[:n]


def test_sweep_picks_are_spread():
    for Bn, _ in SWEEP:
        p = sweep_picks(Bn)
        assert len(p) == 8 and len(set(p)) == 8
        assert (0, 0) in p and (Bn - 1, 31) in p and (Bn // 2, 16) in p


@pytest.mark.parametrize("BL", SWEEP, ids=[f"B{b}_L{l}" for b, l in SWEEP])
def test_sweep_sampled_heads(orc, sweep_buffers, BL):
    """Full-size sweep point in the bench's launch configuration; the oracle
    recomputes eight whole (b,h) sequences (first, last, middle heads of the
    middle batch row, and others spread over rows and heads); adjoint
    identities hold over every head."""
    Bn, L = BL
    xs, _ = sweep_buffers
    x = {n: t.view(Bn, 32, L, 128) for n, t in xs.items()}
    lam = inputs.decay_lambdas(32, DEV)
    o = la2.forward(x["q"], x["k"], x["v"], lam)
    dq, dk, dv = la2.backward(x["q"], x["k"], x["v"], lam, x["dO"])
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    lam_h = lam.double().cpu().numpy()
    picks = sweep_picks(Bn)
    # the sampled sequences go to the oracle as one [1, n, L, .] problem
    sub = {n: np.concatenate([host(t[b:b + 1, h:h + 1]) for b, h in picks], axis=1)
           for n, t in x.items()}
    lh = np.array([lam_h[h] for _, h in picks])
    o_r = orc.forward(sub["q"], sub["k"], sub["v"], lh)
    g_r = orc.backward(sub["q"], sub["k"], sub["v"], lh, sub["dO"])
    for i, (b, h) in enumerate(picks):
        for name, a, r in zip(("o", "dq", "dk", "dv"), (o, dq, dk, dv), (o_r,) + g_r[:3]):
            check(f"sweep B{Bn} L{L} (b={b},h={h}) {name}", a[b:b + 1, h:h + 1],
                  r[:, i:i + 1], torch.bfloat16)
    # adjoint identities (o is linear in q, and in k, and in v):
    # sum dq*q = sum dk*k = sum dv*v = sum dO*o, per head, in fp64
    ref = (o.double() * x["dO"].double()).sum(dim=(2, 3))
    for name, g, t in (("q", dq, x["q"]), ("k", dk, x["k"]), ("v", dv, x["v"])):
        val = (g.double() * t.double()).sum(dim=(2, 3))
        scale = (o.double().abs() * x["dO"].double().abs()).sum(dim=(2, 3))
        rel = ((val - ref).abs() / scale).max().item()
        assert rel < 1e-2, f"adjoint {name}: {rel:.3e}"


# ------------------------------------------ workload: long context (forward)
@pytest.mark.parametrize("de", [(128, 128), (64, 64), (64, 128)], ids=["d128e128", "d64e64", "d64e128"])
def test_split_point_with_state_sampled(orc, de):
    """The L = 32K sweep shape (B = 2, H = 32: each sequence split across
    CTAs, the initial state entering through the chunk-state scan) with an
    initial state kv0 and, for 64-column heads, the zero-padded tensors and
    128 x 128 padded states of the tensor-core path: forward (o, final
    state) and backward (dq, dk, dv, dkv0) of four (b, h) sequences against
    the oracle."""
    d, e = de
    Bn, H, L = 2, 32, 32768
    x = inputs.make_inputs(Bn, H, L, d, e, dtype=torch.bfloat16, device=DEV, seed=d + e + 7,
                           with_kv0=True)
    lam = inputs.decay_lambdas(H, DEV)
    with options(path="tc"):
        got = run_fwd_bwd(x, lam, x["kv0"])
    assert got is not None
    lam_h = lam.double().cpu().numpy()
    picks = [(0, 0), (1, 31), (1, 16), (0, 9)]
    sub = {n: np.concatenate([host(t[b:b + 1, h:h + 1]) for b, h in picks], axis=1)
           for n, t in x.items()}
    lh = np.array([lam_h[h] for _, h in picks])
    ref = oracle_all(orc, {n: torch.from_numpy(v) for n, v in sub.items()},
                     torch.from_numpy(lh), torch.from_numpy(sub["kv0"]))
    for i, (b, h) in enumerate(picks):
        for name, a, r in zip(NAMES, got, ref):
            check(f"L32K d{d} e{e} kv0 (b={b},h={h}) {name}", a[b:b + 1, h:h + 1],
                  r[:, i:i + 1], torch.bfloat16)


def test_long_context_1m_sampled(orc):
    """B=1, H=64, L=1,048,576, forward only (8K+ blocks of on-chip carry);
    the oracle recomputes heads 0, 21, 42 and 63 over the full length."""
    B, H, L = 1, 64, 1 << 20
    free, _ = torch.cuda.mem_get_info()
    if free < 80 * (1 << 30):
        pytest.skip("needs ~70 GB of free device memory")
    x = inputs.make_inputs(B, H, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=0,
                           with_dO=False)
    lam = inputs.decay_lambdas(H, DEV)
    o, st = la2.forward(x["q"], x["k"], x["v"], lam, want_state=True)
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    lam_h = lam.double().cpu().numpy()
    heads = [0, 21, 42, 63]
    sub = {n: np.concatenate([host(t[:, h:h + 1]) for h in heads], axis=1) for n, t in x.items()}
    o_r, st_r = orc.forward(sub["q"], sub["k"], sub["v"], lam_h[heads], want_state=True)
    for i, h in enumerate(heads):
        check(f"1M head {h} o", o[:, h:h + 1], o_r[:, i:i + 1], torch.bfloat16)
        check(f"1M head {h} state", st[:, h:h + 1], st_r[:, i:i + 1], torch.bfloat16)
    del x, o


# ------------------------------------------------------- workload: decode
def test_decode_1024_steps_sampled(orc):
    """batch 256, H=64, d=e=128, fp32 state ~ 0.01 N(0,1), 1024 steps; the
    oracle follows 64 sampled (b,h) states through every step."""
    B, H, d, e, steps = 256, 64, 128, 128, 1024
    lam = inputs.decay_lambdas(H, DEV)
    kv = inputs.decode_state0(B, H, d, e, device=DEV, seed=0)
    rng = np.random.default_rng(0)
    pick = sorted(set([(0, 0), (B - 1, H - 1)] +
                      [(int(rng.integers(B)), int(rng.integers(H))) for _ in range(62)]))
    bi = torch.tensor([p[0] for p in pick], device=DEV)
    hi = torch.tensor([p[1] for p in pick], device=DEV)
    kv_r = np.ascontiguousarray(kv[bi, hi].double().cpu().numpy()[None])
    lam_r = lam[hi].double().cpu().numpy()
    stream = inputs.DecodeStream(B, H, d, e, device=DEV, seed=0)
    for step in range(steps):
        q, k, v = stream.next()
        o = la2.decode_step(q, k, v, lam, kv)
        o_r = orc.decode_step(host(q[bi, hi])[None], host(k[bi, hi])[None],
                              host(v[bi, hi])[None], lam_r, kv_r)
        if step % 64 == 0 or step == steps - 1:
            check(f"decode step {step} o", o[bi, hi][None], o_r, torch.bfloat16)
    check("decode final state", kv[bi, hi][None], kv_r, torch.bfloat16)
    assert la2.last_device_error() == 0


def test_decode_matches_forward(orc):
    """L decode steps from kv0 equal one forward call with kv0 (fp32 I/O)."""
    B, H, L, d, e = 2, 3, 40, 64, 128
    x = inputs.make_inputs(B, H, L, d, e, dtype=torch.float32, device=DEV, seed=4,
                           with_kv0=True, with_dO=False)
    lam = inputs.fixed_lambdas((1.0, 0.9, 0.5), DEV)
    o_f, st_f = la2.forward(x["q"], x["k"], x["v"], lam, x["kv0"], want_state=True)
    kv = x["kv0"].clone()
    outs = []
    for t in range(L):
        outs.append(la2.decode_step(x["q"][:, :, t].contiguous(), x["k"][:, :, t].contiguous(),
                                    x["v"][:, :, t].contiguous(), lam, kv))
    o_d = torch.stack(outs, dim=2)
    check("decode vs forward o", o_d, host(o_f), torch.float32)
    check("decode vs forward state", kv, host(st_f), torch.float32)


# ----------------------------------------------- failure detection (no fault)
def test_bounded_wait_reports_timeout():
    """A tensor-core pass whose completion signal is withheld (test hook) gives
    up after its bounded wait, reports LA2_ERR_TIMEOUT, and leaves the context
    usable: the next call is correct."""
    x = inputs.make_inputs(1, 1, 256, 128, 128, dtype=torch.bfloat16, device=DEV, seed=2,
                           with_dO=False)
    lam = inputs.decay_lambdas(1, DEV)
    with options(path="tc"):
        ref = la2.forward(x["q"], x["k"], x["v"], lam)
        torch.cuda.synchronize()
        assert la2.last_device_error() == 0
        la2.set_option(la2.LA2_OPT_INJECT_TIMEOUT, 1)
        la2.forward(x["q"], x["k"], x["v"], lam)
        assert la2.last_device_error() == 4  # LA2_ERR_TIMEOUT
        again = la2.forward(x["q"], x["k"], x["v"], lam)
        torch.cuda.synchronize()
        assert la2.last_device_error() == 0
    assert torch.equal(again, ref)


# ----------------------------------------------------------------- tracing
def test_trace_instantiation_matches():
    """LA2_OPT_TRACE runs the tensor-core forward through its traced
    instantiation: bit-identical output, an entry/exit stamp for every CTA,
    and per-block stamps of CTA 0 in causal order (S issued after its tiles
    were loaded, the mask after S, the products after the mask, the output
    staged after the products)."""
    B, H, L = 2, 4, 1000
    x = inputs.make_inputs(B, H, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=21)
    lam = inputs.decay_lambdas(H, DEV)
    with options(path="tc", split=1):
        ref = la2.forward(x["q"], x["k"], x["v"], lam)
        torch.cuda.synchronize()
        la2.trace_read()  # clears
        old = la2.set_option(la2.LA2_OPT_TRACE, 1)  # mode 0: forward
        try:
            got = la2.forward(x["q"], x["k"], x["v"], lam)
            torch.cuda.synchronize()
        finally:
            la2.set_option(la2.LA2_OPT_TRACE, old)
    assert torch.equal(got, ref)
    t = la2.trace_read()
    n_cta, nblk = B * H, (L + 127) // 128
    entry, exit_ = t[10, :n_cta], t[11, :n_cta]
    assert bool((entry > 0).all()) and bool((exit_ > entry).all())
    assert int((t[10, n_cta:] > 0).sum()) == 0
    for i in range(nblk):
        s_end, mask_e, p_end, epi_s, oempty = (int(t[e, i]) for e in (1, 4, 2, 5, 6))
        assert 0 < s_end <= mask_e <= p_end, (i, s_end, mask_e, p_end)
        assert p_end <= epi_s <= oempty, (i, p_end, epi_s, oempty)


# --------------------------------------------------- gradient w.r.t. lambda
@pytest.mark.parametrize("split", [0, 1, 3, 7, None])
@pytest.mark.parametrize("dtype,de,L", [(torch.bfloat16, (128, 128), 300),
                                        (torch.float32, (64, 64), 257),
                                        (torch.bfloat16, (64, 128), 33),
                                        (torch.float32, (128, 64), 1000)])
def test_dlambda_matches_oracle(orc, dtype, de, L, split):
    """split: chunks per sequence (0 = the library's choice; None = the
    workspace-free entry point, one chunk per sequence)."""
    d, e = de
    x = inputs.make_inputs(2, 3, L, d, e, dtype=dtype, device=DEV, seed=L, with_kv0=True)
    lam = inputs.fixed_lambdas((1.0, 0.9, 0.0), DEV)
    old = la2.set_option(la2.LA2_OPT_SPLIT, split or 0)
    try:
        got = la2.dlambda(x["q"], x["k"], x["v"], lam, x["dO"], x["kv0"],
                          chunked=split is not None)
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_SPLIT, old)
    assert la2.last_device_error() == 0
    h = {n: host(t) for n, t in x.items()}
    ref = orc.dlambda(h["q"], h["k"], h["v"], lam.double().cpu().numpy(), h["dO"], h["kv0"])
    err = np.max(np.abs(got.double().cpu().numpy() - ref))
    assert err <= 1e-3 * max(float(np.max(np.abs(ref))), 1e-6), (got, ref)


def test_dlambda_b4_h16_l2048(orc):
    """The decay gradient on the training shape the bench times (B=4, H=16,
    L=2,048, bf16 inputs, the recipe's decays), every head against the
    oracle."""
    B, H, L = 4, 16, 2048
    x = inputs.make_inputs(B, H, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=0)
    lam = inputs.decay_lambdas(H, DEV)
    got = la2.dlambda(x["q"], x["k"], x["v"], lam, x["dO"])
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    h = {n: host(t) for n, t in x.items()}
    ref = orc.dlambda(h["q"], h["k"], h["v"], lam.double().cpu().numpy(), h["dO"])
    err = np.max(np.abs(got.double().cpu().numpy() - ref))
    assert err <= 1e-3 * float(np.max(np.abs(ref))), (got, ref)


@pytest.mark.parametrize("case", range(6))
def test_dlambda_random_splits_agree(case):
    """Seeded random shapes and forced splits: the chunked decay gradient
    equals the one-CTA-per-sequence form within the fp32 tolerance."""
    rng = np.random.default_rng(900 + case)
    B, H, L = int(rng.integers(1, 4)), int(rng.integers(1, 5)), int(rng.integers(1, 3000))
    split = int(rng.integers(2, 12))
    x = inputs.make_inputs(B, H, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=case,
                           with_kv0=True)
    lam = inputs.decay_lambdas(H, DEV)
    ref = la2.dlambda(x["q"], x["k"], x["v"], lam, x["dO"], x["kv0"], chunked=False)
    old = la2.set_option(la2.LA2_OPT_SPLIT, split)
    try:
        got = la2.dlambda(x["q"], x["k"], x["v"], lam, x["dO"], x["kv0"])
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_SPLIT, old)
    assert la2.last_device_error() == 0
    err = float((got.double() - ref.double()).abs().max())
    assert err <= 1e-3 * float(ref.double().abs().max()), (B, H, L, split, got, ref)


@pytest.mark.parametrize("case", range(10))
def test_random_shapes_match_oracle(orc, case):
    """Seeded random shapes on the tensor-core path (B 1..3, H 1..4, L
    1..1500 with ragged tails, decays drawn in [0, 1] with one head at 0 and
    one at 1, an initial state, a random forced split or the library's own):
    forward, final state and every gradient against the oracle."""
    rng = np.random.default_rng(4000 + case)
    B, H, L = int(rng.integers(1, 4)), int(rng.integers(1, 5)), int(rng.integers(1, 1501))
    vals = [float(v) for v in rng.uniform(0.0, 1.0, size=H)]
    vals[0] = 0.0
    if H > 1:
        vals[-1] = 1.0
    lam = inputs.fixed_lambdas(tuple(vals), DEV)
    split = int(rng.integers(0, 9))
    x = inputs.make_inputs(B, H, L, 128, 128, dtype=torch.bfloat16, device=DEV,
                           seed=4100 + case, with_kv0=True)
    with options(path="tc", split=split):
        got = run_fwd_bwd(x, lam, x["kv0"])
    compare(got, oracle_all(orc, x, lam, x["kv0"]), torch.bfloat16,
            f"B={B} H={H} L={L} split={split}")


# ------------------------------------------- paired dV/dK reverse launch
@contextlib.contextmanager
def bwd_form(form):
    old = la2.set_option(la2.LA2_OPT_BWD_FORM, form)
    try:
        yield
    finally:
        la2.set_option(la2.LA2_OPT_BWD_FORM, old)


@pytest.mark.parametrize("split", [1, 2, 5])
@pytest.mark.parametrize("L", [127, 1000, 2048])
def test_paired_reverse_matches_two_passes(orc, L, split):
    """dV and dK from the paired launch (two CTAs per chunk, clusters of
    two) are bitwise those of the two separate passes under the same split,
    and the oracle's, dkv0 included."""
    B, H = 2, 3
    x = inputs.make_inputs(B, H, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=L + split,
                           with_kv0=True)
    lam = inputs.fixed_lambdas((1.0, 0.95, 0.0), DEV)
    res = {}
    for form in (0, 1):
        with bwd_form(form), options(path="tc", split=split):
            res[form] = run_fwd_bwd(x, lam, x["kv0"])
    for name, a, b in zip(NAMES, res[0], res[1]):
        assert torch.equal(a, b), name
    compare(res[0], oracle_all(orc, x, lam, x["kv0"]), torch.bfloat16,
            f"paired L={L} S={split}")


@pytest.mark.parametrize("BL", [(1, 32768), (1, 65536), (2, 20000)])
def test_paired_reverse_automatic_split(orc, BL):
    """Under the automatic split the paired form plans its own (coarser)
    reverse chunks; few (b,h) sequences so that the reverse pre-pass runs:
    every gradient of two sampled heads against the oracle, and the
    workspace the binding sizes is the one the call needs."""
    Bn, L = BL
    H = 4
    x = inputs.make_inputs(Bn, H, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=L,
                           with_kv0=True)
    lam = inputs.decay_lambdas(H, DEV)
    n_pair = la2.workspace_size(la2.LA2_OP_BACKWARD, Bn, H, L, 128, 128, torch.bfloat16)
    with bwd_form(1):
        n_two = la2.workspace_size(la2.LA2_OP_BACKWARD, Bn, H, L, 128, 128, torch.bfloat16)
    assert 0 < n_pair <= n_two
    got = run_fwd_bwd(x, lam, x["kv0"])
    picks = [(0, 0), (Bn - 1, H - 1)]
    lam_h = lam.double().cpu().numpy()
    sub = {n: np.concatenate([host(t[b:b + 1, h:h + 1]) for b, h in picks], axis=1)
           for n, t in x.items()}
    lh = np.array([lam_h[h] for _, h in picks])
    ref = (orc.forward(sub["q"], sub["k"], sub["v"], lh, sub["kv0"], want_state=True)
           + tuple(orc.backward(sub["q"], sub["k"], sub["v"], lh, sub["dO"], sub["kv0"])))
    for i, (b, h) in enumerate(picks):
        for name, a, r in zip(NAMES, got, ref):
            check(f"auto split B{Bn} L{L} (b={b},h={h}) {name}", a[b:b + 1, h:h + 1],
                  r[:, i:i + 1], torch.bfloat16)


# ------------------------------------------ decay gradient on the tensor cores
@pytest.mark.parametrize("split", [0, 1, 3])
@pytest.mark.parametrize("L", [1, 127, 129, 1000])
def test_dlambda_tc_decay_range(orc, L, split):
    """The tensor-core decay gradient (bf16, d = e = 128; blocks of 128 rows,
    bf16 copies of the carried KV and W as MMA operands) over decays from 0
    to 1, an initial state, ragged blocks and forced splits, every head
    against the oracle at the 1e-3 bar."""
    x = inputs.make_inputs(2, 6, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=L + 7 * split,
                           with_kv0=True)
    lam = inputs.fixed_lambdas((0.0, 0.3, 0.9, 0.99, 0.999, 1.0), DEV)
    old = la2.set_option(la2.LA2_OPT_SPLIT, split)
    try:
        got = la2.dlambda(x["q"], x["k"], x["v"], lam, x["dO"], x["kv0"])
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_SPLIT, old)
    assert la2.last_device_error() == 0
    h = {n: host(t) for n, t in x.items()}
    ref = orc.dlambda(h["q"], h["k"], h["v"], lam.double().cpu().numpy(), h["dO"], h["kv0"])
    err = np.max(np.abs(got.double().cpu().numpy() - ref))
    assert err <= 1e-3 * max(float(np.max(np.abs(ref))), 1e-6), (got, ref)


def test_dlambda_tc_matches_fp32_form():
    """The tensor-core and fp32-FMA forms of the decay gradient agree on the
    bench's shape (two independent kernels, one chunk plan each)."""
    B, H, L = 4, 16, 2048
    x = inputs.make_inputs(B, H, L, 128, 128, dtype=torch.bfloat16, device=DEV, seed=3)
    lam = inputs.decay_lambdas(H, DEV)
    tc = la2.dlambda(x["q"], x["k"], x["v"], lam, x["dO"])
    with options(path="simt"):
        ref = la2.dlambda(x["q"], x["k"], x["v"], lam, x["dO"])
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    err = float((tc.double() - ref.double()).abs().max())
    assert err <= 1e-3 * float(ref.double().abs().max()), (tc, ref)
