"""Independent pins for the fp64 oracle.

Each ``pin_*`` function takes a loaded oracle (``oracle.Oracle``) and raises
AssertionError when the oracle disagrees with something that is fixed
independently of it: a brute-force quadratic formula, a textbook routine
(``numpy.cumsum``), a closed form, central finite differences, an identity
the mathematics forces, or a hand-derived golden example.  The pins are run
against the real oracle (``test_oracle_pins.py``) and against deliberately
broken copies of it (``test_oracle_mutants.py``) to show they bite.

None of this code is used by the CUDA path.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ----------------------------------------------------------------- helpers
def bf16_exact(shape, seed, scale=1.0):
    """Random normals rounded to bf16, returned as float32 (exact values)."""
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(shape, generator=g, dtype=torch.float32) * scale
    return x.to(torch.bfloat16).to(torch.float32).numpy()


def small_case(B=2, H=3, L=23, d=5, e=4, seed=1, lams=(1.0, 0.9, 0.37), kv0=True):
    q = bf16_exact((B, H, L, d), seed, 0.5)
    k = bf16_exact((B, H, L, d), seed + 1, 0.5)
    v = bf16_exact((B, H, L, e), seed + 2)
    dO = bf16_exact((B, H, L, e), seed + 3)
    lam = np.array(lams[:H], np.float64)
    s0 = bf16_exact((B, H, d, e), seed + 4, 0.3).astype(np.float64) if kv0 else None
    return q, k, v, dO, lam, s0


def decay_mask(L, lam):
    """M[t, j] = lam^(t-j) for j <= t, else 0 (0^0 = 1)."""
    t = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    n = t - j
    with np.errstate(divide="ignore", invalid="ignore"):
        m = np.where(n >= 0, np.power(float(lam), np.maximum(n, 0)), 0.0)
    return m


def assert_close(x, ref, tol, what):
    x = np.asarray(x, np.float64)
    ref = np.asarray(ref, np.float64)
    assert x.shape == ref.shape, (what, x.shape, ref.shape)
    scale = max(1.0, float(np.max(np.abs(ref))) if ref.size else 1.0)
    err = float(np.max(np.abs(x - ref))) if ref.size else 0.0
    assert err <= tol * scale, f"{what}: max err {err:.3e} > {tol:.1e}*{scale:.3e}"


# ------------------------------------------- brute-force quadratic attention
def quadratic_forward(q, k, v, lam, kv0):
    """O = (Q K^T (.) M) V + diag(lam^(t+1)) Q kv0, per (b,h), fp64."""
    B, H, L, d = q.shape
    o = np.zeros(v.shape[:3] + (v.shape[-1],), np.float64)
    for b in range(B):
        for h in range(H):
            Q, K, V = (a[b, h].astype(np.float64) for a in (q, k, v))
            M = decay_mask(L, lam[h])
            o[b, h] = ((Q @ K.T) * M) @ V
            if kv0 is not None:
                a = np.power(float(lam[h]), np.arange(1, L + 1))
                o[b, h] += a[:, None] * (Q @ kv0[b, h])
    return o


def quadratic_state(k, v, lam, kv0):
    """kv_L = lam^L kv0 + sum_j lam^(L-1-j) k_j^T v_j."""
    B, H, L, d = k.shape
    out = np.zeros((B, H, d, v.shape[-1]))
    for b in range(B):
        for h in range(H):
            w = np.power(float(lam[h]), np.arange(L - 1, -1, -1))
            out[b, h] = (k[b, h].astype(np.float64) * w[:, None]).T @ v[b, h]
            if kv0 is not None:
                out[b, h] += float(lam[h]) ** L * kv0[b, h]
    return out


def pin_bruteforce(orc):
    for kv0 in (False, True):
        q, k, v, dO, lam, s0 = small_case(kv0=kv0)
        o, st = orc.forward(q, k, v, lam, s0, want_state=True)
        assert_close(o, quadratic_forward(q, k, v, lam, s0), 1e-12, "o vs quadratic")
        assert_close(st, quadratic_state(k, v, lam, s0), 1e-12, "state vs quadratic")


def pin_prefix_sum(orc):
    """lambda = 1: o_t = q_t . cumsum_j (k_j^T v_j) -- the running sum of the
    causal case, built with numpy's cumsum."""
    q, k, v, dO, _, _ = small_case(H=2, lams=(1.0, 1.0), kv0=False)
    lam = np.ones(2)
    outer = k[..., :, None].astype(np.float64) * v[..., None, :]
    cum = np.cumsum(outer, axis=2)
    ref = np.einsum("bhti,bhtij->bhtj", q.astype(np.float64), cum)
    o, st = orc.forward(q, k, v, lam, want_state=True)
    assert_close(o, ref, 1e-12, "o vs cumsum")
    assert_close(st, cum[:, :, -1], 1e-12, "state vs cumsum")


def pin_lambda_zero(orc):
    """lambda = 0 keeps only the diagonal: o_t = (q_t . k_t) v_t."""
    q, k, v, dO, _, s0 = small_case(H=1, lams=(0.0,), kv0=True)
    lam = np.zeros(1)
    ref = np.sum(q.astype(np.float64) * k, -1, keepdims=True) * v
    o, st = orc.forward(q, k, v, lam, s0, want_state=True)
    assert_close(o, ref, 1e-13, "o, lambda=0")
    last = k[:, :, -1, :, None].astype(np.float64) * v[:, :, -1, None, :]
    assert_close(st, last, 1e-13, "state, lambda=0")
    dq, dk, dv, dkv0 = orc.backward(q, k, v, lam, dO, s0)
    g = np.sum(dO.astype(np.float64) * v, -1, keepdims=True)
    assert_close(dq, g * k, 1e-13, "dq, lambda=0")
    assert_close(dk, g * q, 1e-13, "dk, lambda=0")
    assert_close(dv, np.sum(q.astype(np.float64) * k, -1, keepdims=True) * dO,
                 1e-13, "dv, lambda=0")
    assert_close(dkv0, np.zeros_like(dkv0), 0, "dkv0, lambda=0")


def pin_length_one(orc):
    """L = 1: o_0 = q_0 (lambda kv0 + k_0^T v_0)."""
    q, k, v, dO, lam, s0 = small_case(L=1, kv0=True)
    o = orc.forward(q, k, v, lam, s0)
    for b in range(q.shape[0]):
        for h in range(q.shape[1]):
            S = float(lam[h]) * s0[b, h] + np.outer(k[b, h, 0], v[b, h, 0])
            assert_close(o[b, h, 0], q[b, h, 0].astype(np.float64) @ S, 1e-13, "L=1")


# ------------------------------------------------------- backward closed forms
def quadratic_backward(q, k, v, lam, dO, kv0):
    """dQ = (dO V^T (.) M) K + diag(lam^(t+1)) dO kv0^T,
    dK = (dO V^T (.) M)^T Q,  dV = (Q K^T (.) M)^T dO,
    dkv0 = sum_t lam^(t+1) q_t^T dO_t."""
    B, H, L, d = q.shape
    e = v.shape[-1]
    dq = np.zeros((B, H, L, d)); dk = np.zeros((B, H, L, d))
    dv = np.zeros((B, H, L, e)); dkv0 = np.zeros((B, H, d, e))
    for b in range(B):
        for h in range(H):
            Q, K, V, G = (a[b, h].astype(np.float64) for a in (q, k, v, dO))
            M = decay_mask(L, lam[h])
            dP = (G @ V.T) * M
            P = (Q @ K.T) * M
            dq[b, h] = dP @ K
            dk[b, h] = dP.T @ Q
            dv[b, h] = P.T @ G
            a = np.power(float(lam[h]), np.arange(1, L + 1))
            if kv0 is not None:
                dq[b, h] += a[:, None] * (G @ kv0[b, h].T)
            dkv0[b, h] = (Q * a[:, None]).T @ G
    return dq, dk, dv, dkv0


def pin_backward_closed_form(orc):
    for kv0 in (False, True):
        q, k, v, dO, lam, s0 = small_case(kv0=kv0)
        got = orc.backward(q, k, v, lam, dO, s0)
        ref = quadratic_backward(q, k, v, lam, dO, s0)
        for name, x, r in zip(("dq", "dk", "dv", "dkv0"), got, ref):
            assert_close(x, r, 1e-12, f"{name} vs closed form (kv0={kv0})")


def pin_finite_difference(orc):
    """loss = sum(o * dO) is linear in each input, so a central difference
    with a step that keeps the perturbed inputs exact in fp32 reproduces the
    gradient up to fp64 rounding."""
    q, k, v, dO, lam, s0 = small_case(B=1, H=2, L=9, d=3, e=4, lams=(0.8, 1.0))
    dq, dk, dv, dkv0 = orc.backward(q, k, v, lam, dO, s0)

    def loss(qq, kk, vv, ss):
        return float(np.sum(orc.forward(qq, kk, vv, lam, ss) * dO))

    h = 2.0 ** -6
    rng = np.random.default_rng(0)
    for name, arr, grad in (("q", q, dq), ("k", k, dk), ("v", v, dv), ("kv0", s0, dkv0)):
        for _ in range(6):
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            args = {"q": q, "k": k, "v": v, "kv0": s0}
            args[name] = plus
            lp = loss(args["q"], args["k"], args["v"], args["kv0"])
            args[name] = minus
            lm = loss(args["q"], args["k"], args["v"], args["kv0"])
            fd = (lp - lm) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-9 * max(1.0, abs(fd)), \
                f"finite difference d{name}{idx}: {fd} vs {grad[idx]}"


def pin_adjoint(orc):
    """o is linear in q and bilinear in (k,v) / (q,kv0); Euler's identity for
    homogeneous functions gives
      sum dq*q = sum dO*o,  sum dk*k + sum dkv0*kv0 = sum dO*o,
      sum dv*v + sum dkv0*kv0 = sum dO*o."""
    q, k, v, dO, lam, s0 = small_case(kv0=True)
    o = orc.forward(q, k, v, lam, s0)
    dq, dk, dv, dkv0 = orc.backward(q, k, v, lam, dO, s0)
    ref = float(np.sum(o * dO))
    t0 = float(np.sum(dkv0 * s0))
    for name, val in (("q", float(np.sum(dq * q))),
                      ("k", float(np.sum(dk * k)) + t0),
                      ("v", float(np.sum(dv * v)) + t0)):
        assert abs(val - ref) <= 1e-11 * max(1.0, abs(ref)), (name, val, ref)


def pin_backward_terminal_closed_form(orc):
    """A terminal adjoint G_L (the reverse state flowing in from rows after
    the sequence) adds to the closed form: G_t gains lam^(L-t) G_L, so
    dk_t += lam^(L-t) G_L v_t, dv_t += lam^(L-t) k_t G_L, dkv0 += lam^(L+1)
    G_L; dq does not change."""
    q, k, v, dO, lam, s0 = small_case(kv0=True)
    B, H, L, d = q.shape
    e = v.shape[-1]
    gend = bf16_exact((B, H, d, e), 17, 0.4).astype(np.float64)
    got = orc.backward(q, k, v, lam, dO, s0, dstate_end=gend)
    dq, dk, dv, dkv0 = quadratic_backward(q, k, v, lam, dO, s0)
    for b in range(B):
        for h in range(H):
            w = np.power(float(lam[h]), L - np.arange(L))  # lam^(L-t)
            G = gend[b, h]
            dk[b, h] += w[:, None] * (v[b, h].astype(np.float64) @ G.T)
            dv[b, h] += w[:, None] * (k[b, h].astype(np.float64) @ G)
            dkv0[b, h] += float(lam[h]) ** (L + 1) * G
    for name, x, r in zip(("dq", "dk", "dv", "dkv0"), got, (dq, dk, dv, dkv0)):
        assert_close(x, r, 1e-12, f"{name} with a terminal adjoint vs closed form")


def pin_backward_split(orc):
    """A sequence cut at L1: the second part's backward from the forward state
    at L1, and the first part's backward with the terminal adjoint sum_{s >=
    L1} lam^(s-L1) q_s^T dO_s (the plain sum), reproduce the whole backward."""
    q, k, v, dO, lam, s0 = small_case(L=30, kv0=True)
    full = orc.backward(q, k, v, lam, dO, s0)
    L1 = 13
    _, st1 = orc.forward(q[:, :, :L1], k[:, :, :L1], v[:, :, :L1], lam, s0, want_state=True)
    part2 = orc.backward(q[:, :, L1:], k[:, :, L1:], v[:, :, L1:], lam, dO[:, :, L1:], st1)
    B, H, L, d = q.shape
    e = v.shape[-1]
    gend = np.zeros((B, H, d, e))
    for b in range(B):
        for h in range(H):
            w = np.power(float(lam[h]), np.arange(L - L1))
            gend[b, h] = (q[b, h, L1:].astype(np.float64) * w[:, None]).T @ dO[b, h, L1:]
    part1 = orc.backward(q[:, :, :L1], k[:, :, :L1], v[:, :, :L1], lam, dO[:, :, :L1], s0,
                         dstate_end=gend)
    for i, name in enumerate(("dq", "dk", "dv")):
        assert_close(np.concatenate([part1[i], part2[i]], 2), full[i], 1e-12, f"split {name}")
    assert_close(part1[3], full[3], 1e-12, "split dkv0")


def pin_dlambda_closed_form(orc):
    """dlambda_h = sum_b sum_t dO_t . [ sum_{j<t} (t-j) lam^(t-j-1) (q_t.k_j) v_j
    + (t+1) lam^t q_t kv0 ]: the derivative of the quadratic form entry by
    entry (the diagonal's weight 1 does not depend on lambda); lambda = 0 keeps
    only the j = t-1 terms and, with kv0, the t = 0 one."""
    for lams in ((1.0, 0.9, 0.37), (0.0, 0.5, 1.0)):
        q, k, v, dO, lam, s0 = small_case(lams=lams, kv0=True)
        got = orc.dlambda(q, k, v, lam, dO, s0)
        B, H, L, d = q.shape
        ref = np.zeros(H)
        n = np.arange(L)[:, None] - np.arange(L)[None, :]
        for h in range(H):
            lm = float(lam[h])
            with np.errstate(divide="ignore", invalid="ignore"):
                W = np.where(n >= 1, n * np.power(lm, np.maximum(n - 1, 0)), 0.0)
            a = (np.arange(L) + 1) * np.power(lm, np.arange(L))  # (t+1) lam^t, 0^0 = 1
            for b in range(B):
                Q, K, V, G = (x[b, h].astype(np.float64) for x in (q, k, v, dO))
                ref[h] += np.sum(((Q @ K.T) * W) @ V * G)
                ref[h] += np.sum(a[:, None] * (Q @ s0[b, h]) * G)
        assert_close(got, ref, 1e-12, f"dlambda vs closed form {lams}")


def pin_dlambda_finite_difference(orc):
    """sum(o * dO) as a function of one head's lambda: a central difference
    with step 2^-10 around lambda (a polynomial of degree L in lambda, so the
    error is O(h^2) times its third derivative)."""
    q, k, v, dO, lam, s0 = small_case(B=1, H=2, L=9, d=3, e=4, lams=(0.75, 0.5))
    got = orc.dlambda(q, k, v, lam, dO, s0)
    h = 2.0 ** -10
    for i in range(2):
        lp, lm = lam.copy(), lam.copy()
        lp[i] += h
        lm[i] -= h
        fp = float(np.sum(orc.forward(q, k, v, lp, s0) * dO))
        fm = float(np.sum(orc.forward(q, k, v, lm, s0) * dO))
        fd = (fp - fm) / (2 * h)
        assert abs(fd - got[i]) <= 1e-5 * max(1.0, abs(fd)), (i, fd, got[i])


# --------------------------------------------------------------- state pins
def pin_state_handoff(orc):
    q, k, v, dO, lam, s0 = small_case(L=30, kv0=True)
    o, st = orc.forward(q, k, v, lam, s0, want_state=True)
    L1 = 11
    o1, st1 = orc.forward(q[:, :, :L1], k[:, :, :L1], v[:, :, :L1], lam, s0, want_state=True)
    o2, st2 = orc.forward(q[:, :, L1:], k[:, :, L1:], v[:, :, L1:], lam, st1, want_state=True)
    assert_close(np.concatenate([o1, o2], 2), o, 1e-13, "split forward")
    assert_close(st2, st, 1e-13, "split state")


def pin_decode_equals_forward(orc):
    q, k, v, dO, lam, s0 = small_case(L=12, kv0=True)
    o, st = orc.forward(q, k, v, lam, s0, want_state=True)
    kv = np.ascontiguousarray(s0.copy())
    for t in range(q.shape[2]):
        ot = orc.decode_step(q[:, :, t], k[:, :, t], v[:, :, t], lam, kv)
        assert_close(ot, o[:, :, t], 1e-13, f"decode step {t}")
    assert_close(kv, st, 1e-13, "decode final state")


# ------------------------------------------------------------- golden pins
def pin_golden(orc):
    with open(os.path.join(GOLDEN, "hand_examples.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        L, d, e = c["L"], c["d"], c["e"]
        q = np.array(c["q"], np.float32).reshape(1, 1, L, d)
        k = np.array(c["k"], np.float32).reshape(1, 1, L, d)
        v = np.array(c["v"], np.float32).reshape(1, 1, L, e)
        dO = np.array(c["dO"], np.float32).reshape(1, 1, L, e)
        lam = np.array([c["lambda"]], np.float64)
        s0 = None if c["kv0"] is None else np.array(c["kv0"], np.float64).reshape(1, 1, d, e)
        o, st = orc.forward(q, k, v, lam, s0, want_state=True)
        assert_close(o.reshape(L, e), np.array(c["o"]), 0, c["name"] + " o")
        assert_close(st.reshape(d, e), np.array(c["kv_out"]), 0, c["name"] + " kv_out")
        dq, dk, dv, dkv0 = orc.backward(q, k, v, lam, dO, s0)
        assert_close(dq.reshape(L, d), np.array(c["dq"]), 0, c["name"] + " dq")
        assert_close(dk.reshape(L, d), np.array(c["dk"]), 0, c["name"] + " dk")
        assert_close(dv.reshape(L, e), np.array(c["dv"]), 0, c["name"] + " dv")
        assert_close(dkv0.reshape(d, e), np.array(c["dkv0"]), 0, c["name"] + " dkv0")


# ------------------------------------------------------------- feature map
def pin_feature_map_values(orc):
    """phi(x) = elu(x) + 1 at points where it is known without the oracle:
    exact on the linear side (phi(0) = 1, phi(3) = 4, phi(2.5) = 3.5), and
    on the exponential side e^-1 and e^-30 (their decimal expansions, to
    1e-15 absolute) and
    e^(-ln 2) = 1/2, e^(-ln 4) = 1/4 (the float32 rounding of -ln 2 and
    -ln 4 moves these by under 1e-7 relative)."""
    x = np.array([0.0, 3.0, 2.5, -1.0, -30.0, -np.log(2.0), -np.log(4.0)], np.float32)
    want = np.array([1.0, 4.0, 3.5, 0.36787944117144233, 9.357622968840175e-14, 0.5, 0.25])
    got = orc.feature_map(x)
    assert np.array_equal(got[:3], want[:3]), f"feature map, linear side: {got[:3]}"
    # elu(x) + 1 on the exponential side rounds the sum to 1's spacing, so
    # its error is absolute, about 1e-16 (e^-30 itself is 9.4e-14)
    err = np.abs(got - want)
    assert err[3:5].max() < 1e-15, f"feature map at -1, -30: {got[3:5]} vs {want[3:5]}"
    assert (err[5:] / want[5:]).max() < 1e-7, f"feature map at -ln 2, -ln 4: {got[5:]}"


def pin_feature_map_shape(orc):
    """The map is positive (what lets the numerator stay a sum of positive
    weights), equals 1 + x on the positive side and lies in (0, 1] on the
    other, never below the tangent line 1 + x there (e^x >= 1 + x), and is
    increasing."""
    x = bf16_exact((4096,), 91, 3.0)
    y = orc.feature_map(x)
    xd = x.astype(np.float64)
    assert (y > 0).all(), "feature map not positive"
    pos = xd > 0
    assert np.array_equal(y[pos], xd[pos] + 1.0), "feature map != 1 + x for x > 0"
    assert (y[~pos] <= 1.0).all() and (y[~pos] >= 1.0 + xd[~pos]).all(), \
        "feature map outside [1 + x, 1] for x <= 0"
    order = np.argsort(xd, kind="stable")
    assert (np.diff(y[order]) >= 0).all(), "feature map not increasing"


def pin_feature_map_finite_difference(orc):
    """dL/dx = dL/dphi * phi'(x) against central differences of the
    oracle's own map (the step taken between float32 neighbours of x so
    both evaluation points are exact inputs)."""
    g = np.random.default_rng(17)
    x = (g.standard_normal(512) * 2.0).astype(np.float32)
    x = x[np.abs(x) > 0.05]
    dy = g.standard_normal(x.shape)
    h = np.maximum(1e-3, 1e-3 * np.abs(x)).astype(np.float32)
    xp, xm = (x + h).astype(np.float32), (x - h).astype(np.float32)
    slope = (orc.feature_map(xp) - orc.feature_map(xm)) / (xp.astype(np.float64) - xm)
    got = orc.feature_map_grad(x, dy)
    err = np.abs(got - dy * slope) / (np.abs(dy * slope) + 1e-12)
    assert err.max() < 1e-5, f"feature map gradient vs finite differences: {err.max():.3e}"


def pin_feature_map_chain(orc):
    """The chain rule through the map, end to end: for loss(q, k) =
    sum(forward(phi(q), phi(k), v) * dO) the gradient in the unmapped q is
    backward(phi(q), phi(k), ...)'s dq times phi'(q) (likewise k), against
    central differences of the whole loss.  The steps keep q +- h exact in
    float32; the map's values pass to the attention as float32, which with
    the O(h^2) truncation bounds the agreement near 1e-5; entries within 2h
    of the kink at 0 are skipped."""
    q, k, v, dO, lam, s0 = small_case(B=1, H=2, L=9, d=3, e=4, lams=(0.8, 1.0))
    q, k = q * 4.0, k * 4.0          # both sides of the map; still exact
    g = orc.backward(orc.feature_map(q), orc.feature_map(k), v, lam, dO, s0)
    grads = {"q": orc.feature_map_grad(q, g[0]), "k": orc.feature_map_grad(k, g[1])}

    def loss(qq, kk):
        o = orc.forward(orc.feature_map(qq), orc.feature_map(kk), v, lam, s0)
        return float(np.sum(o * dO))

    h = 2.0 ** -8
    rng = np.random.default_rng(4)
    for name, arr in (("q", q), ("k", k)):
        done = 0
        while done < 6:
            idx = tuple(int(rng.integers(0, n)) for n in arr.shape)
            if abs(arr[idx]) < 2 * h:
                continue
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            if name == "q":
                fd = (loss(plus, k) - loss(minus, k)) / (2 * h)
            else:
                fd = (loss(q, plus) - loss(q, minus)) / (2 * h)
            want = grads[name][idx]
            assert abs(fd - want) <= 1e-4 * max(1.0, abs(fd)), \
                f"feature map chain rule d{name}{idx}: {fd} vs {want}"
            done += 1


ALL_PINS = [pin_bruteforce, pin_prefix_sum, pin_lambda_zero, pin_length_one,
            pin_backward_closed_form, pin_backward_terminal_closed_form, pin_backward_split,
            pin_dlambda_closed_form, pin_dlambda_finite_difference,
            pin_finite_difference, pin_adjoint,
            pin_state_handoff, pin_decode_equals_forward, pin_golden,
            pin_feature_map_values, pin_feature_map_shape, pin_feature_map_finite_difference,
            pin_feature_map_chain]
