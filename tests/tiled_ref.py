"""fp64 tiled restatement of the forward and backward schedule (test-only).

This is NOT the oracle and NOT used by the CUDA path.  It writes out, in
numpy, the block schedule the kernels follow -- the intra-block masked dense
part plus the inter-block part through a carried d x e state, in forward and
backward (Lightning Attention-2 notes page, "Tiling." paragraph) -- together
with the sequence split into chunks whose boundary states are found by a
short scan.  ``test_tiled_schedule.py`` checks it against the oracle for many
block sizes and splits, which pins the per-block decay factors before any
kernel relies on them.

Block i covers rows [p, p+cb) (cb = C except a ragged last block), local
rows s, t in [0, cb):
  M_loc[s,t] = lam^(s-t) (t <= s)
  forward:  O_i = (Q_i K_i^T (.) M_loc) V_i + diag(lam^(s+1)) Q_i KV(p)
            KV(p+cb) = lam^cb KV(p) + (diag(lam^(cb-1-t)) K_i)^T V_i
  dQ:       dQ_i = (dO_i V_i^T (.) M_loc) K_i + diag(lam^(s+1)) dO_i KV(p)^T
  dK, dV:   D(p) = sum_{t >= p} lam^(t-p) q_t^T dO_t  (reverse state)
            dK_i = (dO_i V_i^T (.) M_loc)^T Q_i + diag(lam^(cb-s)) V_i D(p+cb)^T
            dV_i = (Q_i K_i^T (.) M_loc)^T dO_i + diag(lam^(cb-s)) K_i D(p+cb)
            D(p) = lam^cb D(p+cb) + (diag(lam^s) Q_i)^T dO_i
            dkv0 = lam * D(0)
Chunks of Lc rows (a multiple of C): the forward chunk state is the carry
started from zero; chunk entry states follow KV_in[c] = lam^Lc KV_in[c-1] +
dKV[c-1]; the reverse states mirror it.
"""
from __future__ import annotations

import numpy as np


def _pw(lam, n):
    n = np.asarray(n)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(n == 0, 1.0, np.power(float(lam), np.maximum(n, 0)))


def _mask(cb, lam):
    s = np.arange(cb)[:, None]
    t = np.arange(cb)[None, :]
    return np.where(t <= s, _pw(lam, s - t), 0.0)


def _blocks(a, b, C):
    p = a
    while p < b:
        yield p, min(C, b - p)
        p += C


def _chunks(L, C, S):
    """Chunk boundaries: chunk length a multiple of C, S chunks at most."""
    nblk = -(-L // C)
    per = -(-nblk // S)
    Lc = per * C
    bounds = []
    a = 0
    while a < L:
        bounds.append((a, min(L, a + Lc)))
        a += Lc
    return bounds


def forward_one(Q, K, V, lam, kv0, C, S):
    L, d = Q.shape
    e = V.shape[1]
    ch = _chunks(L, C, S)
    # pass 1: chunk states from zero (all but the last chunk)
    dkv = []
    for (a, b) in ch[:-1]:
        st = np.zeros((d, e))
        for p, cb in _blocks(a, b, C):
            bt = _pw(lam, cb - 1 - np.arange(cb))
            st = _pw(lam, cb) * st + (K[p:p + cb] * bt[:, None]).T @ V[p:p + cb]
        dkv.append(st)
    # pass 2: scan of entry states
    kin = [np.zeros((d, e)) if kv0 is None else kv0.copy()]
    for c in range(1, len(ch)):
        a, b = ch[c - 1]
        kin.append(_pw(lam, b - a) * kin[-1] + dkv[c - 1])
    # pass 3: per chunk, intra + inter with the carried state
    O = np.zeros((L, e))
    st = None
    for c, (a, b) in enumerate(ch):
        st = kin[c].copy()
        for p, cb in _blocks(a, b, C):
            Qi, Ki, Vi = Q[p:p + cb], K[p:p + cb], V[p:p + cb]
            a_s = _pw(lam, np.arange(1, cb + 1))
            O[p:p + cb] = ((Qi @ Ki.T) * _mask(cb, lam)) @ Vi + a_s[:, None] * (Qi @ st)
            bt = _pw(lam, cb - 1 - np.arange(cb))
            st = _pw(lam, cb) * st + (Ki * bt[:, None]).T @ Vi
    return O, st


def backward_one(Q, K, V, lam, kv0, dO, C, S):
    L, d = Q.shape
    e = V.shape[1]
    ch = _chunks(L, C, S)
    # ---- dQ: forward scan, same entry states as the forward pass
    dkv = []
    for (a, b) in ch[:-1]:
        st = np.zeros((d, e))
        for p, cb in _blocks(a, b, C):
            bt = _pw(lam, cb - 1 - np.arange(cb))
            st = _pw(lam, cb) * st + (K[p:p + cb] * bt[:, None]).T @ V[p:p + cb]
        dkv.append(st)
    kin = [np.zeros((d, e)) if kv0 is None else kv0.copy()]
    for c in range(1, len(ch)):
        a, b = ch[c - 1]
        kin.append(_pw(lam, b - a) * kin[-1] + dkv[c - 1])
    dQ = np.zeros((L, d))
    for c, (a, b) in enumerate(ch):
        st = kin[c].copy()
        for p, cb in _blocks(a, b, C):
            Gi, Ki, Vi = dO[p:p + cb], K[p:p + cb], V[p:p + cb]
            a_s = _pw(lam, np.arange(1, cb + 1))
            dQ[p:p + cb] = ((Gi @ Vi.T) * _mask(cb, lam)) @ Ki + a_s[:, None] * (Gi @ st.T)
            bt = _pw(lam, cb - 1 - np.arange(cb))
            st = _pw(lam, cb) * st + (Ki * bt[:, None]).T @ Vi
    # ---- dK, dV: reverse scan
    # chunk c's own contribution to D(a_c), for chunks 1..S-1
    dD = {}
    for c in range(1, len(ch)):
        a, b = ch[c]
        st = np.zeros((d, e))
        for p, cb in reversed(list(_blocks(a, b, C))):
            g = _pw(lam, np.arange(cb))
            st = _pw(lam, cb) * st + (Q[p:p + cb] * g[:, None]).T @ dO[p:p + cb]
        dD[c] = st
    din = [None] * len(ch)
    din[-1] = np.zeros((d, e))
    for c in range(len(ch) - 2, -1, -1):
        a1, b1 = ch[c + 1]
        din[c] = _pw(lam, b1 - a1) * din[c + 1] + dD[c + 1]
    dK = np.zeros((L, d))
    dV = np.zeros((L, e))
    D0 = None
    for c, (a, b) in enumerate(ch):
        D = din[c].copy()
        for p, cb in reversed(list(_blocks(a, b, C))):
            Qi, Ki, Vi, Gi = Q[p:p + cb], K[p:p + cb], V[p:p + cb], dO[p:p + cb]
            M = _mask(cb, lam)
            c_s = _pw(lam, cb - np.arange(cb))
            dK[p:p + cb] = ((Gi @ Vi.T) * M).T @ Qi + c_s[:, None] * (Vi @ D.T)
            dV[p:p + cb] = ((Qi @ Ki.T) * M).T @ Gi + c_s[:, None] * (Ki @ D)
            g = _pw(lam, np.arange(cb))
            D = _pw(lam, cb) * D + (Qi * g[:, None]).T @ Gi
        if c == 0:
            D0 = D
    return dQ, dK, dV, float(lam) * D0


def forward(q, k, v, lam, kv0, C, S=1):
    B, H, L, d = q.shape
    o = np.zeros(v.shape, np.float64)
    st = np.zeros((B, H, d, v.shape[-1]))
    for b in range(B):
        for h in range(H):
            o[b, h], st[b, h] = forward_one(
                q[b, h].astype(np.float64), k[b, h].astype(np.float64),
                v[b, h].astype(np.float64), lam[h],
                None if kv0 is None else kv0[b, h], C, S)
    return o, st


def backward(q, k, v, lam, dO, kv0, C, S=1):
    B, H, L, d = q.shape
    e = v.shape[-1]
    out = [np.zeros((B, H, L, d)), np.zeros((B, H, L, d)),
           np.zeros((B, H, L, e)), np.zeros((B, H, d, e))]
    for b in range(B):
        for h in range(H):
            r = backward_one(q[b, h].astype(np.float64), k[b, h].astype(np.float64),
                             v[b, h].astype(np.float64), lam[h],
                             None if kv0 is None else kv0[b, h],
                             dO[b, h].astype(np.float64), C, S)
            for i in range(4):
                out[i][b, h] = r[i]
    return tuple(out)
