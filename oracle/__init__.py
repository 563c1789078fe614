"""fp64 CPU oracle for decayed causal linear attention -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never loads it and it
never loads the CUDA library: the two share no code.

``la2_oracle.c`` holds the arithmetic (the token-by-token recurrence, see its
header); this module only compiles it with gcc and marshals numpy arrays.

Every function here is pinned by tests in ``tests/test_oracle_pins.py``
(brute-force quadratic attention, the lambda=1 prefix-sum identity, lambda=0,
block-size invariance of a tiled restatement, finite differences, adjoint
identities, state hand-off, a hand-derived golden example; for the feature
map: printed constants, closed forms, its shape, finite differences).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "la2_oracle.c")
LIB = os.path.join(_HERE, "_build", "libla2_oracle.so")

_lock = threading.Lock()
_loaded = {}


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile the oracle C file into a shared library (gcc, OpenMP)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(src)):
        return out
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
           "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


class Oracle:
    """ctypes view of one compiled oracle library."""

    def __init__(self, path: str):
        self.path = path
        self._lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i, l = ctypes.c_int, ctypes.c_long
        self._lib.oracle_forward.argtypes = [i, i, l, i, i, P, P, P, P, P, P, P]
        self._lib.oracle_backward.argtypes = [i, i, l, i, i, P, P, P, P, P, P,
                                              P, P, P, P]
        self._lib.oracle_backward_end.argtypes = [i, i, l, i, i, P, P, P, P, P, P,
                                                  P, P, P, P, P]
        self._lib.oracle_dlambda.argtypes = [i, i, l, i, i, P, P, P, P, P, P, P]
        self._lib.oracle_decode_step.argtypes = [i, i, i, i, P, P, P, P, P, P]
        self._lib.oracle_feature_map.argtypes = [l, P, P]
        self._lib.oracle_feature_map_grad.argtypes = [l, P, P, P]
        self._lib.oracle_num_threads.restype = ctypes.c_int
        for f in ("oracle_forward", "oracle_backward", "oracle_backward_end",
                  "oracle_dlambda", "oracle_decode_step", "oracle_feature_map",
                  "oracle_feature_map_grad"):
            getattr(self._lib, f).restype = None

    @staticmethod
    def _f32(a):
        return np.ascontiguousarray(a, dtype=np.float32)

    @staticmethod
    def _f64(a):
        return np.ascontiguousarray(a, dtype=np.float64)

    @staticmethod
    def _p(a):
        return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

    def num_threads(self) -> int:
        return int(self._lib.oracle_num_threads())

    def forward(self, q, k, v, lam, kv0=None, want_state=False):
        """q,k [B,H,L,d], v [B,H,L,e], lam [H] -> o [B,H,L,e] (fp64)
        (and the final state [B,H,d,e] when want_state)."""
        q, k, v = self._f32(q), self._f32(k), self._f32(v)
        B, H, L, d = q.shape
        e = v.shape[-1]
        assert k.shape == (B, H, L, d) and v.shape == (B, H, L, e)
        lam = self._f64(lam).reshape(H)
        kv0 = None if kv0 is None else self._f64(kv0).reshape(B, H, d, e)
        o = np.empty((B, H, L, e), np.float64)
        st = np.empty((B, H, d, e), np.float64) if want_state else None
        self._lib.oracle_forward(B, H, L, d, e, self._p(q), self._p(k),
                                 self._p(v), self._p(lam), self._p(kv0),
                                 self._p(o), self._p(st))
        return (o, st) if want_state else o

    def backward(self, q, k, v, lam, dO, kv0=None, dstate_end=None):
        """Gradients (dq, dk, dv, dkv0) of sum(o * dO); all fp64.
        dstate_end [B,H,d,e]: terminal adjoint G_L (the reverse state flowing
        in from rows after these; default zero)."""
        q, k, v, dO = self._f32(q), self._f32(k), self._f32(v), self._f32(dO)
        B, H, L, d = q.shape
        e = v.shape[-1]
        assert dO.shape == (B, H, L, e)
        lam = self._f64(lam).reshape(H)
        kv0 = None if kv0 is None else self._f64(kv0).reshape(B, H, d, e)
        dq = np.empty((B, H, L, d), np.float64)
        dk = np.empty((B, H, L, d), np.float64)
        dv = np.empty((B, H, L, e), np.float64)
        dkv0 = np.empty((B, H, d, e), np.float64)
        gend = None if dstate_end is None else self._f64(dstate_end).reshape(B, H, d, e)
        self._lib.oracle_backward_end(B, H, L, d, e, self._p(q), self._p(k),
                                      self._p(v), self._p(lam), self._p(kv0),
                                      self._p(dO), self._p(gend), self._p(dq),
                                      self._p(dk), self._p(dv), self._p(dkv0))
        return dq, dk, dv, dkv0

    def dlambda(self, q, k, v, lam, dO, kv0=None):
        """Gradient of sum(o * dO) with respect to lam [H], summed over the
        batch (fp64 [H])."""
        q, k, v, dO = self._f32(q), self._f32(k), self._f32(v), self._f32(dO)
        B, H, L, d = q.shape
        e = v.shape[-1]
        lam = self._f64(lam).reshape(H)
        kv0 = None if kv0 is None else self._f64(kv0).reshape(B, H, d, e)
        out = np.empty(H, np.float64)
        self._lib.oracle_dlambda(B, H, L, d, e, self._p(q), self._p(k), self._p(v),
                                 self._p(lam), self._p(kv0), self._p(dO), self._p(out))
        return out

    def decode_step(self, q, k, v, lam, kv):
        """One step; kv [B,H,d,e] fp64 is updated IN PLACE; returns o [B,H,e]."""
        q, k, v = self._f32(q), self._f32(k), self._f32(v)
        B, H, d = q.shape
        e = v.shape[-1]
        assert kv.dtype == np.float64 and kv.flags["C_CONTIGUOUS"]
        assert kv.shape == (B, H, d, e)
        lam = self._f64(lam).reshape(H)
        o = np.empty((B, H, e), np.float64)
        self._lib.oracle_decode_step(B, H, d, e, self._p(q), self._p(k),
                                     self._p(v), self._p(lam), self._p(kv),
                                     self._p(o))
        return o


    def feature_map(self, x):
        """phi(x) = elu(x) + 1 elementwise (fp64, same shape)."""
        x = self._f32(x)
        y = np.empty(x.shape, np.float64)
        self._lib.oracle_feature_map(x.size, self._p(x), self._p(y))
        return y

    def feature_map_grad(self, x, dy):
        """dL/dx from dL/dphi(x) = dy: dy * elu'(x) (fp64, same shape)."""
        x = self._f32(x)
        dy = self._f64(dy)
        assert dy.shape == x.shape
        dx = np.empty(x.shape, np.float64)
        self._lib.oracle_feature_map_grad(x.size, self._p(x), self._p(dy), self._p(dx))
        return dx


def load(path: str | None = None) -> Oracle:
    """Build (if needed) and load the oracle library."""
    with _lock:
        p = path or build()
        if p not in _loaded:
            _loaded[p] = Oracle(p)
        return _loaded[p]
