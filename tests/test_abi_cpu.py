"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point include/la2.h declares, and rejects bad arguments before
touching the device.  Pointers here are fake addresses that are never
dereferenced: every case returns during validation."""
import ctypes
import os
import re

import pytest

import causal_linear_attention_fwd_b200 as la2
from causal_linear_attention_fwd_b200 import _binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            src = open(os.path.join(ROOT, "include", f)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(la2_\w+)\s*\(", src))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    return la2.library()


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert {"la2_forward", "la2_backward", "la2_decode_step",
            "la2_workspace_size"} <= set(names)
    for n in names:
        assert hasattr(lib, n), f"libla2.so does not export {n}"


def test_status_strings(lib):
    for code, name in enumerate(["LA2_OK", "LA2_ERR_INVALID", "LA2_ERR_UNSUPPORTED",
                                 "LA2_ERR_CUDA", "LA2_ERR_TIMEOUT"]):
        assert la2.status_string(code) == name


def test_set_option_roundtrip(lib):
    old = la2.set_option(la2.LA2_OPT_SPLIT, 5)
    assert la2.set_option(la2.LA2_OPT_SPLIT, old) == 5
    for opt in (la2.LA2_OPT_PATH, la2.LA2_OPT_VARIANT, la2.LA2_OPT_VARLEN_ORDER,
                la2.LA2_OPT_DECODE_BLOCK_TOKENS, la2.LA2_OPT_BWD_FORM):
        old = la2.set_option(opt, 1)
        assert old >= 0
        assert la2.set_option(opt, old) == 1
    assert la2.set_option(99, 1) == -1


# fake, 16-byte aligned, non-overlapping device addresses
MB = 1 << 20
Q, K, V, O, LAM, KV0, KVO, WS, DO, DQ, DK, DV, DKV, CU = [(i + 1) * 64 * MB for i in range(14)]


def fwd(lib, q=Q, k=K, v=V, lam=LAM, kv0=None, o=O, kvo=None, Bn=1, H=2, L=100, d=64, e=64,
        dt=B.LA2_BF16, ws=None, wsb=0):
    return lib.la2_forward(q, k, v, lam, kv0, o, kvo, Bn, H, L, d, e, dt, ws, wsb, None)


def bwd(lib, q=Q, k=K, v=V, lam=LAM, kv0=None, dO=DO, dq=DQ, dk=DK, dv=DV, dkv=None, Bn=1, H=2,
        L=100, d=64, e=64, dt=B.LA2_BF16, ws=None, wsb=0):
    return lib.la2_backward(q, k, v, lam, kv0, dO, dq, dk, dv, dkv, Bn, H, L, d, e, dt, ws, wsb,
                            None)


def test_forward_validation(lib):
    INV, UNS = B.LA2_ERR_INVALID, B.LA2_ERR_UNSUPPORTED
    assert fwd(lib, q=None) == INV
    assert fwd(lib, o=None) == INV
    assert fwd(lib, lam=None) == INV
    assert fwd(lib, Bn=-1) == INV
    assert fwd(lib, L=-5) == INV
    assert fwd(lib, d=96) == UNS
    assert fwd(lib, e=32) == UNS
    assert fwd(lib, dt=7) == UNS
    assert fwd(lib, q=Q + 8) == INV                 # not 16-byte aligned
    assert fwd(lib, kv0=KV0, kvo=KV0) == INV         # kv_out == kv0
    assert fwd(lib, o=Q + 64) == INV                 # o overlaps q
    assert fwd(lib, kvo=V + 1024) == INV             # kv_out overlaps v
    assert fwd(lib, o=V) == INV                      # o exactly aliases v (same span)
    assert fwd(lib, kv0=KV0, kvo=KV0 + 0) == INV
    assert fwd(lib, Bn=0) == B.LA2_OK                # empty batch: nothing to do
    assert fwd(lib, H=0) == B.LA2_OK


def test_backward_validation(lib):
    INV, UNS = B.LA2_ERR_INVALID, B.LA2_ERR_UNSUPPORTED
    assert bwd(lib, dO=None) == INV
    assert bwd(lib, dq=None) == INV
    assert bwd(lib, dk=DQ) == INV                    # two outputs at one address
    assert bwd(lib, dv=DO) == INV                    # output aliases an input
    assert bwd(lib, dq=DO) == INV                    # dq exactly aliases dO (d = e)
    assert bwd(lib, dk=K) == INV                     # dk exactly aliases k
    assert bwd(lib, dkv=DQ + 16) == INV              # dkv0 inside dq
    assert bwd(lib, d=128, e=96) == UNS
    assert bwd(lib, H=-1) == INV
    assert bwd(lib, Bn=0) == B.LA2_OK


def test_decode_validation(lib):
    INV = B.LA2_ERR_INVALID
    f = lib.la2_decode_step
    assert f(None, K, V, LAM, KV0, O, 2, 2, 64, 64, B.LA2_BF16, None) == INV
    assert f(Q, K, V, LAM, KV0, KV0 + 16, 2, 2, 64, 64, B.LA2_BF16, None) == INV
    assert f(Q, K, V, LAM, KV0 + 4, O, 2, 2, 64, 64, B.LA2_BF16, None) == INV
    assert f(Q, K, V, LAM, KV0, O, 2, 2, 64, 80, B.LA2_BF16, None) == B.LA2_ERR_UNSUPPORTED
    assert f(Q, K, V, LAM, KV0, O, 0, 2, 64, 64, B.LA2_BF16, None) == B.LA2_OK


def test_varlen_validation(lib):
    INV, UNS, OK = B.LA2_ERR_INVALID, B.LA2_ERR_UNSUPPORTED, B.LA2_OK

    def fwdv(q=Q, k=K, v=V, lam=LAM, cu=CU, kv0=None, o=O, kvo=None, N=3, H=2, T=100, d=64,
             e=64, dt=B.LA2_BF16):
        return lib.la2_forward_varlen(q, k, v, lam, cu, kv0, o, kvo, N, H, T, d, e, dt, None)

    def bwdv(q=Q, k=K, v=V, lam=LAM, cu=CU, kv0=None, dO=DO, dq=DQ, dk=DK, dv=DV, dkv=None, N=3,
             H=2, T=100, d=64, e=64, dt=B.LA2_BF16):
        return lib.la2_backward_varlen(q, k, v, lam, cu, kv0, dO, dq, dk, dv, dkv, N, H, T, d, e,
                                       dt, None)

    assert fwdv(cu=None) == INV
    assert fwdv(cu=CU + 4) == INV                    # offsets not 8-byte aligned
    assert fwdv(lam=None) == INV
    assert fwdv(q=None) == INV
    assert fwdv(N=-1) == INV and fwdv(T=-1) == INV and fwdv(H=-2) == INV
    assert fwdv(d=96) == UNS and fwdv(dt=5) == UNS
    assert fwdv(kv0=KV0, kvo=KV0) == INV             # kv_out == kv0
    assert fwdv(o=Q + 64) == INV                     # o overlaps q
    assert fwdv(kvo=CU) == INV                       # kv_out overlaps the offsets
    assert fwdv(q=Q + 8) == INV                      # not 16-byte aligned
    assert fwdv(N=0) == OK and fwdv(H=0) == OK       # empty batch
    assert fwdv(T=0, q=None, k=None, v=None, o=None) == OK  # all sequences empty, no state out
    assert bwdv(dO=None) == INV
    assert bwdv(dk=DQ) == INV                        # two outputs at one address
    assert bwdv(dv=CU) == INV                        # output over the offsets
    assert bwdv(d=128, e=80) == UNS
    assert bwdv(N=0) == OK


def test_pool_validation(lib):
    INV, UNS, OK = B.LA2_ERR_INVALID, B.LA2_ERR_UNSUPPORTED, B.LA2_OK
    SL = CU  # a fake slot table address

    def fwdp(q=Q, k=K, v=V, lam=LAM, pool=KV0, slots=SL, P=8, o=O, flags=0, Bn=2, H=2, L=100,
             d=64, e=64, dt=B.LA2_BF16, ws=None, wsb=0):
        return lib.la2_forward_pool(q, k, v, lam, pool, slots, P, o, flags, Bn, H, L, d, e, dt,
                                    ws, wsb, None)

    def dect(q=Q, k=K, v=V, lam=LAM, pool=KV0, slots=SL, P=8, o=O, Bn=2, H=2, T=4, d=64, e=64,
             dt=B.LA2_BF16):
        return lib.la2_decode_tokens(q, k, v, lam, pool, slots, P, o, Bn, H, T, d, e, dt, None)

    assert fwdp(flags=2) == INV                      # unknown flag bit
    assert fwdp(L=0) == INV                          # a prefill has at least one row
    assert fwdp(slots=None) == INV
    assert fwdp(slots=SL + 2) == INV                 # slot table not 4-byte aligned
    assert fwdp(pool=None) == INV
    assert fwdp(o=KV0 + 64) == INV                   # o inside the pool
    assert fwdp(P=-1) == INV
    assert fwdp(d=96) == UNS
    assert fwdp(Bn=0) == OK
    assert dect(T=-1) == INV
    assert dect(slots=None, P=1) == INV              # no slot table: pool must hold B states
    assert dect(o=KV0) == INV                        # o overlaps the pool
    assert dect(q=None) == INV
    assert dect(e=80) == UNS
    assert dect(T=0) == OK and dect(Bn=0) == OK


def test_shard_validation(lib):
    INV, UNS, OK = B.LA2_ERR_INVALID, B.LA2_ERR_UNSUPPORTED, B.LA2_OK
    ss = lambda a=K, b=V, lam=LAM, out=KVO, Bn=1, H=2, L=100, d=64, e=64, rev=0, ws=WS, wsb=MB: \
        lib.la2_shard_state(a, b, lam, out, Bn, H, L, d, e, B.LA2_BF16, rev, ws, wsb, None)
    assert ss(L=0) == INV
    assert ss(ws=None) == INV                        # the workspace is required
    assert ss(out=K + 256) == INV                    # out overlaps an input
    assert ss(d=96) == UNS
    assert ss(wsb=16) == INV                         # workspace too small
    assert ss(Bn=0) == OK
    sp = lambda dl=DQ, kv0=None, lam=LAM, out=DK, R=3, Bn=1, H=2, L=100, d=64, e=64, rev=0: \
        lib.la2_state_prefix(dl, kv0, lam, out, R, Bn, H, L, d, e, rev, None)
    assert sp(R=-1) == INV
    assert sp(out=DQ + 16) == INV                    # out overlaps the deltas
    assert sp(d=96) == UNS
    assert sp(R=0) == OK
    bs = lambda flags=0, dend=None, dq=DQ, L=100: lib.la2_backward_shard(
        Q, K, V, LAM, None, DO, dend, dq, DK, DV, None, 1, 2, L, 64, 64, B.LA2_BF16, None, 0,
        flags, None)
    assert bs(flags=2) == INV
    assert bs(dend=DQ) == INV                        # an output over dstate_end
    assert bs(L=0) == INV


def test_dlambda_validation(lib):
    INV, UNS, OK = B.LA2_ERR_INVALID, B.LA2_ERR_UNSUPPORTED, B.LA2_OK
    f = lambda q=Q, dl=KVO, L=100, d=64, H=2: lib.la2_backward_dlambda(
        q, K, V, LAM, None, DO, dl, 1, H, L, d, 64, B.LA2_BF16, None)
    assert f(L=-1) == INV
    assert f(dl=None) == INV
    assert f(dl=LAM) == INV                          # output over lambda
    assert f(q=None) == INV
    assert f(d=96) == UNS
    assert f(H=0) == OK


def test_dlambda_ex_workspace_rules(lib):
    """The chunked decay gradient: scratch (KV, W) per chunk when the
    sequences are split; too little scratch, or scratch over an input, is
    rejected before any launch."""
    INV = B.LA2_ERR_INVALID
    need = lib.la2_workspace_size(B.LA2_OP_DLAMBDA, 1, 2, 1 << 16, 64, 64, B.LA2_BF16)
    assert need > 0 and need % (2 * 64 * 64 * 4) == 0
    old = la2.set_option(la2.LA2_OPT_SPLIT, 3)
    try:
        n = lib.la2_workspace_size(B.LA2_OP_DLAMBDA, 2, 3, 1000, 64, 128, B.LA2_F32)
        # (KV, W) pairs at the sub-chunk boundaries of the first two chunks
        # plus the initial pair: an odd number of pairs, at least 3
        pairs = n // (2 * 3 * 2 * 64 * 128 * 4)
        assert n == pairs * 2 * 3 * 2 * 64 * 128 * 4 and pairs >= 3 and pairs % 2 == 1
        la2.set_option(la2.LA2_OPT_SPLIT, 1)
        assert lib.la2_workspace_size(B.LA2_OP_DLAMBDA, 2, 3, 1000, 64, 128, B.LA2_F32) == 0
    finally:
        la2.set_option(la2.LA2_OPT_SPLIT, old)
    f = lambda ws=WS, wsb=need, L=1 << 16: lib.la2_backward_dlambda_ex(
        Q, K, V, LAM, None, DO, KVO, 1, 2, L, 64, 64, B.LA2_BF16, ws, wsb, None)
    assert f(wsb=need - 1) == INV
    assert f(ws=None, wsb=0) == INV
    assert f(ws=Q) == INV                            # scratch over an input
    assert f(ws=KVO) == INV                          # scratch over the output


def test_workspace_rules(lib):
    # a long sequence with few (b,h) pairs is split, so scratch is needed ...
    need = lib.la2_workspace_size(B.LA2_OP_FORWARD, 1, 2, 1 << 16, 64, 64, B.LA2_BF16)
    assert need > 0 and need % (64 * 64 * 4) == 0
    bneed = lib.la2_workspace_size(B.LA2_OP_BACKWARD, 1, 2, 1 << 16, 64, 64, B.LA2_BF16)
    assert bneed == 2 * need
    # ... and a call that brings too little is rejected before any launch
    assert fwd(lib, L=1 << 16, ws=WS, wsb=need - 1) == B.LA2_ERR_INVALID
    assert fwd(lib, L=1 << 16, ws=None, wsb=0) == B.LA2_ERR_INVALID
    # invalid arguments size to 0
    assert lib.la2_workspace_size(B.LA2_OP_FORWARD, 1, 2, 100, 64, 96, B.LA2_BF16) == 0
    assert lib.la2_workspace_size(7, 1, 2, 100, 64, 64, B.LA2_BF16) == 0


def test_forced_split_sizes_workspace(lib):
    old = la2.set_option(la2.LA2_OPT_SPLIT, 4)
    try:
        n = lib.la2_workspace_size(B.LA2_OP_FORWARD, 2, 3, 1000, 64, 128, B.LA2_F32)
        assert n == 2 * 3 * 4 * 64 * 128 * 4
        la2.set_option(la2.LA2_OPT_SPLIT, 1)
        assert lib.la2_workspace_size(B.LA2_OP_FORWARD, 2, 3, 1000, 64, 128, B.LA2_F32) == 0
    finally:
        la2.set_option(la2.LA2_OPT_SPLIT, old)


def test_product_path_does_not_reference_oracle():
    """The package never imports or loads the oracle."""
    pkg = os.path.join(ROOT, "causal_linear_attention_fwd_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                for pat in (r"^\s*import\s+oracle", r"^\s*from\s+oracle", r"la2_oracle",
                            r"oracle\.(load|build|Oracle)"):
                    assert not re.search(pat, src, flags=re.M), f"{f} reaches the oracle ({pat})"


def test_feature_map_validation(lib):
    """The elementwise feature-map calls: in-place use is the only overlap
    allowed (an output over its own input, or over its own upstream
    gradient); everything else shared, misaligned, missing or negative is
    rejected before any launch.  Only rejected cases and n = 0 (nothing to
    launch) are called here."""
    INV, UNS, OK = B.LA2_ERR_INVALID, B.LA2_ERR_UNSUPPORTED, B.LA2_OK
    n = 4096
    f = lambda q=Q, k=K, pq=O, pk=DQ, n=n, dt=B.LA2_BF16: lib.la2_feature_map(
        q, k, pq, pk, n, dt, None)
    assert f(n=-1) == INV
    assert f(dt=7) == UNS
    assert f(n=0) == OK
    assert f(q=None) == INV
    assert f(pq=None) == INV
    assert f(pk=None) == INV                         # k given, phi_k missing
    assert f(k=None) == INV                          # phi_k given, k missing
    assert f(q=Q + 8) == INV
    assert f(pq=K) == INV                            # phi_q over k
    assert f(pq=Q + 16) == INV                       # phi_q partly over q
    assert f(pk=O + 16) == INV                       # outputs share bytes
    g = lambda q=Q, k=K, gq=DO, gk=DV, dq=DQ, dk=DK, n=n: lib.la2_feature_map_backward(
        q, k, gq, gk, dq, dk, n, B.LA2_BF16, None)
    assert g(n=-1) == INV
    assert g(n=0) == OK
    assert g(gq=None) == INV
    assert g(gk=None) == INV                         # k given, dphi_k missing
    assert g(dk=None) == INV
    assert g(dq=Q) == INV                            # in place over q: not allowed
    assert g(dq=DV) == INV                           # dq over dphi_k
    assert g(dk=DQ) == INV                           # outputs alias
    assert g(gq=DO + 8) == INV


def test_feature_map_binding_checks(lib):
    """The Python binding refuses host tensors and mismatched arguments before
    calling the library."""
    import torch
    q = torch.zeros(4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        la2.feature_map(q, q.clone())
    with pytest.raises(ValueError, match="both"):
        la2.feature_map_backward(q, q.clone(), q.clone(), None)
    with pytest.raises(ValueError, match="both"):
        la2.feature_map_backward(q, None, q.clone(), q.clone())


class _FakeCuda:
    """A stand-in for a CUDA tensor (no GPU here): only what the binding's
    device checks read."""

    def __init__(self, device):
        import torch
        self.device = torch.device(device)
        self.is_cuda = True

    def is_contiguous(self):
        return True


def test_binding_rejects_mixed_devices():
    """Every tensor argument of a call must live on one device: the library
    launches on the current device, so a tensor on another GPU would be read
    through the wrong device's tensor maps."""
    import torch
    a, b = _FakeCuda("cuda:0"), _FakeCuda("cuda:1")
    assert B._devices(("q", a), ("k", _FakeCuda("cuda:0")), ("kv0", None)) == torch.device("cuda:0")
    with pytest.raises(ValueError, match="k is on cuda:1"):
        B._devices(("q", a), ("k", b))
    with pytest.raises(ValueError, match="CUDA"):
        B._devices(("q", a), ("v", torch.zeros(2)))
    with pytest.raises(ValueError, match="no tensor"):
        B._devices(("kv0", None))


def test_noalloc_binding_checks(lib):
    """forward_noalloc checks its arguments as forward() does, kv0 included,
    before anything reaches the library."""
    import torch
    q = torch.zeros(1, 2, 8, 64, dtype=torch.bfloat16)
    lam = torch.zeros(2)
    with pytest.raises(ValueError, match="CUDA"):
        la2.forward_noalloc(q, q, q, lam)
    with pytest.raises(ValueError, match="CUDA"):
        la2.forward(q, q, q, lam)
