"""GPU parity of the feature map phi(x) = elu(x) + 1 (la2_feature_map) and
its chain rule (la2_feature_map_backward) against the oracle, element by
element, and of the attention behind it: the map, the attention forward
and backward, and the map's backward together against the oracle's
composition of the same steps."""
import numpy as np
import pytest
import torch

import causal_linear_attention_fwd_b200 as la2
from causal_linear_attention_fwd_b200 import inputs
from gpu_util import check, host

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
# the kernel's arithmetic is fp32 with CUDA's expf (2 ulp), its result
# rounded to the I/O type.  For bf16 one rounding errs by at most half an ulp,
# which relative to the value is below 2^-8 (2^-9 at the top of a binade, up
# to just under 2^-8 at its bottom); the fp32 error (~2^-22) fits in the gap
# below 2^-8.  For fp32, a few fp32 ulp.
REL = {torch.bfloat16: 2.0 ** -8, torch.float32: 5e-7}
SPECIAL = [0.0, -0.0, 1.0, -1.0, 50.0, -30.0, -87.0, -100.0, 1e-3, -1e-3]


def sample(n, seed, dtype):
    g = torch.Generator(device=DEV).manual_seed(seed)
    x = torch.randn(n, generator=g, device=DEV, dtype=torch.float32) * 3.0
    x[:len(SPECIAL)] = torch.tensor(SPECIAL[:n], device=DEV)
    return x.to(dtype)


def assert_map(name, got, x, ref, dtype):
    got = host(got).astype(np.float64)
    # the oracle forms elu(x) + 1 in fp64, whose final rounding leaves an
    # absolute error up to 2^-53 (at x = -87, say, it returns 0 for
    # e^-87 = 1.6e-38): compare relatively, above that floor
    err = np.abs(got - ref) - REL[dtype] * np.abs(ref)
    assert err.max(initial=-1.0) <= 2.0 ** -52, f"{name}: worst excess {err.max():.3e}"
    # on the linear side the result is x + 1 rounded once to the I/O type
    # (fp32: one rounding; bf16: x + 1 of a bf16 x in this range is exact
    # in fp32, or rounds to a value that rounds to 1 in bf16 either way)
    pos = host(x) > 0
    want = torch.from_numpy(ref[pos]).to(dtype).float().numpy()
    assert np.array_equal(got[pos], want), f"{name}: linear side not exactly x + 1"


def assert_grad(name, got, ref, dtype):
    """dL/dphi * elu'(x): two fp32 roundings and the output's; results
    in the denormal range are compared in absolute terms."""
    got = host(got).astype(np.float64)
    err = np.abs(got - ref) - 2 * REL[dtype] * np.abs(ref)
    assert err.max(initial=-1.0) <= 1e-37, f"{name}: worst excess {err.max():.3e}"


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("n", [1, 7, 8, 1110, 65536 + 5, (1 << 23) + 3])
def test_map_and_gradient_match_oracle(orc, dtype, n):
    """Both tensors at once, sizes from one value to several grid-stride
    passes, with ragged tails (n not a multiple of the 16-byte vector)."""
    q, k = sample(n, 1, dtype), sample(n, 2, dtype)
    gq, gk = sample(n, 3, dtype), sample(n, 4, dtype)
    pq, pk = la2.feature_map(q, k)
    dq, dk = la2.feature_map_backward(q, k, gq, gk)
    torch.cuda.synchronize()
    for name, x, y in (("phi_q", q, pq), ("phi_k", k, pk)):
        assert_map(f"{name} n={n}", y, x, orc.feature_map(host(x)), dtype)
    for name, x, g, y in (("dq", q, gq, dq), ("dk", k, gk, dk)):
        ref = orc.feature_map_grad(host(x), host(g).astype(np.float64))
        assert_grad(f"{name} n={n}", y, ref, dtype)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_in_place_and_single_tensor(orc, dtype):
    q, k = sample(4099, 5, dtype), sample(4099, 6, dtype)
    ref_q, ref_k = orc.feature_map(host(q)), orc.feature_map(host(k))
    only = la2.feature_map(q)                      # q alone
    q0 = q.clone()
    la2.feature_map(q, k, out=(q, k))              # in place
    g = sample(4099, 7, dtype)
    g0 = g.clone()
    d = la2.feature_map_backward(q0, None, g, None, out=(g, None))   # in place, q alone
    torch.cuda.synchronize()
    assert d.data_ptr() == g.data_ptr()
    assert_map("q alone", only, q0, ref_q, dtype)
    assert_map("q in place", q, q0, ref_q, dtype)
    err = np.abs(host(k).astype(np.float64) - ref_k) - REL[dtype] * np.abs(ref_k)
    assert err.max() <= 2.0 ** -52, "k in place"
    ref_d = orc.feature_map_grad(host(q0), host(g0).astype(np.float64))
    assert_grad("dq in place", d, ref_d, dtype)


def test_non_finite_inputs():
    """-inf maps to 0, +inf to +inf, NaN stays NaN (no value is rejected)."""
    x = torch.tensor([float("-inf"), float("inf"), float("nan"), 0.0] * 4, device=DEV)
    y = la2.feature_map(x)
    torch.cuda.synchronize()
    y = host(y)
    assert (y[0::4] == 0).all() and np.isposinf(y[1::4]).all() and np.isnan(y[2::4]).all()
    assert (y[3::4] == 1).all()


@pytest.mark.parametrize("path,dtype,de", [("tc", torch.bfloat16, (128, 128)),
                                           ("simt", torch.float32, (64, 64))])
def test_attention_with_feature_map_matches_oracle(orc, path, dtype, de):
    """phi on q and k, the attention forward and backward on the mapped
    inputs, then the chain rule back to q and k: against the oracle's
    composition of the same steps (several blocks, a ragged tail, kv0)."""
    d, e = de
    x = inputs.make_inputs(2, 3, 333, d, e, dtype=dtype, device=DEV, seed=21, with_kv0=True)
    lam = inputs.fixed_lambdas((1.0, 0.97, 0.5), DEV)
    old = la2.set_option(la2.LA2_OPT_PATH, {"simt": 1, "tc": 2}[path])
    try:
        pq, pk = la2.feature_map(x["q"], x["k"])
        o, st = la2.forward(pq, pk, x["v"], lam, x["kv0"], want_state=True)
        gpq, gpk, dv = la2.backward(pq, pk, x["v"], lam, x["dO"], x["kv0"])
        dq, dk = la2.feature_map_backward(x["q"], x["k"], gpq, gpk)
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_PATH, old)
    assert la2.last_device_error() == 0
    h = {n: host(t) for n, t in x.items()}
    lam_h = lam.double().cpu().numpy()
    fq, fk = orc.feature_map(h["q"]), orc.feature_map(h["k"])
    o_ref, st_ref = orc.forward(fq, fk, h["v"], lam_h, h["kv0"], want_state=True)
    g = orc.backward(fq, fk, h["v"], lam_h, h["dO"], h["kv0"])
    tag = f"phi {path}"
    check(f"{tag} o", o, o_ref, dtype)
    check(f"{tag} state", st, st_ref, dtype)
    check(f"{tag} dq", dq, orc.feature_map_grad(h["q"], g[0]), dtype)
    check(f"{tag} dk", dk, orc.feature_map_grad(h["k"], g[1]), dtype)
    check(f"{tag} dv", dv, g[2], dtype)


def test_bench_size_sampled(orc):
    """The launch the bench times (q and k of the B=8, H=32, L=8,192 sweep
    point, 268M values each): 1M sampled values of each output against
    the oracle."""
    x = inputs.make_inputs(8, 32, 8192, 128, 128, dtype=torch.bfloat16, device=DEV, seed=0,
                           with_dO=False)
    del x["v"]
    q, k = x["q"].view(-1), x["k"].view(-1)
    pq, pk = la2.feature_map(q, k)
    dq, dk = la2.feature_map_backward(q, k, pk, pq)  # any upstream gradient will do
    torch.cuda.synchronize()
    g = torch.Generator(device=DEV).manual_seed(9)
    idx = torch.randint(0, q.numel(), (1 << 20,), generator=g, device=DEV)
    for name, xin, y in (("phi_q", q, pq), ("phi_k", k, pk)):
        xs = xin[idx]
        assert_map(f"bench {name}", y[idx], xs, orc.feature_map(host(xs)), torch.bfloat16)
    for name, xin, up, y in (("dq", q, pk, dq), ("dk", k, pq, dk)):
        ref = orc.feature_map_grad(host(xin[idx]), host(up[idx]).astype(np.float64))
        assert_grad(f"bench {name}", y[idx], ref, torch.bfloat16)
