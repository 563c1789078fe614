"""la2_forward_noalloc: the forward entry point for callers that cannot
allocate device memory (plug-ins whose host framework owns all device
memory, latency-critical paths that cannot afford cudaMalloc's device
synchronisation, callbacks that only receive device pointers).  It keeps its
chunk-boundary states in the library's own fixed device array instead of a
caller workspace, so it must give the oracle's result, and the same result
as la2_forward.

This file is collected last on purpose: a failure here leaves every other
test already run.  The tests also pass when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import causal_linear_attention_fwd_b200 as la2
from causal_linear_attention_fwd_b200 import _binding, inputs
from gpu_util import check, host

DEV = "cuda:0"
ARRAY_BYTES = 32 << 20


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.gpu
def test_noalloc_forward_matches_oracle_and_workspace_forward(orc):
    """Two calls in a row through the C ABI, chunk split in use (so the fixed
    array really holds the chunk states): each matches the oracle, and
    la2_forward on the same inputs."""
    lib = la2.library()
    B, H, L, d, e = 1, 2, 4096, 128, 128
    assert la2.workspace_size(la2.LA2_OP_FORWARD, B, H, L, d, e, torch.bfloat16) > 0
    lam = inputs.decay_lambdas(H, DEV)
    lam_h = lam.double().cpu().numpy()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for seed in (0, 1):  # two calls in a row, different inputs
        x = inputs.make_inputs(B, H, L, d, e, dtype=torch.bfloat16, device=DEV, seed=seed,
                               with_dO=False, with_kv0=True)
        ref_o, ref_st = la2.forward(x["q"], x["k"], x["v"], lam, x["kv0"], want_state=True)
        o = torch.empty_like(ref_o)
        st = torch.empty_like(ref_st)
        code = lib.la2_forward_noalloc(_ptr(x["q"]), _ptr(x["k"]), _ptr(x["v"]), _ptr(lam),
                                       _ptr(x["kv0"]), _ptr(o), _ptr(st), B, H, L, d, e,
                                       _binding.LA2_BF16, stream)
        assert code == 0, la2.status_string(code)
        torch.cuda.synchronize()
        assert la2.last_device_error() == 0
        h = {n: host(t) for n, t in x.items()}
        o_r, st_r = orc.forward(h["q"], h["k"], h["v"], lam_h, x["kv0"].double().cpu().numpy(),
                                want_state=True)
        check(f"noalloc o vs oracle (call {seed})", o, o_r, torch.bfloat16)
        check(f"noalloc state vs oracle (call {seed})", st, st_r, torch.bfloat16)
        check(f"noalloc o vs la2_forward (call {seed})", o, host(ref_o), torch.bfloat16)
        check(f"noalloc state vs la2_forward (call {seed})", st, host(ref_st), torch.bfloat16)


@pytest.mark.gpu
@pytest.mark.parametrize("de", [(128, 128), (64, 64)])
@pytest.mark.parametrize("with_kv0", [True, False])
def test_noalloc_python_wrapper(orc, with_kv0, de):
    """la2.forward_noalloc (the binding) against la2.forward and the oracle,
    with and without an initial state, outputs allocated by the caller (with
    64-column heads the array also holds the padded states)."""
    B, H, L = 2, 3, 1000
    d, e = de
    x = inputs.make_inputs(B, H, L, d, e, dtype=torch.bfloat16, device=DEV, seed=7,
                           with_dO=False, with_kv0=True)
    kv0 = x["kv0"] if with_kv0 else None
    lam = inputs.fixed_lambdas((1.0, 0.97, 0.5), DEV)
    old = la2.set_option(la2.LA2_OPT_SPLIT, 3)  # chunk states in the array
    try:
        ref_o, ref_st = la2.forward(x["q"], x["k"], x["v"], lam, kv0, want_state=True)
        out = torch.empty_like(ref_o)
        st_out = torch.empty_like(ref_st)
        o, st = la2.forward_noalloc(x["q"], x["k"], x["v"], lam, kv0, want_state=True,
                                    out=out, state_out=st_out)
        torch.cuda.synchronize()
    finally:
        la2.set_option(la2.LA2_OPT_SPLIT, old)
    assert o is out and st is st_out
    assert la2.last_device_error() == 0
    h = {n: host(t) for n, t in x.items()}
    s0 = None if kv0 is None else kv0.double().cpu().numpy()
    o_r, st_r = orc.forward(h["q"], h["k"], h["v"], lam.double().cpu().numpy(), s0,
                            want_state=True)
    check("wrapper o vs oracle", o, o_r, torch.bfloat16)
    check("wrapper state vs oracle", st, st_r, torch.bfloat16)
    check("wrapper o vs la2_forward", o, host(ref_o), torch.bfloat16)
    check("wrapper state vs la2_forward", st, host(ref_st), torch.bfloat16)


@pytest.mark.gpu
def test_noalloc_rejects_plans_beyond_the_array():
    """A plan needing more than the 32 MiB array is refused before launch.
    The split is forced so that the plan exceeds the array at a modest size,
    and the buffers are real: were the size check ever to pass such a call
    on, la2_forward would refuse it in turn (its workspace, the array, too
    small), so nothing is launched either way."""
    lib = la2.library()
    B, H, L, d, e = 1, 4, 128 * 300, 128, 128
    x = inputs.make_inputs(B, H, L, d, e, dtype=torch.bfloat16, device=DEV, seed=3,
                           with_dO=False)
    lam = inputs.decay_lambdas(H, DEV)
    o = torch.empty_like(x["v"])
    old = la2.set_option(la2.LA2_OPT_SPLIT, 300)
    try:
        need = la2.workspace_size(la2.LA2_OP_FORWARD, B, H, L, d, e, torch.bfloat16)
        assert need > ARRAY_BYTES, need
        code = lib.la2_forward_noalloc(_ptr(x["q"]), _ptr(x["k"]), _ptr(x["v"]), _ptr(lam), None,
                                       _ptr(o), None, B, H, L, d, e, _binding.LA2_BF16, None)
        assert code == _binding.LA2_ERR_UNSUPPORTED, la2.status_string(code)
        with pytest.raises(la2.LA2Error) as err:
            la2.forward_noalloc(x["q"], x["k"], x["v"], lam, out=o)
        assert err.value.code == _binding.LA2_ERR_UNSUPPORTED
    finally:
        la2.set_option(la2.LA2_OPT_SPLIT, old)
    torch.cuda.synchronize()
    assert la2.last_device_error() == 0
    # the same call with the automatic plan fits the array and is correct
    o2 = la2.forward_noalloc(x["q"], x["k"], x["v"], lam)
    ref = la2.forward(x["q"], x["k"], x["v"], lam)
    torch.cuda.synchronize()
    check("noalloc after a refusal", o2, host(ref), torch.bfloat16)
    assert np.isfinite(host(o2)).all()
