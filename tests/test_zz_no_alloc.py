"""la2_forward_noalloc: the forward entry point for callers that cannot
allocate device memory (plug-ins whose host framework owns all device
memory, latency-critical paths that cannot afford cudaMalloc's device
synchronisation, callbacks that only receive device pointers).  It keeps its
chunk-boundary states in the library's own fixed device array instead of a
caller workspace, so it must give the same result as la2_forward.

This file is collected last on purpose: a failure here leaves every other
test already run.  The test also passes when run alone in a fresh process.
"""
import ctypes

import pytest
import torch

import causal_linear_attention_fwd_b200 as la2
from causal_linear_attention_fwd_b200 import _binding, inputs
from gpu_util import check, host

DEV = "cuda:0"


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


@pytest.mark.gpu
def test_noalloc_forward_matches_workspace_forward():
    """Two calls in a row through the C ABI agree with la2_forward (same
    plan, chunk split in use, so the fixed array is really used)."""
    lib = la2.library()
    B, H, L, d, e = 1, 2, 4096, 128, 128
    assert la2.workspace_size(la2.LA2_OP_FORWARD, B, H, L, d, e, torch.bfloat16) > 0
    lam = inputs.decay_lambdas(H, DEV)
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
        check(f"noalloc o (call {seed})", o, host(ref_o), torch.bfloat16)
        check(f"noalloc state (call {seed})", st, host(ref_st), torch.bfloat16)


@pytest.mark.gpu
def test_noalloc_rejects_plans_beyond_the_array():
    """A plan needing more than the 32 MiB array is refused before launch."""
    lib = la2.library()
    B, H, L, d, e = 1, 64, 1 << 20, 128, 128
    need = la2.workspace_size(la2.LA2_OP_FORWARD, B, H, L, d, e, torch.bfloat16)
    if need <= (32 << 20):
        pytest.skip("this device's plan fits the array")
    # fake, aligned, distinct addresses: the call must return before using them
    base = 1 << 40
    ptrs = [ctypes.c_void_p(base + i * (1 << 36)) for i in range(5)]
    code = lib.la2_forward_noalloc(ptrs[0], ptrs[1], ptrs[2], ptrs[3], None, ptrs[4], None,
                                   B, H, L, d, e, _binding.LA2_BF16, None)
    assert code == 2  # LA2_ERR_UNSUPPORTED
