"""ctypes binding of libla2 (include/la2.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libla2.so.  PyTorch supplies device memory (outputs, scratch
workspace) and the current CUDA stream.  There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""
from __future__ import annotations

import ctypes
import json
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libla2.so")

LA2_OK, LA2_ERR_INVALID, LA2_ERR_UNSUPPORTED, LA2_ERR_CUDA, LA2_ERR_TIMEOUT = range(5)
LA2_F32, LA2_BF16 = 0, 1
LA2_OP_FORWARD, LA2_OP_BACKWARD, LA2_OP_SHARD_STATE, LA2_OP_DLAMBDA = 0, 1, 2, 3
LA2_OPT_SPLIT, LA2_OPT_PATH, LA2_OPT_INJECT_TIMEOUT, LA2_OPT_VARIANT, LA2_OPT_TRACE = 0, 1, 2, 3, 4
LA2_OPT_VARLEN_ORDER, LA2_OPT_DECODE_BLOCK_TOKENS, LA2_OPT_BWD_FORM = 5, 6, 7

_lock = threading.Lock()
_lib = None


class LA2Error(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {status_string(code)}")


def library():
    """Load libla2.so (built in-tree by ``build.py``); raise if it is absent."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libla2.so is not built ({LIB_PATH}); run "
                "`python -c 'import __graft_entry__ as g; g.build()'` or "
                "`python causal_linear_attention_fwd_b200/build.py`")
        lib = ctypes.CDLL(LIB_PATH)
        P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        lib.la2_workspace_size.argtypes = [I, I, I, I64, I, I, I]
        lib.la2_workspace_size.restype = SZ
        lib.la2_forward.argtypes = [P, P, P, P, P, P, P, I, I, I64, I, I, I, P, SZ, P]
        lib.la2_forward.restype = I
        lib.la2_forward_noalloc.argtypes = [P, P, P, P, P, P, P, I, I, I64, I, I, I, P]
        lib.la2_forward_noalloc.restype = I
        lib.la2_backward.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I64, I, I, I,
                                     P, SZ, P]
        lib.la2_backward.restype = I
        lib.la2_backward_ex.argtypes = [P, P, P, P, P, P, P, P, P, P, I, I, I64, I, I, I,
                                        P, SZ, ctypes.c_uint, P]
        lib.la2_backward_ex.restype = I
        lib.la2_forward_varlen.argtypes = [P, P, P, P, P, P, P, P, I, I, I64, I, I, I, P]
        lib.la2_forward_varlen.restype = I
        lib.la2_backward_varlen.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I, I64, I, I,
                                            I, P]
        lib.la2_backward_varlen.restype = I
        lib.la2_forward_pool.argtypes = [P, P, P, P, P, P, I, P, ctypes.c_uint, I, I, I64, I,
                                         I, I, P, SZ, P]
        lib.la2_forward_pool.restype = I
        lib.la2_decode_tokens.argtypes = [P, P, P, P, P, P, I, P, I, I, I, I, I, I, P]
        lib.la2_decode_tokens.restype = I
        lib.la2_shard_state.argtypes = [P, P, P, P, I, I, I64, I, I, I, I, P, SZ, P]
        lib.la2_shard_state.restype = I
        lib.la2_state_prefix.argtypes = [P, P, P, P, I, I, I, I64, I, I, I, P]
        lib.la2_state_prefix.restype = I
        lib.la2_backward_shard.argtypes = [P, P, P, P, P, P, P, P, P, P, P, I, I, I64, I, I, I,
                                           P, SZ, ctypes.c_uint, P]
        lib.la2_backward_shard.restype = I
        lib.la2_backward_dlambda.argtypes = [P, P, P, P, P, P, P, I, I, I64, I, I, I, P]
        lib.la2_backward_dlambda.restype = I
        lib.la2_backward_dlambda_ex.argtypes = [P, P, P, P, P, P, P, I, I, I64, I, I, I, P, SZ, P]
        lib.la2_backward_dlambda_ex.restype = I
        lib.la2_decode_step.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P]
        lib.la2_decode_step.restype = I
        lib.la2_feature_map.argtypes = [P, P, P, P, I64, I, P]
        lib.la2_feature_map.restype = I
        lib.la2_feature_map_backward.argtypes = [P, P, P, P, P, P, I64, I, P]
        lib.la2_feature_map_backward.restype = I
        lib.la2_last_device_error.argtypes = [P]
        lib.la2_last_device_error.restype = I
        lib.la2_status_string.argtypes = [I]
        lib.la2_status_string.restype = ctypes.c_char_p
        lib.la2_set_option.argtypes = [I, I]
        lib.la2_set_option.restype = I
        lib.la2_profile_enable.argtypes = [I]
        lib.la2_profile_enable.restype = None
        lib.la2_profile_report.argtypes = [ctypes.c_char_p, SZ]
        lib.la2_profile_report.restype = SZ
        lib.la2_trace_read.argtypes = [P, SZ]
        lib.la2_trace_read.restype = SZ
        lib.la2_version.argtypes = []
        lib.la2_version.restype = ctypes.c_char_p
        _lib = lib
        return lib


def status_string(code: int) -> str:
    try:
        return library().la2_status_string(int(code)).decode()
    except Exception:  # library missing: still give a name
        return {0: "LA2_OK", 1: "LA2_ERR_INVALID", 2: "LA2_ERR_UNSUPPORTED",
                3: "LA2_ERR_CUDA", 4: "LA2_ERR_TIMEOUT"}.get(int(code), str(code))


def _check(code: int, what: str):
    if code != LA2_OK:
        raise LA2Error(code, what)


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return LA2_F32
    if t.dtype == torch.bfloat16:
        return LA2_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dev(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _devices(*named):
    """Check (name, tensor) pairs -- None tensors skipped -- as _dev does and
    that all of them live on one device; return that device.  The library
    launches on the CURRENT device, so a call with tensors elsewhere would
    run its kernels and tensor maps over another GPU's memory."""
    dev = None
    for name, t in named:
        if t is None:
            continue
        _dev(t, name)
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"{name} is on {t.device}, other arguments on {dev}")
    if dev is None:
        raise ValueError("no tensor arguments")
    return dev


def _stream(stream, device=None):
    if stream is None:
        s = torch.cuda.current_stream(device)
    else:
        s = stream
        if device is not None and s.device != device:
            raise ValueError(f"stream is on {s.device}, the tensors on {device}")
    return ctypes.c_void_p(s.cuda_stream)


def _out(t, name, shape, dtype, device):
    """A caller-provided output buffer: contiguous, on `device`, of this
    shape and dtype."""
    _dev(t, name)
    if t.device != device or tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype} {tuple(shape)} on {device}")
    return t


def set_option(option: int, value: int) -> int:
    return int(library().la2_set_option(int(option), int(value)))


def version() -> str:
    return library().la2_version().decode()


def workspace_size(op: int, B: int, H: int, L: int, d: int, e: int, dtype) -> int:
    dt = LA2_F32 if dtype == torch.float32 else LA2_BF16
    return int(library().la2_workspace_size(op, B, H, L, d, e, dt))


def _workspace(nbytes: int, device):
    if nbytes == 0:
        return None
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def forward(q, k, v, lam, kv0=None, *, want_state: bool = False, out=None,
            workspace=None, stream=None):
    """o = (Q K^T (.) M) V (+ the kv0 term); optionally the final state."""
    lib = library()
    dev = _devices(("q", q), ("k", k), ("v", v), ("lam", lam), ("kv0", kv0),
                   ("workspace", workspace))
    B, H, L, d = q.shape
    e = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L):
        raise ValueError("shape mismatch among q, k, v")
    if lam.dtype != torch.float32 or lam.numel() != H:
        raise ValueError("lam must be float32 [H]")
    if kv0 is not None and (kv0.dtype != torch.float32 or kv0.shape != (B, H, d, e)):
        raise ValueError("kv0 must be float32 [B,H,d,e]")
    with torch.cuda.device(dev):
        o = (_out(out, "out", (B, H, L, e), q.dtype, dev) if out is not None
             else torch.empty((B, H, L, e), dtype=q.dtype, device=dev))
        st = torch.empty((B, H, d, e), dtype=torch.float32, device=dev) if want_state else None
        ws = workspace
        if ws is None:
            ws = _workspace(workspace_size(LA2_OP_FORWARD, B, H, L, d, e, q.dtype), dev)
        code = lib.la2_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(kv0), _ptr(o),
                               _ptr(st), B, H, L, d, e, _dt(q), _ptr(ws),
                               0 if ws is None else ws.numel() * ws.element_size(),
                               _stream(stream, dev))
    _check(code, "la2_forward")
    return (o, st) if want_state else o


def forward_noalloc(q, k, v, lam, kv0=None, *, want_state: bool = False, out=None,
                    state_out=None, stream=None):
    """forward() for callers that cannot allocate device scratch: the library
    keeps the chunk-boundary states in its own fixed 32 MiB device array
    (see la2_forward_noalloc in include/la2.h).  Outputs are allocated here
    unless the caller passes them: `out` (o) and, with want_state,
    `state_out` (the final state)."""
    lib = library()
    dev = _devices(("q", q), ("k", k), ("v", v), ("lam", lam), ("kv0", kv0))
    B, H, L, d = q.shape
    e = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L):
        raise ValueError("shape mismatch among q, k, v")
    if lam.dtype != torch.float32 or lam.numel() != H:
        raise ValueError("lam must be float32 [H]")
    if kv0 is not None and (kv0.dtype != torch.float32 or kv0.shape != (B, H, d, e)):
        raise ValueError("kv0 must be float32 [B,H,d,e]")
    if state_out is not None and not want_state:
        raise ValueError("state_out is given but want_state is False")
    with torch.cuda.device(dev):
        o = (_out(out, "out", (B, H, L, e), q.dtype, dev) if out is not None
             else torch.empty((B, H, L, e), dtype=q.dtype, device=dev))
        st = None
        if want_state:
            st = (_out(state_out, "state_out", (B, H, d, e), torch.float32, dev)
                  if state_out is not None
                  else torch.empty((B, H, d, e), dtype=torch.float32, device=dev))
        code = lib.la2_forward_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(kv0), _ptr(o),
                                       _ptr(st), B, H, L, d, e, _dt(q), _stream(stream, dev))
    _check(code, "la2_forward_noalloc")
    return (o, st) if want_state else o


def backward(q, k, v, lam, dO, kv0=None, *, want_dkv0: bool = False, outs=None,
             workspace=None, reuse_forward_states: bool = False, stream=None):
    """Gradients (dq, dk, dv[, dkv0]) of sum(o * dO).

    reuse_forward_states: `workspace` (sized for the backward) was passed to
    forward() with the same inputs and still holds the chunk states it wrote,
    so the backward does not recompute them."""
    if reuse_forward_states and workspace is None:
        raise ValueError("reuse_forward_states needs the forward's workspace")
    lib = library()
    dev = _devices(("q", q), ("k", k), ("v", v), ("lam", lam), ("dO", dO), ("kv0", kv0),
                   ("workspace", workspace))
    B, H, L, d = q.shape
    e = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L) or dO.shape != v.shape:
        raise ValueError("shape mismatch among q, k, v, dO")
    if lam.dtype != torch.float32 or lam.numel() != H:
        raise ValueError("lam must be float32 [H]")
    if kv0 is not None and (kv0.dtype != torch.float32 or kv0.shape != (B, H, d, e)):
        raise ValueError("kv0 must be float32 [B,H,d,e]")
    with torch.cuda.device(dev):
        if outs is not None:
            dq, dk, dv = outs
            _out(dq, "dq", q.shape, q.dtype, dev)
            _out(dk, "dk", k.shape, q.dtype, dev)
            _out(dv, "dv", v.shape, q.dtype, dev)
        else:
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dkv0 = torch.empty((B, H, d, e), dtype=torch.float32, device=dev) if want_dkv0 else None
        ws = workspace
        if ws is None:
            ws = _workspace(workspace_size(LA2_OP_BACKWARD, B, H, L, d, e, q.dtype), dev)
        code = lib.la2_backward_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(kv0), _ptr(dO),
                                   _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dkv0), B, H, L, d, e,
                                   _dt(q), _ptr(ws),
                                   0 if ws is None else ws.numel() * ws.element_size(),
                                   1 if reuse_forward_states else 0, _stream(stream, dev))
    _check(code, "la2_backward")
    return (dq, dk, dv, dkv0) if want_dkv0 else (dq, dk, dv)


def _varlen_args(q, k, v, lam, cu_seqlens, kv0, *extra):
    dev = _devices(("q", q), ("k", k), ("v", v), ("lam", lam), ("cu_seqlens", cu_seqlens),
                   ("kv0", kv0), *extra)
    H, T, d = q.shape
    e = v.shape[-1]
    if k.shape != q.shape or v.shape[:2] != (H, T):
        raise ValueError("q, k must be [H, T, d] and v [H, T, e]")
    if lam.dtype != torch.float32 or lam.numel() != H:
        raise ValueError("lam must be float32 [H]")
    if cu_seqlens.dtype != torch.int64 or cu_seqlens.dim() != 1 or cu_seqlens.numel() < 1:
        raise ValueError("cu_seqlens must be int64 [N+1]")
    N = cu_seqlens.numel() - 1
    if kv0 is not None and (kv0.dtype != torch.float32 or kv0.shape != (N, H, d, e)):
        raise ValueError("kv0 must be float32 [N,H,d,e]")
    return dev, N, H, T, d, e


def forward_varlen(q, k, v, lam, cu_seqlens, kv0=None, *, want_state: bool = False,
                   out=None, stream=None):
    """Packed variable-length forward: q, k [H,T,d], v [H,T,e], sequence n on
    rows cu_seqlens[n]..cu_seqlens[n+1] of every head; per-sequence states
    [N,H,d,e].  Returns o [H,T,e] (and the final states)."""
    lib = library()
    dev, N, H, T, d, e = _varlen_args(q, k, v, lam, cu_seqlens, kv0)
    with torch.cuda.device(dev):
        o = (_out(out, "out", (H, T, e), q.dtype, dev) if out is not None
             else torch.empty((H, T, e), dtype=q.dtype, device=dev))
        st = torch.empty((N, H, d, e), dtype=torch.float32, device=dev) if want_state else None
        code = lib.la2_forward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(cu_seqlens),
                                      _ptr(kv0), _ptr(o), _ptr(st), N, H, T, d, e, _dt(q),
                                      _stream(stream, dev))
    _check(code, "la2_forward_varlen")
    return (o, st) if want_state else o


def backward_varlen(q, k, v, lam, cu_seqlens, dO, kv0=None, *, want_dkv0: bool = False,
                    outs=None, stream=None):
    """Gradients (dq, dk, dv[, dkv0]) of sum(o * dO) for forward_varlen."""
    lib = library()
    dev, N, H, T, d, e = _varlen_args(q, k, v, lam, cu_seqlens, kv0, ("dO", dO))
    if dO.shape != v.shape:
        raise ValueError("dO must match v")
    with torch.cuda.device(dev):
        if outs is not None:
            dq, dk, dv = outs
            _out(dq, "dq", q.shape, q.dtype, dev)
            _out(dk, "dk", k.shape, q.dtype, dev)
            _out(dv, "dv", v.shape, q.dtype, dev)
        else:
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dkv0 = torch.empty((N, H, d, e), dtype=torch.float32, device=dev) if want_dkv0 else None
        code = lib.la2_backward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(cu_seqlens),
                                       _ptr(kv0), _ptr(dO), _ptr(dq), _ptr(dk), _ptr(dv),
                                       _ptr(dkv0), N, H, T, d, e, _dt(q), _stream(stream, dev))
    _check(code, "la2_backward_varlen")
    return (dq, dk, dv, dkv0) if want_dkv0 else (dq, dk, dv)


LA2_POOL_CONTINUE = 1


def _slots(slots, B):
    if slots is None:
        return None
    if slots.dtype != torch.int32 or slots.shape != (B,):
        raise ValueError("slots must be int32 [B]")
    return slots


def forward_pool(q, k, v, lam, pool, slots, *, continue_state: bool = False, out=None,
                 workspace=None, stream=None):
    """Prefill into a state pool [P,H,d,e]: request b starts from zero (or,
    with continue_state, from pool[slots[b]]) and leaves its final state in
    pool[slots[b]].  Returns o [B,H,L,e]."""
    lib = library()
    if slots is None:
        raise ValueError("forward_pool needs a slot table")
    dev = _devices(("q", q), ("k", k), ("v", v), ("lam", lam), ("pool", pool),
                   ("slots", slots), ("workspace", workspace))
    B, H, L, d = q.shape
    e = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L):
        raise ValueError("shape mismatch among q, k, v")
    if pool.dtype != torch.float32 or pool.dim() != 4 or pool.shape[1:] != (H, d, e):
        raise ValueError("pool must be float32 [P,H,d,e]")
    slots = _slots(slots, B)
    with torch.cuda.device(dev):
        o = (_out(out, "out", (B, H, L, e), q.dtype, dev) if out is not None
             else torch.empty((B, H, L, e), dtype=q.dtype, device=dev))
        ws = workspace
        if ws is None:
            ws = _workspace(workspace_size(LA2_OP_FORWARD, B, H, L, d, e, q.dtype), dev)
        code = lib.la2_forward_pool(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(pool),
                                    _ptr(slots), pool.shape[0], _ptr(o),
                                    LA2_POOL_CONTINUE if continue_state else 0, B, H, L, d, e,
                                    _dt(q), _ptr(ws),
                                    0 if ws is None else ws.numel() * ws.element_size(),
                                    _stream(stream, dev))
    _check(code, "la2_forward_pool")
    return o


def decode_tokens(q, k, v, lam, pool, slots=None, *, out=None, stream=None):
    """T tokens per request at once: q, k [B,H,T,d], v [B,H,T,e]; the state
    of request b is pool[slots[b]] (pool[b] without a slot table), updated
    in place; returns o [B,H,T,e]."""
    lib = library()
    dev = _devices(("q", q), ("k", k), ("v", v), ("lam", lam), ("pool", pool),
                   ("slots", slots))
    B, H, T, d = q.shape
    e = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, T):
        raise ValueError("shape mismatch among q, k, v")
    if pool.dtype != torch.float32 or pool.dim() != 4 or pool.shape[1:] != (H, d, e):
        raise ValueError("pool must be float32 [P,H,d,e]")
    slots = _slots(slots, B)
    with torch.cuda.device(dev):
        o = (_out(out, "out", (B, H, T, e), q.dtype, dev) if out is not None
             else torch.empty((B, H, T, e), dtype=q.dtype, device=dev))
        code = lib.la2_decode_tokens(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(pool),
                                     _ptr(slots), pool.shape[0], _ptr(o), B, H, T, d, e, _dt(q),
                                     _stream(stream, dev))
    _check(code, "la2_decode_tokens")
    return o


def shard_state(a, b, lam, *, reverse: bool = False, workspace=None, stream=None):
    """One shard's d x e summary: forward (a = k, b = v) sum_t
    lam^(L-1-t) k_t^T v_t, reverse (a = q, b = dO) sum_t lam^t q_t^T dO_t;
    fp32 [B,H,d,e]."""
    lib = library()
    dev = _devices(("a", a), ("b", b), ("lam", lam), ("workspace", workspace))
    B, H, L, d = a.shape
    e = b.shape[-1]
    if b.shape[:3] != (B, H, L):
        raise ValueError("shape mismatch between a and b")
    with torch.cuda.device(dev):
        out = torch.empty((B, H, d, e), dtype=torch.float32, device=dev)
        ws = workspace
        if ws is None:
            ws = _workspace(workspace_size(LA2_OP_SHARD_STATE, B, H, L, d, e, a.dtype), dev)
        code = lib.la2_shard_state(_ptr(a), _ptr(b), _ptr(lam), _ptr(out), B, H, L, d, e,
                                   _dt(a), 1 if reverse else 0, _ptr(ws),
                                   0 if ws is None else ws.numel() * ws.element_size(),
                                   _stream(stream, dev))
    _check(code, "la2_shard_state")
    return out


def state_prefix(delta, lam, L_shard: int, kv0=None, *, reverse: bool = False, stream=None):
    """Every shard's boundary state from the R shards' deltas [R,B,H,d,e]:
    forward, the state entering shard r (from kv0); reverse, the reverse
    state flowing into shard r from the rows after it."""
    lib = library()
    dev = _devices(("delta", delta), ("lam", lam), ("kv0", kv0))
    if delta.dtype != torch.float32 or delta.dim() != 5:
        raise ValueError("delta must be float32 [R,B,H,d,e]")
    R, B, H, d, e = delta.shape
    if kv0 is not None and (kv0.dtype != torch.float32 or kv0.shape != (B, H, d, e)):
        raise ValueError("kv0 must be float32 [B,H,d,e]")
    with torch.cuda.device(dev):
        out = torch.empty_like(delta)
        code = lib.la2_state_prefix(_ptr(delta), _ptr(kv0), _ptr(lam), _ptr(out), R, B, H,
                                    int(L_shard), d, e, 1 if reverse else 0,
                                    _stream(stream, dev))
    _check(code, "la2_state_prefix")
    return out


def backward_shard(q, k, v, lam, dO, kv0=None, dstate_end=None, *, want_dkv0: bool = False,
                   outs=None, workspace=None, stream=None):
    """backward() of one shard of a longer sequence: kv0 its entry state,
    dstate_end the reverse state flowing in from the rows after it."""
    lib = library()
    dev = _devices(("q", q), ("k", k), ("v", v), ("lam", lam), ("dO", dO), ("kv0", kv0),
                   ("dstate_end", dstate_end), ("workspace", workspace))
    B, H, L, d = q.shape
    e = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L) or dO.shape != v.shape:
        raise ValueError("shape mismatch among q, k, v, dO")
    for name, t in (("kv0", kv0), ("dstate_end", dstate_end)):
        if t is not None and (t.dtype != torch.float32 or t.shape != (B, H, d, e)):
            raise ValueError(f"{name} must be float32 [B,H,d,e]")
    with torch.cuda.device(dev):
        if outs is not None:
            dq, dk, dv = outs
            _out(dq, "dq", q.shape, q.dtype, dev)
            _out(dk, "dk", k.shape, q.dtype, dev)
            _out(dv, "dv", v.shape, q.dtype, dev)
        else:
            dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        dkv0 = torch.empty((B, H, d, e), dtype=torch.float32, device=dev) if want_dkv0 else None
        ws = workspace
        if ws is None:
            ws = _workspace(workspace_size(LA2_OP_BACKWARD, B, H, L, d, e, q.dtype), dev)
        code = lib.la2_backward_shard(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(kv0), _ptr(dO),
                                      _ptr(dstate_end), _ptr(dq), _ptr(dk), _ptr(dv),
                                      _ptr(dkv0), B, H, L, d, e, _dt(q), _ptr(ws),
                                      0 if ws is None else ws.numel() * ws.element_size(), 0,
                                      _stream(stream, dev))
    _check(code, "la2_backward_shard")
    return (dq, dk, dv, dkv0) if want_dkv0 else (dq, dk, dv)


def dlambda(q, k, v, lam, dO, kv0=None, *, workspace=None, chunked: bool = True, stream=None):
    """Gradient of sum(o * dO) with respect to lam [H] (float32 [H], summed
    over the batch).  chunked: split the sequences over several CTAs
    (la2_backward_dlambda_ex with `workspace`, allocated here when None);
    False: one CTA per (b,h), no workspace (la2_backward_dlambda)."""
    lib = library()
    dev = _devices(("q", q), ("k", k), ("v", v), ("lam", lam), ("dO", dO), ("kv0", kv0),
                   ("workspace", workspace))
    B, H, L, d = q.shape
    e = v.shape[-1]
    if k.shape != q.shape or v.shape[:3] != (B, H, L) or dO.shape != v.shape:
        raise ValueError("shape mismatch among q, k, v, dO")
    if lam.dtype != torch.float32 or lam.numel() != H:
        raise ValueError("lam must be float32 [H]")
    if kv0 is not None and (kv0.dtype != torch.float32 or kv0.shape != (B, H, d, e)):
        raise ValueError("kv0 must be float32 [B,H,d,e]")
    with torch.cuda.device(dev):
        out = torch.empty(H, dtype=torch.float32, device=dev)
        if not chunked:
            code = lib.la2_backward_dlambda(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(kv0),
                                            _ptr(dO), _ptr(out), B, H, L, d, e, _dt(q),
                                            _stream(stream, dev))
            _check(code, "la2_backward_dlambda")
            return out
        if workspace is None:
            workspace = _workspace(workspace_size(LA2_OP_DLAMBDA, B, H, L, d, e, q.dtype), dev)
        nbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
        code = lib.la2_backward_dlambda_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(kv0),
                                           _ptr(dO), _ptr(out), B, H, L, d, e, _dt(q),
                                           _ptr(workspace), nbytes, _stream(stream, dev))
    _check(code, "la2_backward_dlambda_ex")
    return out


def _fmap_args(q, k, extra):
    dev = _devices(("q", q), ("k", k), *extra)
    if k is not None and (k.shape != q.shape or k.dtype != q.dtype):
        raise ValueError("q and k must have the same shape and dtype")
    for name, t in extra:
        if t is not None and (t.shape != q.shape or t.dtype != q.dtype):
            raise ValueError(f"{name} must match q's shape and dtype")
    return dev


def feature_map(q, k=None, *, out=None, stream=None):
    """phi(x) = elu(x) + 1 applied to q (and k): returns phi_q (and phi_k).
    out: (phi_q, phi_k) buffers, which may be q and k themselves (in place)."""
    lib = library()
    dev = _fmap_args(q, k, ())
    with torch.cuda.device(dev):
        phi_q, phi_k = out if out is not None else (
            torch.empty_like(q), None if k is None else torch.empty_like(k))
        _fmap_args(q, k, (("phi_q", phi_q), ("phi_k", phi_k)))
        code = lib.la2_feature_map(_ptr(q), _ptr(k), _ptr(phi_q), _ptr(phi_k), q.numel(),
                                   _dt(q), _stream(stream, dev))
    _check(code, "la2_feature_map")
    return phi_q if k is None else (phi_q, phi_k)


def feature_map_backward(q, k, dphi_q, dphi_k=None, *, out=None, stream=None):
    """Chain rule through the feature map: dq = dphi_q * phi'(q) (and dk
    likewise), q, k the unmapped inputs, dphi_* the attention's gradients
    with respect to phi(q), phi(k).  out may be (dphi_q, dphi_k) (in place).
    k and dphi_k are both None to map q alone."""
    lib = library()
    if (k is None) != (dphi_k is None):
        raise ValueError("k and dphi_k are both given or both None")
    dev = _fmap_args(q, k, (("dphi_q", dphi_q), ("dphi_k", dphi_k)))
    with torch.cuda.device(dev):
        dq, dk = out if out is not None else (
            torch.empty_like(q), None if k is None else torch.empty_like(k))
        _fmap_args(q, k, (("dphi_q", dphi_q), ("dphi_k", dphi_k), ("dq", dq), ("dk", dk)))
        code = lib.la2_feature_map_backward(_ptr(q), _ptr(k), _ptr(dphi_q), _ptr(dphi_k),
                                            _ptr(dq), _ptr(dk), q.numel(), _dt(q),
                                            _stream(stream, dev))
    _check(code, "la2_feature_map_backward")
    return dq if k is None else (dq, dk)


def decode_step(q, k, v, lam, kv, *, out=None, stream=None):
    """kv <- lam kv + k^T v (in place); returns o = q kv."""
    lib = library()
    dev = _devices(("q", q), ("k", k), ("v", v), ("lam", lam), ("kv", kv))
    B, H, d = q.shape
    e = v.shape[-1]
    if kv.dtype != torch.float32 or kv.shape != (B, H, d, e):
        raise ValueError("kv must be float32 [B,H,d,e]")
    with torch.cuda.device(dev):
        o = (_out(out, "out", (B, H, e), q.dtype, dev) if out is not None
             else torch.empty((B, H, e), dtype=q.dtype, device=dev))
        code = lib.la2_decode_step(_ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(kv), _ptr(o),
                                   B, H, d, e, _dt(q), _stream(stream, dev))
    _check(code, "la2_decode_step")
    return o


def last_device_error(stream=None) -> int:
    return int(library().la2_last_device_error(_stream(stream)))


def trace_read():
    """Trace buffer as a [16 events, 512 blocks] int64 tensor (ns; 0 = unset)."""
    lib = library()
    n = int(lib.la2_trace_read(None, 0))
    buf = torch.zeros(n, dtype=torch.int64)
    lib.la2_trace_read(ctypes.c_void_p(buf.data_ptr()), n)
    return buf.view(16, -1)


def profile_enable(on: bool = True):
    library().la2_profile_enable(1 if on else 0)


def profile_report() -> dict:
    # one report clears the records, so size the buffer generously up front
    n = 1 << 16
    buf = ctypes.create_string_buffer(n)
    library().la2_profile_report(buf, n)
    return json.loads(buf.value.decode() or "{}")
