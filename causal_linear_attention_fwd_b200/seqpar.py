"""Sequence parallelism: one long sequence split across the ranks of a
torch.distributed process group, one contiguous shard of L rows per rank in
rank order (every rank the same L and the same B, H, d, e).

Each shard needs, per (b,h), only two d x e summaries of the other shards:
the state entering it (forward) and the reverse state flowing into it from
the rows after it (backward).  A rank computes its own shard's summary with
the library (la2_shard_state), the ranks exchange them in one all-gather per
direction (NCCL over NVLink on GPUs), every rank forms the lambda-weighted
prefix (la2_state_prefix) and runs its shard's ordinary passes from there
(la2_forward with kv0 = the entry state; la2_backward_shard).  The result on
each rank is its rows' slice of what one device would compute for the whole
sequence; the sequence's final state is the last rank's, dkv0 the first
rank's.  The reassociation is the block schedule's (Lightning Attention-2
notes page, "Tiling." paragraph) applied to shards; the pages do not discuss
splitting a sequence across devices.
"""
import torch
import torch.distributed as dist

from . import _binding as _lib


class Ops:
    """The library calls this module makes (a host-only test substitutes
    stand-ins to exercise the exchange on CPU ranks)."""
    shard_state = staticmethod(_lib.shard_state)
    state_prefix = staticmethod(_lib.state_prefix)
    forward = staticmethod(_lib.forward)
    backward_shard = staticmethod(_lib.backward_shard)


def _all_gather(x, group):
    """[R, ...] stack of every rank's x, in rank order."""
    parts = [torch.empty_like(x) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, x.contiguous(), group=group)
    return torch.stack(parts)


def entry_state(k, v, lam, kv0=None, *, group=None, ops=Ops):
    """The state entering this rank's shard (kv0: the sequence's initial
    state, the same tensor on every rank, or None)."""
    deltas = _all_gather(ops.shard_state(k, v, lam), group)
    return ops.state_prefix(deltas, lam, k.shape[2], kv0)[dist.get_rank(group)].contiguous()


def end_state(q, dO, lam, *, group=None, ops=Ops):
    """The reverse state flowing into this rank's shard from the rows after it."""
    deltas = _all_gather(ops.shard_state(q, dO, lam, reverse=True), group)
    return ops.state_prefix(deltas, lam, q.shape[2], reverse=True)[dist.get_rank(group)].contiguous()


def forward(q, k, v, lam, kv0=None, *, group=None, want_state: bool = False, ops=Ops):
    """This shard's o [B,H,L,e] (and the state after it: the sequence's final
    state on the last rank)."""
    entry = entry_state(k, v, lam, kv0, group=group, ops=ops)
    return ops.forward(q, k, v, lam, entry, want_state=want_state)


def backward(q, k, v, lam, dO, kv0=None, *, group=None, want_dkv0: bool = False, ops=Ops):
    """This shard's (dq, dk, dv[, dkv0]) of the whole sequence's sum(o * dO);
    dkv0 is the gradient with respect to kv0 on the first rank."""
    entry = entry_state(k, v, lam, kv0, group=group, ops=ops)
    end = end_state(q, dO, lam, group=group, ops=ops)
    return ops.backward_shard(q, k, v, lam, dO, entry, end, want_dkv0=want_dkv0)
