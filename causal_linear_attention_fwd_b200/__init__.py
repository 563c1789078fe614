"""B200-native tiled causal linear attention with per-head decay.

O = (Q K^T (.) M) V, M_tj = lambda_h^(t-j) for j <= t (lambda_h = 1: plain
causal linear attention), computed with the Lightning Attention-2 block
schedule -- intra-block dense masked products plus an inter-block carried
d x e state -- in forward and backward, plus the recurrent decode step.

The computation lives in the C-ABI library libla2.so (include/la2.h); this
package is its thin Python binding.  The library is loaded on first use and
its absence raises an error: there is no CPU fallback.
"""
from ._binding import (  # noqa: F401
    LA2Error, LA2_OP_BACKWARD, LA2_OP_FORWARD, LA2_OPT_INJECT_TIMEOUT, LA2_OPT_PATH,
    LA2_POOL_CONTINUE, LA2_OP_SHARD_STATE, LA2_OP_DLAMBDA, backward_shard, decode_tokens, forward_pool,
    shard_state, state_prefix, dlambda,
    LA2_OPT_SPLIT, LA2_OPT_TRACE, LA2_OPT_VARIANT, LA2_OPT_VARLEN_ORDER, LA2_OPT_DECODE_BLOCK_TOKENS, LA2_OPT_BWD_FORM,
    trace_read,
    backward, backward_varlen, decode_step, feature_map, feature_map_backward, forward,
    forward_noalloc, forward_varlen,
    last_device_error, library, profile_enable, profile_report, set_option, status_string,
    version, workspace_size)

__all__ = ["forward", "forward_noalloc", "backward", "forward_varlen", "backward_varlen",
           "forward_pool", "decode_step", "decode_tokens", "shard_state", "state_prefix",
           "backward_shard", "dlambda", "feature_map", "feature_map_backward", "workspace_size",
           "last_device_error", "set_option", "profile_enable", "profile_report",
           "status_string", "version", "library", "LA2Error"]
