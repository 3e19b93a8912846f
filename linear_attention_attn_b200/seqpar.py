"""Sequence parallelism for the state form (bidirectional linear attention and simple_la).

Every rank holds one shard of the sequence along T (the same B, H, D on every rank).  A
shard's state is a sum over its tokens, so the whole sequence's state is the sum of the
shards' states: the forward is a local reduce, one all-reduce of the [B, H, D, D+1] fp32
state, and a local apply; the backward is a local dq pass, one all-reduce of (dS | dz), and a
local dk, dv pass.  The collective is torch.distributed's (NCCL over NVLink for CUDA
tensors); `ops` is the module that provides the four stages, the CUDA binding by default.
"""
from __future__ import annotations


def _all_reduce(t, group):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def forward(q, k, v, o, state, feature="elu1", eps: float = 1e-6, group=None, ops=None, stream=None,
            workspace=None):
    """o <- the op's output for this rank's shard; state <- the whole sequence's (S | z).
    workspace: optional device buffer of la_workspace_size("state_reduce", ...) bytes."""
    if ops is None:
        from linear_attention_attn_b200 import la_state_apply, la_state_reduce
    else:
        la_state_reduce, la_state_apply = ops.la_state_reduce, ops.la_state_apply
    kw = {} if workspace is None else {"workspace": workspace}
    la_state_reduce(k, v, state, feature=feature, stream=stream, **kw)
    _all_reduce(state, group)
    la_state_apply(q, state, o, feature=feature, eps=eps, stream=stream)
    return state


def backward(q, k, v, dout, state, dq, dk, dv, dstate, feature="elu1", eps: float = 1e-6, group=None, ops=None,
             stream=None, workspace=None):
    """dq, dk, dv of this rank's shard from the whole sequence's state (from forward).
    workspace: optional device buffer of la_workspace_size("state_bwd_q", ...) bytes."""
    if ops is None:
        from linear_attention_attn_b200 import la_state_bwd_kv, la_state_bwd_q
    else:
        la_state_bwd_q, la_state_bwd_kv = ops.la_state_bwd_q, ops.la_state_bwd_kv
    kw = {} if workspace is None else {"workspace": workspace}
    la_state_bwd_q(q, dout, state, dq, dstate, feature=feature, eps=eps, stream=stream, **kw)
    _all_reduce(dstate, group)
    la_state_bwd_kv(k, v, dstate, dk, dv, feature=feature, stream=stream)
    return dstate
