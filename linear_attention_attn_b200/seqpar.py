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


def decay_forward(q, k, v, o, decay, state_out=None, group=None, ops=None, stream=None, workspace=None):
    """The decay op (retention) forward for this rank's segment of a sequence split along T
    (rank r holds the r-th segment).  A segment's output needs the state of every token before
    it: pass 1 gives each segment's own end state E_r (from a zero state), an all-gather shares
    them with the segment lengths, rank r forms S_r = sum_{r' < r} (prod of gamma^T over the
    segments between) E_r' as the running state gamma^{T_r'} S + E_r', and pass 2 recomputes the
    segment from S_r.  state_out (optional, [B, H, D, D] fp32) receives the state after this
    rank's segment (on the last rank: after the whole sequence)."""
    import torch
    if ops is None:
        from linear_attention_attn_b200 import la_chunk_decay_fwd_state
    else:
        la_chunk_decay_fwd_state = ops.la_chunk_decay_fwd_state
    import torch.distributed as dist
    B, H, T, D = (int(x) for x in q.shape)
    kw = {} if workspace is None else {"workspace": workspace}
    end = torch.empty((B, H, D, D), dtype=torch.float32 if q.is_cuda else torch.float64, device=q.device)
    la_chunk_decay_fwd_state(q, k, v, o, decay, state_in=None, state_out=end, stream=stream, **kw)
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    if world == 1:
        if state_out is not None:
            state_out.copy_(end)
        return state_out
    rank = dist.get_rank(group)
    ends = [torch.empty_like(end) for _ in range(world)]
    dist.all_gather(ends, end, group=group)
    lens = torch.tensor([T], dtype=torch.int64, device=end.device)
    all_lens = [torch.empty_like(lens) for _ in range(world)]
    dist.all_gather(all_lens, lens, group=group)
    gam = torch.as_tensor([float(x) for x in (decay.tolist() if hasattr(decay, "tolist") else decay)],
                          dtype=torch.float64)
    state = torch.zeros((B, H, D, D), dtype=torch.float64, device=end.device)
    for r in range(rank):
        f = torch.pow(gam, float(all_lens[r].item())).to(end.device)
        state = f[None, :, None, None] * state + ends[r].to(torch.float64)
    sin = state.to(end.dtype).contiguous()
    la_chunk_decay_fwd_state(q, k, v, o, decay, state_in=sin, state_out=state_out, stream=stream, **kw)
    return state_out
