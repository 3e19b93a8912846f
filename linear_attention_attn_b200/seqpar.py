"""Sequence parallelism for the state form (bidirectional linear attention and simple_la) and
for the decay op (retention).

Every rank holds one shard of the sequence along T (the same B, H, D on every rank).  A
shard's state is a sum over its tokens, so the whole sequence's state is the sum of the
shards' states: the forward is a local reduce, one all-reduce of the [B, H, D, D+1] fp32
state, and a local apply; the backward is a local dq pass, one all-reduce of (dS | dz), and a
local dk, dv pass.  The decay op's segments are not a sum but a scan (the state entering a
segment decays across the segments in between): its end states are all-gathered and
combined per rank (decay_forward, decay_backward).  The collective is torch.distributed's
(NCCL over NVLink for CUDA tensors); `ops` is the module that provides the stages, the CUDA
binding by default.  The collectives and the stages run in the order of torch's current stream:
pass stream=None, or that stream.
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


def _world(group):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        return dist.get_world_size(group), dist.get_rank(group)
    return 1, 0


def _gather_states(x, T, group):
    """All-gather this rank's [B, H, D, D] state and segment length: ([world, B, H, D, D], lengths)."""
    import torch
    import torch.distributed as dist
    world, _ = _world(group)
    buf = torch.empty((world,) + tuple(x.shape), dtype=x.dtype, device=x.device)
    dist.all_gather(list(buf.unbind(0)), x, group=group)
    lens = torch.tensor([T], dtype=torch.int64, device=x.device)
    all_lens = [torch.empty_like(lens) for _ in range(world)]
    dist.all_gather(all_lens, lens, group=group)
    return buf, [int(t.item()) for t in all_lens]


def entering_gaps(lens, rank):
    """Gaps for the state entering segment `rank`: segment i < rank is followed by the tokens of
    segments i+1 .. rank-1 before it reaches `rank` (-1: segment not included)."""
    return [sum(lens[i + 1:rank]) if i < rank else -1 for i in range(len(lens))]


def leaving_gaps(lens, rank):
    """Gaps for the reverse-sweep state R arriving at segment `rank` from the right: segment
    i > rank is preceded by the tokens of segments rank+1 .. i-1 (-1: not included)."""
    return [sum(lens[rank + 1:i]) if i > rank else -1 for i in range(len(lens))]


def _decay_ops(ops):
    if ops is None:
        import linear_attention_attn_b200 as ops
    return ops


def decay_forward(q, k, v, o, decay, state_out=None, entering=None, group=None, ops=None, stream=None,
                  workspace=None):
    """The decay op (retention) forward for this rank's segment of a sequence split along T
    (rank r holds the r-th segment).  A segment's output needs the state of every token before
    it: pass 1 gives each segment's own end state E_r from a zero state (a state-only pass, o
    not computed; on rank 0, whose entering state is zero, the whole forward, which is final);
    an all-gather shares the E_r and the segment lengths; la_chunk_decay_scan forms
    S_r = sum_{r' < r} gamma^(tokens between) E_r'; the forward then runs once from S_r.
    state_out (optional, [B, H, D, D] fp32) receives the state after this rank's segment (on the
    last rank: after the whole sequence); entering (optional, same shape) receives S_r, which
    decay_backward needs."""
    import torch
    ops = _decay_ops(ops)
    B, H, T, D = (int(x) for x in k.shape)
    kw = {} if workspace is None else {"workspace": workspace}
    world, rank = _world(group)
    sdt = torch.float32 if k.is_cuda else torch.float64
    end = state_out if state_out is not None else torch.empty((B, H, D, D), dtype=sdt, device=k.device)
    if entering is not None:
        entering.zero_()
    if world == 1 or rank == 0:                    # nothing enters the first segment: this pass is final
        ops.la_chunk_decay_fwd_state(q, k, v, o, decay, state_in=None, state_out=end, stream=stream, **kw)
    else:                                          # this segment's own end state only
        ops.la_chunk_decay_fwd_state(None, k, v, None, decay, state_in=None, state_out=end, stream=stream, **kw)
    if world == 1:
        return state_out
    ends, lens = _gather_states(end, T, group)
    if rank == 0:
        return state_out
    sin = entering if entering is not None else torch.empty_like(end)
    ops.la_chunk_decay_scan(ends, entering_gaps(lens, rank), decay, sin, stream=stream)
    ops.la_chunk_decay_fwd_state(q, k, v, o, decay, state_in=sin, state_out=state_out, stream=stream, **kw)
    return state_out


def decay_backward(q, k, v, dout, decay, dq, dk, dv, entering=None, group=None, ops=None, stream=None,
                   workspace=None):
    """The decay op's backward for this rank's segment, with `entering` the state S_r entering it
    (from decay_forward; None for zero).  dk and dv need R, which arrives from the segments to the
    right: pass 1 gives each segment's own reverse-sweep state F_r at its first token from a zero
    R (a state-only pass; on the last rank, where nothing arrives, the whole backward, which is
    final); an all-gather shares the F_r; la_chunk_decay_scan forms
    R_r = sum_{r' > r} gamma^(tokens between) F_r'; the backward then runs once from S_r and R_r."""
    import torch
    ops = _decay_ops(ops)
    B, H, T, D = (int(x) for x in q.shape)
    kw = {} if workspace is None else {"workspace": workspace}
    world, rank = _world(group)
    f = torch.empty((B, H, D, D), dtype=torch.float32 if q.is_cuda else torch.float64, device=q.device)
    if rank == world - 1:                          # nothing arrives after the last segment: final
        ops.la_chunk_decay_bwd_state(q, k, v, dout, decay, dq, dk, dv, state_in=entering, dstate_in=None,
                                     dstate_out=f, stream=stream, **kw)
    else:                                          # this segment's own R at its first token only
        ops.la_chunk_decay_bwd_state(q, None, None, dout, decay, None, None, None, dstate_out=f, stream=stream,
                                     **kw)
    if world == 1:
        return
    fs, lens = _gather_states(f, T, group)
    if rank == world - 1:
        return
    rin = torch.empty_like(f)
    ops.la_chunk_decay_scan(fs, leaving_gaps(lens, rank), decay, rin, stream=stream)
    ops.la_chunk_decay_bwd_state(q, k, v, dout, decay, dq, dk, dv, state_in=entering, dstate_in=rin,
                                 stream=stream, **kw)
