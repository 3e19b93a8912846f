"""Sequence parallelism on CPU: two gloo ranks each hold half of a sequence and run
linear_attention_attn_b200.seqpar with a float64 torch implementation of the four stages
(written here from their definitions); the shards' outputs and gradients must equal the
oracle's on the whole sequence.  This checks the split (local reduce, all-reduce, local
apply; local dq pass, all-reduce of (dS | dz), local dk, dv pass) and the collective plumbing."""
import os
import socket
import sys
import types

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _phi(x, feature):
    return torch.where(x > 0, x + 1.0, torch.exp(torch.clamp(x, max=0.0))) if feature == "elu1" else x


def _dphi(x, feature):
    return torch.where(x > 0, torch.ones_like(x), torch.exp(torch.clamp(x, max=0.0))) if feature == "elu1" \
        else torch.ones_like(x)


def _stages():
    """The four stages on float64 CPU tensors, from the formulas of include/la.h."""
    def la_state_reduce(k, v, state, feature="elu1", stream=None):
        D = k.shape[-1]
        fk = _phi(k, feature)
        state[..., :D] = torch.einsum("bhti,bhtj->bhij", fk, v)
        state[..., D] = fk.sum(2) if feature == "elu1" else 0.0

    def la_state_apply(q, state, o, feature="elu1", eps=1e-6, stream=None):
        D = q.shape[-1]
        fq = _phi(q, feature)
        u = torch.einsum("bhti,bhij->bhtj", fq, state[..., :D])
        if feature == "elu1":
            u = u / (torch.einsum("bhti,bhi->bht", fq, state[..., D]) + eps)[..., None]
        o.copy_(u)

    def la_state_bwd_q(q, dout, state, dq, dstate, feature="elu1", eps=1e-6, stream=None):
        D = q.shape[-1]
        S, z = state[..., :D], state[..., D]
        fq = _phi(q, feature)
        gs = torch.einsum("bhtj,bhij->bhti", dout, S)                 # dout S^T
        if feature == "elu1":
            n = torch.einsum("bhti,bhi->bht", fq, z) + eps
            o = torch.einsum("bhti,bhij->bhtj", fq, S) / n[..., None]
            go = (dout * o).sum(-1)
            dq.copy_((gs - go[..., None] * z[:, :, None, :]) / n[..., None] * _dphi(q, feature))
            dstate[..., :D] = torch.einsum("bhti,bhtj->bhij", fq, dout / n[..., None])
            dstate[..., D] = -torch.einsum("bhti,bht->bhi", fq, go / n)
        else:
            dq.copy_(gs)
            dstate[..., :D] = torch.einsum("bhti,bhtj->bhij", q, dout)
            dstate[..., D] = 0.0

    def la_state_bwd_kv(k, v, dstate, dk, dv, feature="elu1", stream=None):
        D = k.shape[-1]
        dS, dz = dstate[..., :D], dstate[..., D]
        dk.copy_((torch.einsum("bhsj,bhij->bhsi", v, dS) + dz[:, :, None, :]) * _dphi(k, feature))
        dv.copy_(torch.einsum("bhsi,bhij->bhsj", _phi(k, feature), dS))

    return types.SimpleNamespace(la_state_reduce=la_state_reduce, la_state_apply=la_state_apply,
                                 la_state_bwd_q=la_state_bwd_q, la_state_bwd_kv=la_state_bwd_kv)


def _inputs(B, H, T, D):
    g = torch.Generator().manual_seed(7)
    return [torch.randn(B, H, T, D, generator=g, dtype=torch.float64) * s for s in (0.5, 0.5, 1.0, 1.0)]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, feature, cuts, out):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from linear_attention_attn_b200 import seqpar
    B, H, T, D = 2, 3, cuts[-1], 8
    q, k, v, g = _inputs(B, H, T, D)
    sl = slice(cuts[rank], cuts[rank + 1])
    qs, ks, vs, gs = (x[:, :, sl].contiguous() for x in (q, k, v, g))
    ops = _stages()
    state = torch.empty(B, H, D, D + 1, dtype=torch.float64)
    o = torch.empty_like(qs)
    seqpar.forward(qs, ks, vs, o, state, feature=feature, eps=1e-3, ops=ops)
    dq, dk, dv = torch.empty_like(qs), torch.empty_like(qs), torch.empty_like(qs)
    dstate = torch.empty_like(state)
    seqpar.backward(qs, ks, vs, gs, state, dq, dk, dv, dstate, feature=feature, eps=1e-3, ops=ops)
    out[rank] = [t.numpy() for t in (o, dq, dk, dv)]
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("feature", ["elu1", "identity"])
def test_two_ranks_match_the_whole_sequence(feature):
    import oracle
    cuts = [0, 11, 30]                    # uneven shards
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, feature, cuts, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    q, k, v, g = (x.numpy() for x in _inputs(2, 3, cuts[-1], 8))
    if feature == "elu1":
        want = [oracle.bidir_fwd(q, k, v, eps=1e-3)] + list(oracle.bidir_bwd(q, k, v, g, eps=1e-3))
    else:
        want = [oracle.simple_fwd(q, k, v)] + list(oracle.simple_bwd(q, k, v, g))
    for i, name in enumerate(("o", "dq", "dk", "dv")):
        got = np.concatenate([out[0][i], out[1][i]], axis=2)
        np.testing.assert_allclose(got, want[i], rtol=1e-10, atol=1e-12, err_msg=name)


def _decay_ops(calls):
    """The decay op's segment calls on float64 CPU tensors, from their definitions in
    include/la.h: the recurrent form forwards (S) and backwards (R), the state-only forms (o, or
    dq, dk and dv, None), and the combine.  `calls` records which form each call took."""
    def gam4(decay):
        return torch.as_tensor(list(decay), dtype=torch.float64)[None, :, None, None]

    def la_chunk_decay_fwd_state(q, k, v, o, decay, state_in=None, state_out=None, stream=None):
        calls.append("fwd" if o is not None else "fwd_state")
        B, H, T, D = k.shape
        g = gam4(decay)
        S = state_in.clone() if state_in is not None else torch.zeros(B, H, D, D, dtype=torch.float64)
        for t in range(T):
            S = g * S + torch.einsum("bhi,bhj->bhij", k[:, :, t], v[:, :, t])
            if o is not None:
                o[:, :, t] = torch.einsum("bhi,bhij->bhj", q[:, :, t], S)
        if state_out is not None:
            state_out.copy_(S)

    def la_chunk_decay_bwd_state(q, k, v, dout, decay, dq, dk, dv, state_in=None, dstate_in=None,
                                 dstate_out=None, stream=None):
        sonly = dq is None and dk is None and dv is None
        calls.append("bwd_state" if sonly else "bwd")
        B, H, T, D = q.shape
        g = gam4(decay)
        if dq is not None:
            S = state_in.clone() if state_in is not None else torch.zeros(B, H, D, D, dtype=torch.float64)
            for t in range(T):
                S = g * S + torch.einsum("bhi,bhj->bhij", k[:, :, t], v[:, :, t])
                dq[:, :, t] = torch.einsum("bhij,bhj->bhi", S, dout[:, :, t])
        R = dstate_in.clone() if dstate_in is not None else torch.zeros(B, H, D, D, dtype=torch.float64)
        for s in reversed(range(T)):
            R = g * R + torch.einsum("bhi,bhj->bhij", q[:, :, s], dout[:, :, s])
            if not sonly:
                dk[:, :, s] = torch.einsum("bhij,bhj->bhi", R, v[:, :, s])
                dv[:, :, s] = torch.einsum("bhi,bhij->bhj", k[:, :, s], R)
        if dstate_out is not None:
            dstate_out.copy_(R)

    def la_chunk_decay_scan(states, gaps, decay, out, stream=None):
        g = gam4(decay)
        acc = torch.zeros_like(out)
        for i, gap in enumerate(gaps):
            if gap >= 0:
                acc += g ** gap * states[i]
        out.copy_(acc)

    return types.SimpleNamespace(la_chunk_decay_fwd_state=la_chunk_decay_fwd_state,
                                 la_chunk_decay_bwd_state=la_chunk_decay_bwd_state,
                                 la_chunk_decay_scan=la_chunk_decay_scan)


def _decay_rank_main(rank, world, port, cuts, gam, out):
    sys.path.insert(0, ROOT)
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    from linear_attention_attn_b200 import seqpar
    q, k, v, g = _inputs(2, 3, cuts[-1], 6)
    sl = slice(cuts[rank], cuts[rank + 1])
    qs, ks, vs, gs = (x[:, :, sl].contiguous() for x in (q, k, v, g))
    o = torch.empty_like(qs)
    st = torch.empty(2, 3, 6, 6, dtype=torch.float64)
    ent = torch.empty_like(st)
    calls = []
    ops = _decay_ops(calls)
    seqpar.decay_forward(qs, ks, vs, o, gam, state_out=st, entering=ent, ops=ops)
    dq, dk, dv = (torch.empty_like(qs) for _ in range(3))
    seqpar.decay_backward(qs, ks, vs, gs, gam, dq, dk, dv, entering=ent, ops=ops)
    out[rank] = (o.numpy(), st.numpy(), dq.numpy(), dk.numpy(), dv.numpy(), list(calls))
    dist.barrier()
    dist.destroy_process_group()


def test_segment_gaps():
    from linear_attention_attn_b200 import seqpar
    lens = [5, 7, 0, 4]
    assert seqpar.entering_gaps(lens, 0) == [-1, -1, -1, -1]
    assert seqpar.entering_gaps(lens, 3) == [7, 0, 0, -1]
    assert seqpar.leaving_gaps(lens, 0) == [-1, 0, 7, 7]
    assert seqpar.leaving_gaps(lens, 3) == [-1, -1, -1, -1]


def test_decay_forward_and_backward_over_three_ranks():
    import oracle
    cuts = [0, 7, 19, 30]
    gam = [0.6, 0.9, 1.0]
    ctx = mp.get_context("spawn")
    out = ctx.Manager().dict()
    port = _free_port()
    procs = [ctx.Process(target=_decay_rank_main, args=(r, 3, port, cuts, gam, out)) for r in range(3)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    q, k, v, g = (x.numpy() for x in _inputs(2, 3, cuts[-1], 6))
    want_o, want_s = oracle.retention_fwd_state(q, k, v, np.array(gam))
    got = np.concatenate([out[r][0] for r in range(3)], axis=2)
    np.testing.assert_allclose(got, want_o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out[2][1], want_s, rtol=1e-10, atol=1e-12)    # the last rank: whole sequence
    want = oracle.retention_bwd(q, k, v, g, np.array(gam))
    for i, name in enumerate(("dq", "dk", "dv")):
        got = np.concatenate([out[r][2 + i] for r in range(3)], axis=2)
        np.testing.assert_allclose(got, want[i], rtol=1e-10, atol=1e-12, err_msg=name)
    # each rank runs the whole forward and the whole backward once; a state-only pass
    # precedes them where the neighbours' states are needed
    assert out[0][5] == ["fwd", "bwd_state", "bwd"]
    assert out[1][5] == ["fwd_state", "fwd", "bwd_state", "bwd"]
    assert out[2][5] == ["fwd_state", "fwd", "bwd"]
