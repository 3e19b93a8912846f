"""GPU parity of the decay op (retention) over segments of one sequence, through the C ABI,
against the fp64 oracle: the backward of one segment given the state of the tokens before it
(S_in) and the reverse-sweep state of the tokens after it (R_in), and whole sequences cut into
ragged segments and chained through S (forwards) and R (backwards)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

STATE_REL_L2 = 5e-3     # R_0 is a sum of T products of 16-bit inputs in fp32: the gradients' bound


def _rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _dev():
    return torch.device("cuda", 0)


@pytest.mark.parametrize("dtype,D,T", [("bf16", 128, 300), ("bf16", 128, 37), ("bf16", 128, 128),
                                       ("f16", 64, 300), ("f32", 128, 300), ("bf16", 64, 77)])
def test_backward_of_a_segment(dtype, D, T):
    """Random S_in and R_in: dq, dk, dv and R_0 against the oracle.  T = 37 is one partial chunk,
    the first one the backward sweep visits; 300 ends in a partial chunk of 44 rows."""
    import linear_attention_attn_b200 as la
    w = synth.Workload("case", "retention", 2, 3, T, D, dtype, q_scale=D ** -0.5)
    inp = synth.make_inputs(w, seed=21, with_grad=True)
    dev = _dev()
    sin = synth.normal((w.B, w.H, D, D), 22, 0) * 4.0
    rin = synth.normal((w.B, w.H, D, D), 22, 1) * 4.0 * D ** -0.5
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
    rout = torch.empty((w.B, w.H, D, D), dtype=torch.float32, device=dev)
    la.la_chunk_decay_bwd_state(q, k, v, g, inp["gamma"], dq, dk, dv, state_in=sin.to(dev), dstate_in=rin.to(dev),
                                dstate_out=rout)
    torch.cuda.synchronize()
    ref = oracle.retention_bwd_state(inp["q"], inp["k"], inp["v"], inp["do"], inp["gamma"], sin.double().numpy(),
                                     rin.double().numpy())
    for name, got, want in zip(("dq", "dk", "dv"), (dq, dk, dv), ref[:3]):
        pu.assert_grad(got.cpu().double().numpy(), want, "segment %s" % name)
    assert _rel_l2(rout.cpu().numpy(), ref[3]) <= STATE_REL_L2


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("bf16", 64), ("f32", 64)])
def test_segments_chained_forwards_and_backwards(dtype, D):
    """One sequence of 700 tokens cut at 257 and 513: the forward hands S from segment to segment,
    the backward runs last segment first and hands R back; the concatenated outputs and gradients
    match the op on the whole sequence."""
    import linear_attention_attn_b200 as la
    w = synth.Workload("case", "retention", 2, 4, 700, D, dtype, q_scale=D ** -0.5)
    inp = synth.make_inputs(w, seed=23, with_grad=True)
    dev = _dev()
    cuts = [0, 257, 513, w.T]
    segs = [{n: inp[n][:, :, a:b].contiguous().to(dev) for n in ("q", "k", "v", "do")}
            for a, b in zip(cuts[:-1], cuts[1:])]
    states = []                                   # S entering each segment
    st = None
    outs = []
    for s in segs:
        states.append(st)
        o = torch.empty_like(s["q"])
        nxt = torch.empty((w.B, w.H, D, D), dtype=torch.float32, device=dev)
        la.la_chunk_decay_fwd_state(s["q"], s["k"], s["v"], o, inp["gamma"], state_in=st, state_out=nxt)
        outs.append(o)
        st = nxt
    grads = [None] * len(segs)
    r = None
    for i in reversed(range(len(segs))):
        s = segs[i]
        dq, dk, dv = (torch.empty_like(s["q"]) for _ in range(3))
        rout = torch.empty((w.B, w.H, D, D), dtype=torch.float32, device=dev)
        la.la_chunk_decay_bwd_state(s["q"], s["k"], s["v"], s["do"], inp["gamma"], dq, dk, dv,
                                    state_in=states[i], dstate_in=r, dstate_out=rout)
        grads[i] = (dq, dk, dv)
        r = rout
    torch.cuda.synchronize()
    pu.assert_fwd(torch.cat(outs, dim=2),
                  oracle.retention_fwd(inp["q"], inp["k"], inp["v"], inp["gamma"]), "three segments o")
    whole = oracle.retention_bwd(inp["q"], inp["k"], inp["v"], inp["do"], inp["gamma"])
    for j, name in enumerate(("dq", "dk", "dv")):
        got = torch.cat([gr[j] for gr in grads], dim=2).cpu().double().numpy()
        pu.assert_grad(got, whole[j], "three segments %s" % name)
    # R at the first token of the sequence: sum_t gamma^t q_t^T dO_t
    _, _, _, r0 = oracle.retention_bwd_state(inp["q"], inp["k"], inp["v"], inp["do"], inp["gamma"])
    assert _rel_l2(r.cpu().numpy(), r0) <= STATE_REL_L2


def test_backward_of_an_empty_segment_passes_r_through():
    import linear_attention_attn_b200 as la
    dev = _dev()
    B, H, D = 1, 2, 128
    z = torch.empty((B, H, 0, D), dtype=torch.bfloat16, device=dev)
    rin = torch.randn((B, H, D, D), device=dev)
    rout = torch.full_like(rin, 7.0)
    la.la_chunk_decay_bwd_state(z, z, z, z, [0.5, 0.9], z, z, z, dstate_in=rin, dstate_out=rout)
    torch.cuda.synchronize()
    assert torch.equal(rout, rin)
    la.la_chunk_decay_bwd_state(z, z, z, z, [0.5, 0.9], z, z, z, dstate_out=rout)
    torch.cuda.synchronize()
    assert torch.count_nonzero(rout).item() == 0


def test_backward_segment_is_deterministic():
    """Two runs of the tensor-core backward from the same states give the same bits."""
    import linear_attention_attn_b200 as la
    w = synth.Workload("case", "retention", 2, 3, 333, 128, "bf16", q_scale=128 ** -0.5)
    inp = synth.make_inputs(w, seed=24, with_grad=True)
    dev = _dev()
    sin = (synth.normal((w.B, w.H, 128, 128), 25, 0) * 4.0).to(dev)
    rin = (synth.normal((w.B, w.H, 128, 128), 25, 1) * 0.3).to(dev)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    runs = []
    for _ in range(2):
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        rout = torch.empty_like(sin)
        la.la_chunk_decay_bwd_state(q, k, v, g, inp["gamma"], dq, dk, dv, state_in=sin, dstate_in=rin,
                                    dstate_out=rout)
        runs.append((dq, dk, dv, rout))
    torch.cuda.synchronize()
    for a, b in zip(*runs):
        assert torch.equal(a, b)


def test_scan_matches_its_definition():
    """out = sum_i gamma^gap_i states[i] over gap_i >= 0, in fp32, against the sum in float64."""
    import linear_attention_attn_b200 as la
    dev = _dev()
    n, B, H, D = 5, 2, 4, 128
    states = synth.normal((n, B, H, D, D), 26, 0)
    gaps = [3, -1, 0, 1000, 7]
    gam = [0.5, 0.9, 0.999, 1.0]
    out = torch.empty((B, H, D, D), dtype=torch.float32, device=dev)
    la.la_chunk_decay_scan(states.to(dev), gaps, gam, out)
    torch.cuda.synchronize()
    g = np.asarray(gam, dtype=np.float32).astype(np.float64)[None, :, None, None]
    want = sum(g ** gp * states[i].double().numpy() for i, gp in enumerate(gaps) if gp >= 0)
    assert _rel_l2(out.cpu().numpy(), want) <= 1e-6
    # in place: out may be one of the states
    st = states.to(dev)
    la.la_chunk_decay_scan(st, gaps, gam, st[2])
    torch.cuda.synchronize()
    assert _rel_l2(st[2].cpu().numpy(), want) <= 1e-6


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f16", 64)])
def test_sequence_split_across_emulated_ranks(dtype, D):
    """The steps of seqpar.decay_forward / decay_backward for four ranks, run one rank after
    another on one GPU (the all-gather is a stack): segment end states from a zero state, the
    combine for each rank, the second passes; outputs and gradients match the whole sequence."""
    import linear_attention_attn_b200 as la
    from linear_attention_attn_b200 import seqpar
    w = synth.Workload("case", "retention", 2, 4, 1000, D, dtype, q_scale=D ** -0.5)
    inp = synth.make_inputs(w, seed=27, with_grad=True)
    dev = _dev()
    cuts = [0, 300, 301, 777, w.T]
    W = len(cuts) - 1
    lens = [b - a for a, b in zip(cuts[:-1], cuts[1:])]
    segs = [{n: inp[n][:, :, a:b].contiguous().to(dev) for n in ("q", "k", "v", "do")}
            for a, b in zip(cuts[:-1], cuts[1:])]
    gam = inp["gamma"]
    sshape = (w.B, w.H, D, D)
    ends = torch.empty((W,) + sshape, dtype=torch.float32, device=dev)
    outs = []
    for r, s in enumerate(segs):
        o = torch.empty_like(s["q"])
        la.la_chunk_decay_fwd_state(s["q"], s["k"], s["v"], o, gam, state_out=ends[r])
        outs.append(o)
    entering = [torch.zeros(sshape, dtype=torch.float32, device=dev) for _ in range(W)]
    for r in range(1, W):
        la.la_chunk_decay_scan(ends, seqpar.entering_gaps(lens, r), gam, entering[r])
        s = segs[r]
        la.la_chunk_decay_fwd_state(s["q"], s["k"], s["v"], outs[r], gam, state_in=entering[r])
    fs = torch.empty((W,) + sshape, dtype=torch.float32, device=dev)
    grads = []
    for r, s in enumerate(segs):
        dq, dk, dv = (torch.empty_like(s["q"]) for _ in range(3))
        la.la_chunk_decay_bwd_state(s["q"], s["k"], s["v"], s["do"], gam, dq, dk, dv, state_in=entering[r],
                                    dstate_out=fs[r])
        grads.append((dq, dk, dv))
    for r in range(W - 1):
        rin = torch.empty(sshape, dtype=torch.float32, device=dev)
        la.la_chunk_decay_scan(fs, seqpar.leaving_gaps(lens, r), gam, rin)
        s = segs[r]
        la.la_chunk_decay_bwd_state(s["q"], s["k"], s["v"], s["do"], gam, None, grads[r][1], grads[r][2],
                                    dstate_in=rin)
    torch.cuda.synchronize()
    pu.assert_fwd(torch.cat(outs, dim=2),
                  oracle.retention_fwd(inp["q"], inp["k"], inp["v"], gam), "emulated ranks o")
    whole = oracle.retention_bwd(inp["q"], inp["k"], inp["v"], inp["do"], gam)
    for j, name in enumerate(("dq", "dk", "dv")):
        got = torch.cat([gr[j] for gr in grads], dim=2).cpu().double().numpy()
        pu.assert_grad(got, whole[j], "emulated ranks %s" % name)


@pytest.mark.parametrize("dtype,D,T", [("bf16", 128, 300), ("bf16", 128, 37), ("bf16", 64, 300), ("f32", 64, 300),
                                       ("f16", 128, 129)])
def test_state_only_passes(dtype, D, T):
    """The state-only forms (o None; dq, dk, dv None) give exactly the states of the whole passes
    (the same arithmetic computes them) and the oracle's; q and o, resp. k, v, dq, dk and dv are
    not needed.  bf16 (D = 64 and 128) runs on the tensor cores, the rest on the CUDA cores."""
    import linear_attention_attn_b200 as la
    w = synth.Workload("case", "retention", 2, 3, T, D, dtype, q_scale=D ** -0.5)
    inp = synth.make_inputs(w, seed=25, with_grad=True)
    dev = _dev()
    sin = (synth.normal((w.B, w.H, D, D), 26, 0) * 4.0).to(dev)
    rin = (synth.normal((w.B, w.H, D, D), 26, 1) * 4.0 * D ** -0.5).to(dev)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    gam = inp["gamma"]
    st = lambda: torch.full((w.B, w.H, D, D), float("nan"), dtype=torch.float32, device=dev)
    s_full, s_only, r_full, r_only = st(), st(), st(), st()
    la.la_chunk_decay_fwd_state(q, k, v, torch.empty_like(q), gam, state_in=sin, state_out=s_full)
    la.la_chunk_decay_fwd_state(None, k, v, None, gam, state_in=sin, state_out=s_only)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    la.la_chunk_decay_bwd_state(q, k, v, g, gam, dq, dk, dv, state_in=sin, dstate_in=rin, dstate_out=r_full)
    la.la_chunk_decay_bwd_state(q, None, None, g, gam, None, None, None, dstate_in=rin, dstate_out=r_only)
    torch.cuda.synchronize()
    assert torch.equal(s_only, s_full)
    assert torch.equal(r_only, r_full)
    _, want_s = oracle.retention_fwd_state(inp["q"], inp["k"], inp["v"], gam, sin.double().cpu().numpy())
    want_r = oracle.retention_bwd_state(inp["q"], inp["k"], inp["v"], inp["do"], gam, sin.double().cpu().numpy(),
                                        rin.double().cpu().numpy())[3]
    assert _rel_l2(s_only.cpu().numpy(), want_s) <= STATE_REL_L2
    assert _rel_l2(r_only.cpu().numpy(), want_r) <= STATE_REL_L2


def test_state_only_calls_need_an_output():
    import linear_attention_attn_b200 as la
    dev = _dev()
    k = torch.zeros((1, 1, 64, 128), dtype=torch.bfloat16, device=dev)
    with pytest.raises(la.LAError):
        la.la_chunk_decay_fwd_state(None, k, k, None, [0.9])
    with pytest.raises(la.LAError):
        la.la_chunk_decay_bwd_state(k, None, None, k, [0.9], None, None, None)
