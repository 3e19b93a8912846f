"""GPU parity of the recurrent (decode) step and of plain causal linear attention (the decay
op at gamma = 1), through the C ABI, against the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

STATE_REL_L2 = 1e-5     # the state is carried in fp32 on both sides' inputs; fp32 vs fp64 rounding only


def _rel_l2(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f16", 64), ("f32", 128), ("bf16", 64)])
def test_decode_steps_match_oracle(dtype, D):
    """Three chained steps from a random fp32 state: every output and the final state."""
    import linear_attention_attn_b200 as la
    B, H, steps = 3, 5, 3
    dt = synth.DTYPES[dtype]
    dev = torch.device("cuda", 0)
    gam = synth.retention_gammas(H)
    state0 = synth.normal((B, H, D, D), 7, 0) * (D ** -0.5)
    st_gpu = state0.clone().to(dev)
    st_ref = state0.double().numpy()
    for t in range(steps):
        q, k, v = (synth.normal((B, H, D), 11 + t, i).mul(s).to(dt) for i, s in enumerate((D ** -0.5, 1.0, 1.0)))
        o = torch.empty((B, H, D), dtype=dt, device=dev)
        la.la_chunk_decay_step(q.to(dev), k.to(dev), v.to(dev), o, st_gpu, gam)
        o_ref, st_ref = oracle.retention_step(q.double().numpy(), k.double().numpy(), v.double().numpy(),
                                              gam.double().numpy(), st_ref)
        torch.cuda.synchronize()
        pu.assert_fwd(o, o_ref, "decode step %d o" % t)
    assert _rel_l2(st_gpu.cpu().numpy(), st_ref) <= STATE_REL_L2


def test_decode_continues_the_chunked_op():
    """State of a T-token prefix (oracle, fp32) + one GPU step == the last output of the op on T+1 tokens."""
    import linear_attention_attn_b200 as la
    w = synth.Workload("case", "retention", 2, 4, 201, 128, "bf16", q_scale=128 ** -0.5)
    inp = synth.make_inputs(w, seed=3, with_grad=False)
    q, k, v, gam = (inp[n] for n in ("q", "k", "v", "gamma"))
    T = w.T - 1
    g64 = gam.double().numpy()
    wts = g64[None, :, None] ** (T - 1 - np.arange(T))[None, None, :]
    kk, vv = k[:, :, :T].double().numpy(), v[:, :, :T].double().numpy()
    prefix = np.einsum("bhs,bhsi,bhsj->bhij", wts, kk, vv)
    dev = torch.device("cuda", 0)
    st = torch.from_numpy(prefix).float().to(dev)
    o = torch.empty((w.B, w.H, w.D), dtype=q.dtype, device=dev)
    la.la_chunk_decay_step(q[:, :, T].contiguous().to(dev), k[:, :, T].contiguous().to(dev),
                           v[:, :, T].contiguous().to(dev), o, st, gam)
    torch.cuda.synchronize()
    full = oracle.retention_fwd(q, k, v, gam)
    pu.assert_fwd(o, full[:, :, T], "step after a prefix")


@pytest.mark.parametrize("dtype,D,T", [("bf16", 128, 300), ("bf16", 128, 1000), ("f16", 64, 257)])
def test_plain_causal_linear_attention(dtype, D, T):
    """gamma = 1: o_t = q_t sum_{s<=t} k_s^T v_s (plain causal linear attention), fwd and bwd."""
    w = synth.Workload("case", "retention", 2, 3, T, D, dtype, q_scale=D ** -0.5, k_scale=D ** -0.5)
    inp = synth.make_inputs(w, seed=5, with_grad=True)
    inp["gamma"] = torch.ones(w.H, dtype=torch.float32)
    got = pu.gpu_run("retention", inp)
    pu.compare("retention", got, pu.oracle_run("retention", inp))


def test_decode_rejects_bad_state_shape():
    import linear_attention_attn_b200 as la
    dev = torch.device("cuda", 0)
    q = torch.zeros((1, 2, 64), dtype=torch.bfloat16, device=dev)
    with pytest.raises(ValueError):
        la.la_chunk_decay_step(q, q, q, torch.empty_like(q), torch.zeros((1, 2, 64, 65), device=dev), [0.5, 0.5])


@pytest.mark.parametrize("dtype,D", [("bf16", 128), ("f16", 64), ("f32", 128)])
def test_forward_from_a_state(dtype, D):
    """A random entering state: outputs and the state after the sequence against the oracle."""
    import linear_attention_attn_b200 as la
    w = synth.Workload("case", "retention", 2, 3, 300, D, dtype, q_scale=D ** -0.5)
    inp = synth.make_inputs(w, seed=6, with_grad=False)
    dev = torch.device("cuda", 0)
    sin = synth.normal((w.B, w.H, D, D), 8, 0) * (D ** -0.5)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    sout = torch.empty_like(sin, device=dev)
    la.la_chunk_decay_fwd_state(q, k, v, o, inp["gamma"], state_in=sin.to(dev), state_out=sout)
    torch.cuda.synchronize()
    o_ref, s_ref = oracle.retention_fwd_state(inp["q"], inp["k"], inp["v"], inp["gamma"], sin.double().numpy())
    pu.assert_fwd(o, o_ref, "o from a state")
    assert _rel_l2(sout.cpu().numpy(), s_ref) <= 2e-3


def test_segments_chained_through_the_state():
    """Two segments of one sequence, the second starting from the first's state (the same
    buffer in and out), match the op on the whole sequence."""
    import linear_attention_attn_b200 as la
    w = synth.Workload("case", "retention", 2, 4, 700, 128, "bf16", q_scale=128 ** -0.5)
    inp = synth.make_inputs(w, seed=9, with_grad=False)
    dev = torch.device("cuda", 0)
    cut = 257
    st = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)
    outs = []
    for a, b, sin in ((0, cut, None), (cut, w.T, st)):
        q, k, v = (inp[n][:, :, a:b].contiguous().to(dev) for n in ("q", "k", "v"))
        o = torch.empty_like(q)
        la.la_chunk_decay_fwd_state(q, k, v, o, inp["gamma"], state_in=sin, state_out=st)
        outs.append(o)
    torch.cuda.synchronize()
    got = torch.cat(outs, dim=2)
    pu.assert_fwd(got, oracle.retention_fwd(inp["q"], inp["k"], inp["v"], inp["gamma"]), "two segments")


def test_prefill_then_decode():
    """Chunked prefill of T tokens hands its state to the decode step for token T + 1."""
    import linear_attention_attn_b200 as la
    w = synth.Workload("case", "retention", 2, 4, 401, 128, "bf16", q_scale=128 ** -0.5)
    inp = synth.make_inputs(w, seed=10, with_grad=False)
    dev = torch.device("cuda", 0)
    T = w.T - 1
    q, k, v = (inp[n][:, :, :T].contiguous().to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    st = torch.empty((w.B, w.H, w.D, w.D), dtype=torch.float32, device=dev)
    la.la_chunk_decay_fwd_state(q, k, v, o, inp["gamma"], state_out=st)
    o1 = torch.empty((w.B, w.H, w.D), dtype=q.dtype, device=dev)
    la.la_chunk_decay_step(*(inp[n][:, :, T].contiguous().to(dev) for n in ("q", "k", "v")), o1, st, inp["gamma"])
    torch.cuda.synchronize()
    full = oracle.retention_fwd(inp["q"], inp["k"], inp["v"], inp["gamma"])
    pu.assert_fwd(o, full[:, :, :T], "prefill")
    pu.assert_fwd(o1, full[:, :, T], "decode after prefill")
