"""GPU parity of the state-form stages used for a sequence split along T, through the C ABI:
one shard reproduces the fused ops bit for bit; several uneven shards, with their states
summed in between, match the fp64 oracle on the whole sequence."""
import pytest
import torch

import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

CASES = [   # op, dtype, B, H, T, D: tensor-core (fp16 / bf16, D = 64) and CUDA-core paths
    ("bidir", "f16", 2, 4, 1000, 64),
    ("simple", "bf16", 2, 3, 700, 64),
    ("bidir", "bf16", 1, 3, 513, 64),
    ("bidir", "f32", 1, 2, 300, 64),
    ("simple", "f16", 1, 2, 300, 128),
]


def _workload(op, dtype, B, H, T, D):
    sc = (0.5, 0.5, 0.5) if op == "bidir" else (D ** -0.5, D ** -0.5, 1.0)
    return synth.Workload("case", op, B, H, T, D, dtype, eps=1e-6, q_scale=sc[0], k_scale=sc[1], v_scale=sc[2])


def _stages(la, op, shards, eps):
    """Reduce per shard, sum (in shard order), apply per shard; then the backward likewise."""
    feature = "elu1" if op == "bidir" else "identity"
    q0 = shards[0]["q"]
    B, H, _, D = q0.shape
    dev = q0.device
    states = []
    for sh in shards:
        st = torch.empty((B, H, D, D + 1), dtype=torch.float32, device=dev)
        la.la_state_reduce(sh["k"], sh["v"], st, feature=feature)
        states.append(st)
    state = states[0].clone()
    for st in states[1:]:
        state += st
    outs = {"o": [], "dq": [], "dk": [], "dv": []}
    for sh in shards:
        o = torch.empty_like(sh["q"])
        la.la_state_apply(sh["q"], state, o, feature=feature, eps=eps)
        outs["o"].append(o)
    dstates = []
    for sh in shards:
        dq = torch.empty_like(sh["q"])
        ds = torch.empty_like(state)
        la.la_state_bwd_q(sh["q"], sh["do"], state, dq, ds, feature=feature, eps=eps)
        outs["dq"].append(dq)
        dstates.append(ds)
    dstate = dstates[0].clone()
    for ds in dstates[1:]:
        dstate += ds
    for sh in shards:
        dk, dv = torch.empty_like(sh["k"]), torch.empty_like(sh["v"])
        la.la_state_bwd_kv(sh["k"], sh["v"], dstate, dk, dv, feature=feature)
        outs["dk"].append(dk)
        outs["dv"].append(dv)
    torch.cuda.synchronize()
    res = {n: torch.cat(v, dim=2).cpu() for n, v in outs.items()}
    res["state"] = state.cpu()
    return res


def _split(inp, cuts, dev):
    return [{n: inp[n][:, :, a:b].contiguous().to(dev) for n in ("q", "k", "v", "do")}
            for a, b in zip(cuts[:-1], cuts[1:])]


@pytest.mark.parametrize("op,dtype,B,H,T,D", CASES, ids=lambda x: str(x))
def test_one_shard_is_the_fused_op(op, dtype, B, H, T, D):
    import linear_attention_attn_b200 as la
    w = _workload(op, dtype, B, H, T, D)
    inp = synth.make_inputs(w, seed=1, with_grad=True)
    dev = torch.device("cuda", 0)
    got = _stages(la, op, _split(inp, [0, T], dev), w.eps)
    fused = pu.gpu_run(op, inp, eps=w.eps)
    for n in ("o", "dq", "dk", "dv", "state"):
        assert torch.equal(got[n], fused[n]), n


@pytest.mark.parametrize("op,dtype,B,H,T,D", CASES, ids=lambda x: str(x))
def test_uneven_shards_match_oracle(op, dtype, B, H, T, D):
    import linear_attention_attn_b200 as la
    w = _workload(op, dtype, B, H, T, D)
    inp = synth.make_inputs(w, seed=2, with_grad=True)
    dev = torch.device("cuda", 0)
    cuts = [0, T // 3, T // 3 + 129, T]            # three shards, one of them 129 tokens
    got = _stages(la, op, _split(inp, cuts, dev), w.eps)
    pu.compare(op, got, pu.oracle_run(op, inp, eps=w.eps))


def test_empty_shard_reduces_to_zero():
    import linear_attention_attn_b200 as la
    dev = torch.device("cuda", 0)
    k = torch.empty((1, 2, 0, 64), dtype=torch.float16, device=dev)
    st = torch.full((1, 2, 64, 65), 7.0, device=dev)
    la.la_state_reduce(k, k, st, feature="elu1")
    torch.cuda.synchronize()
    assert torch.count_nonzero(st).item() == 0
