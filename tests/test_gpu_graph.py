"""The library's calls can be captured into a CUDA graph (workspace passed in, explicit stream)
and replayed: the replay reproduces the eager results bit for bit."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("op", ["bidir", "simple", "retention"])
def test_graph_replay_matches_eager(op):
    import linear_attention_attn_b200 as la
    dev = torch.device("cuda", 0)
    if op == "retention":
        w = synth.Workload("case", op, 1, 4, 300, 128, "bf16", q_scale=128 ** -0.5)
    else:
        w = synth.Workload("case", op, 2, 3, 1000, 64, "f16" if op == "bidir" else "bf16",
                           q_scale=0.5, k_scale=0.5, v_scale=0.5)
    inp = synth.make_inputs(w, seed=4, with_grad=True)
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    st = torch.empty((w.B, w.H, w.D, w.D + 1), dtype=torch.float32, device=dev)
    names = {"bidir": ("bidir_fwd", "bidir_bwd"), "simple": ("simple_fwd", "simple_bwd"),
             "retention": ("chunk_decay_fwd", "chunk_decay_bwd")}[op]
    nws = max(la.la_workspace_size(n, w.B, w.H, w.T, w.D, q.dtype) for n in names)
    ws = torch.empty(max(256, nws), dtype=torch.uint8, device=dev)
    s = torch.cuda.Stream(dev)
    s.wait_stream(torch.cuda.current_stream(dev))

    def step():
        if op == "bidir":
            la.la_bidir_fwd(q, k, v, o, st, eps=w.eps, workspace=ws, stream=s)
            la.la_bidir_bwd(q, k, v, g, dq, dk, dv, st, eps=w.eps, workspace=ws, stream=s)
        elif op == "simple":
            la.la_simple_fwd(q, k, v, o, st, workspace=ws, stream=s)
            la.la_simple_bwd(q, k, v, g, dq, dk, dv, st, workspace=ws, stream=s)
        else:
            la.la_chunk_decay_fwd(q, k, v, o, inp["gamma"], workspace=ws, stream=s)
            la.la_chunk_decay_bwd(q, k, v, g, inp["gamma"], dq, dk, dv, workspace=ws, stream=s)

    step()
    torch.cuda.synchronize(dev)
    eager = [t.clone() for t in (o, dq, dk, dv)]
    for t in (o, dq, dk, dv):
        t.zero_()
    torch.cuda.synchronize(dev)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        step()
    with torch.cuda.stream(s):
        graph.replay()
    torch.cuda.synchronize(dev)
    for a, b in zip(eager, (o, dq, dk, dv)):
        assert torch.equal(a, b)
    del graph
