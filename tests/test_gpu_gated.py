"""GPU parity of gated linear attention (la_gated_*), through the C ABI, against the fp64 oracle:
every dtype, D = 64 and 128, lengths of one chunk (256 tokens) and of several, whole or ragged;
constant gates against the decay op; sampled heads at the benchmark size."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def _inputs(dtype, B, H, T, D, seed):
    """q ~ N(0,1) D^-1/2, k, v, dO ~ N(0,1); log gates g = log(sigmoid(N(0,1))) / 16 (about -0.04,
    a per-token decay near 0.96 in every key dimension), all rounded to the storage dtype."""
    dt = synth.DTYPES[dtype]
    n = lambda s, scale=1.0: (synth.normal((B, H, T, D), seed, s) * scale).to(dt).contiguous()
    g = (torch.nn.functional.logsigmoid(synth.normal((B, H, T, D), seed, 4)) / 16.0).to(dt).contiguous()
    return {"q": n(0, D ** -0.5), "k": n(1), "v": n(2), "do": n(3), "g": g}


def _run(inp):
    import linear_attention_attn_b200 as la
    dev = _dev()
    q, k, v, g, do = (inp[n].to(dev) for n in ("q", "k", "v", "g", "do"))
    o, dq, dk, dv, dg = (torch.empty_like(q) for _ in range(5))
    la.la_gated_fwd(q, k, v, g, o)
    la.la_gated_bwd(q, k, v, g, do, dq, dk, dv, dg)
    torch.cuda.synchronize()
    return [t.cpu().double().numpy() for t in (o, dq, dk, dv, dg)]


def _ref(inp):
    a = [inp[n].double().numpy() for n in ("q", "k", "v", "g", "do")]
    return [oracle.gated_fwd(*a[:4])] + list(oracle.gated_bwd(*a))


@pytest.mark.parametrize("dtype,D,T", [("bf16", 64, 300), ("f16", 128, 300), ("f32", 64, 37), ("f32", 128, 129),
                                       ("bf16", 128, 2), ("bf16", 64, 1024), ("f16", 64, 517), ("f32", 128, 512)])
def test_matches_oracle(dtype, D, T):
    inp = _inputs(dtype, 2, 3, T, D, seed=61)
    got, want = _run(inp), _ref(inp)
    pu.assert_fwd(got[0], want[0], "o", dtype=inp["q"].dtype)
    for name, a, b in zip(("dq", "dk", "dv", "dg"), got[1:], want[1:]):
        pu.assert_grad(a, b, name)


def test_constant_gates_are_the_decay_op():
    """g_t = log gamma_h everywhere: la_gated_fwd equals la_chunk_decay_fwd (CUDA-core path, f32)."""
    import linear_attention_attn_b200 as la
    B, H, T, D = 2, 3, 600, 64
    inp = _inputs("f32", B, H, T, D, seed=62)
    gam = [0.5, 0.9, 0.999]
    g = torch.log(torch.tensor(gam, dtype=torch.float32))[None, :, None, None].expand(B, H, T, D).contiguous()
    dev = _dev()
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    o1, o2 = torch.empty_like(q), torch.empty_like(q)
    la.la_gated_fwd(q, k, v, g.to(dev), o1)
    la.la_chunk_decay_fwd(q, k, v, o2, gam)
    torch.cuda.synchronize()
    a, b = o1.cpu().double().numpy(), o2.cpu().double().numpy()
    assert np.linalg.norm(a - b) / np.linalg.norm(b) < 1e-5


def test_benchmark_size_sampled_heads():
    """B8 H16 T4096 D64 bf16 (the benchmark's gated workload): three heads against the oracle."""
    inp = _inputs("bf16", 8, 16, 4096, 64, seed=0)
    got = _run(inp)
    for b, h in ((0, 0), (4, 9), (7, 15)):
        sel = {n: inp[n][b:b + 1, h:h + 1] for n in inp}
        want = _ref(sel)
        pu.assert_fwd(got[0][b:b + 1, h:h + 1], want[0], "o (%d,%d)" % (b, h), dtype=inp["q"].dtype)
        for name, a, r in zip(("dq", "dk", "dv", "dg"), got[1:], want[1:]):
            pu.assert_grad(a[b:b + 1, h:h + 1], r, "%s (%d,%d)" % (name, b, h))


def test_deterministic_and_empty():
    import linear_attention_attn_b200 as la
    inp = _inputs("bf16", 1, 2, 333, 64, seed=63)
    a, b = _run(inp), _run(inp)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
    z = torch.empty((1, 2, 0, 64), dtype=torch.bfloat16, device=_dev())
    la.la_gated_fwd(z, z, z, z, z)
    la.la_gated_bwd(z, z, z, z, z, z, z, z, z)
    torch.cuda.synchronize()
