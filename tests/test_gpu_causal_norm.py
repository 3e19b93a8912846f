"""GPU parity of causal linear attention with the norm term (la_causal_norm_*), through the C
ABI, against the fp64 oracle: both feature maps, with and without a per-head decay, every
dtype, D = 64 and 128, lengths of one chunk and of several, whole or with ragged tails; sampled
heads at the benchmark's size.  fp16 and bf16 at D = 64 run on the tensor cores, the rest on the
CUDA cores."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def _inputs(dtype, B, H, T, D, seed, feature):
    """q, k, v ~ 0.5 N(0,1) (the bidirectional recipe); with the identity feature map q and k are
    taken in absolute value, so that f(q) . z stays positive."""
    w = synth.Workload("case", "bidir", B, H, T, D, dtype, q_scale=0.5, k_scale=0.5, v_scale=0.5)
    inp = synth.make_inputs(w, seed=seed, with_grad=True)
    if feature == "identity":
        for n in ("q", "k"):
            inp[n] = inp[n].abs()
    return inp


def _run(inp, decay, feature, eps):
    import linear_attention_attn_b200 as la
    dev = _dev()
    q, k, v, g = (inp[n].to(dev) for n in ("q", "k", "v", "do"))
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    la.la_causal_norm_fwd(q, k, v, o, decay, feature, eps)
    la.la_causal_norm_bwd(q, k, v, g, dq, dk, dv, decay, feature, eps)
    torch.cuda.synchronize()
    return [t.cpu().double().numpy() for t in (o, dq, dk, dv)]


@pytest.mark.parametrize("dtype,D,T", [("f16", 64, 300), ("bf16", 128, 300), ("f32", 64, 37), ("f32", 128, 130),
                                       ("bf16", 64, 2), ("f16", 128, 517), ("f16", 64, 1024), ("bf16", 128, 512),
                                       ("bf16", 64, 700), ("f16", 64, 64), ("f16", 64, 3)])
@pytest.mark.parametrize("feature", ["elu1", "identity"])
@pytest.mark.parametrize("decayed", [False, True])
def test_matches_oracle(dtype, D, T, feature, decayed):
    B, H = 2, 3
    inp = _inputs(dtype, B, H, T, D, seed=41, feature=feature)
    decay = [0.9, 0.99, 1.0] if decayed else None
    eps = 1e-6 if feature == "elu1" else 1e-3
    o, dq, dk, dv = _run(inp, decay, feature, eps)
    want_o = oracle.causal_norm_fwd(inp["q"], inp["k"], inp["v"], decay, feature, eps)
    want = oracle.causal_norm_bwd(inp["q"], inp["k"], inp["v"], inp["do"], decay, feature, eps)
    pu.assert_fwd(o, want_o, "o", dtype=inp["q"].dtype)
    for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
        pu.assert_grad(got, ref, name)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_single_token(dtype):
    """T = 1: o = v a / (a + eps) with a = f(q).f(k), so dq and dk are O(eps) and come out of
    differences of O(1) terms (as in la_bidir_* at T = 1): they are held to an absolute bound of
    1e-3, o and dv to the usual relative ones."""
    inp = _inputs(dtype, 1, 3, 1, 64, seed=44, feature="elu1")
    o, dq, dk, dv = _run(inp, None, "elu1", 1e-6)
    want_o = oracle.causal_norm_fwd(inp["q"], inp["k"], inp["v"], None, "elu1", 1e-6)
    want = oracle.causal_norm_bwd(inp["q"], inp["k"], inp["v"], inp["do"], None, "elu1", 1e-6)
    pu.assert_fwd(o, want_o, "o", dtype=inp["q"].dtype)
    pu.assert_grad(dv, want[2], "dv")
    assert pu.max_abs(dq, want[0]) < 1e-3 and pu.max_abs(dk, want[1]) < 1e-3


def test_benchmark_size_sampled_heads():
    """B8 H16 T4096 D64 fp16 (the benchmark's causal-norm workload): three heads against the oracle."""
    w = synth.WORKLOADS["causal_norm_f16"]
    inp = synth.make_inputs(w, seed=0)
    o, dq, dk, dv = _run(inp, None, "elu1", w.eps)
    for b, h in ((0, 0), (3, 7), (7, 15)):
        sel = {n: inp[n][b:b + 1, h:h + 1] for n in ("q", "k", "v", "do")}
        want_o = oracle.causal_norm_fwd(sel["q"], sel["k"], sel["v"], None, "elu1", w.eps)
        want = oracle.causal_norm_bwd(sel["q"], sel["k"], sel["v"], sel["do"], None, "elu1", w.eps)
        pu.assert_fwd(o[b:b + 1, h:h + 1], want_o, "o (%d,%d)" % (b, h), dtype=inp["q"].dtype)
        for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
            pu.assert_grad(got[b:b + 1, h:h + 1], ref, "%s (%d,%d)" % (name, b, h))


def test_last_row_is_the_bidirectional_output():
    """Without decay the last token sees the whole sequence: its output is la_bidir_fwd's."""
    import linear_attention_attn_b200 as la
    inp = _inputs("f32", 1, 4, 333, 64, seed=42, feature="elu1")
    dev = _dev()
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    o, ob = torch.empty_like(q), torch.empty_like(q)
    la.la_causal_norm_fwd(q, k, v, o, None, "elu1", 1e-6)
    la.la_bidir_fwd(q, k, v, ob, None, eps=1e-6)
    torch.cuda.synchronize()
    a, b = o[:, :, -1].cpu().double().numpy(), ob[:, :, -1].cpu().double().numpy()
    assert np.linalg.norm(a - b) / np.linalg.norm(b) < 1e-5


def test_deterministic():
    inp = _inputs("bf16", 2, 3, 700, 128, seed=43, feature="elu1")
    a = _run(inp, [0.9, 0.95, 1.0], "elu1", 1e-6)
    b = _run(inp, [0.9, 0.95, 1.0], "elu1", 1e-6)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


def test_empty_sequence_is_a_no_op():
    import linear_attention_attn_b200 as la
    z = torch.empty((1, 2, 0, 64), dtype=torch.float16, device=_dev())
    la.la_causal_norm_fwd(z, z, z, z)
    la.la_causal_norm_bwd(z, z, z, z, z, z, z)
    torch.cuda.synchronize()


@pytest.mark.parametrize("T", [300, 1000])
def test_strong_decays_fp16(T):
    """fp16 at D = 64 with a decay below 0.9 takes the tensor-core kernel with two output
    accumulators (the folded one needs gamma >= 0.9 in fp16): o and the gradients against the
    oracle, both feature maps."""
    for feature, eps in (("elu1", 1e-6), ("identity", 1e-3)):
        inp = _inputs("f16", 2, 3, T, 64, seed=45, feature=feature)
        decay = [0.5, 0.85, 0.95]
        o, dq, dk, dv = _run(inp, decay, feature, eps)
        want_o = oracle.causal_norm_fwd(inp["q"], inp["k"], inp["v"], decay, feature, eps)
        want = oracle.causal_norm_bwd(inp["q"], inp["k"], inp["v"], inp["do"], decay, feature, eps)
        pu.assert_fwd(o, want_o, "o " + feature, dtype=inp["q"].dtype)
        for name, got, ref in zip(("dq", "dk", "dv"), (dq, dk, dv), want):
            pu.assert_grad(got, ref, name + " " + feature)
