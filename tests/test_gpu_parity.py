"""GPU parity: the CUDA path through the C ABI against the fp64 oracle, element by element.

Small shapes are compared in full; the full-size workloads are compared in full where the
oracle finishes in seconds and on sampled (b, h) heads otherwise (every output element of a
sampled head is checked).  Tolerances are those of the method's specification (see
parity_util): forward rel-L2 <= 2e-3 and max-abs <= 1e-2, gradients rel-L2 <= 5e-3.
"""
import numpy as np
import pytest
import torch

import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

SCALES = {  # input recipe per op and dtype, as in the named workloads
    ("bidir", "f32"): (1.0, 1.0, 1.0),
    ("bidir", "f16"): (0.5, 0.5, 0.5), ("bidir", "bf16"): (0.5, 0.5, 0.5),
}


def _workload(op, dtype, B, H, T, D, eps=1e-6):
    if op == "bidir":
        qs, ks, vs = SCALES.get((op, dtype), (0.5, 0.5, 0.5))
    elif op == "simple":
        qs, ks, vs = D ** -0.5, D ** -0.5, 1.0
    else:
        qs, ks, vs = D ** -0.5, 1.0, 1.0
    return synth.Workload("case", op, B, H, T, D, dtype, eps=eps, q_scale=qs, k_scale=ks, v_scale=vs)


SMALL_CASES = [
    ("bidir", "f32", 1, 2, 256, 64),
    ("bidir", "f16", 2, 3, 1000, 64),
    ("bidir", "f16", 1, 1, 7, 64),
    ("bidir", "bf16", 1, 2, 129, 128),
    ("bidir", "f16", 2, 2, 300, 128),
    ("bidir", "bf16", 2, 3, 1000, 64),
    ("bidir", "f16", 1, 1, 256, 64),
    ("bidir", "f16", 3, 5, 2000, 64),
    ("simple", "bf16", 2, 2, 257, 64),
    ("simple", "f16", 1, 3, 100, 128),
    ("simple", "f32", 1, 2, 77, 64),
    ("simple", "bf16", 1, 1, 1, 64),
    ("simple", "f16", 1, 2, 2, 128),
    ("simple", "f16", 1, 1, 256, 64),
    ("simple", "bf16", 4, 40, 300, 64),
    ("retention", "bf16", 1, 4, 300, 128),
    ("retention", "bf16", 2, 2, 129, 64),
    ("retention", "f32", 1, 2, 200, 64),
    ("retention", "f16", 1, 2, 64, 128),
    ("retention", "bf16", 1, 2, 1, 128),
]


@pytest.mark.parametrize("op,dtype,B,H,T,D", SMALL_CASES, ids=lambda x: str(x))
def test_small_shapes(op, dtype, B, H, T, D):
    w = _workload(op, dtype, B, H, T, D)
    inp = synth.make_inputs(w, seed=1)
    got = pu.gpu_run(op, inp, eps=w.eps)
    want = pu.oracle_run(op, inp, eps=w.eps)
    pu.compare(op, got, want)


@pytest.mark.parametrize("dtype", ["f16", "f32"])
def test_bidir_single_token(dtype):
    """T = 1 is the degenerate case of the normalised form: o = v a / (a + eps) with
    a = phi(q).phi(k), so o hardly depends on q or k and the exact dq, dk are O(eps).  The
    kernels form them as differences of O(1) terms, (dout S^T - (dout.o) z) / n and
    v dS^T + dz, which cancel to O(eps); so dq and dk are held to an absolute bound of
    1e-3 (rounding of the O(1) terms, with a margin), while o and dv keep the usual
    bounds."""
    w = _workload("bidir", dtype, 1, 3, 1, 64)
    inp = synth.make_inputs(w, seed=2)
    got = pu.gpu_run("bidir", inp, eps=w.eps)
    want = pu.oracle_run("bidir", inp, eps=w.eps)
    pu.assert_fwd(got["o"], want["o"], "o")
    pu.assert_grad(pu.to64(got["dv"]), want["dv"], "dv")
    assert pu.max_abs(pu.to64(got["dq"]), want["dq"]) < 1e-3
    assert pu.max_abs(pu.to64(got["dk"]), want["dk"]) < 1e-3
    # with eps comparable to phi(q).phi(k) (about D) the case is well conditioned and dq, dk
    # meet the usual bounds
    got = pu.gpu_run("bidir", inp, eps=64.0)
    pu.compare("bidir", got, pu.oracle_run("bidir", inp, eps=64.0))


def test_bidir_f32_small_workload():
    w = synth.WORKLOADS["bidir_f32_small"]
    inp = synth.make_inputs(w, seed=0)
    pu.compare("bidir", pu.gpu_run("bidir", inp, eps=w.eps), pu.oracle_run("bidir", inp, eps=w.eps))


def test_bidir_f16_workload_full():
    """B8 H16 T4096 D64 fp16, every head, forward and backward."""
    w = synth.WORKLOADS["bidir_f16"]
    inp = synth.make_inputs(w, seed=0)
    got = pu.gpu_run("bidir", inp, eps=w.eps)
    pu.compare("bidir", got, pu.oracle_run("bidir", inp, eps=w.eps))
    # the stored state matches the oracle's (S | z) too
    import oracle
    _, st = oracle.bidir_fwd(inp["q"][:1, :2], inp["k"][:1, :2], inp["v"][:1, :2], eps=w.eps, want_state=True)
    assert pu.rel_l2(pu.to64(got["state"][:1, :2]), st) < 1e-3


@pytest.mark.parametrize("T", [8192, 16384])
def test_bidir_f16_long_sampled(T):
    w = synth.WORKLOADS["bidir_f16"].with_T(T)
    inp = synth.make_inputs(w, seed=0)
    heads = [(0, 0), (3, 9), (7, 15)]
    got = pu.gpu_run("bidir", inp, eps=w.eps)
    pu.compare("bidir", got, pu.oracle_run("bidir", inp, eps=w.eps, heads=heads), heads=heads)


@pytest.mark.parametrize("T", synth.SIMPLE_T_SWEEP)
def test_simple_bf16_sweep(T):
    w = synth.WORKLOADS["simple_bf16"].with_T(T)
    inp = synth.make_inputs(w, seed=0)
    heads = None if T <= 1024 else [(0, 0), (3, 7), (7, 15)]
    got = pu.gpu_run("simple", inp)
    pu.compare("simple", got, pu.oracle_run("simple", inp, heads=heads), heads=heads)


@pytest.mark.parametrize("T", synth.RETENTION_T_SWEEP)
def test_retention_bf16_sweep(T):
    w = synth.WORKLOADS["retention_bf16"].with_T(T)
    inp = synth.make_inputs(w, seed=0)
    heads = None if T <= 256 else [(0, 0), (4, 16), (7, 31)]
    got = pu.gpu_run("retention", inp)
    pu.compare("retention", got, pu.oracle_run("retention", inp, heads=heads), heads=heads)


def test_vision_f16_forward_sampled():
    w = synth.WORKLOADS["vision_f16"]
    inp = synth.make_inputs(w, seed=0)
    heads = [(0, 0), (1, 9)]
    got = pu.gpu_run("bidir", inp, eps=w.eps, bwd=False)
    pu.compare("bidir", got, pu.oracle_run("bidir", inp, eps=w.eps, bwd=False, heads=heads), heads=heads, bwd=False)


@pytest.mark.parametrize("op", ["bidir", "simple", "retention"])
def test_deterministic(op):
    w = _workload(op, "bf16" if op != "bidir" else "f16", 2, 4, 3000, 64 if op != "retention" else 128)
    inp = synth.make_inputs(w, seed=3)
    a = pu.gpu_run(op, inp, eps=w.eps)
    b = pu.gpu_run(op, inp, eps=w.eps)
    for n in a:
        assert torch.equal(a[n], b[n]), "%s %s differs between runs" % (op, n)


@pytest.mark.parametrize("op", ["bidir", "simple"])
def test_bwd_recomputes_state(op):
    w = _workload(op, "f16", 1, 3, 777, 64)
    inp = synth.make_inputs(w, seed=4)
    a = pu.gpu_run(op, inp, eps=w.eps, state_to_bwd=True)
    b = pu.gpu_run(op, inp, eps=w.eps, state_to_bwd=False)
    for n in ("dq", "dk", "dv"):
        assert pu.rel_l2(pu.to64(a[n]), pu.to64(b[n])) < 1e-6


def test_empty_sequence_zeroes_state():
    import linear_attention_attn_b200 as la
    q = torch.zeros((1, 2, 0, 64), dtype=torch.float16, device="cuda")
    st = torch.full((1, 2, 64, 65), 7.0, device="cuda")
    la.la_bidir_fwd(q, q, q, q.clone(), st)
    torch.cuda.synchronize()
    assert (st == 0).all()


def test_undersized_workspace_is_rejected():
    import linear_attention_attn_b200 as la
    q = torch.randn((1, 2, 64, 64), device="cuda").half()
    need = la.la_workspace_size("bidir_fwd", 1, 2, 64, 64, torch.float16)
    if need == 0:
        pytest.skip("path needs no workspace")
    ws = torch.empty(need // 2, dtype=torch.uint8, device="cuda")
    with pytest.raises(la.LAError) as e:
        la.la_bidir_fwd(q, q, q, torch.empty_like(q), workspace=ws)
    assert e.value.status == 4


def test_other_stream():
    w = _workload("bidir", "f16", 1, 2, 500, 64)
    inp = synth.make_inputs(w, seed=5)
    s = torch.cuda.Stream()
    got = pu.gpu_run("bidir", inp, eps=w.eps, stream=s)
    pu.compare("bidir", got, pu.oracle_run("bidir", inp, eps=w.eps))


# Strong per-head decays on the tensor-core path: gamma >= 1/8 folds the two output parts of
# a chunk into one accumulator (every factor gamma^k with |k| <= 64 in range); smaller decays
# keep the two parts apart.  Heads of both kinds in one call, and each kind alone; several
# chunks with a ragged tail, so the row scales and the state carried between chunks count.
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("gammas", [(0.05, 0.3, 0.9, 0.999), (0.125, 0.5, 0.75, 1.0), (0.06, 0.1, 0.11, 0.02),
                                    (0.9, 0.95, 0.999, 1.0)],
                         ids=["mixed", "folded", "unfolded", "folded_f16"])
def test_retention_strong_decays(gammas, D, dtype):
    w = _workload("retention", dtype, 2, len(gammas), 300, D)
    inp = synth.make_inputs(w, seed=3)
    inp["gamma"] = torch.tensor(gammas, dtype=torch.float32)
    got = pu.gpu_run("retention", inp)
    pu.compare("retention", got, pu.oracle_run("retention", inp))


# D = 64 on the tensor cores: the kernel loads and stores only the first 64-column box of each
# tile and keeps the second one zero.  Plain causal linear attention (gamma = 1 on every head)
# and the retention decays, over several chunks with a ragged tail; then the B8 H16 T4096 D64
# shape of the causal workloads on sampled heads.
@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("gamma", [1.0, None], ids=["causal", "retention"])
def test_decay_d64(gamma, dtype):
    w = _workload("retention", dtype, 2, 3, 1000, 64)
    inp = synth.make_inputs(w, seed=4)
    if gamma is not None:
        inp["gamma"] = torch.full((w.H,), gamma, dtype=torch.float32)
    got = pu.gpu_run("retention", inp)
    pu.compare("retention", got, pu.oracle_run("retention", inp))


@pytest.mark.parametrize("gamma", [1.0, None], ids=["causal", "retention"])
def test_decay_d64_full_size_sampled(gamma):
    w = _workload("retention", "bf16", 8, 16, 4096, 64)
    inp = synth.make_inputs(w, seed=0)
    if gamma is not None:
        inp["gamma"] = torch.full((w.H,), gamma, dtype=torch.float32)
    heads = [(0, 0), (3, 7), (7, 15)]
    got = pu.gpu_run("retention", inp)
    pu.compare("retention", got, pu.oracle_run("retention", inp, heads=heads), heads=heads)
