"""GPU parity of the caller-formed feature maps (la_feature_map_*) and of the state-form stages
with the norm term on given features (feature "norm"), through the C ABI, against the fp64
oracle; then focused linear attention and one polarity-split attention end to end (feature map,
normed attention, gradients back through the map)."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu


def _dev():
    return torch.device("cuda", 0)


def _x(dtype, B, H, T, D, seed, stream, scale=1.0):
    return (synth.normal((B, H, T, D), seed, stream) * scale).to(synth.DTYPES[dtype]).contiguous()


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("D", [32, 64, 128])
@pytest.mark.parametrize("kind,p", [("focused", 3.0), ("focused", 1.0), ("polarity", 1.0), ("polarity_swap", 2.0)])
def test_feature_map_matches_oracle(dtype, D, kind, p):
    import linear_attention_attn_b200 as la
    dev = _dev()
    x = _x(dtype, 2, 3, 37, D, 51, 0)
    W = D if kind == "focused" else 2 * D
    dy = _x(dtype, 2, 3, 37, W, 51, 1)
    y = torch.empty((2, 3, 37, W), dtype=x.dtype, device=dev)
    dx = torch.empty_like(x, device=dev)
    xd, dyd = x.to(dev), dy.to(dev)
    la.la_feature_map_fwd(kind, xd, y, p)
    la.la_feature_map_bwd(kind, xd, dyd, dx, p)
    torch.cuda.synchronize()
    want_y = oracle.feature_map_fwd(kind, x.double().numpy(), p)
    want_dx = oracle.feature_map_bwd(kind, x.double().numpy(), dy.double().numpy(), p)
    pu.assert_fwd(y, want_y, "%s y" % kind)
    pu.assert_grad(dx.cpu().double().numpy(), want_dx, "%s dx" % kind)


def _stored(a, dtype):
    """An fp64 oracle result rounded to the storage dtype: the features travel between the two
    calls as tensors of that dtype, so the reference rounds its own features the same way."""
    return torch.from_numpy(np.ascontiguousarray(a)).to(synth.DTYPES[dtype]).double().numpy()


def _stages(la, q, k, v, g, eps):
    """The single-GPU use of the stages: reduce then apply, bwd_q then bwd_kv (feature 'norm')."""
    B, H, T, D = q.shape
    dev = q.device
    st = torch.empty((B, H, D, D + 1), dtype=torch.float32, device=dev)
    dst = torch.empty_like(st)
    o, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    la.la_state_reduce(k, v, st, feature="norm")
    la.la_state_apply(q, st, o, feature="norm", eps=eps)
    la.la_state_bwd_q(q, g, st, dq, dst, feature="norm", eps=eps)
    la.la_state_bwd_kv(k, v, dst, dk, dv, feature="norm")
    return o, dq, dk, dv


@pytest.mark.parametrize("dtype,D", [("f16", 64), ("bf16", 64), ("f32", 128), ("bf16", 128)])
def test_normed_stages_match_oracle(dtype, D):
    """Features q, k >= 0 (|N(0,1)|): o = q S / (q . z + eps) and its gradients."""
    import linear_attention_attn_b200 as la
    q = _x(dtype, 2, 3, 300, D, 52, 0).abs()
    k = _x(dtype, 2, 3, 300, D, 52, 1).abs()
    v, g = _x(dtype, 2, 3, 300, D, 52, 2), _x(dtype, 2, 3, 300, D, 52, 3)
    dev = _dev()
    got = _stages(la, *(t.to(dev) for t in (q, k, v, g)), 1e-6)
    torch.cuda.synchronize()
    qn, kn, vn, gn = (t.double().numpy() for t in (q, k, v, g))
    pu.assert_fwd(got[0], oracle.normed_fwd(qn, kn, vn, eps=1e-6), "o")
    for name, t, r in zip(("dq", "dk", "dv"), got[1:], oracle.normed_bwd(qn, kn, vn, gn, eps=1e-6)):
        pu.assert_grad(t.cpu().double().numpy(), r, name)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_focused_linear_attention_end_to_end(dtype):
    """q, k -> focusing function (p = 3) -> normed attention -> dq, dk back through the map."""
    import linear_attention_attn_b200 as la
    B, H, T, D, p, eps = 2, 4, 517, 64, 3.0, 1e-6
    q, k = _x(dtype, B, H, T, D, 53, 0), _x(dtype, B, H, T, D, 53, 1)
    v, g = _x(dtype, B, H, T, D, 53, 2), _x(dtype, B, H, T, D, 53, 3)
    dev = _dev()
    qd, kd, vd, gd = (t.to(dev) for t in (q, k, v, g))
    fq, fk = torch.empty_like(qd), torch.empty_like(kd)
    la.la_feature_map_fwd("focused", qd, fq, p)
    la.la_feature_map_fwd("focused", kd, fk, p)
    o, dfq, dfk, dv = _stages(la, fq, fk, vd, gd, eps)
    dq, dk = torch.empty_like(qd), torch.empty_like(kd)
    la.la_feature_map_bwd("focused", qd, dfq, dq, p)
    la.la_feature_map_bwd("focused", kd, dfk, dk, p)
    torch.cuda.synchronize()
    qn, kn, vn, gn = (t.double().numpy() for t in (q, k, v, g))
    fqn = _stored(oracle.feature_map_fwd("focused", qn, p), dtype)
    fkn = _stored(oracle.feature_map_fwd("focused", kn, p), dtype)
    pu.assert_fwd(o, oracle.normed_fwd(fqn, fkn, vn, eps=eps), "o")
    wdfq, wdfk, wdv = oracle.normed_bwd(fqn, fkn, vn, gn, eps=eps)
    pu.assert_grad(dv.cpu().double().numpy(), wdv, "dv")
    pu.assert_grad(dq.cpu().double().numpy(), oracle.feature_map_bwd("focused", qn, wdfq, p), "dq")
    pu.assert_grad(dk.cpu().double().numpy(), oracle.feature_map_bwd("focused", kn, wdfk, p), "dk")


def test_polarity_split_attention_end_to_end():
    """q, k of width 32 -> polarity split (width 64; the key side swapped for the opposite-sign
    map) -> normed attention with v of width 64 -> gradients back through the splits."""
    import linear_attention_attn_b200 as la
    B, H, T, D, eps = 1, 4, 300, 32, 1e-6
    q, k = _x("bf16", B, H, T, D, 54, 0), _x("bf16", B, H, T, D, 54, 1)
    v, g = _x("bf16", B, H, T, 2 * D, 54, 2), _x("bf16", B, H, T, 2 * D, 54, 3)
    dev = _dev()
    qd, kd, vd, gd = (t.to(dev) for t in (q, k, v, g))
    fq = torch.empty((B, H, T, 2 * D), dtype=qd.dtype, device=dev)
    fk = torch.empty_like(fq)
    la.la_feature_map_fwd("polarity", qd, fq)
    la.la_feature_map_fwd("polarity_swap", kd, fk)
    o, dfq, dfk, dv = _stages(la, fq, fk, vd, gd, eps)
    dq, dk = torch.empty_like(qd), torch.empty_like(kd)
    la.la_feature_map_bwd("polarity", qd, dfq, dq)
    la.la_feature_map_bwd("polarity_swap", kd, dfk, dk)
    torch.cuda.synchronize()
    qn, kn, vn, gn = (t.double().numpy() for t in (q, k, v, g))
    fqn = _stored(oracle.feature_map_fwd("polarity", qn), "bf16")          # exact: relu of bf16 values
    fkn = _stored(oracle.feature_map_fwd("polarity_swap", kn), "bf16")
    pu.assert_fwd(o, oracle.normed_fwd(fqn, fkn, vn, eps=eps), "o")
    wdfq, wdfk, wdv = oracle.normed_bwd(fqn, fkn, vn, gn, eps=eps)
    pu.assert_grad(dv.cpu().double().numpy(), wdv, "dv")
    pu.assert_grad(dq.cpu().double().numpy(), oracle.feature_map_bwd("polarity", qn, wdfq), "dq")
    pu.assert_grad(dk.cpu().double().numpy(), oracle.feature_map_bwd("polarity_swap", kn, wdfk), "dk")
