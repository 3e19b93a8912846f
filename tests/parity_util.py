"""Helpers of the GPU-vs-oracle parity tests: error metrics, tolerances, runners."""
from __future__ import annotations

import numpy as np
import torch

# Tolerances of the method's specification: forward outputs of 16-bit runs within a
# relative L2 error of 2e-3 and a max abs error of 1e-2 of the fp64 oracle; gradients
# within a relative L2 error of 5e-3.  fp32 runs are held to the same bounds.
# Two max-abs readings are checked on every forward output:
#  - against the fp64 oracle, at unit output scale: rounding an output of magnitude m
#    to bf16 alone moves it by up to half an ulp, between 2^-9 m and 2^-8 m (more than
#    1e-2 once m > 2.56), so that bound is max|gpu - oracle| <= 1e-2 * max(1, max|oracle|);
#  - against the oracle rounded to the storage dtype (round to nearest even), element by
#    element: what the kernel adds beyond storage rounding, |gpu - rne(oracle)| <= 1e-2
#    plus one ulp of the element (an fp32 result within a hair of a rounding boundary
#    may round to the neighbouring value).
FWD_REL_L2 = 2e-3
FWD_MAX_ABS = 1e-2
GRAD_REL_L2 = 5e-3


def rel_l2(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = np.linalg.norm(want.ravel())
    num = np.linalg.norm((got - want).ravel())
    return float(num / den) if den > 0 else float(num)


def max_abs(got, want) -> float:
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    return float(np.max(np.abs(got - want))) if got.size else 0.0


def to64(t) -> np.ndarray:
    return t.detach().to("cpu").double().numpy()


def max_abs_bound(want) -> float:
    want = np.asarray(want, dtype=np.float64)
    scale = float(np.max(np.abs(want))) if want.size else 0.0
    return FWD_MAX_ABS * max(1.0, scale)


_TORCH_DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def rne(want, dtype) -> np.ndarray:
    """The float64 values rounded to `dtype` (round to nearest even), widened back."""
    return torch.from_numpy(np.ascontiguousarray(want, dtype=np.float64)).to(dtype).double().numpy()


def ulp(x, dtype) -> np.ndarray:
    """Spacing of `dtype` values at |x|: 2^(e - p) for |x| in [2^e, 2^(e+1)), p the
    fraction bits (7 bf16, 10 fp16, 23 fp32), never below the smallest subnormal."""
    p, emin = {torch.bfloat16: (7, -126), torch.float16: (10, -14), torch.float32: (23, -126)}[dtype]
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, emin)
    return np.exp2(e - p)


def beyond_rounding(got, want, dtype) -> float:
    """max over elements of |gpu - rne(oracle)| minus one ulp of the element (<= 1e-2 passes)."""
    got = np.asarray(got, dtype=np.float64)
    if not got.size:
        return 0.0
    r = rne(want, dtype)
    return float(np.max(np.abs(got - r) - ulp(r, dtype)))


def assert_fwd(got, want, what="", dtype=None):
    """Forward output within tolerance.  `got` is a torch tensor (its dtype is the storage
    dtype) or a float64 array with `dtype` given (a torch dtype or "f32"/"f16"/"bf16")."""
    if isinstance(got, torch.Tensor):
        dtype = dtype or got.dtype
        got = to64(got)
    if isinstance(dtype, str):
        dtype = _TORCH_DT[dtype]
    if dtype is None:
        raise TypeError("assert_fwd needs the storage dtype of a float64 array")
    r, m = rel_l2(got, want), max_abs(got, want)
    lim = max_abs_bound(want)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), "%s: non-finite output" % what
    assert r <= FWD_REL_L2 and m <= lim, "%s: rel_l2=%.3e (<= %.0e) max_abs=%.3e (<= %.3e)" % (
        what, r, FWD_REL_L2, m, lim)
    b = beyond_rounding(got, want, dtype)
    assert b <= FWD_MAX_ABS, "%s: |gpu - rne(oracle)| exceeds one ulp by %.3e (<= %.0e)" % (what, b, FWD_MAX_ABS)
    return r, m


def assert_grad(got, want, what=""):
    r = rel_l2(got, want)
    assert np.all(np.isfinite(np.asarray(got, dtype=np.float64))), "%s: non-finite gradient" % what
    assert r <= GRAD_REL_L2, "%s: rel_l2=%.3e (<= %.0e)" % (what, r, GRAD_REL_L2)
    return r


def gpu_run(op, inp, eps=1e-6, bwd=True, state_to_bwd=True, stream=None):
    """Run the library on CUDA copies of `inp` (from synth.make_inputs); returns CPU tensors."""
    import linear_attention_attn_b200 as la
    dev = torch.device("cuda", 0)
    q, k, v = (inp[n].to(dev) for n in ("q", "k", "v"))
    if stream is not None:
        stream.wait_stream(torch.cuda.current_stream(dev))
    B, H, T, D = q.shape
    out = {}
    o = torch.empty_like(q)
    st = torch.empty((B, H, D, D + 1), dtype=torch.float32, device=dev) if op != "retention" else None
    if op == "bidir":
        la.la_bidir_fwd(q, k, v, o, st, eps=eps, stream=stream)
    elif op == "simple":
        la.la_simple_fwd(q, k, v, o, st, stream=stream)
    else:
        la.la_chunk_decay_fwd(q, k, v, o, inp["gamma"], stream=stream)
    out["o"] = o
    if st is not None:
        out["state"] = st
    if bwd:
        g = inp["do"].to(dev)
        if stream is not None:
            stream.wait_stream(torch.cuda.current_stream(dev))
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        sarg = st if state_to_bwd else None
        if op == "bidir":
            la.la_bidir_bwd(q, k, v, g, dq, dk, dv, sarg, eps=eps, stream=stream)
        elif op == "simple":
            la.la_simple_bwd(q, k, v, g, dq, dk, dv, sarg, stream=stream)
        else:
            la.la_chunk_decay_bwd(q, k, v, g, inp["gamma"], dq, dk, dv, stream=stream)
        out.update(dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    return {n: t.cpu() for n, t in out.items()}


def oracle_run(op, inp, eps=1e-6, bwd=True, heads=None):
    """fp64 oracle on the same inputs; `heads` = list of (b, h) to restrict to (sampled parity)."""
    import oracle
    sel = dict(inp)
    if heads is not None:
        idx_b = [b for b, _ in heads]
        idx_h = [h for _, h in heads]
        for n in ("q", "k", "v", "do"):
            if n in sel:
                sel[n] = inp[n][idx_b, idx_h].unsqueeze(0)   # [1, n_sel, T, D]
        if "gamma" in sel:
            sel["gamma"] = inp["gamma"][idx_h]
    q, k, v = sel["q"], sel["k"], sel["v"]
    res = {}
    if op == "bidir":
        res["o"] = oracle.bidir_fwd(q, k, v, eps=eps)
        if bwd:
            res["dq"], res["dk"], res["dv"] = oracle.bidir_bwd(q, k, v, sel["do"], eps=eps)
    elif op == "simple":
        res["o"] = oracle.simple_fwd(q, k, v)
        if bwd:
            res["dq"], res["dk"], res["dv"] = oracle.simple_bwd(q, k, v, sel["do"])
    else:
        res["o"] = oracle.retention_fwd(q, k, v, sel["gamma"])
        if bwd:
            res["dq"], res["dk"], res["dv"] = oracle.retention_bwd(q, k, v, sel["do"], sel["gamma"])
    return res


def select_heads(t, heads):
    idx_b = [b for b, _ in heads]
    idx_h = [h for _, h in heads]
    return t[idx_b, idx_h].unsqueeze(0)


def compare(op, got, want, heads=None, bwd=True):
    """Assert every output within tolerance; returns a dict of the measured errors."""
    errs = {}
    names = ["o"] + (["dq", "dk", "dv"] if bwd else [])
    for n in names:
        g = got[n] if heads is None else select_heads(got[n], heads)
        if n == "o":
            errs[n] = assert_fwd(g, want[n], "%s %s" % (op, n))
        else:
            errs[n] = assert_grad(to64(g), want[n], "%s %s" % (op, n))
    return errs
