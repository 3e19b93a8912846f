"""Pins for the fp64 oracle: checks against facts that do not come from the oracle itself.

Each check takes an ``oracle.Oracle`` instance and raises AssertionError on a
mismatch, so the same checks run against the real oracle (test_oracle_pins.py)
and against deliberately broken copies of it (test_oracle_mutations.py, which
shows that a dropped term, a wrong sign, index or transposed operand fails at
least one of them).

The facts used:
  * hand-worked examples (tests/golden/hand_examples.json);
  * brute force on tiny inputs in the pairwise ("Parallel", O(T^2)) form, a
    different computation from the oracle's state / recurrent forms;
  * closed forms: all-zero q,k (phi = 1 -> plain mean), inputs whose feature
    values are 0.5 / 1 / 2 (weighted mean), V = 1 with eps = 0 (output 1),
    gamma = 1 (prefix sums), gamma -> 0 (diagonal only);
  * invariances: permutation of tokens, linearity in V, per-head independence,
    thread-count independence;
  * gradients: central finite differences of the oracle's forward, and torch
    autograd through an independently written pairwise form in float64;
  * the decode step: T steps from a zero state against the pairwise causal form.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "hand_examples.json")


def _close(a, b, rtol=1e-12, atol=1e-12, what=""):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    if a.shape != b.shape:
        raise AssertionError("%s: shape %r vs %r" % (what, a.shape, b.shape))
    err = np.abs(a - b)
    lim = atol + rtol * np.abs(b)
    if not np.all(err <= lim):
        i = int(np.argmax(err - lim))
        raise AssertionError("%s: max excess at flat index %d: got %r want %r" % (
            what, i, a.reshape(-1)[i], b.reshape(-1)[i]))


def _feature(x):
    """phi = elu + 1, written independently of the oracle (numpy)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def _rand(shape, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return rng.standard_normal(shape) * scale


def _as4(a):
    a = np.asarray(a, dtype=np.float64)
    return a.reshape(1, 1, *a.shape)


def _parse(x):
    if isinstance(x, list):
        return [_parse(e) for e in x]
    if isinstance(x, str):
        return {"-ln2": -math.log(2.0), "ln2": math.log(2.0)}[x]
    return float(x)


# ------------------------------------------------------------------ golden --

def check_golden(orc):
    cases = json.load(open(GOLDEN))["cases"]
    for c in cases:
        if c["op"] == "retention_step":
            q, k, v = (np.asarray(_parse(c[n]), dtype=np.float64)[None, None] for n in ("q", "k", "v"))
            st = np.asarray(_parse(c["state"]), dtype=np.float64)[None, None]
            o, st2 = orc.retention_step(q, k, v, np.array([c["gamma"]]), st)
            _close(o[0, 0], _parse(c["o"]), what=c["name"] + " o")
            _close(st2[0, 0], _parse(c["state_out"]), what=c["name"] + " state")
            continue
        q, k, v = (_as4(_parse(c[n])) for n in ("q", "k", "v"))
        if c["op"] == "bidir":
            o = orc.bidir_fwd(q, k, v, eps=c["eps"])
        elif c["op"] == "simple":
            o = orc.simple_fwd(q, k, v)
        else:
            o = orc.retention_fwd(q, k, v, np.array([c["gamma"]]))
        _close(o[0, 0], _parse(c["o"]), what=c["name"] + " o")
        if "do" in c:
            g = _as4(_parse(c["do"]))
            if c["op"] == "bidir":
                grads = orc.bidir_bwd(q, k, v, g, eps=c["eps"])
            elif c["op"] == "simple":
                grads = orc.simple_bwd(q, k, v, g)
            else:
                grads = orc.retention_bwd(q, k, v, g, np.array([c["gamma"]]))
            for name, got in zip(("dq", "dk", "dv"), grads):
                _close(got[0, 0], _parse(c[name]), what=c["name"] + " " + name)


# ------------------------------------------------------------- brute force --

def brute_bidir(q, k, v, eps):
    """Pairwise form: o_t = sum_s a_ts v_s / (sum_s a_ts + eps), a_ts = phi(q_t).phi(k_s)."""
    a = np.einsum("bhti,bhsi->bhts", _feature(q), _feature(k))
    return np.einsum("bhts,bhsj->bhtj", a, v) / (a.sum(-1, keepdims=True) + eps)


def brute_simple(q, k, v):
    a = np.einsum("bhti,bhsi->bhts", q, k)
    return np.einsum("bhts,bhsj->bhtj", a, v)


def brute_retention(q, k, v, gamma):
    """Pairwise causal form with an explicit decay matrix gamma^(t-s) [t >= s]."""
    B, H, T, D = q.shape
    t = np.arange(T)
    diff = t[:, None] - t[None, :]
    out = np.empty_like(q)
    for h in range(H):
        m = np.where(diff >= 0, np.power(float(gamma[h]), np.maximum(diff, 0).astype(np.float64)), 0.0)
        a = np.einsum("bti,bsi->bts", q[:, h], k[:, h]) * m
        out[:, h] = np.einsum("bts,bsj->btj", a, v[:, h])
    return out


def check_brute(orc):
    B, H, T, D = 2, 3, 13, 5
    q, k, v = _rand((B, H, T, D), 1), _rand((B, H, T, D), 2), _rand((B, H, T, D), 3)
    _close(orc.bidir_fwd(q, k, v, eps=1e-3), brute_bidir(q, k, v, 1e-3), rtol=1e-11, atol=1e-13,
           what="bidir vs pairwise")
    _close(orc.simple_fwd(q, k, v), brute_simple(q, k, v), rtol=1e-11, atol=1e-12,
           what="simple vs pairwise")
    gam = np.array([0.5, 0.9, 0.999])
    _close(orc.retention_fwd(q, k, v, gam), brute_retention(q, k, v, gam), rtol=1e-11, atol=1e-12,
           what="retention vs pairwise")


# ------------------------------------------------------------ closed forms --

def check_closed_forms(orc):
    T, D = 11, 4
    v = _rand((1, 1, T, D), 7)
    # all-zero q, k: phi = 1 everywhere, every weight equal -> o_t = D sum_s v_s / (T D + eps)
    z = np.zeros((1, 1, T, D))
    eps = 0.3
    want = np.broadcast_to(v.sum(2, keepdims=True) * D / (T * D + eps), v.shape)
    _close(orc.bidir_fwd(z, z, v, eps=eps), want, what="phi(0)=1 mean")
    # per-token feature values 0.5 / 1 / 2 (k = -ln2 / 0 / 1), q = 0, eps = 0 -> weighted mean
    kv = np.array([-math.log(2.0), 0.0, 1.0])[np.arange(T) % 3]
    w = np.array([0.5, 1.0, 2.0])[np.arange(T) % 3]
    k = np.broadcast_to(kv[None, None, :, None], (1, 1, T, D)).copy()
    want = np.broadcast_to((w[:, None] * v[0, 0]).sum(0) / w.sum(), (1, 1, T, D))
    _close(orc.bidir_fwd(z, k, v, eps=0.0), want, what="weighted mean (phi = 0.5/1/2)")
    # V = 1 and eps = 0: every output is exactly 1 (numerator and denominator coincide)
    q, k = _rand((2, 2, T, D), 8), _rand((2, 2, T, D), 9)
    _close(orc.bidir_fwd(q, k, np.ones((2, 2, T, D)), eps=0.0), np.ones((2, 2, T, D)),
           rtol=1e-14, atol=1e-14, what="V=1 identity")
    # V = 1 with eps > 0 stays strictly below 1
    o = orc.bidir_fwd(q, k, np.ones((2, 2, T, D)), eps=0.5)
    if not np.all(o < 1.0):
        raise AssertionError("V=1 with eps>0 must give o < 1")
    # simple_la with q = e_a, k = e_b one-hot rows: o_t = sum_{s: k_s = e_a} v_s
    qs = np.zeros((1, 1, T, D)); qs[..., 0] = 1.0
    ks = np.zeros((1, 1, T, D)); ks[0, 0, ::2, 0] = 1.0; ks[0, 0, 1::2, 1] = 1.0
    want = np.broadcast_to(v[0, 0, ::2].sum(0), (1, 1, T, D))
    _close(orc.simple_fwd(qs, ks, v), want, what="simple one-hot selection")
    # retention, gamma = 1: o_t = q_t (sum_{s<=t} k_s^T v_s)  (prefix sums)
    q, k = _rand((1, 1, T, D), 10), _rand((1, 1, T, D), 11)
    pref = np.cumsum(np.einsum("ti,tj->tij", k[0, 0], v[0, 0]), axis=0)
    want = np.einsum("ti,tij->tj", q[0, 0], pref)[None, None]
    _close(orc.retention_fwd(q, k, v, np.array([1.0])), want, rtol=1e-12, atol=1e-12, what="gamma=1 prefix")
    # retention, gamma -> 0: only the diagonal survives, o_t = (q_t . k_t) v_t
    want = ((q * k).sum(-1, keepdims=True) * v)
    _close(orc.retention_fwd(q, k, v, np.array([1e-30])), want, rtol=1e-12, atol=1e-12, what="gamma=0 diagonal")
    # T = 1: bidir o = v (a / (a + eps)) with a = phi(q).phi(k)
    q1, k1, v1 = _rand((1, 1, 1, D), 12), _rand((1, 1, 1, D), 13), _rand((1, 1, 1, D), 14)
    a = float((_feature(q1) * _feature(k1)).sum())
    _close(orc.bidir_fwd(q1, k1, v1, eps=0.1), v1 * a / (a + 0.1), what="T=1")


# -------------------------------------------------------------- invariances --

def check_invariances(orc):
    B, H, T, D = 1, 2, 17, 6
    q, k, v = _rand((B, H, T, D), 20), _rand((B, H, T, D), 21), _rand((B, H, T, D), 22)
    perm = np.random.default_rng(23).permutation(T)
    o = orc.bidir_fwd(q, k, v, eps=1e-6)
    _close(orc.bidir_fwd(q[:, :, perm], k, v, eps=1e-6), o[:, :, perm], rtol=1e-13, atol=1e-14,
           what="permute queries")
    _close(orc.bidir_fwd(q, k[:, :, perm], v[:, :, perm], eps=1e-6), o, rtol=1e-12, atol=1e-14,
           what="permute keys/values jointly")
    v2 = _rand((B, H, T, D), 24)
    for fn in (lambda vv: orc.bidir_fwd(q, k, vv, eps=1e-6), lambda vv: orc.simple_fwd(q, k, vv),
               lambda vv: orc.retention_fwd(q, k, vv, np.array([0.8, 0.95]))):
        _close(fn(v + 2.0 * v2), fn(v) + 2.0 * fn(v2), rtol=1e-10, atol=1e-11, what="linear in V")
    # per-head independence and indexing: each head equals a single-head call on its slice
    B, H = 2, 3
    q, k, v = _rand((B, H, 9, 4), 25), _rand((B, H, 9, 4), 26), _rand((B, H, 9, 4), 27)
    g = _rand((B, H, 9, 4), 28)
    gam = np.array([0.3, 0.7, 0.95])
    full = [orc.bidir_fwd(q, k, v, eps=1e-2), orc.retention_fwd(q, k, v, gam)]
    fullg = [orc.bidir_bwd(q, k, v, g, eps=1e-2), orc.retention_bwd(q, k, v, g, gam)]
    for b in range(B):
        for h in range(H):
            s = (slice(b, b + 1), slice(h, h + 1))
            _close(full[0][s], orc.bidir_fwd(q[s], k[s], v[s], eps=1e-2), rtol=0, atol=0, what="head slice bidir")
            _close(full[1][s], orc.retention_fwd(q[s], k[s], v[s], gam[h:h + 1]), rtol=0, atol=0,
                   what="head slice retention")
            for a_full, a_one in zip(fullg[1], orc.retention_bwd(q[s], k[s], v[s], g[s], gam[h:h + 1])):
                _close(a_full[s], a_one, rtol=0, atol=0, what="head slice retention bwd")
    # thread count does not change a single bit
    _close(orc.bidir_bwd(q, k, v, g, eps=1e-2, nthreads=1)[1], fullg[0][1], rtol=0, atol=0, what="threads")
    # stored state = (sum_s phi(k_s)^T v_s | sum_s phi(k_s))
    o, st = orc.bidir_fwd(q, k, v, eps=1e-2, want_state=True)
    fk = _feature(k)
    _close(st[..., :-1], np.einsum("bhsi,bhsj->bhij", fk, v), rtol=1e-12, atol=1e-12, what="state S")
    _close(st[..., -1], fk.sum(2), rtol=1e-12, atol=1e-12, what="state z")
    o, st = orc.simple_fwd(q, k, v, want_state=True)
    _close(st[..., :-1], np.einsum("bhsi,bhsj->bhij", k, v), rtol=1e-12, atol=1e-12, what="simple state S")
    _close(st[..., -1], np.zeros_like(st[..., -1]), rtol=0, atol=0, what="simple state z")


# --------------------------------------------------------------- gradients --

def _fd_grads(fwd, q, k, v, g, h=1e-6):
    """Central finite differences of L = sum(fwd(q,k,v) * g) with respect to q, k, v."""
    out = []
    for idx in range(3):
        args = [q.copy(), k.copy(), v.copy()]
        grad = np.zeros_like(args[idx])
        it = np.nditer(args[idx], flags=["multi_index"])
        for _ in it:
            mi = it.multi_index
            base = args[idx][mi]
            args[idx][mi] = base + h
            lp = float((fwd(*args) * g).sum())
            args[idx][mi] = base - h
            lm = float((fwd(*args) * g).sum())
            args[idx][mi] = base
            grad[mi] = (lp - lm) / (2 * h)
        out.append(grad)
    return out


def _keep_off_zero(x, margin=1e-2):
    """Move entries away from 0, where phi' has a kink, so central differences are smooth."""
    return np.where(np.abs(x) < margin, np.sign(x + 1e-30) * margin + x, x)


def check_fd_gradients(orc):
    B, H, T, D = 1, 2, 6, 3
    q = _keep_off_zero(_rand((B, H, T, D), 30))
    k = _keep_off_zero(_rand((B, H, T, D), 31))
    v, g = _rand((B, H, T, D), 32), _rand((B, H, T, D), 33)
    gam = np.array([0.6, 0.9])
    cases = [
        ("bidir", lambda a, b, c: orc.bidir_fwd(a, b, c, eps=0.05), orc.bidir_bwd(q, k, v, g, eps=0.05)),
        ("simple", lambda a, b, c: orc.simple_fwd(a, b, c), orc.simple_bwd(q, k, v, g)),
        ("retention", lambda a, b, c: orc.retention_fwd(a, b, c, gam), orc.retention_bwd(q, k, v, g, gam)),
    ]
    for name, fwd, grads in cases:
        fd = _fd_grads(fwd, q, k, v, g)
        for n, a, b in zip(("dq", "dk", "dv"), grads, fd):
            _close(a, b, rtol=1e-6, atol=1e-7, what="%s %s vs finite differences" % (name, n))


def _torch_pairwise(op, q, k, v, eps=0.0, gamma=None):
    """Independent float64 torch forms used only through autograd."""
    if op in ("bidir",):
        fq = torch.where(q > 0, q + 1.0, torch.exp(torch.clamp(q, max=0.0)))
        fk = torch.where(k > 0, k + 1.0, torch.exp(torch.clamp(k, max=0.0)))
        a = fq @ fk.transpose(-1, -2)
        return (a @ v) / (a.sum(-1, keepdim=True) + eps)
    if op == "simple":
        return (q @ k.transpose(-1, -2)) @ v
    T = q.shape[-2]
    t = torch.arange(T, dtype=torch.float64)
    diff = t[:, None] - t[None, :]
    outs = []
    for h in range(q.shape[1]):
        m = torch.where(diff >= 0, torch.pow(torch.tensor(float(gamma[h]), dtype=torch.float64),
                                             torch.clamp(diff, min=0.0)), torch.zeros(()))
        a = (q[:, h] @ k[:, h].transpose(-1, -2)) * m
        outs.append(a @ v[:, h])
    return torch.stack(outs, 1)


def check_autograd(orc):
    B, H, T, D = 2, 2, 9, 4
    q, k, v, g = (_rand((B, H, T, D), s) for s in (40, 41, 42, 43))
    gam = np.array([0.7, 0.97])
    for op in ("bidir", "simple", "retention"):
        tq, tk, tv = (torch.tensor(a, dtype=torch.float64, requires_grad=True) for a in (q, k, v))
        out = _torch_pairwise(op, tq, tk, tv, eps=0.02, gamma=gam)
        (out * torch.tensor(g)).sum().backward()
        if op == "bidir":
            got = orc.bidir_bwd(q, k, v, g, eps=0.02)
        elif op == "simple":
            got = orc.simple_bwd(q, k, v, g)
        else:
            got = orc.retention_bwd(q, k, v, g, gam)
        for n, a, b in zip(("dq", "dk", "dv"), got, (tq.grad, tk.grad, tv.grad)):
            _close(a, b.numpy(), rtol=1e-10, atol=1e-11, what="%s %s vs autograd" % (op, n))


# ------------------------------------------------------------- decode step --

def check_decode_step(orc):
    """T recurrent steps from a zero state give the pairwise causal outputs, and leave the
    state sum_s gamma^(T-1-s) k_s^T v_s; a step from a nonzero state continues a prefix."""
    B, H, T, D = 2, 3, 9, 5
    q, k, v = _rand((B, H, T, D), 41), _rand((B, H, T, D), 42), _rand((B, H, T, D), 43)
    gam = np.array([0.5, 0.9, 1.0])
    want = brute_retention(q, k, v, gam)
    st = np.zeros((B, H, D, D))
    for t in range(T):
        o, st = orc.retention_step(q[:, :, t], k[:, :, t], v[:, :, t], gam, st)
        _close(o, want[:, :, t], rtol=1e-11, atol=1e-12, what="step %d vs pairwise" % t)
    w = gam[None, :, None] ** (T - 1 - np.arange(T))[None, None, :]
    _close(st, np.einsum("bhs,bhsi,bhsj->bhij", w, k, v), rtol=1e-12, atol=1e-12, what="state after T steps")
    # a prefix of T - 3 tokens as the state, then the last 3 tokens one by one
    p = T - 3
    wp = gam[None, :, None] ** (p - 1 - np.arange(p))[None, None, :]
    st = np.einsum("bhs,bhsi,bhsj->bhij", wp, k[:, :, :p], v[:, :, :p])
    for t in range(p, T):
        o, st = orc.retention_step(q[:, :, t], k[:, :, t], v[:, :, t], gam, st)
        _close(o, want[:, :, t], rtol=1e-11, atol=1e-12, what="step %d after a prefix state" % t)


def check_state_segments(orc):
    """The forward from a given state: o_t = pairwise output + gamma^(t+1) q_t S_in, the state
    after T tokens is gamma^T S_in + sum_s gamma^(T-1-s) k_s^T v_s, and two segments chained
    through the state give the whole sequence."""
    B, H, T, D = 2, 3, 11, 5
    q, k, v = _rand((B, H, T, D), 51), _rand((B, H, T, D), 52), _rand((B, H, T, D), 53)
    gam = np.array([0.5, 0.9, 1.0])
    sin = _rand((B, H, D, D), 54)
    o, sout = orc.retention_fwd_state(q, k, v, gam, sin)
    decay_t = gam[None, :, None] ** (np.arange(T) + 1)[None, None, :]            # gamma^(t+1)
    want = brute_retention(q, k, v, gam) + decay_t[..., None] * np.einsum("bhti,bhij->bhtj", q, sin)
    _close(o, want, rtol=1e-11, atol=1e-12, what="fwd from a state")
    w = gam[None, :, None] ** (T - 1 - np.arange(T))[None, None, :]
    want_s = (gam ** T)[None, :, None, None] * sin + np.einsum("bhs,bhsi,bhsj->bhij", w, k, v)
    _close(sout, want_s, rtol=1e-12, atol=1e-12, what="state after the sequence")
    p = 4
    o1, s1 = orc.retention_fwd_state(q[:, :, :p], k[:, :, :p], v[:, :, :p], gam)
    o2, s2 = orc.retention_fwd_state(q[:, :, p:].copy(), k[:, :, p:].copy(), v[:, :, p:].copy(), gam, s1)
    _close(np.concatenate([o1, o2], axis=2), orc.retention_fwd(q, k, v, gam), rtol=1e-12, atol=1e-12,
           what="two segments vs the whole")


def check_segment_backward(orc):
    """The backward of one segment, with S_in from the tokens before it and R_in from the tokens
    after it.  The tokens after the segment see its state only through S_out, and their loss
    changes by gamma <R_in, dS_out> to first order, so the segment's gradients are those of
    L = sum(o * g) + gamma <R_in, S_out>: finite differences of the forward from a state give
    dq, dk, dv and, with respect to S_in, gamma R_0.  Then R_0 of a lone segment is
    sum_t gamma^t q_t^T g_t, and two segments chained (S forwards, R backwards) give the whole
    sequence's gradients."""
    B, H, T, D = 1, 2, 5, 3
    q, k, v, g = (_rand((B, H, T, D), 61 + i) for i in range(4))
    gam = np.array([0.6, 0.95])
    gm = gam[None, :, None, None]
    sin, rin = _rand((B, H, D, D), 65), _rand((B, H, D, D), 66)
    dq, dk, dv, r0 = orc.retention_bwd_state(q, k, v, g, gam, sin, rin)

    def loss(a, b, c, s):
        o, so = orc.retention_fwd_state(a, b, c, gam, s)
        return float((o * g).sum() + (gm * rin * so).sum())

    h = 1e-6
    args = [q, k, v, sin]
    for idx, (name, got) in enumerate((("dq", dq), ("dk", dk), ("dv", dv), ("dS_in", gm * r0))):
        fd = np.zeros_like(args[idx])
        for mi in np.ndindex(*args[idx].shape):
            a = [x.copy() for x in args]
            a[idx][mi] += h
            lp = loss(*a)
            a[idx][mi] -= 2 * h
            fd[mi] = (lp - loss(*a)) / (2 * h)
        _close(got, fd, rtol=1e-6, atol=1e-7, what="segment backward %s vs finite differences" % name)
    # a lone segment: R_0 = sum_t gamma^t q_t^T g_t
    _, _, _, r_lone = orc.retention_bwd_state(q, k, v, g, gam)
    w = gam[None, :, None] ** np.arange(T)[None, None, :]
    _close(r_lone, np.einsum("bht,bhti,bhtj->bhij", w, q, g), rtol=1e-12, atol=1e-13, what="R_0 closed form")
    # two segments of a sequence of 11 chained through S (forwards) and R (backwards)
    T2, p = 11, 4
    q, k, v, g = (_rand((B, H, T2, D), 71 + i) for i in range(4))
    cut = lambda x, a, b: np.ascontiguousarray(x[:, :, a:b])
    _, s1 = orc.retention_fwd_state(cut(q, 0, p), cut(k, 0, p), cut(v, 0, p), gam)
    dq2, dk2, dv2, r2 = orc.retention_bwd_state(cut(q, p, T2), cut(k, p, T2), cut(v, p, T2), cut(g, p, T2), gam, s1)
    dq1, dk1, dv1, _ = orc.retention_bwd_state(cut(q, 0, p), cut(k, 0, p), cut(v, 0, p), cut(g, 0, p), gam, None, r2)
    whole = orc.retention_bwd(q, k, v, g, gam)
    for n, a, b, c in zip(("dq", "dk", "dv"), (dq1, dk1, dv1), (dq2, dk2, dv2), whole):
        _close(np.concatenate([a, b], axis=2), c, rtol=1e-12, atol=1e-12, what="segments vs whole %s" % n)


def brute_causal_norm(q, k, v, gamma, eps, use_phi=True):
    """Pairwise causal form: o_t = sum_{s<=t} a_ts v_s / (sum_{s<=t} a_ts + eps) with
    a_ts = gamma^(t-s) f(q_t).f(k_s), f = phi or the identity (gamma None: 1)."""
    f = _feature if use_phi else (lambda x: np.asarray(x, dtype=np.float64))
    T = q.shape[2]
    gm = np.ones(q.shape[1]) if gamma is None else np.asarray(gamma, dtype=np.float64)
    dt = np.arange(T)[:, None] - np.arange(T)[None, :]
    mask = np.where(dt[None] >= 0, gm[:, None, None] ** np.maximum(dt, 0)[None], 0.0)    # [H, T, T]
    a = np.einsum("bhti,bhsi->bhts", f(q), f(k)) * mask[None]
    return np.einsum("bhts,bhsj->bhtj", a, v) / (a.sum(-1, keepdims=True) + eps)


def check_causal_norm(orc):
    """Causal linear attention with the norm term: the pairwise form for both feature maps and
    several decays; at gamma = 1 its last row is the bidirectional output's last row (the prefix
    is the whole sequence there); v = 1 gives (n - eps) / n in every column; gradients of both
    feature maps by finite differences."""
    B, H, T, D = 2, 3, 9, 4
    q, k, v = _rand((B, H, T, D), 81), _rand((B, H, T, D), 82), _rand((B, H, T, D), 83)
    for gamma in (None, [0.5, 0.9, 1.0]):
        for feature, up in (("elu1", True), ("identity", False)):
            eps = 1e-3 if up else 50.0      # identity: keep the denominator away from 0
            got = orc.causal_norm_fwd(q, k, v, gamma, feature, eps)
            _close(got, brute_causal_norm(q, k, v, gamma, eps, up), rtol=1e-11, atol=1e-12,
                   what="causal norm %s gamma=%s vs the pairwise form" % (feature, gamma))
    last = orc.causal_norm_fwd(q, k, v, None, "elu1", 1e-3)[:, :, -1]
    _close(last, orc.bidir_fwd(q, k, v, eps=1e-3)[:, :, -1], rtol=1e-12, atol=1e-13,
           what="causal norm last row vs bidirectional")
    ones = np.ones_like(v)
    o1 = orc.causal_norm_fwd(q, k, ones, [0.5, 0.9, 1.0], "elu1", 0.25)
    gm = np.array([0.5, 0.9, 1.0])
    n = np.zeros((B, H, T))
    for t in range(T):
        w = gm[:, None] ** (t - np.arange(t + 1))[None, :]                                     # [H, t+1]
        n[:, :, t] = np.einsum("bhi,bhsi,hs->bh", _feature(q[:, :, t]), _feature(k[:, :, :t + 1]), w) + 0.25
    _close(o1, np.broadcast_to(((n - 0.25) / n)[..., None], o1.shape), rtol=1e-12, atol=1e-13, what="v = 1")
    Bs, Hs, Ts, Ds = 1, 2, 5, 3
    qs = _keep_off_zero(_rand((Bs, Hs, Ts, Ds), 84))
    ks = _keep_off_zero(_rand((Bs, Hs, Ts, Ds), 85))
    vs, gs = _rand((Bs, Hs, Ts, Ds), 86), _rand((Bs, Hs, Ts, Ds), 87)
    for gamma, feature, eps in (([0.6, 0.95], "elu1", 0.05), (None, "identity", 20.0)):
        fwd = lambda a, b, c: orc.causal_norm_fwd(a, b, c, gamma, feature, eps)
        fd = _fd_grads(fwd, qs, ks, vs, gs)
        got = orc.causal_norm_bwd(qs, ks, vs, gs, gamma, feature, eps)
        for name, a, b in zip(("dq", "dk", "dv"), got, fd):
            _close(a, b, rtol=1e-6, atol=1e-7, what="causal norm %s %s vs finite differences" % (feature, name))


def _focus_np(x, p):
    """The focusing function written independently (numpy): y = relu(x), (|y| / |y^p|) y^p per row."""
    y = np.maximum(np.asarray(x, dtype=np.float64), 0.0)
    yp = y ** p
    a = np.linalg.norm(y, axis=-1, keepdims=True)
    b = np.linalg.norm(yp, axis=-1, keepdims=True)
    return np.where(b > 0, a / np.where(b > 0, b, 1.0) * yp, 0.0)


def _fd_rows(fn, x, dy, h=1e-6):
    """Central differences of sum(fn(x) * dy) with respect to x."""
    g = np.zeros_like(x)
    for mi in np.ndindex(*x.shape):
        a = x.copy()
        a[mi] += h
        lp = float((fn(a) * dy).sum())
        a[mi] -= 2 * h
        g[mi] = (lp - float((fn(a) * dy).sum())) / (2 * h)
    return g


def check_feature_maps(orc):
    """The focusing function and the polarity split: a hand-worked row, the norm of relu(x) kept,
    degree-1 homogeneity, p = 1 giving relu(x), the split recovering x, finite-difference gradients,
    and agreement with an independent numpy restatement."""
    # hand-worked: x = (1, 2, -1), p = 2: y = (1, 2, 0), |y| = sqrt 5, y^2 = (1, 4, 0), |y^2| = sqrt 17
    _close(orc.feature_map_fwd("focused", np.array([[1.0, 2.0, -1.0]]), 2.0),
           np.array([[1.0, 4.0, 0.0]]) * np.sqrt(5.0 / 17.0), rtol=1e-15, atol=0, what="focusing, hand-worked")
    x = _rand((5, 7), 91)
    x[2] = -np.abs(x[2])                                   # a row with no positive entry maps to 0
    for p in (1.0, 2.0, 3.0):
        f = orc.feature_map_fwd("focused", x, p)
        _close(f, _focus_np(x, p), rtol=1e-13, atol=1e-15, what="focusing vs numpy, p=%g" % p)
        _close(np.linalg.norm(f, axis=-1), np.linalg.norm(np.maximum(x, 0), axis=-1), rtol=1e-13, atol=1e-15,
               what="focusing keeps |relu(x)|")
        _close(orc.feature_map_fwd("focused", 2.5 * x, p), 2.5 * f, rtol=1e-13, atol=1e-15, what="degree 1")
    _close(orc.feature_map_fwd("focused", x, 1.0), np.maximum(x, 0), rtol=1e-15, atol=0, what="p = 1 is relu")
    s1, s2 = orc.feature_map_fwd("polarity", x, 1.0), orc.feature_map_fwd("polarity_swap", x, 1.0)
    _close(s1[:, :7] - s1[:, 7:], x, rtol=0, atol=0, what="polarity split recovers x")
    _close(s2, np.concatenate([s1[:, 7:], s1[:, :7]], axis=1), rtol=0, atol=0, what="swapped halves")
    _close(orc.feature_map_fwd("polarity", x, 3.0)[:, :7], np.maximum(x, 0) ** 3, rtol=1e-15, atol=0,
           what="polarity power")
    xs = _keep_off_zero(_rand((3, 5), 92), 5e-2)
    for kind, p, w in (("focused", 3.0, 5), ("focused", 1.5, 5), ("polarity", 2.0, 10), ("polarity_swap", 1.0, 10)):
        dy = _rand((3, w), 93)
        fd = _fd_rows(lambda a: orc.feature_map_fwd(kind, a, p), xs, dy)
        _close(orc.feature_map_bwd(kind, xs, dy, p), fd, rtol=1e-6, atol=1e-8,
               what="%s p=%g gradient vs finite differences" % (kind, p))


def check_normed(orc):
    """The bidirectional op on caller-formed features: the pairwise form; phi applied outside gives
    the elu+1 op exactly; focused linear attention (the focusing function then this op) against an
    independent numpy pairwise form; finite-difference gradients."""
    B, H, T, D = 2, 2, 9, 4
    q, k, v = np.abs(_rand((B, H, T, D), 94)), np.abs(_rand((B, H, T, D), 95)), _rand((B, H, T, D), 96)
    a = np.einsum("bhti,bhsi->bhts", q, k)
    _close(orc.normed_fwd(q, k, v, eps=1e-3), np.einsum("bhts,bhsj->bhtj", a, v) / (a.sum(-1, keepdims=True) + 1e-3),
           rtol=1e-12, atol=1e-13, what="normed vs pairwise")
    qr, kr = _rand((B, H, T, D), 97), _rand((B, H, T, D), 98)
    _close(orc.normed_fwd(_feature(qr), _feature(kr), v, eps=1e-3), orc.bidir_fwd(qr, kr, v, eps=1e-3),
           rtol=1e-12, atol=1e-13, what="normed on phi(q), phi(k) = bidir")
    fq, fk = _focus_np(qr, 3.0), _focus_np(kr, 3.0)
    a = np.einsum("bhti,bhsi->bhts", fq, fk)
    want = np.einsum("bhts,bhsj->bhtj", a, v) / (a.sum(-1, keepdims=True) + 1e-2)
    got = orc.normed_fwd(orc.feature_map_fwd("focused", qr, 3.0), orc.feature_map_fwd("focused", kr, 3.0), v, eps=1e-2)
    _close(got, want, rtol=1e-11, atol=1e-12, what="focused linear attention")
    qs, ks = np.abs(_rand((1, 2, 5, 3), 99)) + 0.1, np.abs(_rand((1, 2, 5, 3), 100)) + 0.1
    vs, gs = _rand((1, 2, 5, 3), 101), _rand((1, 2, 5, 3), 102)
    fd = _fd_grads(lambda x, y, z: orc.normed_fwd(x, y, z, eps=0.05), qs, ks, vs, gs)
    for name, a, b in zip(("dq", "dk", "dv"), orc.normed_bwd(qs, ks, vs, gs, eps=0.05), fd):
        _close(a, b, rtol=1e-6, atol=1e-7, what="normed %s vs finite differences" % name)


def brute_gated(q, k, v, lg):
    """Pairwise form: o_t = sum_{s<=t} sum_i q_t[i] k_s[i] exp(sum_{s<r<=t} lg_r[i]) v_s."""
    B, H, T, D = q.shape
    G = np.cumsum(lg, axis=2)                                   # G_t = sum_{r<=t} lg_r
    o = np.zeros_like(v, dtype=np.float64)
    for t in range(T):
        w = np.exp(G[:, :, t:t + 1, :] - G[:, :, :t + 1, :])     # [B, H, t+1, D]
        a = np.einsum("bhi,bhsi->bhs", q[:, :, t], k[:, :, :t + 1] * w)
        o[:, :, t] = np.einsum("bhs,bhsj->bhj", a, v[:, :, :t + 1])
    return o


def check_gated(orc):
    """Gated linear attention: the pairwise form; constant gates log gamma_h give retention; zero
    gates the causal prefix sums; finite differences of dq, dk, dv and of the log gates."""
    B, H, T, D = 2, 3, 8, 4
    q, k, v = _rand((B, H, T, D), 111), _rand((B, H, T, D), 112), _rand((B, H, T, D), 113)
    lg = -np.abs(_rand((B, H, T, D), 114)) * 0.4
    _close(orc.gated_fwd(q, k, v, lg), brute_gated(q, k, v, lg), rtol=1e-12, atol=1e-13, what="gated vs pairwise")
    gam = np.array([0.5, 0.9, 1.0])
    lgc = np.broadcast_to(np.log(gam)[None, :, None, None], q.shape).copy()
    _close(orc.gated_fwd(q, k, v, lgc), orc.retention_fwd(q, k, v, gam), rtol=1e-12, atol=1e-13,
           what="constant gates = retention")
    a = np.tril(np.einsum("bhti,bhsi->bhts", q, k))
    _close(orc.gated_fwd(q, k, v, np.zeros_like(q)), np.einsum("bhts,bhsj->bhtj", a, v), rtol=1e-12, atol=1e-13,
           what="zero gates = causal prefix sums")
    Bs, Hs, Ts, Ds = 1, 2, 5, 3
    qs, ks, vs, gs = (_rand((Bs, Hs, Ts, Ds), 115 + i) for i in range(4))
    ls = -np.abs(_rand((Bs, Hs, Ts, Ds), 119)) * 0.5
    got = orc.gated_bwd(qs, ks, vs, ls, gs)
    fd = _fd_grads(lambda x, y, z: orc.gated_fwd(x, y, z, ls), qs, ks, vs, gs)
    for name, a, b in zip(("dq", "dk", "dv"), got[:3], fd):
        _close(a, b, rtol=1e-6, atol=1e-7, what="gated %s vs finite differences" % name)
    fdg = _fd_rows(lambda x: orc.gated_fwd(qs, ks, vs, x), ls, gs)
    _close(got[3], fdg, rtol=1e-6, atol=1e-7, what="gated dlog-gate vs finite differences")


ALL_CHECKS = (check_golden, check_brute, check_closed_forms, check_invariances,
              check_fd_gradients, check_autograd, check_decode_step, check_state_segments,
              check_segment_backward, check_causal_norm, check_feature_maps, check_normed, check_gated)
