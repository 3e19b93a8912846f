"""The chunk algebra of the causal-norm and gated kernels, restated in float64 numpy and checked
against the oracle's whole-sequence results (CPU, no GPU).

The kernels cut the sequence into chunks: each chunk's own state from a zero state (a weighted sum
of outer products), a scan over the chunks for the state entering each one, and a walk of each
chunk from its entering state; the backward does the same in reverse.  These tests take the same
steps at small, odd sizes (D = 5, ragged lengths, chunks of 1 token up to longer than the
sequence) so that a wrong weight, a missing boundary term or a transposed index in the algebra
shows up against the oracle's recurrent form."""
import numpy as np
import pytest

import oracle

REL = 1e-10


def _rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def _chunks(T, L):
    return [(s0, min(T, s0 + L)) for s0 in range(0, T, L)]


def _f(x):          # elu + 1
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def _fprime(x):
    return np.where(x > 0, 1.0, np.exp(np.minimum(x, 0.0)))


# ------------------------------------------------------------------ causal norm ---

def _causal_norm_chunked(q, k, v, dout, gam, eps, L):
    """One head ([T, D] arrays): o, dq, dk, dv by chunk states, scans and chunk walks."""
    T, D = q.shape
    fq, fk = _f(q), _f(k)
    vb = np.concatenate([v, np.ones((T, 1))], axis=1)            # [v | 1]
    ch = _chunks(T, L)
    nc = len(ch)
    # forward: chunk states from zero, then the entering states
    E = [np.zeros((D, D + 1)) for _ in range(nc)]
    for c, (s0, s1) in enumerate(ch[:-1]):
        for t in range(s0, s1):
            E[c] += gam ** (s1 - 1 - t) * np.outer(fk[t], vb[t])
    S_in = [np.zeros((D, D + 1))]
    for c in range(nc - 1):
        S_in.append(gam ** L * S_in[c] + E[c])
    o, dq = np.zeros((T, D)), np.zeros((T, D))
    n, dn = np.zeros(T), np.zeros(T)
    for c, (s0, s1) in enumerate(ch):
        S = S_in[c].copy()
        for t in range(s0, s1):
            S = gam * S + np.outer(fk[t], vb[t])
            u = fq[t] @ S
            n[t] = u[D] + eps
            o[t] = u[:D] / n[t]
            dn[t] = -(dout[t] @ u[:D]) / n[t] ** 2
            dq[t] = (S[:, :D] @ dout[t] / n[t] + S[:, D] * dn[t]) * _fprime(q[t])
    # reverse: chunk states from zero after each chunk, then the entering (later) states
    db = np.concatenate([dout / n[:, None], dn[:, None]], axis=1)  # [dout / n | dn]
    F = [np.zeros((D, D + 1)) for _ in range(nc)]
    for c, (s0, s1) in enumerate(ch):
        if c == 0:
            continue
        for t in range(s0, s1):
            F[c] += gam ** (t - s0) * np.outer(fq[t], db[t])
    R_in = [None] * nc
    R_in[nc - 1] = np.zeros((D, D + 1))
    for c in range(nc - 1, 0, -1):
        R_in[c - 1] = F[c] + gam ** L * R_in[c]
    dk, dv = np.zeros((T, D)), np.zeros((T, D))
    for c, (s0, s1) in enumerate(ch):
        R = R_in[c].copy()
        for t in range(s1 - 1, s0 - 1, -1):
            R = gam * R + np.outer(fq[t], db[t])
            dk[t] = (R[:, :D] @ v[t] + R[:, D]) * _fprime(k[t])
            dv[t] = fk[t] @ R[:, :D]
    return o, dq, dk, dv


@pytest.mark.parametrize("L", [1, 3, 8, 29, 100])
def test_causal_norm_chunks_reproduce_the_oracle(L):
    rng = np.random.default_rng(91)
    B, H, T, D = 1, 2, 29, 5
    q, k, v, g = (rng.standard_normal((B, H, T, D)) * 0.5 for _ in range(4))
    gammas, eps = [0.9, 1.0], 1e-6
    want_o = oracle.causal_norm_fwd(q, k, v, gammas, "elu1", eps)
    want = oracle.causal_norm_bwd(q, k, v, g, gammas, "elu1", eps)
    for h in range(H):
        got = _causal_norm_chunked(q[0, h], k[0, h], v[0, h], g[0, h], gammas[h], eps, L)
        assert _rel(got[0], want_o[0, h]) < REL
        for a, b in zip(got[1:], want):
            assert _rel(a, b[0, h]) < REL


# ------------------------------------------------------------------------ gated ---

def _gated_chunked(q, k, v, lg, dout, L, reach_next=True):
    """One head: o, dq, dk, dv, dlg of gated linear attention by chunk states, scans and walks
    (reach_next False plants a slip: the reverse factor stops at the chunk's own last token)."""
    T, D = q.shape
    ch = _chunks(T, L)
    nc = len(ch)
    E = [np.zeros((D, D)) for _ in range(nc)]
    A = [np.ones(D) for _ in range(nc)]
    for c, (s0, s1) in enumerate(ch[:-1]):
        for t in range(s0, s1):
            w = np.exp(lg[t + 1:s1].sum(axis=0))                 # gates between t and the chunk's end
            E[c] += np.outer(w * k[t], v[t])
        A[c] = np.exp(lg[s0:s1].sum(axis=0))
    S_in = [np.zeros((D, D))]
    for c in range(nc - 1):
        S_in.append(A[c][:, None] * S_in[c] + E[c])
    o, dq = np.zeros((T, D)), np.zeros((T, D))
    for c, (s0, s1) in enumerate(ch):
        S = S_in[c].copy()
        for t in range(s0, s1):
            S = np.exp(lg[t])[:, None] * S + np.outer(k[t], v[t])
            o[t] = q[t] @ S
            dq[t] = S @ dout[t]
    # reverse chunk states: gates from the chunk's start; the product reaches g at s1 (the first
    # token after the chunk), since R_t decays by the gates of t + 1
    F = [np.zeros((D, D)) for _ in range(nc)]
    A2 = [np.ones(D) for _ in range(nc)]
    for c, (s0, s1) in enumerate(ch):
        if c == 0:
            continue
        for t in range(s0, s1):
            w = np.exp(lg[s0 + 1:t + 1].sum(axis=0))
            F[c] += np.outer(w * q[t], dout[t])
        A2[c] = np.exp(lg[s0 + 1:min(s1 + 1 if reach_next else s1, T)].sum(axis=0))
    R_in = [None] * nc
    R_in[nc - 1] = np.zeros((D, D))
    for c in range(nc - 1, 0, -1):
        R_in[c - 1] = F[c] + A2[c][:, None] * R_in[c]
    dk, dv, part = np.zeros((T, D)), np.zeros((T, D)), np.zeros((T, D))
    totals = np.zeros((nc, D))
    for c, (s0, s1) in enumerate(ch):
        R = R_in[c].copy()
        acc = np.zeros(D)
        for t in range(s1 - 1, s0 - 1, -1):
            a_next = np.exp(lg[t + 1]) if t + 1 < T else np.zeros(D)
            R = np.outer(q[t], dout[t]) + a_next[:, None] * R
            dk[t] = R @ v[t]
            dv[t] = k[t] @ R
            acc += q[t] * dq[t] - k[t] * dk[t]
            part[t] = acc
        totals[c] = acc
    dlg = part.copy()
    for c, (s0, s1) in enumerate(ch):
        dlg[s0:s1] += totals[c + 1:].sum(axis=0)
    return o, dq, dk, dv, dlg


@pytest.mark.parametrize("L", [1, 3, 8, 29, 100])
def test_gated_chunks_reproduce_the_oracle(L):
    rng = np.random.default_rng(92)
    B, H, T, D = 1, 2, 29, 5
    q, k, v, g = (rng.standard_normal((B, H, T, D)) for _ in range(4))
    lg = np.log(1.0 / (1.0 + np.exp(-rng.standard_normal((B, H, T, D))))) / 4.0
    want_o = oracle.gated_fwd(q, k, v, lg)
    want = oracle.gated_bwd(q, k, v, lg, g)
    for h in range(H):
        got = _gated_chunked(q[0, h], k[0, h], v[0, h], lg[0, h], g[0, h], L)
        assert _rel(got[0], want_o[0, h]) < REL
        for a, b in zip(got[1:], want):
            assert _rel(a, b[0, h]) < REL


def test_gated_reverse_factor_needs_the_next_chunks_first_gate():
    """Leaving g at the first token after a chunk out of its reverse factor (a plausible slip at
    the boundary) breaks the reverse states entering the earlier chunks: dk, dv and dlg then miss
    the oracle."""
    rng = np.random.default_rng(93)
    T, D, L = 20, 4, 5
    q, k, v, g = (rng.standard_normal((T, D)) for _ in range(4))
    lg = -np.abs(rng.standard_normal((T, D))) / 2.0
    want = oracle.gated_bwd(q[None, None], k[None, None], v[None, None], lg[None, None], g[None, None])
    good = _gated_chunked(q, k, v, lg, g, L)
    bad = _gated_chunked(q, k, v, lg, g, L, reach_next=False)
    for j in (2, 3, 4):                          # dk, dv, dlg
        assert _rel(good[j], want[j - 1][0, 0]) < REL
        assert _rel(bad[j], want[j - 1][0, 0]) > 1e-3
