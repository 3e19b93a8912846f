"""fp64 CPU oracle for linear attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline /
reference arm may import this package.  The CUDA library never does, and this
package never imports the CUDA library: the two share nothing but the seeded
input generators in ``synth``.

The arithmetic lives in ``la_oracle.c`` (plain C, double precision); this module
compiles it with gcc on first use (``build()``) and marshals numpy arrays.
Every array is [B, H, T, D] float64, C-contiguous.

Definitions (see the header of ``la_oracle.c`` for the derivations):
  * ``bidir_fwd``  -- "Flash Bi-directional Linear Attention" README, intro:
    non-causal linear attention with phi = elu + 1 and the norm term,
    o_t = phi(q_t) S / (phi(q_t) . z + eps).
  * ``simple_fwd`` -- same README, "Update" list (simple_la): identity phi,
    no norm term.
  * ``retention_fwd`` -- "flash-linear-attention" README, "Benchmarks" (RetNet)
    and "Different forms of linear attention" (FusedRecurrent): causal, per-head
    scalar decay, o_t = sum_{s<=t} gamma^(t-s) (q_t . k_s) v_s.
  * the ``*_bwd`` functions are the hand-derived gradients of those forwards.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "la_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_default = None


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile la_oracle.c into liboracle.so (plain gcc, -O2, no fast-math, no FMA contraction)."""
    stale = (not os.path.exists(out)) or os.path.getmtime(out) < os.path.getmtime(src)
    if force or stale:
        tmp = out + ".tmp%d" % os.getpid()
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math",
               "-ffp-contract=off", "-o", tmp, src, "-lm", "-lpthread"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


def _bind(lib):
    P = ctypes.c_void_p
    L = ctypes.c_long
    Dbl = ctypes.c_double
    I = ctypes.c_int
    lib.oracle_bidir_fwd.argtypes = [P, P, P, P, P, L, L, L, L, Dbl, I]
    lib.oracle_simple_fwd.argtypes = [P, P, P, P, P, L, L, L, L, I]
    lib.oracle_bidir_bwd.argtypes = [P, P, P, P, P, P, P, L, L, L, L, Dbl, I]
    lib.oracle_simple_bwd.argtypes = [P, P, P, P, P, P, P, L, L, L, L, I]
    lib.oracle_retention_fwd.argtypes = [P, P, P, P, P, L, L, L, L, I]
    lib.oracle_retention_bwd.argtypes = [P, P, P, P, P, P, P, P, L, L, L, L, I]
    lib.oracle_retention_step.argtypes = [P, P, P, P, P, P, L, L, L]
    lib.oracle_retention_fwd_state.argtypes = [P, P, P, P, P, P, P, L, L, L, L, I]
    lib.oracle_retention_bwd_state.argtypes = [P, P, P, P, P, P, P, P, P, P, P, L, L, L, L, I]
    lib.oracle_causal_norm_fwd.argtypes = [P, P, P, P, I, Dbl, P, L, L, L, L, I]
    lib.oracle_normed_fwd.argtypes = [P, P, P, P, P, L, L, L, L, Dbl, I]
    lib.oracle_normed_bwd.argtypes = [P, P, P, P, P, P, P, L, L, L, L, Dbl, I]
    lib.oracle_feature_map_fwd.argtypes = [I, Dbl, P, P, L, L]
    lib.oracle_gated_fwd.argtypes = [P, P, P, P, P, L, L, L, L, I]
    lib.oracle_gated_bwd.argtypes = [P, P, P, P, P, P, P, P, P, L, L, L, L, I]
    lib.oracle_feature_map_bwd.argtypes = [I, Dbl, P, P, P, L, L]
    lib.oracle_causal_norm_bwd.argtypes = [P, P, P, P, P, I, Dbl, P, P, P, L, L, L, L, I]
    for name in ("oracle_bidir_fwd", "oracle_simple_fwd", "oracle_bidir_bwd",
                 "oracle_simple_bwd", "oracle_retention_fwd", "oracle_retention_bwd",
                 "oracle_retention_step", "oracle_retention_fwd_state", "oracle_retention_bwd_state",
                 "oracle_causal_norm_fwd", "oracle_causal_norm_bwd", "oracle_normed_fwd", "oracle_normed_bwd",
                 "oracle_feature_map_fwd", "oracle_feature_map_bwd", "oracle_gated_fwd", "oracle_gated_bwd"):
        getattr(lib, name).restype = ctypes.c_int
    return lib


def _load():
    global _default
    with _lock:
        if _default is None:
            build()
            _default = _bind(ctypes.CDLL(_LIB))
    return _default


def default_threads() -> int:
    return os.cpu_count() or 1


def _f64(a) -> np.ndarray:
    """Widen to a C-contiguous float64 numpy array (exact for f16/bf16/f32)."""
    if hasattr(a, "detach"):  # torch tensor (CPU); widen through float64 exactly
        a = a.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def _shape4(q):
    if q.ndim != 4:
        raise ValueError("expected a [B, H, T, D] array, got shape %r" % (q.shape,))
    return q.shape


def _check(rc, name):
    if rc != 0:
        raise RuntimeError("%s failed (rc=%d)" % (name, rc))


class Oracle:
    """The oracle's functions, bound to one compiled library (the default one, or a
    variant compiled from an edited copy of la_oracle.c by the oracle's own tests)."""

    def __init__(self, lib=None):
        self._lib = lib if lib is not None else _load()

    def bidir_fwd(self, q, k, v, eps: float = 1e-6, nthreads: int | None = None, want_state: bool = False):
        """o = phi(q) S / (phi(q) . z + eps);  returns o (and state [B,H,D,D+1] if asked)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, T, D = _shape4(q)
        o = np.empty_like(q)
        st = np.empty((B, H, D, D + 1)) if want_state else None
        rc = self._lib.oracle_bidir_fwd(_p(q), _p(k), _p(v), _p(o), _p(st) if st is not None else None,
                                      B, H, T, D, float(eps), nthreads or default_threads())
        _check(rc, "oracle_bidir_fwd")
        return (o, st) if want_state else o

    def simple_fwd(self, q, k, v, nthreads: int | None = None, want_state: bool = False):
        """o = q (k^T v): identity feature map, no norm term."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, T, D = _shape4(q)
        o = np.empty_like(q)
        st = np.empty((B, H, D, D + 1)) if want_state else None
        rc = self._lib.oracle_simple_fwd(_p(q), _p(k), _p(v), _p(o), _p(st) if st is not None else None,
                                       B, H, T, D, nthreads or default_threads())
        _check(rc, "oracle_simple_fwd")
        return (o, st) if want_state else o

    def bidir_bwd(self, q, k, v, dout, eps: float = 1e-6, nthreads: int | None = None):
        """Gradients (dq, dk, dv) of sum(o * dout) for bidir_fwd."""
        q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, H, T, D = _shape4(q)
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        rc = self._lib.oracle_bidir_bwd(_p(q), _p(k), _p(v), _p(g), _p(dq), _p(dk), _p(dv),
                                      B, H, T, D, float(eps), nthreads or default_threads())
        _check(rc, "oracle_bidir_bwd")
        return dq, dk, dv

    def simple_bwd(self, q, k, v, dout, nthreads: int | None = None):
        """Gradients (dq, dk, dv) of sum(o * dout) for simple_fwd."""
        q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, H, T, D = _shape4(q)
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        rc = self._lib.oracle_simple_bwd(_p(q), _p(k), _p(v), _p(g), _p(dq), _p(dk), _p(dv),
                                       B, H, T, D, nthreads or default_threads())
        _check(rc, "oracle_simple_bwd")
        return dq, dk, dv

    def retention_fwd(self, q, k, v, gamma, nthreads: int | None = None):
        """o_t = sum_{s<=t} gamma_h^(t-s) (q_t . k_s) v_s, recurrent form; gamma is [H]."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, T, D = _shape4(q)
        gm = _f64(gamma).reshape(-1)
        if gm.shape[0] != H:
            raise ValueError("gamma must have H=%d entries" % H)
        o = np.empty_like(q)
        rc = self._lib.oracle_retention_fwd(_p(q), _p(k), _p(v), _p(gm), _p(o), B, H, T, D,
                                          nthreads or default_threads())
        _check(rc, "oracle_retention_fwd")
        return o

    def retention_bwd(self, q, k, v, dout, gamma, nthreads: int | None = None):
        """Gradients (dq, dk, dv) of sum(o * dout) for retention_fwd."""
        q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, H, T, D = _shape4(q)
        gm = _f64(gamma).reshape(-1)
        if gm.shape[0] != H:
            raise ValueError("gamma must have H=%d entries" % H)
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        rc = self._lib.oracle_retention_bwd(_p(q), _p(k), _p(v), _p(g), _p(gm), _p(dq), _p(dk), _p(dv),
                                          B, H, T, D, nthreads or default_threads())
        _check(rc, "oracle_retention_bwd")
        return dq, dk, dv

    def retention_fwd_state(self, q, k, v, gamma, state_in=None, nthreads: int | None = None):
        """retention_fwd starting from state_in ([B, H, D, D], zero if None); returns
        (o, state after the last token)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, T, D = _shape4(q)
        gm = _f64(gamma).reshape(-1)
        if gm.shape[0] != H:
            raise ValueError("gamma must have H=%d entries" % H)
        sin = None if state_in is None else np.ascontiguousarray(_f64(state_in))
        if sin is not None and sin.shape != (B, H, D, D):
            raise ValueError("state_in must be [B, H, D, D]")
        o = np.empty_like(q)
        sout = np.empty((B, H, D, D))
        rc = self._lib.oracle_retention_fwd_state(_p(q), _p(k), _p(v), _p(gm), None if sin is None else _p(sin),
                                                 _p(o), _p(sout), B, H, T, D, nthreads or default_threads())
        _check(rc, "oracle_retention_fwd_state")
        return o, sout

    def retention_bwd_state(self, q, k, v, dout, gamma, state_in=None, dstate_in=None,
                            nthreads: int | None = None):
        """retention_bwd of one segment of a longer sequence: state_in is the state of the
        tokens before it, dstate_in the reverse-sweep R = sum_u gamma^(u-T) q_u^T dout_u of the
        tokens after it ([B, H, D, D], zero if None).  Returns (dq, dk, dv, R at the segment's
        first token)."""
        q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, H, T, D = _shape4(q)
        gm = _f64(gamma).reshape(-1)
        if gm.shape[0] != H:
            raise ValueError("gamma must have H=%d entries" % H)
        ins = []
        for a, name in ((state_in, "state_in"), (dstate_in, "dstate_in")):
            a = None if a is None else np.ascontiguousarray(_f64(a))
            if a is not None and a.shape != (B, H, D, D):
                raise ValueError("%s must be [B, H, D, D]" % name)
            ins.append(a)
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        rout = np.empty((B, H, D, D))
        rc = self._lib.oracle_retention_bwd_state(
            _p(q), _p(k), _p(v), _p(g), _p(gm), None if ins[0] is None else _p(ins[0]),
            None if ins[1] is None else _p(ins[1]), _p(dq), _p(dk), _p(dv), _p(rout), B, H, T, D,
            nthreads or default_threads())
        _check(rc, "oracle_retention_bwd_state")
        return dq, dk, dv, rout

    def normed_fwd(self, q, k, v, eps: float = 1e-6, nthreads: int | None = None, want_state: bool = False):
        """The bidirectional op with the identity feature map (q, k are features formed by the
        caller): o = q S / (q . z + eps), S = sum_s k_s^T v_s, z = sum_s k_s."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        B, H, T, D = _shape4(q)
        o = np.empty_like(q)
        st = np.empty((B, H, D, D + 1)) if want_state else None
        rc = self._lib.oracle_normed_fwd(_p(q), _p(k), _p(v), _p(o), _p(st) if st is not None else None,
                                         B, H, T, D, float(eps), nthreads or default_threads())
        _check(rc, "oracle_normed_fwd")
        return (o, st) if want_state else o

    def normed_bwd(self, q, k, v, dout, eps: float = 1e-6, nthreads: int | None = None):
        """Gradients (dq, dk, dv) of sum(o * dout) for normed_fwd."""
        q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
        B, H, T, D = _shape4(q)
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        rc = self._lib.oracle_normed_bwd(_p(q), _p(k), _p(v), _p(g), _p(dq), _p(dk), _p(dv),
                                         B, H, T, D, float(eps), nthreads or default_threads())
        _check(rc, "oracle_normed_bwd")
        return dq, dk, dv

    def gated_fwd(self, q, k, v, lg, nthreads: int | None = None):
        """Gated linear attention: S_t = diag(exp(lg_t)) S_{t-1} + k_t^T v_t, o_t = q_t S_t."""
        q, k, v, lg = _f64(q), _f64(k), _f64(v), _f64(lg)
        B, H, T, D = _shape4(q)
        o = np.empty_like(q)
        rc = self._lib.oracle_gated_fwd(_p(q), _p(k), _p(v), _p(lg), _p(o), B, H, T, D, nthreads or default_threads())
        _check(rc, "oracle_gated_fwd")
        return o

    def gated_bwd(self, q, k, v, lg, dout, nthreads: int | None = None):
        """Gradients (dq, dk, dv, dlg) of sum(o * dout) for gated_fwd."""
        q, k, v, lg, g = _f64(q), _f64(k), _f64(v), _f64(lg), _f64(dout)
        B, H, T, D = _shape4(q)
        dq, dk, dv, dg = (np.empty_like(q) for _ in range(4))
        rc = self._lib.oracle_gated_bwd(_p(q), _p(k), _p(v), _p(lg), _p(g), _p(dq), _p(dk), _p(dv), _p(dg),
                                        B, H, T, D, nthreads or default_threads())
        _check(rc, "oracle_gated_bwd")
        return dq, dk, dv, dg

    FMAPS = {"focused": 0, "polarity": 1, "polarity_swap": 2}

    def feature_map_fwd(self, kind, x, p: float = 1.0):
        """Row-wise feature map of x [..., D]: 'focused' (width D) or 'polarity' / 'polarity_swap'
        (width 2D)."""
        x = np.ascontiguousarray(_f64(x))
        D = x.shape[-1]
        kd = self.FMAPS[kind]
        w = D if kd == 0 else 2 * D
        y = np.empty(x.shape[:-1] + (w,))
        rc = self._lib.oracle_feature_map_fwd(kd, float(p), _p(x), _p(y), int(x.size // D), D)
        _check(rc, "oracle_feature_map_fwd")
        return y

    def feature_map_bwd(self, kind, x, dy, p: float = 1.0):
        """dx = J^T dy for feature_map_fwd."""
        x = np.ascontiguousarray(_f64(x))
        dy = np.ascontiguousarray(_f64(dy))
        D = x.shape[-1]
        dx = np.empty_like(x)
        rc = self._lib.oracle_feature_map_bwd(self.FMAPS[kind], float(p), _p(x), _p(dy), _p(dx), int(x.size // D), D)
        _check(rc, "oracle_feature_map_bwd")
        return dx

    def _causal_args(self, q, gamma, feature):
        B, H, T, D = _shape4(q)
        gm = None if gamma is None else _f64(gamma).reshape(-1)
        if gm is not None and gm.shape[0] != H:
            raise ValueError("gamma must have H=%d entries" % H)
        if feature not in ("elu1", "identity"):
            raise ValueError("feature must be 'elu1' or 'identity'")
        return (B, H, T, D), gm, 1 if feature == "elu1" else 0

    def causal_norm_fwd(self, q, k, v, gamma=None, feature="elu1", eps: float = 1e-6, nthreads: int | None = None):
        """Causal linear attention with the norm term: o_t = f(q_t) S_t / (f(q_t) . z_t + eps) with
        S_t, z_t the gamma-decayed sums over s <= t of f(k_s)^T v_s and f(k_s) (gamma None: 1)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        (B, H, T, D), gm, up = self._causal_args(q, gamma, feature)
        o = np.empty_like(q)
        rc = self._lib.oracle_causal_norm_fwd(_p(q), _p(k), _p(v), None if gm is None else _p(gm), up, float(eps),
                                              _p(o), B, H, T, D, nthreads or default_threads())
        _check(rc, "oracle_causal_norm_fwd")
        return o

    def causal_norm_bwd(self, q, k, v, dout, gamma=None, feature="elu1", eps: float = 1e-6,
                        nthreads: int | None = None):
        """Gradients (dq, dk, dv) of sum(o * dout) for causal_norm_fwd."""
        q, k, v, g = _f64(q), _f64(k), _f64(v), _f64(dout)
        (B, H, T, D), gm, up = self._causal_args(q, gamma, feature)
        dq, dk, dv = np.empty_like(q), np.empty_like(q), np.empty_like(q)
        rc = self._lib.oracle_causal_norm_bwd(_p(q), _p(k), _p(v), _p(g), None if gm is None else _p(gm), up,
                                              float(eps), _p(dq), _p(dk), _p(dv), B, H, T, D,
                                              nthreads or default_threads())
        _check(rc, "oracle_causal_norm_bwd")
        return dq, dk, dv

    def retention_step(self, q, k, v, gamma, state):
        """One decode step: returns (o, new_state) with new_state = gamma_h state + k^T v and
        o = q new_state; q, k, v are [B, H, D], state is [B, H, D, D] (not modified)."""
        q, k, v = _f64(q), _f64(k), _f64(v)
        if q.ndim != 3:
            raise ValueError("expected [B, H, D] arrays")
        B, H, D = q.shape
        S = np.array(_f64(state), dtype=np.float64, copy=True, order="C")
        if S.shape != (B, H, D, D):
            raise ValueError("state must be [B, H, D, D]")
        gm = _f64(gamma).reshape(-1)
        if gm.shape[0] != H:
            raise ValueError("gamma must have H=%d entries" % H)
        o = np.empty_like(q)
        rc = self._lib.oracle_retention_step(_p(q), _p(k), _p(v), _p(gm), _p(S), _p(o), B, H, D)
        _check(rc, "oracle_retention_step")
        return o, S


_inst = None


def _instance() -> Oracle:
    global _inst
    if _inst is None:
        _inst = Oracle()
    return _inst


def load_variant(path: str) -> Oracle:
    """Bind an Oracle to another compiled copy of la_oracle.c (used by the oracle's tests)."""
    return Oracle(_bind(ctypes.CDLL(path)))


def bidir_fwd(*a, **kw):
    return _instance().bidir_fwd(*a, **kw)


def simple_fwd(*a, **kw):
    return _instance().simple_fwd(*a, **kw)


def bidir_bwd(*a, **kw):
    return _instance().bidir_bwd(*a, **kw)


def simple_bwd(*a, **kw):
    return _instance().simple_bwd(*a, **kw)


def retention_fwd(*a, **kw):
    return _instance().retention_fwd(*a, **kw)


def retention_bwd(*a, **kw):
    return _instance().retention_bwd(*a, **kw)


def retention_step(*a, **kw):
    return _instance().retention_step(*a, **kw)


def retention_fwd_state(*a, **kw):
    return _instance().retention_fwd_state(*a, **kw)


def retention_bwd_state(*a, **kw):
    return _instance().retention_bwd_state(*a, **kw)


def causal_norm_fwd(*a, **kw):
    return _instance().causal_norm_fwd(*a, **kw)


def causal_norm_bwd(*a, **kw):
    return _instance().causal_norm_bwd(*a, **kw)


def normed_fwd(*a, **kw):
    return _instance().normed_fwd(*a, **kw)


def normed_bwd(*a, **kw):
    return _instance().normed_bwd(*a, **kw)


def feature_map_fwd(*a, **kw):
    return _instance().feature_map_fwd(*a, **kw)


def feature_map_bwd(*a, **kw):
    return _instance().feature_map_bwd(*a, **kw)


def gated_fwd(*a, **kw):
    return _instance().gated_fwd(*a, **kw)


def gated_bwd(*a, **kw):
    return _instance().gated_bwd(*a, **kw)
