"""Python binding of libla_b200.so: B200 (sm_100a) linear attention, forward and backward.

Argument marshalling only: each function checks the tensors, takes their device
pointers and calls the C entry point of the same name (``include/la.h``).  All
arithmetic runs in the library's CUDA kernels; there is no CPU or PyTorch
fallback -- importing this package fails if the compiled library is missing.

Tensors are torch CUDA tensors, contiguous [B, H, T, D], dtype float32, float16
or bfloat16, 16-byte aligned.  ``state`` tensors are float32 [B, H, D, D+1].
When ``workspace`` is omitted, a torch uint8 buffer of la_workspace_size()
bytes is allocated (torch's allocator is the only allocator involved).  When
``stream`` is omitted the current torch stream is used.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libla_b200.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libla_b200.so is not built: run `python -m linear_attention_attn_b200.build` "
                      "(or __graft_entry__.build()) first")

_lib = ctypes.CDLL(LIB_PATH)

LA_F32, LA_F16, LA_BF16 = 0, 1, 2
OPS = {"bidir_fwd": 0, "bidir_bwd": 1, "simple_fwd": 2, "simple_bwd": 3,
       "chunk_decay_fwd": 4, "chunk_decay_bwd": 5, "state_reduce": 6, "state_apply": 7,
       "state_bwd_q": 8, "state_bwd_kv": 9, "causal_norm_fwd": 10, "causal_norm_bwd": 11, "gated_fwd": 12,
       "gated_bwd": 13}
FEATURES = {"identity": 0, "elu1": 1, "norm": 2}
STATUS = {0: "LA_OK", 1: "LA_ERR_INVALID_ARG", 2: "LA_ERR_UNSUPPORTED", 3: "LA_ERR_ALIGNMENT",
          4: "LA_ERR_WORKSPACE", 5: "LA_ERR_CUDA", 6: "LA_ERR_TIMEOUT"}
MAX_DECAY_HEADS = 512

_P = ctypes.c_void_p
_I = ctypes.c_int
_F = ctypes.c_float
_Z = ctypes.c_size_t


class _ProfRecord(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_longlong), ("total_ms", ctypes.c_double)]


_lib.la_workspace_size.argtypes = [_I, _I, _I, _I, _I, _I]
_lib.la_workspace_size.restype = _Z
_lib.la_bidir_fwd.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _Z, _P]
_lib.la_simple_fwd.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_bidir_bwd.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P, _Z, _P]
_lib.la_simple_bwd.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_chunk_decay_fwd.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_chunk_decay_bwd.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_chunk_decay_step.argtypes = [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]
_lib.la_chunk_decay_fwd_state.argtypes = [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_chunk_decay_bwd_state.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z,
                                          _P]
_lib.la_chunk_decay_scan.argtypes = [_P, _P, _I, _P, _P, _I, _I, _I, _P]
_lib.la_gated_fwd.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_gated_bwd.argtypes = [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_feature_map_fwd.argtypes = [_I, _F, _P, _P, _I, _I, _I, _I, _I, _P]
_lib.la_feature_map_bwd.argtypes = [_I, _F, _P, _P, _P, _I, _I, _I, _I, _I, _P]
_lib.la_causal_norm_fwd.argtypes = [_P, _P, _P, _P, _P, _I, _F, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_causal_norm_bwd.argtypes = [_P, _P, _P, _P, _P, _I, _F, _P, _P, _P, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_state_reduce.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _Z, _P]
_lib.la_state_apply.argtypes = [_P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P]
_lib.la_state_bwd_q.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _F, _P, _Z, _P]
_lib.la_state_bwd_kv.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P]
for _n in ("la_bidir_fwd", "la_simple_fwd", "la_bidir_bwd", "la_simple_bwd", "la_chunk_decay_fwd",
           "la_chunk_decay_bwd", "la_chunk_decay_step", "la_chunk_decay_fwd_state", "la_chunk_decay_bwd_state",
           "la_chunk_decay_scan", "la_state_reduce", "la_state_apply", "la_state_bwd_q", "la_state_bwd_kv",
           "la_causal_norm_fwd", "la_causal_norm_bwd", "la_feature_map_fwd", "la_feature_map_bwd", "la_gated_fwd",
           "la_gated_bwd"):
    getattr(_lib, _n).restype = _I
_lib.la_bidir_fwd_static.argtypes = [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _F, _P]
_lib.la_bidir_fwd_static.restype = _I
_lib.la_debug_fail_launch.argtypes = [_I]
_lib.la_debug_fail_launch.restype = _I
_lib.la_debug_wait_timeout.argtypes = [ctypes.c_uint, _P, _P]
_lib.la_debug_wait_timeout.restype = _I
_lib.la_static_scratch_bytes.argtypes = []
_lib.la_static_scratch_bytes.restype = _Z
_lib.la_status_string.argtypes = [_I]
_lib.la_status_string.restype = ctypes.c_char_p
_lib.la_last_error.argtypes = []
_lib.la_last_error.restype = ctypes.c_char_p
_lib.la_device_check.argtypes = []
_lib.la_device_check.restype = _I
_lib.la_launch_count.argtypes = []
_lib.la_launch_count.restype = ctypes.c_longlong
_lib.la_prof_enable.argtypes = [_I]
_lib.la_prof_enable.restype = _I
_lib.la_prof_collect.argtypes = [ctypes.POINTER(_ProfRecord), _I]
_lib.la_prof_collect.restype = _I


class LAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = _lib.la_last_error().decode(errors="replace")
        super().__init__("%s: %s: %s" % (where, STATUS.get(status, status), msg))


def _check(rc: int, where: str):
    if rc != 0:
        raise LAError(rc, where)


def _dtype_code(t) -> int:
    import torch
    codes = {torch.float32: LA_F32, torch.float16: LA_F16, torch.bfloat16: LA_BF16}
    if t.dtype not in codes:
        raise TypeError("unsupported dtype %s" % t.dtype)
    return codes[t.dtype]


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _shape(q, *others):
    if q.dim() != 4:
        raise ValueError("expected [B, H, T, D] tensors, got %r" % (tuple(q.shape),))
    for o in others:
        if o is None:
            continue
        if tuple(o.shape) != tuple(q.shape) or o.dtype != q.dtype or o.device != q.device:
            raise ValueError("all tensors must share shape, dtype and device")
    for o in (q,) + others:
        if o is not None and (not o.is_cuda or not o.is_contiguous()):
            raise ValueError("tensors must be contiguous CUDA tensors")
    return tuple(int(x) for x in q.shape)


def _stream(stream, dev):
    import torch
    if stream is None:
        return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    if isinstance(stream, int):
        return ctypes.c_void_p(stream)
    return ctypes.c_void_p(stream.cuda_stream)


def _state_check(state, B, H, D, dev):
    import torch
    if state is None:
        return
    if (tuple(state.shape) != (B, H, D, D + 1) or state.dtype != torch.float32 or not state.is_cuda
            or not state.is_contiguous() or state.device != dev):
        raise ValueError("state must be a contiguous float32 CUDA tensor [B, H, D, D+1] on the inputs' device")


def la_workspace_size(op, B: int, H: int, T: int, D: int, dtype) -> int:
    """Bytes of workspace the op needs (op is a name from OPS or its code; dtype a torch dtype or code)."""
    import torch
    code = OPS[op] if isinstance(op, str) else int(op)
    if isinstance(dtype, torch.dtype):
        dtype = {torch.float32: LA_F32, torch.float16: LA_F16, torch.bfloat16: LA_BF16}[dtype]
    return int(_lib.la_workspace_size(code, B, H, T, D, int(dtype)))


def _workspace(op, shape, dt, workspace, dev, stream):
    import torch
    need = _lib.la_workspace_size(OPS[op], *shape, dt)
    if workspace is not None:
        return ctypes.c_void_p(workspace.data_ptr()), workspace.numel() * workspace.element_size(), workspace
    if need == 0:
        return None, 0, None
    buf = torch.empty(need + 256, dtype=torch.uint8, device=dev)
    if isinstance(stream, torch.cuda.Stream):
        buf.record_stream(stream)   # the kernels run on `stream`, not torch's current one
    off = (-buf.data_ptr()) % 256
    buf = buf[off:off + need]
    return ctypes.c_void_p(buf.data_ptr()), need, buf


def la_bidir_fwd(q, k, v, o, state=None, eps: float = 1e-6, workspace=None, stream=None):
    """o <- phi(q) S / (phi(q) . z + eps); optionally state <- (S | z). See include/la.h."""
    B, H, T, D = _shape(q, k, v, o)
    _state_check(state, B, H, D, q.device)
    dt = _dtype_code(q)
    wp, wn, _keep = _workspace("bidir_fwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_bidir_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(state), B, H, T, D, dt, float(eps),
                             wp, wn, _stream(stream, q.device)), "la_bidir_fwd")


def la_bidir_fwd_static(q, k, v, o, state=None, eps: float = 1e-6, stream=None):
    """la_bidir_fwd for callers that cannot allocate device memory: the scratch is a fixed
    LA_STATIC_SCRATCH_BYTES array inside the library (shared by all calls; calls that
    overlap on the GPU race).  No workspace is allocated here either."""
    B, H, T, D = _shape(q, k, v, o)
    _state_check(state, B, H, D, q.device)
    dt = _dtype_code(q)
    _check(_lib.la_bidir_fwd_static(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(state), B, H, T, D, dt, float(eps),
                                    _stream(stream, q.device)), "la_bidir_fwd_static")


def la_static_scratch_bytes() -> int:
    """Bytes of the scratch array built into the library for la_bidir_fwd_static."""
    return int(_lib.la_static_scratch_bytes())


STATIC_SCRATCH_BYTES = la_static_scratch_bytes()


def la_simple_fwd(q, k, v, o, state=None, workspace=None, stream=None):
    """o <- q (k^T v). See include/la.h."""
    B, H, T, D = _shape(q, k, v, o)
    _state_check(state, B, H, D, q.device)
    dt = _dtype_code(q)
    wp, wn, _keep = _workspace("simple_fwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_simple_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(state), B, H, T, D, dt,
                              wp, wn, _stream(stream, q.device)), "la_simple_fwd")


def la_bidir_bwd(q, k, v, dout, dq, dk, dv, state=None, eps: float = 1e-6, workspace=None, stream=None):
    """dq, dk, dv <- gradients of sum(o * dout) for la_bidir_fwd. See include/la.h."""
    B, H, T, D = _shape(q, k, v, dout, dq, dk, dv)
    _state_check(state, B, H, D, q.device)
    dt = _dtype_code(q)
    wp, wn, _keep = _workspace("bidir_bwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_bidir_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(state), _ptr(dq), _ptr(dk), _ptr(dv),
                             B, H, T, D, dt, float(eps), wp, wn, _stream(stream, q.device)), "la_bidir_bwd")


def la_simple_bwd(q, k, v, dout, dq, dk, dv, state=None, workspace=None, stream=None):
    """dq, dk, dv <- gradients of sum(o * dout) for la_simple_fwd. See include/la.h."""
    B, H, T, D = _shape(q, k, v, dout, dq, dk, dv)
    _state_check(state, B, H, D, q.device)
    dt = _dtype_code(q)
    wp, wn, _keep = _workspace("simple_bwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_simple_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(state), _ptr(dq), _ptr(dk), _ptr(dv),
                              B, H, T, D, dt, wp, wn, _stream(stream, q.device)), "la_simple_bwd")


def _decay(decay, H):
    vals = [float(x) for x in (decay.tolist() if hasattr(decay, "tolist") else decay)]
    if len(vals) != H:
        raise ValueError("decay must have H=%d entries" % H)
    return (ctypes.c_float * H)(*vals)


def la_chunk_decay_fwd(q, k, v, o, decay, workspace=None, stream=None):
    """o_t <- sum_{s<=t} decay[h]^(t-s) (q_t . k_s) v_s; decay is a length-H host sequence."""
    B, H, T, D = _shape(q, k, v, o)
    dt = _dtype_code(q)
    dec = _decay(decay, H)
    wp, wn, _keep = _workspace("chunk_decay_fwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_chunk_decay_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), ctypes.cast(dec, _P), B, H, T, D, dt,
                                   wp, wn, _stream(stream, q.device)), "la_chunk_decay_fwd")


def la_chunk_decay_fwd_state(q, k, v, o, decay, state_in=None, state_out=None, workspace=None, stream=None):
    """la_chunk_decay_fwd continuing from state_in ([B, H, D, D] float32, zero if None) and
    writing the state after the last token to state_out (if given); they may be the same tensor.
    o may be None: then only state_out is computed (q is not read and may be None)."""
    import torch
    B, H, T, D = _shape(k, v, q, o)
    for st, name in ((state_in, "state_in"), (state_out, "state_out")):
        if st is not None and (tuple(st.shape) != (B, H, D, D) or st.dtype != torch.float32 or not st.is_cuda
                               or not st.is_contiguous() or st.device != k.device):
            raise ValueError("%s must be a contiguous float32 CUDA tensor [B, H, D, D] on the inputs' device" % name)
    dt = _dtype_code(k)
    dec = _decay(decay, H)
    wp, wn, _keep = _workspace("chunk_decay_fwd", (B, H, T, D), dt, workspace, k.device, stream)
    _check(_lib.la_chunk_decay_fwd_state(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(state_in), _ptr(state_out),
                                         ctypes.cast(dec, _P), B, H, T, D, dt, wp, wn, _stream(stream, k.device)),
           "la_chunk_decay_fwd_state")


def la_chunk_decay_bwd_state(q, k, v, dout, decay, dq, dk, dv, state_in=None, dstate_in=None, dstate_out=None,
                             workspace=None, stream=None):
    """la_chunk_decay_bwd of one segment: state_in is the state of the tokens before it,
    dstate_in R = sum gamma^(u-T) q_u^T dout_u of the tokens after it (both [B, H, D, D] float32,
    zero if None); dstate_out (if given, not overlapping either) receives R at the segment's
    first row.  dq may be None: then only dk and dv are computed; dq, dk and dv may all be
    None: then only dstate_out is computed (k and v are not read and may be None)."""
    import torch
    B, H, T, D = _shape(q, dout, k, v, dq, dk, dv)
    for st, name in ((state_in, "state_in"), (dstate_in, "dstate_in"), (dstate_out, "dstate_out")):
        if st is not None and (tuple(st.shape) != (B, H, D, D) or st.dtype != torch.float32 or not st.is_cuda
                               or not st.is_contiguous() or st.device != q.device):
            raise ValueError("%s must be a contiguous float32 CUDA tensor [B, H, D, D] on the inputs' device" % name)
    dt = _dtype_code(q)
    dec = _decay(decay, H)
    wp, wn, _keep = _workspace("chunk_decay_bwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_chunk_decay_bwd_state(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), _ptr(state_in), _ptr(dstate_in),
                                         _ptr(dstate_out), ctypes.cast(dec, _P), _ptr(dq), _ptr(dk), _ptr(dv), B, H,
                                         T, D, dt, wp, wn, _stream(stream, q.device)),
           "la_chunk_decay_bwd_state")


def la_chunk_decay_bwd(q, k, v, dout, decay, dq, dk, dv, workspace=None, stream=None):
    """dq, dk, dv <- gradients of sum(o * dout) for la_chunk_decay_fwd."""
    B, H, T, D = _shape(q, k, v, dout, dq, dk, dv)
    dt = _dtype_code(q)
    dec = _decay(decay, H)
    wp, wn, _keep = _workspace("chunk_decay_bwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_chunk_decay_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), ctypes.cast(dec, _P), _ptr(dq),
                                   _ptr(dk), _ptr(dv), B, H, T, D, dt, wp, wn, _stream(stream, q.device)),
           "la_chunk_decay_bwd")


def la_chunk_decay_scan(states, gaps, decay, out, stream=None):
    """out[b, h] <- sum over i with gaps[i] >= 0 of decay[h]^gaps[i] * states[i, b, h]: the state
    entering (or, backwards, the R leaving into) one segment of a sequence split into segments.
    states is a float32 [n, B, H, D, D] CUDA tensor, out a float32 [B, H, D, D] one, gaps a
    length-n host sequence of ints (-1 = leave segment i out)."""
    import torch
    if states.dim() != 5 or states.dtype != torch.float32 or not states.is_cuda or not states.is_contiguous():
        raise ValueError("states must be a contiguous float32 CUDA tensor [n, B, H, D, D]")
    n, B, H, D, D2 = (int(x) for x in states.shape)
    if D2 != D or tuple(out.shape) != (B, H, D, D) or out.dtype != torch.float32 or not out.is_cuda \
            or not out.is_contiguous() or out.device != states.device:
        raise ValueError("out must be a contiguous float32 CUDA tensor [B, H, D, D] on the states' device")
    g = [int(x) for x in gaps]
    if len(g) != n:
        raise ValueError("gaps must have n=%d entries" % n)
    garr = (ctypes.c_longlong * n)(*g)
    dec = _decay(decay, H)
    _check(_lib.la_chunk_decay_scan(_ptr(states), ctypes.cast(garr, _P), n, ctypes.cast(dec, _P), _ptr(out), B, H,
                                    D, _stream(stream, states.device)), "la_chunk_decay_scan")


def _decay_or_null(decay, H):
    return (None, None) if decay is None else (lambda a: (ctypes.cast(a, _P), a))(_decay(decay, H))


def la_gated_fwd(q, k, v, g, o, workspace=None, stream=None):
    """Gated linear attention: S_t = diag(exp(g_t)) S_{t-1} + k_t^T v_t, o_t <- q_t S_t; g holds the
    log gates, [B, H, T, D] like q."""
    B, H, T, D = _shape(q, k, v, g, o)
    dt = _dtype_code(q)
    wp, wn, _keep = _workspace("gated_fwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_gated_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), B, H, T, D, dt, wp, wn,
                             _stream(stream, q.device)), "la_gated_fwd")


def la_gated_bwd(q, k, v, g, dout, dq, dk, dv, dg, workspace=None, stream=None):
    """dq, dk, dv, dg <- gradients of sum(o * dout) for la_gated_fwd."""
    B, H, T, D = _shape(q, k, v, g, dout, dq, dk, dv, dg)
    dt = _dtype_code(q)
    wp, wn, _keep = _workspace("gated_bwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_gated_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
                             B, H, T, D, dt, wp, wn, _stream(stream, q.device)), "la_gated_bwd")


FMAPS = {"focused": 0, "polarity": 1, "polarity_swap": 2}


def _fmap_args(kind, x, out, out_width):
    if kind not in FMAPS:
        raise ValueError("kind must be one of %s" % sorted(FMAPS))
    if x.dim() != 4 or out.dim() != 4:
        raise ValueError("expected [B, H, T, D] tensors")
    B, H, T, D = (int(n) for n in x.shape)
    if tuple(out.shape) != (B, H, T, out_width(D)) or out.dtype != x.dtype or out.device != x.device:
        raise ValueError("output must be [B, H, T, %s] of the input's dtype and device" % ("D" if kind == "focused" else "2D"))
    for t in (x, out):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    return B, H, T, D


def la_feature_map_fwd(kind, x, y, p: float = 1.0, stream=None):
    """y <- f(x) row by row: kind 'focused' (y = relu(x), (|y| / |y^p|) y^p; y [B,H,T,D]), 'polarity'
    ([relu(x)^p, relu(-x)^p]; y [B,H,T,2D]) or 'polarity_swap' (the halves swapped)."""
    width = (lambda D: D) if kind == "focused" else (lambda D: 2 * D)
    B, H, T, D = _fmap_args(kind, x, y, width)
    _check(_lib.la_feature_map_fwd(FMAPS[kind], ctypes.c_float(p), _ptr(x), _ptr(y), B, H, T, D, _dtype_code(x),
                                   _stream(stream, x.device)), "la_feature_map_fwd")


def la_feature_map_bwd(kind, x, dy, dx, p: float = 1.0, stream=None):
    """dx <- J(x)^T dy, the gradient through la_feature_map_fwd."""
    width = (lambda D: D) if kind == "focused" else (lambda D: 2 * D)
    B, H, T, D = _fmap_args(kind, x, dy, width)
    if tuple(dx.shape) != tuple(x.shape) or dx.dtype != x.dtype or not dx.is_cuda or not dx.is_contiguous():
        raise ValueError("dx must be a contiguous CUDA tensor like x")
    _check(_lib.la_feature_map_bwd(FMAPS[kind], ctypes.c_float(p), _ptr(x), _ptr(dy), _ptr(dx), B, H, T, D,
                                   _dtype_code(x), _stream(stream, x.device)), "la_feature_map_bwd")


def la_causal_norm_fwd(q, k, v, o, decay=None, feature="elu1", eps: float = 1e-6, workspace=None, stream=None):
    """Causal linear attention with the norm term: o_t <- f(q_t) S_t / (f(q_t) . z_t + eps), S_t and
    z_t the decay[h]-weighted sums over s <= t of f(k_s)^T v_s and f(k_s) (decay None: 1)."""
    B, H, T, D = _shape(q, k, v, o)
    dp, _keep = _decay_or_null(decay, H)
    dt = _dtype_code(q)
    wp, wn, _wkeep = _workspace("causal_norm_fwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_causal_norm_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), dp, _feature(feature),
                                   ctypes.c_float(eps), B, H, T, D, dt, wp, wn, _stream(stream, q.device)),
           "la_causal_norm_fwd")


def la_causal_norm_bwd(q, k, v, dout, dq, dk, dv, decay=None, feature="elu1", eps: float = 1e-6, workspace=None,
                       stream=None):
    """dq, dk, dv <- gradients of sum(o * dout) for la_causal_norm_fwd."""
    B, H, T, D = _shape(q, k, v, dout, dq, dk, dv)
    dp, _keep = _decay_or_null(decay, H)
    dt = _dtype_code(q)
    wp, wn, _wkeep = _workspace("causal_norm_bwd", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_causal_norm_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(dout), dp, _feature(feature),
                                   ctypes.c_float(eps), _ptr(dq), _ptr(dk), _ptr(dv), B, H, T, D, dt, wp, wn,
                                   _stream(stream, q.device)),
           "la_causal_norm_bwd")


def la_chunk_decay_step(q, k, v, o, state, decay, stream=None):
    """One decode step: state <- decay[h] state + k^T v, o <- q state.  q, k, v, o are [B, H, D]
    tensors of one dtype; state is a float32 [B, H, D, D] tensor updated in place."""
    import torch
    if q.dim() != 3:
        raise ValueError("expected [B, H, D] tensors, got %r" % (tuple(q.shape),))
    for t in (k, v, o):
        if tuple(t.shape) != tuple(q.shape) or t.dtype != q.dtype or t.device != q.device:
            raise ValueError("q, k, v, o must share shape, dtype and device")
    for t in (q, k, v, o, state):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
    B, H, D = (int(x) for x in q.shape)
    if tuple(state.shape) != (B, H, D, D) or state.dtype != torch.float32 or state.device != q.device:
        raise ValueError("state must be a float32 [B, H, D, D] tensor on the inputs' device")
    dec = _decay(decay, H)
    _check(_lib.la_chunk_decay_step(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(state), ctypes.cast(dec, _P), B, H, D,
                                    _dtype_code(q), _stream(stream, q.device)), "la_chunk_decay_step")


def _feature(feature):
    if isinstance(feature, str):
        if feature not in FEATURES:
            raise ValueError("feature must be one of %s" % sorted(FEATURES))
        return FEATURES[feature]
    return int(feature)


def _full_state_check(state, B, H, D, dev, name="state"):
    import torch
    if (state is None or tuple(state.shape) != (B, H, D, D + 1) or state.dtype != torch.float32
            or not state.is_cuda or not state.is_contiguous() or state.device != dev):
        raise ValueError("%s must be a contiguous float32 CUDA tensor [B, H, D, D+1] on the inputs' device" % name)


def la_state_reduce(k, v, state, feature="elu1", workspace=None, stream=None):
    """state <- (S | z) of the tokens of k, v (one shard of a sequence split along T)."""
    B, H, T, D = _shape(k, v)
    _full_state_check(state, B, H, D, k.device)
    dt = _dtype_code(k)
    wp, wn, _keep = _workspace("state_reduce", (B, H, T, D), dt, workspace, k.device, stream)
    _check(_lib.la_state_reduce(_ptr(k), _ptr(v), _ptr(state), B, H, T, D, dt, _feature(feature), wp, wn,
                                _stream(stream, k.device)), "la_state_reduce")


def la_state_apply(q, state, o, feature="elu1", eps: float = 1e-6, stream=None):
    """o <- the op's output for the tokens of q, given the whole sequence's (S | z)."""
    B, H, T, D = _shape(q, o)
    _full_state_check(state, B, H, D, q.device)
    _check(_lib.la_state_apply(_ptr(q), _ptr(state), _ptr(o), B, H, T, D, _dtype_code(q), _feature(feature),
                               float(eps), _stream(stream, q.device)), "la_state_apply")


def la_state_bwd_q(q, dout, state, dq, dstate, feature="elu1", eps: float = 1e-6, workspace=None, stream=None):
    """dq of the shard and its (dS | dz) into dstate, given the whole sequence's (S | z)."""
    B, H, T, D = _shape(q, dout, dq)
    _full_state_check(state, B, H, D, q.device)
    _full_state_check(dstate, B, H, D, q.device, "dstate")
    dt = _dtype_code(q)
    wp, wn, _keep = _workspace("state_bwd_q", (B, H, T, D), dt, workspace, q.device, stream)
    _check(_lib.la_state_bwd_q(_ptr(q), _ptr(dout), _ptr(state), _ptr(dq), _ptr(dstate), B, H, T, D, dt,
                               _feature(feature), float(eps), wp, wn, _stream(stream, q.device)), "la_state_bwd_q")


def la_state_bwd_kv(k, v, dstate, dk, dv, feature="elu1", stream=None):
    """dk, dv of the shard given the whole sequence's (dS | dz)."""
    B, H, T, D = _shape(k, v, dk, dv)
    _full_state_check(dstate, B, H, D, k.device, "dstate")
    _check(_lib.la_state_bwd_kv(_ptr(k), _ptr(v), _ptr(dstate), _ptr(dk), _ptr(dv), B, H, T, D, _dtype_code(k),
                                _feature(feature), _stream(stream, k.device)), "la_state_bwd_kv")


def la_status_string(status: int) -> str:
    return _lib.la_status_string(int(status)).decode()


def la_last_error() -> str:
    return _lib.la_last_error().decode(errors="replace")


def la_device_check() -> None:
    """Raise LAError if a tensor-core kernel gave up waiting since the last check."""
    _check(_lib.la_device_check(), "la_device_check")


def la_debug_fail_launch(after: int) -> None:
    """Test hook: the launch after `after` further launches of the library fails (-1 disarms)."""
    _check(_lib.la_debug_fail_launch(int(after)), "la_debug_fail_launch")


def la_debug_wait_timeout(limit_us: int, waited_out=None, stream=None) -> None:
    """Test hook: a kernel whose bounded wait runs out after limit_us (see include/la.h)."""
    dev = waited_out.device if waited_out is not None else None
    _check(_lib.la_debug_wait_timeout(int(limit_us), _ptr(waited_out), _stream(stream, dev)),
           "la_debug_wait_timeout")


def la_launch_count() -> int:
    return int(_lib.la_launch_count())


def la_prof_enable(enabled: bool) -> bool:
    return bool(_lib.la_prof_enable(1 if enabled else 0))


def la_prof_collect(max_records: int = 64):
    """[(kernel name, launches, total ms)] for launches made while profiling was on."""
    recs = (_ProfRecord * max_records)()
    n = _lib.la_prof_collect(recs, max_records)
    if n < 0:
        raise RuntimeError("la_prof_collect failed: " + la_last_error())
    return [(recs[i].name.decode(), int(recs[i].launches), float(recs[i].total_ms)) for i in range(min(n, max_records))]


def raw_lib():
    """The ctypes handle of libla_b200.so (for callers passing raw pointers)."""
    return _lib
