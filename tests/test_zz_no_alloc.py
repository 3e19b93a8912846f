"""la_bidir_fwd_static: the bidirectional forward for callers that cannot allocate device
memory (code inside a framework that owns the CUDA allocator, plugins in a serving
process, runtimes that may not call cudaMalloc after start-up).  Its scratch is a fixed
array inside the library, so these tests call it through the C ABI with nothing but
input and output pointers, and compare it with la_bidir_fwd run with a caller-provided
workspace.  The file sorts last so that a run stopping at its first failure has already
run every other test.
"""
import ctypes
import os
import subprocess
import sys
import textwrap

import pytest
import torch

import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

LA_ERR_WORKSPACE = 4
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _static_call(lib, q, k, v, o, st, eps):
    B, H, T, D = q.shape
    dt = {torch.float16: 1, torch.bfloat16: 2, torch.float32: 0}[q.dtype]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.la_bidir_fwd_static(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(st), B, H, T, D, dt,
                                   ctypes.c_float(eps), stream)


def _check_close(got, want):
    got, want = pu.to64(got), pu.to64(want)
    assert pu.rel_l2(got, want) <= pu.FWD_REL_L2
    assert pu.max_abs(got, want) <= pu.max_abs_bound(want)


def _cuda_inputs(shape, dtype, seed):
    B, H, T, D = shape
    w = synth.Workload("noalloc", "bidir", B, H, T, D, dtype, q_scale=0.5, k_scale=0.5, v_scale=0.5)
    inp = synth.make_inputs(w, seed=seed, with_grad=False)
    return w, inp, tuple(inp[n].cuda() for n in ("q", "k", "v"))


# f16/bf16 at D = 64 run on the tensor-core kernels; fp32 and D = 128 on the CUDA-core
# kernels, whose scratch layout differs.
@pytest.mark.parametrize("shape,dtype", [((2, 4, 1000, 64), "f16"), ((1, 3, 777, 64), "bf16"),
                                         ((1, 2, 256, 64), "f32"), ((2, 2, 300, 128), "f16")])
def test_static_scratch_matches_workspace_entry(shape, dtype):
    import linear_attention_attn_b200 as la
    lib = la.raw_lib()
    B, H, T, D = shape
    # a call of another shape first leaves its partial states in the shared array: a
    # kernel reading scratch it has not written in the same call would pick them up
    _, _, (q2, k2, v2) = _cuda_inputs((3, 5, 513, D), dtype, seed=5)
    assert _static_call(lib, q2, k2, v2, torch.empty_like(q2), None, 1e-6) == 0, la.la_last_error()
    w, inp, (q, k, v) = _cuda_inputs(shape, dtype, seed=11)
    o_ref = torch.empty_like(q)
    st_ref = torch.empty((B, H, D, D + 1), dtype=torch.float32, device="cuda")
    la.la_bidir_fwd(q, k, v, o_ref, st_ref, eps=w.eps)          # caller-provided workspace
    torch.cuda.synchronize()
    for _ in range(2):                                          # two calls in a row share the array
        o = torch.full_like(q, float("nan"))
        st = torch.full_like(st_ref, float("nan"))
        rc = _static_call(lib, q, k, v, o, st, w.eps)
        assert rc == 0, la.la_last_error()
        torch.cuda.synchronize()
        _check_close(o, o_ref)
        assert pu.rel_l2(pu.to64(st), pu.to64(st_ref)) <= 1e-6
    # and the result is right, not merely equal to the other entry point
    want = pu.oracle_run("bidir", inp, eps=w.eps, bwd=False)
    pu.assert_fwd(o, want["o"], "o")


def test_static_scratch_rejects_oversized_shapes():
    import linear_attention_attn_b200 as la
    lib = la.raw_lib()
    assert la.STATIC_SCRATCH_BYTES == 32 << 20                   # the size the library reports
    B, H, T, D = 8, 64, 4096, 128              # needs more scratch than the array holds
    need = la.la_workspace_size("bidir_fwd", B, H, T, D, torch.float16)
    assert need > la.STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)             # never dereferenced: the call stops at the size check
    rc = lib.la_bidir_fwd_static(fake, fake, fake, fake, ctypes.c_void_p(0), B, H, T, D, 1,
                                 ctypes.c_float(1e-6), ctypes.c_void_p(0))
    assert rc == LA_ERR_WORKSPACE
    assert "static scratch" in la.la_last_error()


# Runs in a fresh process: a first call in torch's context, then calls from a second
# driver-API context made current on the thread (the array has another address there),
# then again in torch's context once the second one is destroyed.  Each call's output
# must equal the first bit for bit.  Inputs of the second context are allocated by the
# test itself: the entry point still allocates nothing.
_CTX_SCRIPT = textwrap.dedent("""
    import ctypes, sys
    import numpy as np
    import torch
    sys.path.insert(0, {root!r})
    import linear_attention_attn_b200 as la
    import synth
    from cuda.bindings import driver as drv

    def ok(res):
        err = res[0] if isinstance(res, tuple) else res
        assert int(err) == 0, "driver call failed: %r" % (err,)
        return res[1] if isinstance(res, tuple) and len(res) > 1 else None

    lib = la.raw_lib()
    B, H, T, D = 2, 3, 700, 64
    w = synth.Workload("ctx", "bidir", B, H, T, D, "f16", q_scale=0.5, k_scale=0.5, v_scale=0.5)
    inp = synth.make_inputs(w, seed=3, with_grad=False)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))

    def call(ptrs, stream):
        rc = lib.la_bidir_fwd_static(*[ctypes.c_void_p(int(p)) for p in ptrs], ctypes.c_void_p(0),
                                     B, H, T, D, 1, ctypes.c_float(w.eps), ctypes.c_void_p(stream))
        assert rc == 0, la.la_last_error()

    o = torch.empty_like(q)
    call([q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr()], torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    ref = o.cpu().numpy().copy()

    ok(drv.cuInit(0))
    dev = ok(drv.cuDeviceGet(0))
    ctx = ok(drv.cuCtxCreate(0, dev))            # now current on this thread
    nbytes = ref.nbytes
    bufs = []
    for n in ("q", "k", "v"):
        h = np.ascontiguousarray(inp[n].numpy())
        p = ok(drv.cuMemAlloc(nbytes))
        ok(drv.cuMemcpyHtoD(p, h.ctypes.data, nbytes))
        bufs.append(p)
    po = ok(drv.cuMemAlloc(nbytes))
    for _ in range(2):
        ok(drv.cuMemsetD8(po, 0xFF, nbytes))
        call([int(bufs[0]), int(bufs[1]), int(bufs[2]), int(po)], 0)
        ok(drv.cuCtxSynchronize())
        out = np.empty_like(ref)
        ok(drv.cuMemcpyDtoH(out.ctypes.data, po, nbytes))
        assert np.array_equal(out.view(np.uint16), ref.view(np.uint16)), "second context differs"
    for p in bufs + [po]:
        ok(drv.cuMemFree(p))
    ok(drv.cuCtxDestroy(ctx))                    # torch's context is current again

    o2 = torch.full_like(q, float("nan"))
    call([q.data_ptr(), k.data_ptr(), v.data_ptr(), o2.data_ptr()], torch.cuda.current_stream().cuda_stream)
    torch.cuda.synchronize()
    assert np.array_equal(o2.cpu().numpy().view(np.uint16), ref.view(np.uint16)), "back in torch's context"
    print("CTX_OK")
""")


def test_static_scratch_follows_the_current_context():
    r = subprocess.run([sys.executable, "-c", _CTX_SCRIPT.format(root=ROOT)], capture_output=True, text=True,
                       timeout=300, cwd=ROOT)
    assert r.returncode == 0 and "CTX_OK" in r.stdout, r.stdout[-2000:] + r.stderr[-4000:]
