"""la_bidir_fwd_static: the bidirectional forward for callers that cannot allocate device
memory (code inside a framework that owns the CUDA allocator, plugins in a serving
process, runtimes that may not call cudaMalloc after start-up).  Its scratch is a fixed
array inside the library, so these tests call it through the C ABI with nothing but
input and output pointers, and compare it with la_bidir_fwd run with a caller-provided
workspace.  The file sorts last so that a run stopping at its first failure has already
run every other test.
"""
import ctypes

import pytest
import torch

import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

LA_ERR_WORKSPACE = 4


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


@pytest.mark.parametrize("shape,dtype", [((2, 4, 1000, 64), "f16"), ((1, 3, 777, 64), "bf16")])
def test_static_scratch_matches_workspace_entry(shape, dtype):
    import linear_attention_attn_b200 as la
    lib = la.raw_lib()
    B, H, T, D = shape
    w = synth.Workload("noalloc", "bidir", B, H, T, D, dtype, q_scale=0.5, k_scale=0.5, v_scale=0.5)
    inp = synth.make_inputs(w, seed=11, with_grad=False)
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
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
    pu.assert_fwd(pu.to64(o), want["o"], "o")


def test_static_scratch_rejects_oversized_shapes():
    import linear_attention_attn_b200 as la
    lib = la.raw_lib()
    B, H, T, D = 8, 64, 4096, 128              # needs more scratch than the array holds
    need = la.la_workspace_size("bidir_fwd", B, H, T, D, torch.float16)
    assert need > la.STATIC_SCRATCH_BYTES
    fake = ctypes.c_void_p(1 << 20)             # never dereferenced: the call stops at the size check
    rc = lib.la_bidir_fwd_static(fake, fake, fake, fake, ctypes.c_void_p(0), B, H, T, D, 1,
                                 ctypes.c_float(1e-6), ctypes.c_void_p(0))
    assert rc == LA_ERR_WORKSPACE
    assert "static scratch" in la.la_last_error()
