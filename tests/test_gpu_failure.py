"""Failure detection without a GPU fault: a launch made to fail on the host, and a bounded
device wait made to run out.  Both paths must report their error through the C ABI and
leave the context usable: a correct call follows each.
"""
import pytest
import torch

import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

LA_ERR_CUDA, LA_ERR_TIMEOUT = 5, 6


def _small_bidir(seed=4):
    w = synth.Workload("fail", "bidir", 1, 2, 300, 64, "f16", q_scale=0.5, k_scale=0.5, v_scale=0.5)
    return w, synth.make_inputs(w, seed=seed)


def _check_still_correct():
    w, inp = _small_bidir()
    got = pu.gpu_run("bidir", inp, eps=w.eps)
    pu.compare("bidir", got, pu.oracle_run("bidir", inp, eps=w.eps))


def test_injected_launch_failure_is_reported():
    import linear_attention_attn_b200 as la
    w, inp = _small_bidir()
    q, k, v = (inp[n].cuda() for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    launches = la.la_launch_count()
    la.la_debug_fail_launch(0)                   # the next launch fails
    with pytest.raises(la.LAError) as err:
        la.la_bidir_fwd(q, k, v, o, eps=w.eps)
    assert err.value.status == LA_ERR_CUDA
    assert "injected launch failure" in la.la_last_error()
    assert la.la_launch_count() == launches       # nothing reached the GPU
    torch.cuda.synchronize()
    _check_still_correct()                        # the hook fired once and disarmed


def test_injected_failure_between_the_kernels_of_a_call():
    import linear_attention_attn_b200 as la
    w, inp = _small_bidir()
    q, k, v, g = (inp[n].cuda() for n in ("q", "k", "v", "do"))
    st = torch.empty((1, 2, 64, 65), dtype=torch.float32, device="cuda")
    o = torch.empty_like(q)
    la.la_bidir_fwd(q, k, v, o, st, eps=w.eps)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    la.la_debug_fail_launch(1)                   # the backward's first kernel runs, its second fails
    with pytest.raises(la.LAError) as err:
        la.la_bidir_bwd(q, k, v, g, dq, dk, dv, None, eps=w.eps)
    assert err.value.status == LA_ERR_CUDA
    assert "injected launch failure" in la.la_last_error()
    la.la_debug_fail_launch(-1)
    torch.cuda.synchronize()
    _check_still_correct()


def test_disarmed_hook_does_nothing():
    import linear_attention_attn_b200 as la
    la.la_debug_fail_launch(3)
    la.la_debug_fail_launch(-1)
    _check_still_correct()


def test_bounded_wait_runs_out_and_is_reported():
    import linear_attention_attn_b200 as la
    la.la_device_check()                          # nothing pending
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    la.la_debug_wait_timeout(2000, flag)          # a 2 ms wait that nothing ends
    torch.cuda.synchronize()                      # the kernel returned: no hang
    assert int(flag.item()) == 1
    with pytest.raises(la.LAError) as err:
        la.la_device_check()
    assert err.value.status == LA_ERR_TIMEOUT
    assert "wait ran out" in la.la_last_error()
    la.la_device_check()                          # the report was cleared
    _check_still_correct()                        # and the context still works
    la.la_device_check()


def test_wait_limit_is_validated():
    import linear_attention_attn_b200 as la
    with pytest.raises(la.LAError):
        la.la_debug_wait_timeout(0)
