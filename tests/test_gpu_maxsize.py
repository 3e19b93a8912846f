"""Parity at the largest tensor the ABI accepts (B*H*T*D just under 2^31 elements).

The oracle cannot run 16.8 M tokens, so the test uses a property that holds at any size: with
eps = 0 the bidirectional op on a sequence made of N copies of a P-token block gives, token
for token, the outputs and gradients of the P-token block (S, z and every n scale by N and
cancel).  The block is checked against the fp64 oracle; every copy of it in the long sequence
is checked against the block."""
import numpy as np
import pytest
import torch

import oracle
import synth
from tests import parity_util as pu

pytestmark = pytest.mark.gpu

B, H, D, P = 1, 2, 64, 1000
N = ((2 ** 31 - 1) // (B * H * D)) // P          # 16777 copies: T = 16,777,000 (ragged: T % 128 = 40)


def test_periodic_sequence_at_the_size_limit():
    import linear_attention_attn_b200 as la
    T = N * P
    assert B * H * T * D < 2 ** 31 and T % 128 != 0
    w = synth.Workload("case", "bidir", B, H, P, D, "f16", eps=0.0, q_scale=0.5, k_scale=0.5, v_scale=0.5)
    blk = synth.make_inputs(w, seed=12, with_grad=True)
    want = pu.oracle_run("bidir", blk, eps=0.0)
    dev = torch.device("cuda", 0)
    big = {n: blk[n].to(dev).repeat(1, 1, N, 1).contiguous() for n in ("q", "k", "v", "do")}
    outs = {n: torch.empty_like(big["q"]) for n in ("o", "dq", "dk", "dv")}
    st = torch.empty((B, H, D, D + 1), dtype=torch.float32, device=dev)
    la.la_bidir_fwd(big["q"], big["k"], big["v"], outs["o"], st, eps=0.0)
    la.la_bidir_bwd(big["q"], big["k"], big["v"], big["do"], outs["dq"], outs["dk"], outs["dv"], st, eps=0.0)
    torch.cuda.synchronize()
    del big
    for n in ("o", "dq", "dk", "dv"):
        x = outs[n].view(B, H, N, P, D).float()
        ref = torch.from_numpy(want[n]).to(dev).float().view(B, H, 1, P, D)
        err = (x - ref).pow(2).sum().sqrt() / (ref.pow(2).sum().sqrt() * N ** 0.5)
        lim = pu.FWD_REL_L2 if n == "o" else pu.GRAD_REL_L2
        assert err.item() <= lim, "%s: rel-L2 %.3g over all %d copies" % (n, err.item(), N)
        worst = (x - ref).abs().amax().item()
        if n == "o":
            assert worst <= pu.max_abs_bound(want[n]), "o: max-abs %.3g" % worst
        del x
