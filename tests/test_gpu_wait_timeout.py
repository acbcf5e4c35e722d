"""Failure detection without a GPU fault: every pipeline wait of the tensor-core kernels
is bounded, and a wait that gives up records a code in the call's error word, drains the
block's copies and products, frees its tensor memory and returns.  The test hook makes
the sparse forward's softmax warps wait on a barrier that nothing completes (with a
20 us limit), then checks that the host reads ELSAA_ERR_TIMEOUT with that wait's code,
and that the next calls on the same stream are correct."""
import re

import numpy as np
import pytest
import torch

from sparse_rank_approximation_b200 import binding as bd
from sparse_rank_approximation_b200.workloads import make_inputs, small_workload
from tests.harness import check, device_inputs, gpu_op, np64, oracle_params
from oracle import elsaa_oracle as orc

pytestmark = pytest.mark.gpu

STALL_CODE = 0x40000     # the softmax warps' stalled wait (attn_fwd_tc)


def test_a_wait_that_runs_out_reports_timeout_and_the_context_stays_usable():
    w = small_workload(N=128 * 4 + 37, d=128, block_size=128, topk=2, rank_r=128, H=2)
    inp = make_inputs(w, 0)
    dev = device_inputs(w, inp)
    op = gpu_op(w)
    try:
        bd.set_wait_limit(20_000, stall=True)
        op.forward(dev["Q"], dev["K"], dev["V"], dev["W"])
        st = op.check_device_flags()
        msg = bd.lib().elsaa_last_error_message().decode()
    finally:
        bd.set_wait_limit(0, stall=False)
    assert st == bd.ELSAA_ERR_TIMEOUT, (st, msg)
    flag = int(re.search(r"flag 0x([0-9a-f]+)", msg).group(1), 16)
    assert flag & STALL_CODE, msg
    # the flag was cleared by the read; the same stream now runs normally
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"])
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"])
    assert op.check_device_flags() == bd.ELSAA_OK
    torch.cuda.synchronize()
    p = oracle_params(w)
    W = inp["W"].double().numpy()
    for h in range(w.H):
        get = lambda n: inp[n][0, h].double().numpy()
        fw = orc.forward_head(get("Q"), get("K"), get("V"), W, p)
        dq, dk, dv = orc.backward_head(get("Q"), get("K"), get("V"), W, get("dO"), fw, p)
        check(w, f"O[{h}]", np64(O[0, h]), fw["O"])
        check(w, f"dQ[{h}]", np64(dQ[0, h]), dq)
        check(w, f"dK[{h}]", np64(dK[0, h]), dk)
        check(w, f"dV[{h}]", np64(dV[0, h]), dv)


def test_the_hook_rejects_bad_arguments():
    assert bd.lib().elsaa_debug_set_wait_limit(0, 2) == bd.ELSAA_ERR_INVALID_ARG
    assert bd.lib().elsaa_debug_set_wait_limit(0, 0) == bd.ELSAA_OK
