"""elsaa_select_noalloc: selection for callers that cannot allocate device memory
(inside CUDA-graph capture, under a fully reserved memory pool, or in runtimes
that forbid allocation after start-up).  Its scratch is a static array inside
the library; the test checks, through the C ABI, that two calls in a row give
exactly the indices of elsaa_debug_select (which uses caller scratch)."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import elsaa_oracle as orc
from sparse_rank_approximation_b200 import binding as bd
from sparse_rank_approximation_b200.workloads import WORKLOADS, make_inputs, small_workload
from tests.harness import device_inputs, gpu_op

pytestmark = pytest.mark.gpu

CASES = [WORKLOADS["n16k_d128"], WORKLOADS["n2k_d64"], WORKLOADS["tiny_f32"],
         small_workload(N=64 * 7 + 13, d=64, block_size=64, topk=3, rank_r=32, H=3, causal=False)]


def _noalloc(op, q, k):
    n_t = -(-op.p.N // op.p.block_size)
    idx = torch.full((op.p.B, op.p.H, n_t, max(op.p.topk, 1)), -7, dtype=torch.int32, device=q.device)
    st = bd.lib().elsaa_select_noalloc(ctypes.byref(op.p), q.data_ptr(), k.data_ptr(), idx.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == bd.ELSAA_OK, bd.lib().elsaa_last_error_message()
    return idx[..., :op.p.topk]


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_noalloc_selection_matches_workspace_selection_twice(w):
    op = gpu_op(w)
    for seed in (0, 1):                      # two calls in a row, different inputs
        dev = device_inputs(w, make_inputs(w, seed))
        _, ref = op.debug_select(dev["Q"], dev["K"])
        scores, _ = op.debug_select(dev["Q"], dev["K"])
        got = _noalloc(op, dev["Q"], dev["K"])
        torch.cuda.synchronize()
        assert torch.equal(got, ref), f"seed {seed}: selection differs"
        # and the oracle's selection rule fed the same float32 scores picks the same blocks
        sc, ix = scores.cpu().numpy(), got.cpu().numpy()
        for b in range(w.B):
            for h in range(w.H):
                assert np.array_equal(orc.select_from_scores(sc[b, h], w.topk, w.causal), ix[b, h]), (b, h)


def test_noalloc_selection_replays_from_a_cuda_graph():
    """The reason for the entry point: it can be captured, since it allocates nothing.
    One eager call first (it resolves the array's address), then a capture on a side
    stream; new inputs copied into the captured buffers give the new selection."""
    w = small_workload(N=128 * 6 + 21, d=128, block_size=128, topk=3, rank_r=16, H=2)
    op = gpu_op(w)
    a = device_inputs(w, make_inputs(w, 0))
    q, k = a["Q"].clone(), a["K"].clone()
    _noalloc(op, q, k)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        out = _noalloc(op, q, k)
    for seed in (3, 4):
        b = device_inputs(w, make_inputs(w, seed))
        q.copy_(b["Q"])
        k.copy_(b["K"])
        g.replay()
        _, ref = op.debug_select(b["Q"], b["K"])
        torch.cuda.synchronize()
        assert torch.equal(out, ref), f"seed {seed}: replayed selection differs"
    del g


def test_noalloc_rejects_problems_beyond_its_static_scratch():
    p = bd.make_params(1, 8, 65536, 128, rank_r=256, block_size=64, topk=32)   # needs about 50 MiB
    x = torch.empty(16, dtype=torch.uint8, device="cuda")
    st = bd.lib().elsaa_select_noalloc(ctypes.byref(p), x.data_ptr(), x.data_ptr(), x.data_ptr(), None)
    assert st == bd.ELSAA_ERR_UNSUPPORTED
    assert b"static scratch" in bd.lib().elsaa_last_error_message()
