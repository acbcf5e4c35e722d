"""The operator's calls are stream-ordered with no host synchronisation, so a whole
forward + backward step can be captured in a CUDA graph and replayed on new inputs.
Every kernel is deterministic (no atomics on floating-point data), so a replay must
match eager calls on the same inputs bit for bit."""
import pytest
import torch

from sparse_rank_approximation_b200 import binding as bd
from sparse_rank_approximation_b200.workloads import make_inputs, small_workload
from tests.harness import device_inputs, gpu_op

pytestmark = pytest.mark.gpu

CASES = {
    "topk_tcgen05": (dict(N=128 * 4 + 37, d=128, block_size=128, topk=2, rank_r=128), {}),
    "topk_d64_pairs": (dict(N=64 * 5 + 11, d=64, block_size=64, topk=2, rank_r=32), {}),
    "sortlsh": (dict(N=128 * 4 + 37, d=128, block_size=128, topk=1, rank_r=128, causal=False),
                dict(selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=5)),
    "sortlsh_causal": (dict(N=128 * 8, d=128, block_size=128, topk=2, rank_r=128),
                       dict(selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=5)),
}


@pytest.mark.parametrize("case", list(CASES))
def test_graph_replay_matches_eager(case):
    shape, kw = CASES[case]
    w = small_workload(H=2, **shape)
    planes = torch.randn(w.d, 5, generator=torch.Generator().manual_seed(9)).cuda() if kw else None
    op = gpu_op(w, lsh_planes=planes, **kw)
    a = device_inputs(w, make_inputs(w, 0))
    b = device_inputs(w, make_inputs(w, 1))
    static = {n: t.clone() for n, t in a.items()}
    O = op._empty_like_io()
    grads = tuple(op._empty_like_io() for _ in range(3))

    def step():
        op.forward(static["Q"], static["K"], static["V"], static["W"], out=O)
        op.backward(static["Q"], static["K"], static["V"], static["W"], static["dO"], grads=grads)

    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        step()
    torch.cuda.current_stream().wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    for inp in (b, a, b):
        for n, t in inp.items():
            static[n].copy_(t)
        graph.replay()
        replayed = [x.clone() for x in (O,) + grads]
        step()                                        # eager, same inputs
        torch.cuda.synchronize()
        assert op.check_device_flags() == 0
        for name, r, e in zip(("O", "dQ", "dK", "dV"), replayed, (O,) + grads):
            assert torch.equal(r, e), f"{case}: {name} differs between graph replay and eager"
