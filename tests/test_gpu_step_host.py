"""The end-to-end entry elsaa_step_host copies a step's inputs from pinned host memory,
runs the forward and backward and copies O, dQ, dK, dV back, on three streams ordered by
the caller's events. With two device sets alternating and different inputs each step,
every step's host results must equal the device path's on the same inputs: bit for bit on
the bf16 path (its kernels are deterministic), to float32 rounding on the float32 path."""
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
    # no low-rank branch: W is not passed at all
    "rank0": (dict(N=128 * 3 + 5, d=128, block_size=128, topk=2, rank_r=0), {}),
    # the float32 path: single-key blocks, non-causal
    "f32": (dict(N=256, d=64, block_size=1, topk=32, rank_r=16, causal=False, dtype="f32"), {}),
}


@pytest.mark.parametrize("case", list(CASES))
def test_step_host_matches_the_device_path(case):
    shape, kw = CASES[case]
    w = small_workload(H=2, **shape)
    planes_h = torch.randn(w.d, 5, generator=torch.Generator().manual_seed(9)) if kw else None
    planes = planes_h.cuda() if kw else None
    op = gpu_op(w, lsh_planes=planes, **kw)
    steps = [device_inputs(w, make_inputs(w, seed)) for seed in range(4)]
    names = ("Q", "K", "V", "dO", "W") if w.rank_r > 0 else ("Q", "K", "V", "dO")
    host = [[steps[i][n].cpu().pin_memory() for n in names] for i in range(4)]
    if kw:
        host = [h + [planes_h.pin_memory()] for h in host]
    elif w.rank_r == 0:
        host = [h + [None] for h in host]
    dev_in = [[torch.empty_like(steps[0][n]) for n in names] + ([] if w.rank_r > 0 else [None]) for _ in range(2)]
    dev_out = [[op._empty_like_io() for _ in range(4)] for _ in range(2)]
    host_out = [[torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in dev_out[0]] for _ in range(4)]
    stream, s_in, s_out = torch.cuda.current_stream(), torch.cuda.Stream(), torch.cuda.Stream()
    events = [[torch.cuda.Event() for _ in range(3)] for _ in range(2)]
    for evs in events:                                # create the events (waiting on them is then a no-op)
        for e in evs:
            e.record(stream)
    for i in range(4):
        j = i % 2
        op.step_host(host[i], host_out[i], dev_in[j], dev_out[j], events[j], stream, s_in, s_out)
    torch.cuda.synchronize()
    assert op.check_device_flags() == 0
    for i in range(4):
        d = steps[i]
        O = op.forward(d["Q"], d["K"], d["V"], d["W"])
        grads = op.backward(d["Q"], d["K"], d["V"], d["W"], d["dO"])
        torch.cuda.synchronize()
        for name, h, ref in zip(("O", "dQ", "dK", "dV"), host_out[i], (O,) + grads):
            msg = f"{case}: step {i} {name} differs from the device path"
            if w.dtype == "f32":
                torch.testing.assert_close(h, ref.cpu(), rtol=1e-5, atol=1e-6, msg=msg)
            else:
                assert torch.equal(h, ref.cpu()), msg
