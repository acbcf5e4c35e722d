"""sortLSH selector [ELSAA §3.2] through the C ABI against the float64 oracle.

The hash codes are compared bit for bit (a mismatch is allowed only where a projection
is within float32 rounding of zero); the outputs and gradients are compared with the
oracle run on the same sorted orders, for the tensor-core (every bf16 shape) and float32 paths.
"""
import numpy as np
import pytest
import torch

from oracle import elsaa_oracle as orc
from sparse_rank_approximation_b200 import binding as bd
from sparse_rank_approximation_b200.workloads import WORKLOADS, make_inputs, small_workload
from tests.harness import check, check_fusion_grads, device_inputs, gpu_op, np64, oracle_params

pytestmark = pytest.mark.gpu

GEOMS = {
    "bf16_d128_T128_r128": dict(N=128 * 4 + 44, d=128, block_size=128, rank_r=128, dtype="bf16"),
    "bf16_d64_T64_r32": dict(N=64 * 5 + 11, d=64, block_size=64, rank_r=32, dtype="bf16"),
    "f32_d64_T64_r16": dict(N=64 * 3 + 20, d=64, block_size=64, rank_r=16, dtype="f32"),
}


def _setup(geom, bits, seed=0, fixed_m=False):
    w = small_workload(topk=1, causal=False, H=2, **GEOMS[geom])
    inp = make_inputs(w, seed)
    dev = device_inputs(w, inp)
    g = torch.Generator().manual_seed(seed + 7)
    R = torch.randn(w.d, bits, generator=g)
    p = bd.make_params(w.B, w.H, w.N, w.d, dtype=bd.ELSAA_DTYPE_BF16 if w.dtype == "bf16" else bd.ELSAA_DTYPE_F32,
                       causal=False, rank_r=w.rank_r, block_size=w.block_size, topk=1, scale=w.scale,
                       fixed_m=fixed_m, selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=bits)
    op = bd.Elsaa(p, torch.device("cuda", 0), lsh_planes=R.cuda())
    return w, inp, dev, R, op


def _oracle_params(w, R, orders, fixed_m=False):
    p = oracle_params(w, fixed_m=fixed_m)
    p.selector = "sortlsh"
    p.lsh_planes = R.double().numpy()
    p.lsh_orders = orders
    return p


@pytest.mark.parametrize("geom", list(GEOMS))
@pytest.mark.parametrize("bits", [1, 4, 9, 16])
def test_codes_and_orders(geom, bits):
    w, inp, dev, R, op = _setup(geom, bits)
    codes, order = op.debug_sortlsh(dev["Q"], dev["K"])
    torch.cuda.synchronize()
    Rn = R.double().numpy()
    for h in range(w.H):
        for side, name in ((0, "Q"), (1, "K")):
            X = inp[name][0, h].double().numpy()
            ref = orc.simhash_codes(X, Rn)
            got = codes[0, h, side].cpu().numpy()
            proj = X @ Rn
            near = np.abs(proj) <= 1e-5 * np.linalg.norm(X, axis=1)[:, None] * np.linalg.norm(Rn, axis=0)[None, :]
            diff = (got ^ ref)[:, None] >> np.arange(bits)[None, :] & 1
            assert not np.any(diff.astype(bool) & ~near), f"{name}[{h}]: code bits differ away from zero"
            if np.array_equal(got, ref):
                assert np.array_equal(order[0, h, side].cpu().numpy(), orc.sortlsh_order(X, Rn))
            # the order is a permutation sorted by Gray position of the GPU's own codes, ties by row
            o = order[0, h, side].cpu().numpy()
            assert np.array_equal(np.sort(o), np.arange(w.N))
            pos = orc.gray_rank(got)[o]
            assert np.all(np.diff(pos) >= 0) and np.all(np.diff(o)[np.diff(pos) == 0] > 0)


@pytest.mark.parametrize("geom", list(GEOMS))
@pytest.mark.parametrize("gates,fixed_m", [(False, False), (True, False), (True, True)])
def test_forward_backward(geom, gates, fixed_m):
    w, inp, dev, R, op = _setup(geom, 6, seed=1, fixed_m=fixed_m)
    BH = (w.B, w.H, w.N)
    g = torch.Generator().manual_seed(11)
    extra = {}
    if gates:
        extra = {"lam": torch.rand(BH, generator=g) * 2.0, "g_s": torch.rand(BH, generator=g),
                 "g_lr": torch.rand(BH, generator=g)}
    ex_dev = {k: v.cuda() for k, v in extra.items()}
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"], ex_dev.get("lam"), ex_dev.get("g_s"), ex_dev.get("g_lr"))
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"], ex_dev.get("lam"),
                             ex_dev.get("g_s"), ex_dev.get("g_lr"))
    dl, dgs, dgl = op.fusion_grads(dev["dO"], ex_dev.get("lam"), ex_dev.get("g_s"), ex_dev.get("g_lr"))
    _, order = op.debug_sortlsh(dev["Q"], dev["K"])
    torch.cuda.synchronize()
    W = inp["W"].double().numpy()
    for h in range(w.H):
        orders = (order[0, h, 0].cpu().numpy(), order[0, h, 1].cpu().numpy())
        p = _oracle_params(w, R, orders, fixed_m)
        get = lambda n: inp[n][0, h].double().numpy()
        ex = {k: v[0, h].double().numpy() for k, v in extra.items()}
        fw = orc.forward_head(get("Q"), get("K"), get("V"), W, p, ex.get("lam"), ex.get("g_s"), ex.get("g_lr"))
        dq, dk, dv = orc.backward_head(get("Q"), get("K"), get("V"), W, get("dO"), fw, p, ex.get("lam"),
                                       ex.get("g_s"), ex.get("g_lr"))
        check(w, f"O[{h}]", np64(O[0, h]), fw["O"])
        check(w, f"dQ[{h}]", np64(dQ[0, h]), dq)
        check(w, f"dK[{h}]", np64(dK[0, h]), dk)
        check(w, f"dV[{h}]", np64(dV[0, h]), dv)
        ref = orc.fusion_param_grads(get("dO"), fw, p, ex.get("lam"), ex.get("g_s"), ex.get("g_lr"))
        check_fusion_grads(w, h, p, fw, ex, get("dO"), (dl, dgs, dgl), ref)


def test_full_size():
    """The full-length sortLSH workload (B1 H32 N16384 d128, 7-bit codes), launched as the
    benchmark launches it; every row of two heads against the oracle on the GPU's orders."""
    w = WORKLOADS["n16k_d128_sortlsh"]
    inp = make_inputs(w, 0)
    dev = device_inputs(w, inp)
    R = inp["R"]
    op = gpu_op(w, selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=w.lsh_bits, lsh_planes=R.cuda())
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"])
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"])
    _, order = op.debug_sortlsh(dev["Q"], dev["K"])
    torch.cuda.synchronize()
    W = inp["W"].double().numpy()
    for h in (0, w.H - 1):
        get = lambda n: inp[n][0, h].double().numpy()
        p = _oracle_params(w, R, (order[0, h, 0].cpu().numpy(), order[0, h, 1].cpu().numpy()))
        fw = orc.forward_head(get("Q"), get("K"), get("V"), W, p)
        dq, dk, dv = orc.backward_head(get("Q"), get("K"), get("V"), W, get("dO"), fw, p)
        check(w, f"O[{h}]", np64(O[0, h]), fw["O"])
        # at this length sorted blocks put most of a row's mass on a few keys, where
        # dP_ij and Delta_i nearly cancel: Delta comes from the fp32 O_s
        check(w, f"dQ[{h}]", np64(dQ[0, h]), dq)
        check(w, f"dK[{h}]", np64(dK[0, h]), dk)
        check(w, f"dV[{h}]", np64(dV[0, h]), dv)


@pytest.mark.parametrize("N", [20000, 65536])
def test_long_heads_sort_through_global_memory(N):
    """Heads longer than a shared-memory sort takes (N > 16384) are sorted through global
    memory, one 8-bit pass after another: the orders are permutations sorted by the Gray
    position of the GPU's own codes, ties by row, and equal the oracle's where the codes agree."""
    w = small_workload(N=N, d=64, block_size=64, topk=1, rank_r=16, causal=False, dtype="bf16", H=1)
    inp = make_inputs(w, 5)
    dev = device_inputs(w, inp)
    R = torch.randn(w.d, 12, generator=torch.Generator().manual_seed(12))
    op = gpu_op(w, selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=12, lsh_planes=R.cuda())
    codes, order = op.debug_sortlsh(dev["Q"], dev["K"])
    torch.cuda.synchronize()
    Rn = R.double().numpy()
    for side, name in ((0, "Q"), (1, "K")):
        got = codes[0, 0, side].cpu().numpy()
        o = order[0, 0, side].cpu().numpy()
        assert np.array_equal(np.sort(o), np.arange(w.N))
        pos = orc.gray_rank(got)[o]
        assert np.all(np.diff(pos) >= 0) and np.all(np.diff(o)[np.diff(pos) == 0] > 0)
        X = inp[name][0, 0].double().numpy()
        if np.array_equal(got, orc.simhash_codes(X, Rn)):
            assert np.array_equal(o, orc.sortlsh_order(X, Rn))


def test_long_forward_backward():
    """Non-causal sortLSH at N = 32768 (its sort goes through global memory): every row of one
    head's O, and dQ on every 16th sorted query block, against the oracle on the GPU's orders (sparse
    branch only: the low-rank branch does not depend on the length of the sort, and the oracle's
    at this length takes minutes)."""
    w = small_workload(N=32768, d=128, block_size=128, topk=1, rank_r=0, causal=False, dtype="bf16", H=1)
    inp = make_inputs(w, 2)
    dev = device_inputs(w, inp)
    R = torch.randn(w.d, 8, generator=torch.Generator().manual_seed(3))
    op = gpu_op(w, selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=8, lsh_planes=R.cuda())
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"])
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"])
    _, order = op.debug_sortlsh(dev["Q"], dev["K"])
    assert op.check_device_flags() == 0
    torch.cuda.synchronize()
    W = inp["W"].double().numpy()
    get = lambda n: inp[n][0, 0].double().numpy()
    p = _oracle_params(w, R, (order[0, 0, 0].cpu().numpy(), order[0, 0, 1].cpu().numpy()))
    fw = orc.forward_head(get("Q"), get("K"), get("V"), W, p)
    check(w, "O", np64(O[0, 0]), fw["O"])
    # dQ of a row comes from that row's support alone: every 16th sorted query block, all its rows
    tiles = list(range(0, w.n_tiles, 16))
    dq, _, _ = orc.backward_head(get("Q"), get("K"), get("V"), W, get("dO"), fw, p, tiles=tiles)
    oq = p.lsh_orders[0]
    rows = np.concatenate([oq[t * w.block_size:(t + 1) * w.block_size] for t in tiles])
    check(w, "dQ", np64(dQ[0, 0])[rows], dq[rows])


# ---- the causal recursion (bf16, d = 128, block 128 on the tensor-core kernels) ----

def _causal_setup(N, r, seed, fixed_m=False, bits=6, H=2, d=128, T=128):
    w = small_workload(N=N, d=d, block_size=T, topk=2, rank_r=r, causal=True, dtype="bf16", H=H)
    inp = make_inputs(w, seed)
    dev = device_inputs(w, inp)
    g = torch.Generator().manual_seed(seed + 7)
    R = torch.randn(w.d, bits, generator=g)
    op = gpu_op(w, fixed_m=fixed_m, selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=bits, lsh_planes=R.cuda())
    return w, inp, dev, R, op


def _causal_oracle_params(w, R, codes, h, fixed_m=False):
    p = oracle_params(w, fixed_m=fixed_m)
    p.selector = "sortlsh"
    p.lsh_planes = R.double().numpy()
    p.lsh_codes = (codes[0, h, 0].cpu().numpy(), codes[0, h, 1].cpu().numpy())
    return p


@pytest.mark.parametrize("bits", [1, 12])
def test_causal_hash_widths(bits):
    """The causal recursion with 1-bit codes (one sort pass, two buckets) and 12-bit codes
    (two 8-bit passes in every level sort)."""
    w, inp, dev, R, op = _causal_setup(1024, 128, seed=4, bits=bits)
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"])
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"])
    codes, _ = op.debug_sortlsh(dev["Q"], dev["K"])
    assert op.check_device_flags() == 0
    torch.cuda.synchronize()
    W = inp["W"].double().numpy()
    for h in range(w.H):
        p = _causal_oracle_params(w, R, codes, h)
        get = lambda n: inp[n][0, h].double().numpy()
        fw = orc.forward_head(get("Q"), get("K"), get("V"), W, p)
        dq, dk, dv = orc.backward_head(get("Q"), get("K"), get("V"), W, get("dO"), fw, p)
        check(w, f"O[{h}]", np64(O[0, h]), fw["O"])
        check(w, f"dQ[{h}]", np64(dQ[0, h]), dq)
        check(w, f"dK[{h}]", np64(dK[0, h]), dk)
        check(w, f"dV[{h}]", np64(dV[0, h]), dv)


@pytest.mark.parametrize("N,r,gates,fixed_m,d,T", [(1024, 128, False, False, 128, 128),
                                                   (1024, 128, True, False, 128, 128),
                                                   (2048, 64, False, False, 128, 128),
                                                   (1024, 0, False, False, 128, 128),
                                                   (1024, 128, True, True, 128, 128),
                                                   (128, 128, False, False, 128, 128),
                                                   (256, 128, False, False, 128, 128),
                                                   (1024, 32, False, False, 64, 64),
                                                   (512, 64, True, False, 64, 64),
                                                   (1024, 0, False, True, 64, 64),
                                                   (1024, 64, False, False, 64, 128),
                                                   (512, 64, True, False, 128, 64)])
def test_causal_forward_backward(N, r, gates, fixed_m, d, T):
    """O, dQ, dK, dV and the fusion gradients against the oracle's recursion run on the GPU's
    hash codes (every level's sorted order follows from them), for d = 64 and 128 and blocks of 64
    and 128 keys (pair mode at 64); N = 128 and 256 at block 128 are the single-block and
    two-block cases (exact causal attention)."""
    w, inp, dev, R, op = _causal_setup(N, r, seed=3, fixed_m=fixed_m, d=d, T=T)
    BH = (w.B, w.H, w.N)
    g = torch.Generator().manual_seed(13)
    extra = {}
    if gates:
        extra = {"lam": torch.rand(BH, generator=g) * 2.0, "g_s": torch.rand(BH, generator=g),
                 "g_lr": torch.rand(BH, generator=g)}
    ex_dev = {k: v.cuda() for k, v in extra.items()}
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"], ex_dev.get("lam"), ex_dev.get("g_s"), ex_dev.get("g_lr"))
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"], ex_dev.get("lam"),
                             ex_dev.get("g_s"), ex_dev.get("g_lr"))
    dl, dgs, dgl = op.fusion_grads(dev["dO"], ex_dev.get("lam"), ex_dev.get("g_s"), ex_dev.get("g_lr"))
    codes, _ = op.debug_sortlsh(dev["Q"], dev["K"])
    assert op.check_device_flags() == 0
    torch.cuda.synchronize()
    W = inp["W"].double().numpy()
    for h in range(w.H):
        p = _causal_oracle_params(w, R, codes, h, fixed_m)
        get = lambda n: inp[n][0, h].double().numpy()
        ex = {k: v[0, h].double().numpy() for k, v in extra.items()}
        fw = orc.forward_head(get("Q"), get("K"), get("V"), W, p, ex.get("lam"), ex.get("g_s"), ex.get("g_lr"))
        dq, dk, dv = orc.backward_head(get("Q"), get("K"), get("V"), W, get("dO"), fw, p, ex.get("lam"),
                                       ex.get("g_s"), ex.get("g_lr"))
        check(w, f"O[{h}]", np64(O[0, h]), fw["O"])
        check(w, f"dQ[{h}]", np64(dQ[0, h]), dq)
        check(w, f"dK[{h}]", np64(dK[0, h]), dk)
        check(w, f"dV[{h}]", np64(dV[0, h]), dv)
        ref = orc.fusion_param_grads(get("dO"), fw, p, ex.get("lam"), ex.get("g_s"), ex.get("g_lr"))
        check_fusion_grads(w, h, p, fw, ex, get("dO"), (dl, dgs, dgl), ref)


def test_causal_long_halves_sort_through_global_memory():
    """The causal recursion at N = 65536 (8 sorted levels; the first level's halves of 32768
    rows sort through global memory): one head's O, and dQ on every 16th query tile, against the
    oracle on the GPU's codes (sparse branch only, as in the long non-causal test)."""
    w, inp, dev, R, op = _causal_setup(65536, 0, seed=6, bits=7, H=1)
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"])
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"])
    codes, _ = op.debug_sortlsh(dev["Q"], dev["K"])
    assert op.check_device_flags() == 0
    torch.cuda.synchronize()
    W = inp["W"].double().numpy()
    get = lambda n: inp[n][0, 0].double().numpy()
    p = _causal_oracle_params(w, R, codes, 0)
    fw = orc.forward_head(get("Q"), get("K"), get("V"), W, p)
    check(w, "O", np64(O[0, 0]), fw["O"])
    # dQ of a row comes from that row's support alone: every 16th query tile, all its rows
    tiles = list(range(0, w.n_tiles, 16))
    dq, _, _ = orc.backward_head(get("Q"), get("K"), get("V"), W, get("dO"), fw, p, tiles=tiles)
    rows = np.concatenate([np.arange(t * w.block_size, min(w.N, (t + 1) * w.block_size)) for t in tiles])
    check(w, "dQ", np64(dQ[0, 0])[rows], dq[rows])


def test_causal_full_size():
    """The full-length causal sortLSH workload (B1 H32 N16384 d128, 7-bit codes, six sorted
    levels), launched as the benchmark launches it; every row of two heads."""
    w = WORKLOADS["n16k_d128_sortlsh_causal"]
    inp = make_inputs(w, 0)
    dev = device_inputs(w, inp)
    R = inp["R"]
    op = gpu_op(w, selector=bd.ELSAA_SEL_SORTLSH, lsh_bits=w.lsh_bits, lsh_planes=R.cuda())
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"])
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"])
    codes, _ = op.debug_sortlsh(dev["Q"], dev["K"])
    assert op.check_device_flags() == 0
    torch.cuda.synchronize()
    W = inp["W"].double().numpy()
    for h in (0, w.H - 1):
        get = lambda n: inp[n][0, h].double().numpy()
        p = _causal_oracle_params(w, R, codes, h)
        fw = orc.forward_head(get("Q"), get("K"), get("V"), W, p)
        dq, dk, dv = orc.backward_head(get("Q"), get("K"), get("V"), W, get("dO"), fw, p)
        check(w, f"O[{h}]", np64(O[0, h]), fw["O"])
        check(w, f"dQ[{h}]", np64(dQ[0, h]), dq)
        check(w, f"dK[{h}]", np64(dK[0, h]), dk)
        check(w, f"dV[{h}]", np64(dV[0, h]), dv)
