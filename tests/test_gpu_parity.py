"""CUDA path vs the float64 oracle, through the C ABI, on seeded inputs.

Small problems span several tiles and a ragged last tile and are compared
element by element; the named full-size workloads are compared on every
selected index and on sampled rows of O, dQ, dK and dV.
"""
import numpy as np
import pytest
import torch

from oracle import elsaa_oracle as orc
from sparse_rank_approximation_b200.workloads import WORKLOADS, make_inputs, small_workload
from tests.harness import check, check_fusion_grads, device_inputs, gpu_op, np64, oracle_params

pytestmark = pytest.mark.gpu

SMALL = {
    "bf16_d64_T64_causal_ragged": small_workload(N=64 * 5 + 37, d=64, block_size=64, topk=3, rank_r=32, H=2),
    "bf16_d128_T128_causal_ragged": small_workload(N=128 * 4 + 5, d=128, block_size=128, topk=2, rank_r=64, H=2),
    "bf16_d64_T128_noncausal": small_workload(N=128 * 3 + 50, d=64, block_size=128, topk=2, rank_r=16,
                                              causal=False),
    "bf16_d128_T128_r128_causal_ragged": small_workload(N=128 * 6 + 5, d=128, block_size=128, topk=3, rank_r=128,
                                                        H=2),
    "bf16_d128_T128_r128_noncausal": small_workload(N=128 * 3 + 50, d=128, block_size=128, topk=2, rank_r=128,
                                                    causal=False),
    "bf16_d128_T64_r256": small_workload(N=64 * 6, d=128, block_size=64, topk=4, rank_r=256, B=2, H=1),
    # feature counts that are not one group of 128 on the tensor-core RACE path: two groups,
    # a padded second group, and a single padded group
    "bf16_d128_T128_r256_causal_ragged": small_workload(N=128 * 5 + 9, d=128, block_size=128, topk=2, rank_r=256,
                                                        H=2),
    "bf16_d128_T128_r192_noncausal": small_workload(N=128 * 3 + 50, d=128, block_size=128, topk=2, rank_r=192,
                                                    causal=False),
    "bf16_d128_T128_r48_causal": small_workload(N=128 * 4, d=128, block_size=128, topk=3, rank_r=48, H=2),
    "bf16_all_blocks": small_workload(N=64 * 4, d=64, block_size=64, topk=4, rank_r=16, causal=False),
    "f32_config_tiny": WORKLOADS["tiny_f32"],
    "f32_T64_causal_ragged": small_workload(N=64 * 3 + 11, d=64, block_size=64, topk=2, rank_r=32, dtype="f32"),
    "f32_T1_causal": small_workload(N=200, d=128, block_size=1, topk=24, rank_r=48, dtype="f32", kind="iid"),
    "f32_T128_noncausal": small_workload(N=300, d=128, block_size=128, topk=2, rank_r=16, dtype="f32",
                                         causal=False),
}


def _run(w, seed=0, lam_vec=False, gates=False, **over):
    inp = make_inputs(w, seed)
    dev = device_inputs(w, inp)
    op = gpu_op(w, **{k: v for k, v in over.items() if k in ("lam", "eps", "tau", "fixed_m")})
    BH = (w.B, w.H, w.N)
    g = torch.Generator().manual_seed(seed + 100)
    extra_cpu = {}
    if lam_vec:
        extra_cpu["lam"] = torch.rand(BH, generator=g) * 2.0
    if gates:
        extra_cpu["g_s"] = torch.rand(BH, generator=g)
        extra_cpu["g_lr"] = torch.rand(BH, generator=g)
    extra = {k: v.cuda() for k, v in extra_cpu.items()}
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"], extra.get("lam"), extra.get("g_s"), extra.get("g_lr"))
    scores, idx = op.debug_select(dev["Q"], dev["K"])
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"], extra.get("lam"),
                             extra.get("g_s"), extra.get("g_lr"))
    torch.cuda.synchronize()
    _run.last = (op, dev, extra)
    return inp, extra_cpu, O, scores, idx, (dQ, dK, dV)


def _oracle_head(w, inp, extra, scores, b, h, **over):
    p = oracle_params(w, **over)
    get = lambda n: inp[n][b, h].double().numpy()
    ex = {k: v[b, h].double().numpy() for k, v in extra.items()}
    W = inp["W"].double().numpy()
    fw = orc.forward_head(get("Q"), get("K"), get("V"), W, p, ex.get("lam"), ex.get("g_s"), ex.get("g_lr"),
                          scores=np64(scores[b, h]))
    grads = orc.backward_head(get("Q"), get("K"), get("V"), W, get("dO"), fw, p, ex.get("lam"), ex.get("g_s"),
                              ex.get("g_lr"))
    return fw, grads


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_backward_small(name):
    w = SMALL[name]
    inp, extra, O, scores, idx, grads = _run(w)
    for b in range(w.B):
        for h in range(w.H):
            fw, (dq, dk, dv) = _oracle_head(w, inp, extra, scores, b, h)
            assert np.array_equal(idx[b, h].cpu().numpy(), fw["idx"]), "selection differs"
            check(w, f"O[{b},{h}]", np64(O[b, h]), fw["O"])
            check(w, f"dQ[{b},{h}]", np64(grads[0][b, h]), dq)
            check(w, f"dK[{b},{h}]", np64(grads[1][b, h]), dk)
            check(w, f"dV[{b},{h}]", np64(grads[2][b, h]), dv)


@pytest.mark.parametrize("case", ["k0", "r0_eps0", "lam_gates", "tau_lam", "noncausal", "fixed_m", "fixed_m_gates"])
@pytest.mark.parametrize("geom", ["bf16_d64_T64", "bf16_d128_T128", "bf16_d128_T128_r128", "f32_d64_T64"])
def test_branch_switches_and_options(case, geom):
    parts = geom.split("_")
    dtype, d, T = parts[0], int(parts[1][1:]), int(parts[2][1:])
    r = int(parts[3][1:]) if len(parts) > 3 else 32
    base = dict(N=T * 3 + 20, d=d, block_size=T, topk=2, rank_r=r, dtype=dtype, H=2)
    kw, over, lam_vec, gates = {}, {}, False, False
    if case == "k0":
        base["topk"] = 0
    elif case == "r0_eps0":
        base["rank_r"] = 0
        over["eps"] = 0.0
    elif case == "lam_gates":
        lam_vec = gates = True
    elif case == "tau_lam":
        over.update(tau=0.5, lam=3.0, eps=0.01)
    elif case == "noncausal":
        base["causal"] = False
    elif case == "fixed_m":
        over["fixed_m"] = True
    elif case == "fixed_m_gates":
        over["fixed_m"] = True
        lam_vec = gates = True
    w = small_workload(**base)
    inp, extra, O, scores, idx, grads = _run(w, lam_vec=lam_vec, gates=gates, **over)
    for h in range(w.H):
        fw, (dq, dk, dv) = _oracle_head(w, inp, extra, scores, 0, h, **over)
        check(w, "O", np64(O[0, h]), fw["O"])
        check(w, "dQ", np64(grads[0][0, h]), dq)
        check(w, "dK", np64(grads[1][0, h]), dk)
        check(w, "dV", np64(grads[2][0, h]), dv)


@pytest.mark.parametrize("gates", [False, True])
@pytest.mark.parametrize("fixed_m", [False, True])
@pytest.mark.parametrize("geom", ["bf16_d128_T128_r128", "bf16_d64_T64", "f32_d64_T64"])
def test_fusion_parameter_gradients(geom, fixed_m, gates):
    """elsaa_fusion_grads (per-row d/dlambda, d/dg_s, d/dg_lr) against the oracle's."""
    parts = geom.split("_")
    dtype, d, T = parts[0], int(parts[1][1:]), int(parts[2][1:])
    r = int(parts[3][1:]) if len(parts) > 3 else 32
    w = small_workload(N=T * 3 + 20, d=d, block_size=T, topk=2, rank_r=r, dtype=dtype, H=2)
    over = {"fixed_m": fixed_m}
    inp, extra, O, scores, idx, grads = _run(w, lam_vec=True, gates=gates, **over)
    op, dev, extra_dev = _run.last
    dl, dgs, dgl = op.fusion_grads(dev["dO"], extra_dev.get("lam"), extra_dev.get("g_s"), extra_dev.get("g_lr"))
    torch.cuda.synchronize()
    for h in range(w.H):
        p = oracle_params(w, **over)
        fw, _ = _oracle_head(w, inp, extra, scores, 0, h, **over)
        ex = {k: v[0, h].double().numpy() for k, v in extra.items()}
        dO_h = inp["dO"][0, h].double().numpy()
        ref = orc.fusion_param_grads(dO_h, fw, p, ex.get("lam"), ex.get("g_s"), ex.get("g_lr"))
        check_fusion_grads(w, h, p, fw, ex, dO_h, (dl, dgs, dgl), ref)


@pytest.mark.parametrize("causal,k,r", [(False, 1, 0), (False, 1, 24), (False, 2, 0), (True, 2, 16)])
def test_rank_of_sparse_plus_low_rank_on_gpu_selection(causal, k, r):
    """[ELSAA §4] rank(S_Omega + B A) = min(n, nu(Omega) + r) on the support the GPU selector
    realised (elsaa_debug_select), evaluated in float64."""
    w = small_workload(N=256, d=64, block_size=64, topk=k, rank_r=16, causal=causal, H=2)
    inp = make_inputs(w, 3)
    dev = device_inputs(w, inp)
    op = gpu_op(w)
    _, idx = op.debug_select(dev["Q"], dev["K"])
    torch.cuda.synchronize()
    p = oracle_params(w)
    for h in range(w.H):
        out = orc.rank_diagnostic(np64(inp["Q"][0, h]), np64(inp["K"][0, h]), idx[0, h].cpu().numpy(), p, r,
                                  seed=h)
        assert out["rank"] == out["predicted"], out


@pytest.mark.parametrize("name", ["n2k_d64", "n8k_d64", "n16k_d128", "n64k_d128"])
def test_selection_full_size(name):
    """Bit-exact against the oracle fed the GPU's float32 scores; against the
    oracle's own float64 scores, differences only at near-ties (1e-6 relative)."""
    w = WORKLOADS[name]
    inp = make_inputs(w, 0)
    dev = device_inputs(w, inp)
    op = gpu_op(w)
    scores, idx = op.debug_select(dev["Q"], dev["K"])
    torch.cuda.synchronize()
    sc, ix = scores.cpu().numpy(), idx.cpu().numpy()
    p = oracle_params(w)
    for b in range(w.B):
        for h in range(w.H):
            assert np.array_equal(orc.select_from_scores(sc[b, h], w.topk, w.causal), ix[b, h])
    for b, h in [(0, 0), (w.B - 1, w.H - 1)]:
        s64 = orc.block_scores(inp["Q"][b, h].double().numpy(), inp["K"][b, h].double().numpy(), p)
        np.testing.assert_allclose(sc[b, h], s64, rtol=0, atol=2e-6 * max(1.0, np.abs(s64).max()))
        own = orc.select_from_scores(s64, w.topk, w.causal)
        for t in np.nonzero(np.any(own != ix[b, h], axis=1))[0]:
            a = set(own[t]) - set(ix[b, h, t])
            g = set(ix[b, h, t]) - set(own[t])
            for x, y in zip(sorted(a), sorted(g)):
                assert abs(s64[t, x] - s64[t, y]) <= 1e-6 * max(abs(s64[t, x]), abs(s64[t, y])), (t, x, y)


@pytest.mark.parametrize("name", ["n2k_d64", "n8k_d64", "n16k_d128", "n64k_d128"])
def test_forward_backward_full_size_sampled(name):
    """Full-size workload, launched exactly as the benchmark launches it; outputs
    compared on sampled rows of two heads."""
    w = WORKLOADS[name]
    inp = make_inputs(w, 0)
    dev = device_inputs(w, inp)
    op = gpu_op(w)
    O = op.forward(dev["Q"], dev["K"], dev["V"], dev["W"])
    scores, _ = op.debug_select(dev["Q"], dev["K"])
    dQ, dK, dV = op.backward(dev["Q"], dev["K"], dev["V"], dev["W"], dev["dO"])
    torch.cuda.synchronize()
    p = oracle_params(w)
    rng = np.random.default_rng(1)
    heads = [(0, 0), (w.B - 1, w.H - 1)] if name != "n64k_d128" else [(0, w.H - 1)]
    for b, h in heads:
        get = lambda n: inp[n][b, h].double().numpy()
        q, k, v, dO = get("Q"), get("K"), get("V"), get("dO")
        W = inp["W"].double().numpy()
        sc = np64(scores[b, h])
        rows = np.unique(np.concatenate([[0, w.N - 1, w.block_size - 1, w.block_size],
                                         rng.integers(0, w.N, 12)]))
        fr = orc.forward_rows_head(q, k, v, W, p, rows, scores=sc)
        check(w, "O rows", np64(O[b, h][rows]), fr["O"])
        fw = orc.forward_head(q, k, v, W, p, scores=sc)
        krows = np.unique(np.concatenate([[0, w.N - 1], rng.integers(0, w.N, 6)]))
        dq, dk, dv = orc.backward_rows_head(q, k, v, W, dO, fw, p, rows, krows)
        check(w, "dQ rows", np64(dQ[b, h][rows]), dq)
        check(w, "dK rows", np64(dK[b, h][krows]), dk)
        check(w, "dV rows", np64(dV[b, h][krows]), dv)


@pytest.mark.parametrize("causal", [True, False])
def test_race_statistics_in_multi_chunk_segments(causal):
    """Enough heads that the tensor-core RACE statistics walk segments of several chunks
    (40 heads: 3 segments per head, of 3, 3 and 1 chunks, the last one ragged), so the
    carried prefix inside a segment and the scanned carry between segments both matter;
    three heads against the oracle."""
    w = small_workload(N=128 * 6 + 5, d=128, block_size=128, topk=2, rank_r=128, H=40, causal=causal)
    inp, extra, O, scores, idx, grads = _run(w)
    for h in (0, 17, w.H - 1):
        fw, (dq, dk, dv) = _oracle_head(w, inp, extra, scores, 0, h)
        check(w, f"O[{h}]", np64(O[0, h]), fw["O"])
        check(w, f"dQ[{h}]", np64(grads[0][0, h]), dq)
        check(w, f"dK[{h}]", np64(grads[1][0, h]), dk)
        check(w, f"dV[{h}]", np64(grads[2][0, h]), dv)
