"""Host logic of bench.py: the work model behind the roofline line (no GPU needed)."""
import bench
from sparse_rank_approximation_b200.workloads import WORKLOADS

PEAKS = {"hbm_gbs": 6551.0, "bf16_tflops": 1646.8, "bf16_tflops_sustained": 1398.0}


def _bound(entry):
    t_f = entry["flops"] / (PEAKS["bf16_tflops_sustained"] * 1e12)
    t_b = entry["bytes"] / (PEAKS["hbm_gbs"] * 1e9)
    return "tensor" if t_f >= t_b else "hbm"


def test_selected_pairs_count_the_causal_triangle():
    """Causal top-k: tile t has min(k, t + 1) eligible blocks; non-causal: k each."""
    for name in ("n2k_d64", "n16k_d128", "n64k_d128"):
        w = WORKLOADS[name]
        brute = sum(min(w.topk, t + 1) for t in range(w.n_tiles))
        assert bench.selected_blocks_per_head(w) == brute
    w = WORKLOADS["n16k_d128_sortlsh"]
    assert bench.selected_blocks_per_head(w) == w.n_tiles


def test_every_dominant_kernel_has_a_work_model_entry():
    """The kernels that dominate some workload's step get a roofline (positive bytes; the
    tensor-core ones positive flops too)."""
    for name, w in WORKLOADS.items():
        m, tot = bench.work_model(w)
        for k in ("attn_fwd_tc", "dq_tc", "dkdv_tc", "race_k_bwd_tc", "race_q_bwd_tc", "race_readout_tc",
                  "race_features_tc", "race_stats_fwd_totals", "race_stats_bwd_totals"):
            assert m[k]["bytes"] > 0, (name, k)
        for k in ("attn_fwd_tc", "dq_tc", "dkdv_tc"):
            assert m[k]["flops"] > 0 or w.topk == 0, (name, k)
        if w.selector == "sortlsh":
            assert {"sortlsh_order", "sortlsh_gather", "sortlsh_scatter"} <= set(m)


def test_bound_follows_the_longer_of_flop_and_byte_time():
    """At the headline dK/dV is tensor-bound; with one key block per tile (sortLSH) the same
    kernel is bound by HBM."""
    m, _ = bench.work_model(WORKLOADS["n16k_d128"])
    assert _bound(m["dkdv_tc"]) == "tensor"
    m, _ = bench.work_model(WORKLOADS["n16k_d128_sortlsh"])
    assert _bound(m["dkdv_tc"]) == "hbm"


def test_whole_step_roofline_is_consistent():
    w = WORKLOADS["n16k_d128"]
    r = bench.whole_step_roofline(w, PEAKS, 5.0)
    assert r["t_roof_ms"] > 0 and 0 < r["frac"] < 1
    assert abs(r["frac"] - r["t_roof_ms"] / 5.0) < 1e-12
    assert r["bound"] in ("tensor", "hbm")
