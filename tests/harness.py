"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and measure the differences."""
import numpy as np
import torch

from oracle import elsaa_oracle as orc
from sparse_rank_approximation_b200 import binding as bd
from sparse_rank_approximation_b200.workloads import Workload, make_inputs

# Tolerances (relative to the oracle, float64):
#   float32 path: max |gpu - oracle| / max |oracle| <= 1e-4 per output tensor;
#   bf16 path:    |gpu - oracle| <= 2e-2 + 2^-8 |oracle| element-wise (unit-variance
#                 V and dO): 2e-2 for the arithmetic plus the rounding of the bf16
#                 output itself, whose half-ulp is up to 2^-8 of the value (an
#                 output of magnitude 8 is already 0.03 away from its exact value).
F32_REL_TOL = 1e-4
BF16_ABS_TOL = 2e-2
BF16_STORE_REL = 2.0 ** -8


def oracle_params(w: Workload, **kw) -> orc.Params:
    p = orc.Params(N=w.N, d=w.d, block_size=w.block_size, topk=w.topk, rank_r=w.rank_r,
                   causal=w.causal, scale=w.scale, hash_bits=w.hash_bits)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def gpu_op(w: Workload, lsh_planes=None, **kw) -> bd.Elsaa:
    p = bd.make_params(w.B, w.H, w.N, w.d,
                       dtype=bd.ELSAA_DTYPE_BF16 if w.dtype == "bf16" else bd.ELSAA_DTYPE_F32,
                       causal=w.causal, rank_r=w.rank_r, block_size=w.block_size, topk=w.topk,
                       scale=w.scale, **kw)
    return bd.Elsaa(p, torch.device("cuda", 0), lsh_planes=lsh_planes)


def device_inputs(w: Workload, inp: dict) -> dict:
    dev = torch.device("cuda", 0)
    suffix = "16" if w.dtype == "bf16" else ""
    out = {n: inp[n + suffix].to(dev) for n in ("Q", "K", "V", "dO")}
    out["W"] = inp["W"].to(dev)
    return out


def np64(t) -> np.ndarray:
    return t.detach().cpu().double().numpy()


def check(w: Workload, name: str, gpu: np.ndarray, ref: np.ndarray):
    err = np.abs(gpu - ref).max()
    assert np.all(np.isfinite(gpu)), f"{name}: non-finite values"
    if w.dtype == "f32":
        rel = err / max(np.abs(ref).max(), 1e-30)
        assert rel <= F32_REL_TOL, f"{name}: max rel err {rel:.3e} > {F32_REL_TOL}"
        return rel
    excess = (np.abs(gpu - ref) - BF16_STORE_REL * np.abs(ref)).max()
    assert excess <= BF16_ABS_TOL, (f"{name}: max abs err {err:.3e}, beyond bf16 storage {excess:.3e} > "
                                    f"{BF16_ABS_TOL} (max |ref| {np.abs(ref).max():.3f})")
    return err


def check_fusion_grads(w: Workload, h: int, p: orc.Params, fw: dict, ex: dict, dO_h: np.ndarray, got, ref):
    """elsaa_fusion_grads outputs (dlambda, dg_s, dg_lr) of head h against the oracle's.

    float32: the usual relative bound.  bf16: the GPU reduces over the saved bf16 O_s and
    O_lr, each element within half an ulp (2^-9 relative) of the exact value, so row i's
    dot product is off by at most 2^-9 sum_k |dO_ik O_ik|; the bound doubles that, carries
    it through d m / d lambda, and adds the usual 2e-2.
    """
    if w.dtype == "f32":
        for name, g, want in zip(("dlambda", "dg_s", "dg_lr"), got, ref):
            check(w, f"{name}[{h}]", np64(g[0, h]), want)
        return
    sa = np.abs(dO_h * fw["O_s"]).sum(axis=1)
    sb = np.abs(dO_h * fw["O_lr"]).sum(axis=1)
    gs = ex.get("g_s", np.ones(w.N))
    ds = np.exp(fw["logd_s"])
    lam = ex.get("lam", np.full(w.N, p.lam))
    D = ds + lam * fw["d_lr"] + p.eps
    dm_bound = gs * sa + (0.0 if "g_lr" in ex else sb)
    bounds = (np.where(p.fixed_m, 0.0, ds * fw["d_lr"] / D ** 2 * dm_bound), fw["m"] * sa, sb)
    for name, g, want, bnd in zip(("dlambda", "dg_s", "dg_lr"), got, ref, bounds):
        err = np.abs(np64(g[0, h]) - want)
        assert np.all(err <= BF16_ABS_TOL + 2.0 ** -8 * bnd), f"{name}[{h}]: max err {err.max():.3e}"


def sparse_rounding_scales(q, k, v, dO, fw, p, lam=None, g_s=None, g_lr=None):
    """Per-element scales of the bf16 rounding inside the sparse backward, from the oracle's
    own quantities: dS is rounded before dS K and dS^T Q, P before P^T dO_s, and Delta is a
    row sum over the bf16-saved O_s, so it is off by up to 2^-9 sum_c |dO_s,ic O_s,ic|, which
    every dS_ij = P_ij (dP_ij - Delta_i) inherits times P_ij.  When one key dominates a row,
    dP_ij and Delta_i nearly cancel and that last term is the whole of dS_ij's error."""
    dOs, _, dds_ds, _ = orc._fusion_adjoints(dO, fw, p, lam, g_s, g_lr)
    Delta = (dOs * fw["O_s"]).sum(axis=1) - dds_ds
    eD = (np.abs(dOs) * np.abs(fw["O_s"])).sum(axis=1)
    Bq, Bk, Bv = np.zeros_like(q), np.zeros_like(k), np.zeros_like(v)
    sup = orc.lsh_support(q, k, p) if p.selector == "sortlsh" else orc.support(fw["idx"], p)
    for i, keys in enumerate(sup):
        if keys.size == 0:
            continue
        P = np.exp(p.scale * (k[keys] @ q[i]) - fw["logd_s"][i])
        dz = np.abs(P * (v[keys] @ dOs[i] - Delta[i])) + P * eD[i]
        Bq[i] += p.scale * dz @ np.abs(k[keys])
        Bk[keys] += p.scale * np.outer(dz, np.abs(q[i]))
        Bv[keys] += np.outer(P, np.abs(dOs[i]))
    return Bq, Bk, Bv
