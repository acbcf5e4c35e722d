"""Shared helpers for the GPU parity tests: run the CUDA path through the C ABI
and the oracle on the same seeded inputs, and measure the differences."""
import os

import numpy as np
import torch

from oracle import elsaa_oracle as orc
from sparse_rank_approximation_b200 import binding as bd
from sparse_rank_approximation_b200.workloads import Workload, make_inputs

# Tolerances against the float64 oracle (unit-variance V and dO):
#   float32 path: max |gpu - oracle| / max |oracle| <= 1e-4 per output tensor (the
#                 relative error of the tensor as a whole: element-wise relative
#                 error has no meaning at gradient entries that cancel to ~0);
#   bf16 path, O: |gpu - oracle| <= 2e-2 element-wise;
#   bf16 path, dQ, dK, dV: |gpu - oracle| <= 2e-2 + 2^-8 |oracle| element-wise: 2e-2 for
#                 the arithmetic plus the rounding of the bf16 gradient itself, whose
#                 half-ulp is up to 2^-8 of its value (a gradient of magnitude 8 is
#                 already 0.03 away from its exact value once stored in bf16).
F32_REL_TOL = 1e-4
BF16_ABS_TOL = 2e-2
BF16_STORE_REL = 2.0 ** -8

# (test, workload, tensor, max abs error, margin used of the bound) of every check, for
# the summary table conftest prints at the end of the run
RECORDS = []


def _record(w, name, err, used):
    test = os.environ.get("PYTEST_CURRENT_TEST", "").split(" ")[0]
    RECORDS.append((test, w.describe(), name, float(err), float(used)))


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
    """One output tensor against the oracle; a name starting with "O" is the operator's
    output (strict bound), anything else a gradient."""
    err = np.abs(gpu - ref).max()
    assert np.all(np.isfinite(gpu)), f"{name}: non-finite values"
    if w.dtype == "f32":
        rel = err / max(np.abs(ref).max(), 1e-30)
        _record(w, name, rel, rel / F32_REL_TOL)
        assert rel <= F32_REL_TOL, f"{name}: max rel err {rel:.3e} > {F32_REL_TOL}"
        return rel
    if name.startswith("O"):
        _record(w, name, err, err / BF16_ABS_TOL)
        assert err <= BF16_ABS_TOL, f"{name}: max abs err {err:.3e} > {BF16_ABS_TOL}"
        return err
    excess = (np.abs(gpu - ref) - BF16_STORE_REL * np.abs(ref)).max()
    _record(w, name, err, excess / BF16_ABS_TOL)
    assert excess <= BF16_ABS_TOL, (f"{name}: max abs err {err:.3e}, beyond the gradient's own bf16 rounding "
                                    f"{excess:.3e} > {BF16_ABS_TOL} (max |ref| {np.abs(ref).max():.3f})")
    return err


def check_fusion_grads(w: Workload, h: int, p: orc.Params, fw: dict, ex: dict, dO_h: np.ndarray, got, ref):
    """elsaa_fusion_grads outputs (dlambda, dg_s, dg_lr) of head h against the oracle's.

    float32: the usual relative bound.  bf16 (a reading of the bf16 bar for these per-row
    scalars): the GPU reduces dO against the saved bf16 O_lr, each element within half an
    ulp (2^-9 relative), so that dot product is off by up to 2^-9 sum_k |dO_ik O_lr,ik|;
    against O_s it reduces over an fp32 copy whose forward products rounded the softmax
    weights to bf16 (2^-9 relative each), and the same form over O_s is the allowance for
    that.  The bound doubles both, carries them through d m / d lambda, and adds 2e-2.
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
        _record(w, f"{name}[{h}]", err.max(), (err - 2.0 ** -8 * bnd).max() / BF16_ABS_TOL)
        assert np.all(err <= BF16_ABS_TOL + 2.0 ** -8 * bnd), f"{name}[{h}]: max err {err.max():.3e}"
