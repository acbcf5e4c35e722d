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


def gpu_op(w: Workload, **kw) -> bd.Elsaa:
    p = bd.make_params(w.B, w.H, w.N, w.d,
                       dtype=bd.ELSAA_DTYPE_BF16 if w.dtype == "bf16" else bd.ELSAA_DTYPE_F32,
                       causal=w.causal, rank_r=w.rank_r, block_size=w.block_size, topk=w.topk,
                       scale=w.scale, **kw)
    return bd.Elsaa(p, torch.device("cuda", 0))


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
