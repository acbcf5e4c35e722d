"""Seeded synthetic workloads for the ELSAA attention operator.

This module only draws random numbers and describes shapes.  It holds none of
the operator's arithmetic, so the CPU oracle (test infrastructure) and the CUDA
path can both take their inputs from it without sharing any of the method.

Recipe (all draws from one ``torch.Generator`` seeded with ``seed``, in this
fixed order, on the CPU, in float32; bf16 workloads round the float32 draws):

* ``iid``: Q, K, V ~ N(0, 1) element-wise.
* ``clustered``: per (batch, head) ``n_centroids`` centroids ~ N(0, 1)^d; each
  query row and each key row picks a centroid uniformly at random (independent
  for Q and K, natural token order); Q_i = c[a_i] + sigma * N(0, 1),
  K_j = c[b_j] + sigma * N(0, 1); V ~ N(0, 1).
* then dO ~ N(0, 1) (same shape as Q), then the RACE hash hyperplanes
  W ~ N(0, 1) of shape [L, d, gamma] shared by every batch and head.

The five named workloads follow the long-context training shapes the operator
is meant for: a tiny fp32 check instance and four clustered bf16 causal ones,
the largest at N = 65536.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import torch

HASH_BITS = 4  # gamma: bits per RACE table, so each table has 2**gamma buckets


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    dtype: str            # "f32" or "bf16"
    causal: bool
    rank_r: int           # r = L * 2**gamma
    block_size: int       # keys per block == queries per tile
    topk: int             # selected blocks per query tile
    kind: str = "clustered"   # "iid" or "clustered"
    n_centroids: int = 0
    sigma: float = 0.3
    backward: bool = True
    hash_bits: int = HASH_BITS
    selector: str = "topk"    # "topk" (top-k blocks by pooled score) or "sortlsh"
    lsh_bits: int = 0         # sortLSH: bits of the angular hash code

    @property
    def n_tables(self) -> int:
        return self.rank_r // (1 << self.hash_bits)

    @property
    def scale(self) -> float:
        return 1.0 / (self.d ** 0.5)

    @property
    def n_tiles(self) -> int:
        return -(-self.N // self.block_size)

    def describe(self) -> str:
        return (f"B{self.B} H{self.H} N{self.N} d{self.d} {self.dtype} "
                f"{'causal' if self.causal else 'non-causal'} r{self.rank_r} "
                + (f"block{self.block_size} sortLSH{self.lsh_bits}" if self.selector == "sortlsh"
                   else f"block{self.block_size} top{self.topk}"))


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", 1, 1, 256, 64, "f32", False, 16, 1, 32,
                         kind="iid", backward=False),
    "n2k_d64": Workload("n2k_d64", 2, 8, 2048, 64, "bf16", True, 64, 64, 8,
                        n_centroids=32, sigma=0.3),
    "n8k_d64": Workload("n8k_d64", 4, 16, 8192, 64, "bf16", True, 128, 64, 16,
                        n_centroids=128, sigma=0.3),
    "n16k_d128": Workload("n16k_d128", 1, 32, 16384, 128, "bf16", True, 128, 128, 16,
                          n_centroids=256, sigma=0.5),
    # the headline shape, non-causal, with the sortLSH selector: 2^7 hash buckets for the
    # 128 blocks of 128 rows
    "n16k_d128_sortlsh": Workload("n16k_d128_sortlsh", 1, 32, 16384, 128, "bf16", False, 128, 128, 1,
                                  n_centroids=256, sigma=0.5, selector="sortlsh", lsh_bits=7),
    # the headline shape with the causal sortLSH recursion (halves down to single blocks)
    "n16k_d128_sortlsh_causal": Workload("n16k_d128_sortlsh_causal", 1, 32, 16384, 128, "bf16", True, 128, 128, 2,
                                         n_centroids=256, sigma=0.5, selector="sortlsh", lsh_bits=7),
    # config 3's shape (d = 64, blocks of 64) with the causal sortLSH recursion
    "n8k_d64_sortlsh_causal": Workload("n8k_d64_sortlsh_causal", 4, 16, 8192, 64, "bf16", True, 128, 64, 2,
                                       n_centroids=128, sigma=0.3, selector="sortlsh", lsh_bits=7),
    "n64k_d128": Workload("n64k_d128", 1, 8, 65536, 128, "bf16", True, 256, 128, 32,
                          n_centroids=512, sigma=0.3),
    # config 5's shape with the causal sortLSH recursion (eight sorted levels; the first
    # level's halves of 32768 rows sort through global memory): 2^9 buckets for 512 blocks
    "n64k_d128_sortlsh_causal": Workload("n64k_d128_sortlsh_causal", 1, 8, 65536, 128, "bf16", True, 256, 128, 2,
                                         n_centroids=512, sigma=0.3, selector="sortlsh", lsh_bits=9),
}
HEADLINE = "n16k_d128"


def make_inputs(w: Workload, seed: int = 0, heads: Optional[range] = None) -> dict:
    """Draw Q, K, V, dO (shape [B, H, N, d]) and W_hash ([L, d, gamma]) on the CPU.

    Returns float32 tensors; ``Q16``/``K16``/... bf16 copies are added for bf16
    workloads (the float32 tensors then hold the bf16 values exactly, so both
    sides see identical inputs).  ``heads`` keeps only a subset of the (b, h)
    pairs after drawing, so a sample sees the same numbers as the full run.
    """
    g = torch.Generator().manual_seed(seed)
    B, H, N, d = w.B, w.H, w.N, w.d
    BH = B * H
    if w.kind == "iid":
        Q = torch.randn(BH, N, d, generator=g)
        K = torch.randn(BH, N, d, generator=g)
    elif w.kind == "clustered":
        cent = torch.randn(BH, w.n_centroids, d, generator=g)
        aq = torch.randint(0, w.n_centroids, (BH, N), generator=g)
        ak = torch.randint(0, w.n_centroids, (BH, N), generator=g)
        Q = torch.gather(cent, 1, aq[..., None].expand(BH, N, d))
        Q += w.sigma * torch.randn(BH, N, d, generator=g)
        K = torch.gather(cent, 1, ak[..., None].expand(BH, N, d))
        K += w.sigma * torch.randn(BH, N, d, generator=g)
        del cent, aq, ak
    else:
        raise ValueError(f"unknown workload kind {w.kind!r}")
    V = torch.randn(BH, N, d, generator=g)
    dO = torch.randn(BH, N, d, generator=g)
    W = torch.randn(w.n_tables, d, w.hash_bits, generator=g)
    out = {}
    for name, t in (("Q", Q), ("K", K), ("V", V), ("dO", dO)):
        t = t.view(B, H, N, d)
        if heads is not None:
            t = t.view(BH, N, d)[list(heads)].view(1, len(heads), N, d)
        if w.dtype == "bf16":
            t16 = t.to(torch.bfloat16)
            out[name + "16"] = t16.contiguous()
            t = t16.float()
        out[name] = t.contiguous()
    out["W"] = W.contiguous()
    if w.selector == "sortlsh":   # hyperplanes of the angular hash, drawn after everything else
        out["R"] = torch.randn(d, w.lsh_bits, generator=g).contiguous()
    return out


def small_workload(N=192, d=64, block_size=64, topk=2, rank_r=32, causal=True,
                   dtype="bf16", B=1, H=2, kind="clustered", n_centroids=8,
                   sigma=0.3, name="small") -> Workload:
    """A reduced workload with the same construction, for parity tests."""
    return Workload(name, B, H, N, d, dtype, causal, rank_r, block_size, topk,
                    kind=kind, n_centroids=n_centroids, sigma=sigma)
