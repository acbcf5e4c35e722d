"""ELSAA oracle: a plain, slow, float64 CPU statement of what the operator computes.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` use it.  It shares no code with the CUDA path;
its inputs come from the seeded generators (numbers only, no method arithmetic).

Source: the paper page "ELSAA: Efficient Low-Rank and Sparse Attention
Approximation for Training Transformers" (arXiv 2607.20214), cited below as
[ELSAA <section>, <equation>].  Everything is float64; bf16 inputs enter as
their exact values.

Readings taken where the page is silent:
  * selector: the page allows "any efficient important-key selector that
    returns an exact sparse output and a denominator" [ELSAA §3.3, Practical
    notes]; this operator uses top-k key blocks per query tile, scored by the
    mean-pooled logit  s_tb = scale * mean(Q_t) . mean(K_b)  (exact logit when
    the block size is 1); ties go to the lower block index.
  * causal: the diagonal block is always selected (the causal sortLSH recursion
    always attends its diagonal blocks [ELSAA §3.2]), then the best k-1 earlier
    blocks; keys j > i are masked.
  * RACE soft assignment: unit-normalised input u = x/max(|x|, 1e-12); table l
    projects h_l = W_l^T u (gamma values); the bucket probabilities are the
    softmax over the 2^gamma hypercube corners c of <c, h_l>/tau; the feature
    vector is Phi(x) = [p_l(c|x) / sqrt(L)], so Phi(q).Phi(k) is the bucket
    co-assignment probability averaged over the L tables.  Algorithm 2 of the
    paper is not on the page, so this form is parity unpinned against the
    paper itself; it is pinned here to its own definition (brute force), the
    corner-softmax/sigmoid-product identity and the hard-hash collision limit.
  * rank r = L * 2^gamma, the RACE sketch size S_R = L_s 2^gamma [ELSAA §6].
  * gates: optional per-row inputs; default g_sparse = 1, g_lr = 1 - m.
  * epsilon default 1e-6, lambda default 1 (scalar or per row).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import numpy as np

NORM_FLOOR = 1e-12


@dataclasses.dataclass
class Params:
    N: int
    d: int
    block_size: int          # T = B: queries per tile and keys per block
    topk: int                # k: blocks per query tile (0 disables the sparse branch)
    rank_r: int              # r = L * 2^gamma (0 disables the low-rank branch)
    causal: bool
    scale: float
    hash_bits: int = 4       # gamma
    lam: float = 1.0
    eps: float = 1e-6
    tau: float = 1.0
    chunk: Optional[int] = None   # RACE causal chunk size; defaults to block_size
    fixed_m: bool = False    # ablation without denominator-aware fusion: m = 1, default g_lr = 1
    selector: str = "topk"   # "topk" (blocks by pooled score) or "sortlsh" (§3.2; causal: the recursion)
    lsh_planes: Optional[np.ndarray] = None   # sortLSH hyperplanes [d, bits] (selector "sortlsh")
    lsh_orders: Optional[tuple] = None        # non-causal sortLSH: externally decided (query, key) orders
    lsh_codes: Optional[tuple] = None         # causal sortLSH: externally decided (query, key) hash codes

    @property
    def n_tables(self) -> int:
        return self.rank_r >> self.hash_bits if self.rank_r else 0

    @property
    def n_tiles(self) -> int:
        return -(-self.N // self.block_size)

    @property
    def race_chunk(self) -> int:
        return self.chunk or max(self.block_size, 1)


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):
        x = x.detach().cpu().double().numpy()
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------
# Selection [ELSAA §3.3 Practical notes; §1 names approximate large-entry
# detection and §3 learned top-k selectors as instantiations]
# ----------------------------------------------------------------------------

def pooled_means(X: np.ndarray, T: int) -> np.ndarray:
    """Mean of each group of T consecutive rows (the last group may be short)."""
    N = X.shape[0]
    n = -(-N // T)
    out = np.zeros((n, X.shape[1]))
    for t in range(n):
        out[t] = X[t * T:min(N, (t + 1) * T)].mean(axis=0)
    return out


def block_scores(q: np.ndarray, k: np.ndarray, p: Params) -> np.ndarray:
    """s_tb = scale * qbar_t . kbar_b, the mean logit over the tile x block rectangle."""
    return p.scale * (pooled_means(q, p.block_size) @ pooled_means(k, p.block_size).T)


def select_from_scores(scores: np.ndarray, topk: int, causal: bool) -> np.ndarray:
    """Top-k blocks per tile row of ``scores``: highest score first, lower index on ties.

    Causal: the diagonal block t is always taken, then the best k-1 of blocks < t
    (all of 0..t when t+1 <= k).  Returns int64 [n_t, topk] in ascending block
    order, padded with -1.
    """
    scores = _f64(scores)
    n_t, n_b = scores.shape
    idx = -np.ones((n_t, topk), dtype=np.int64)
    if topk == 0:
        return idx
    for t in range(n_t):
        if causal:
            chosen = [t]
            cand = list(range(t))
            need = topk - 1
        else:
            chosen = []
            cand = list(range(n_b))
            need = topk
        cand.sort(key=lambda b: (-scores[t, b], b))
        chosen += cand[:need]
        chosen.sort()
        idx[t, :len(chosen)] = chosen
    return idx


def support(idx: np.ndarray, p: Params) -> list:
    """Per query row i, the sorted array of key indices in Omega_i."""
    T, N = p.block_size, p.N
    out = []
    for i in range(N):
        t = i // T
        keys = []
        for b in idx[t]:
            if b < 0:
                continue
            for j in range(b * T, min(N, (b + 1) * T)):
                if not p.causal or j <= i:
                    keys.append(j)
        out.append(np.array(sorted(keys), dtype=np.int64))
    return out


# ----------------------------------------------------------------------------
# sortLSH selector [ELSAA §3.2]: queries and keys are hashed, sorted by hash value
# and grouped into equal-size blocks; query block t attends exactly key block t.
# Reading (the page has no pseudocode): angular LSH with the caller's hyperplanes
# R [d, b], bit c of a row's code set when x . R_c > 0; rows are ordered by the
# position of their code in the reflected Gray sequence (neighbouring buckets
# differ in one bit), ties by row index.  The causal selector is the recursion
# further down.
# ----------------------------------------------------------------------------

def simhash_codes(X, R) -> np.ndarray:
    """b-bit angular hash code of every row: bit c is [x . R_c > 0]."""
    bits = (_f64(X) @ _f64(R)) > 0
    return (bits.astype(np.int64) << np.arange(bits.shape[1])[None, :]).sum(axis=1)


def gray_rank(code: np.ndarray) -> np.ndarray:
    """Position of ``code`` in the reflected Gray sequence g(n) = n ^ (n >> 1): the
    inverse map, n = code ^ (code >> 1) ^ (code >> 2) ^ ..."""
    code = np.asarray(code, dtype=np.int64)
    n = code.copy()
    shift = code >> 1
    while np.any(shift):
        n ^= shift
        shift >>= 1
    return n


def sortlsh_order(X, R) -> np.ndarray:
    """Row indices in sorted order: by Gray position of the code, then by index."""
    return np.argsort(gray_rank(simhash_codes(X, R)), kind="stable")


def sortlsh_support(q, k, p: Params, tiles=None) -> list:
    """Per query row i, the sorted key indices of the key block that shares its
    position with i's query block in the two sorted orders.  ``tiles`` keeps only
    those sorted query blocks (a timing sample); other rows get an empty support."""
    assert not p.causal, "the sortLSH selector here is the non-causal one"
    T, N = p.block_size, p.N
    if p.lsh_orders is not None:      # orders decided elsewhere (the hash signs of another precision)
        oq, ok = (np.asarray(o) for o in p.lsh_orders)
    else:
        oq, ok = sortlsh_order(q, p.lsh_planes), sortlsh_order(k, p.lsh_planes)
    out = [np.zeros(0, dtype=np.int64)] * N
    for t in (range(p.n_tiles) if tiles is None else tiles):
        keys = np.sort(ok[t * T:(t + 1) * T])
        for i in oq[t * T:(t + 1) * T]:
            out[i] = keys
    return out


# ----------------------------------------------------------------------------
# Causal sortLSH [ELSAA §3.2, "For the causal setting"]: divide and conquer.  A
# segment is split into a past and a future half; each half recurses (its own
# causal problem); the future queries against the past keys are a non-causal
# sortLSH problem (every such key precedes every such query); the future half's
# two results are merged by log-sum-exp, which keeps the softmax exact over the
# union of the two supports.
# Readings (Algorithm 5 is not on the page): the split is on block boundaries
# with the extra block of an odd count going to the past half, so the past half
# has at least as many sorted key blocks as the future half has query blocks; a
# single block is the leaf, attended exactly under the mask j <= i; every level
# hashes with the same planes, and the off-diagonal problem is the non-causal
# selector above restricted to the two halves.
# ----------------------------------------------------------------------------

def _lsh_codes(q, k, p: Params):
    if p.lsh_codes is not None:       # codes decided elsewhere (the hash signs of another precision)
        return tuple(np.asarray(c, dtype=np.int64) for c in p.lsh_codes)
    return simhash_codes(q, p.lsh_planes), simhash_codes(k, p.lsh_planes)


def _split(a: int, b: int, T: int):
    """Past/future boundary of the row segment [a, b), or None for a leaf."""
    nb = -(-(b - a) // T)
    return None if nb <= 1 else a + -(-nb // 2) * T


def _sorted_rows(codes, a: int, b: int) -> np.ndarray:
    """Rows a..b-1 by Gray position of their code, ties by row."""
    return a + np.argsort(gray_rank(codes[a:b]), kind="stable")


def causal_sortlsh(q, k, v, p: Params):
    """Sparse branch (O_s, log d_s) of the causal recursion, taken in its own steps:
    recurse on both halves, attend the future queries' sorted blocks to the past
    keys' sorted blocks, merge the future half by log-sum-exp."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    N, d = q.shape
    T = p.block_size
    cq, ck = _lsh_codes(q, k, p)

    def rec(a, b):
        mid = _split(a, b, T)
        if mid is None:                                   # leaf: one block, exact under j <= i
            O = np.zeros((b - a, d))
            logd = np.zeros(b - a)
            for i in range(a, b):
                z = p.scale * (k[a:i + 1] @ q[i])
                mx = z.max()
                e = np.exp(z - mx)
                O[i - a] = e @ v[a:i + 1] / e.sum()
                logd[i - a] = mx + np.log(e.sum())
            return O, logd
        O_past, l_past = rec(a, mid)
        O_ff, l_ff = rec(mid, b)
        # future queries x past keys: non-causal sortLSH on the two halves
        oq, ok = _sorted_rows(cq, mid, b), _sorted_rows(ck, a, mid)
        O_fp = np.zeros((b - mid, d))
        l_fp = np.full(b - mid, -np.inf)
        for t in range(-(-(b - mid) // T)):
            rows, keys = oq[t * T:(t + 1) * T], ok[t * T:(t + 1) * T]
            if keys.size == 0:
                continue
            z = p.scale * (q[rows] @ k[keys].T)
            mx = z.max(axis=1, keepdims=True)
            e = np.exp(z - mx)
            O_fp[rows - mid] = e @ v[keys] / e.sum(axis=1, keepdims=True)
            l_fp[rows - mid] = mx[:, 0] + np.log(e.sum(axis=1))
        # log-sum-exp merge of the future half's two contributions
        l_f = np.logaddexp(l_ff, l_fp)
        O_f = np.exp(l_ff - l_f)[:, None] * O_ff + np.exp(l_fp - l_f)[:, None] * O_fp
        return np.concatenate([O_past, O_f]), np.concatenate([l_past, l_f])

    return rec(0, N)


def causal_sortlsh_support(q, k, p: Params, tiles=None) -> list:
    """Per query row i, its keys under the causal recursion: the union over the
    levels of the sorted key block its sorted query block meets, plus its own
    block's keys j <= i.  ``tiles`` keeps only the rows of those query tiles (a
    timing sample); other rows get an empty support."""
    N, T = p.N, p.block_size
    cq, ck = _lsh_codes(q, k, p)
    parts = [[] for _ in range(N)]

    def rec(a, b):
        mid = _split(a, b, T)
        if mid is None:
            for i in range(a, b):
                parts[i].append(np.arange(a, i + 1))
            return
        rec(a, mid)
        rec(mid, b)
        oq, ok = _sorted_rows(cq, mid, b), _sorted_rows(ck, a, mid)
        for t in range(-(-(b - mid) // T)):
            keys = ok[t * T:(t + 1) * T]
            for i in oq[t * T:(t + 1) * T]:
                parts[i].append(keys)

    rec(0, N)
    keep = None if tiles is None else {i for t in tiles for i in range(t * T, min(N, (t + 1) * T))}
    return [np.sort(np.concatenate(parts[i])) if keep is None or i in keep else np.zeros(0, dtype=np.int64)
            for i in range(N)]


def lsh_support(q, k, p: Params, tiles=None) -> list:
    """Per-row support of the sortLSH selector (the recursion when causal)."""
    return causal_sortlsh_support(q, k, p, tiles) if p.causal else sortlsh_support(q, k, p, tiles)


def sparse_from_support(q, k, v, sup, p: Params):
    """O_s and log d_s row by row over an explicit support (list of key arrays)."""
    N, d = q.shape
    O_s = np.zeros((N, d))
    logd = np.full(N, -np.inf)
    for i, keys in enumerate(sup):
        if keys.size == 0:
            continue
        z = p.scale * (k[keys] @ q[i])
        mx = z.max()
        e = np.exp(z - mx)
        O_s[i] = e @ v[keys] / e.sum()
        logd[i] = mx + np.log(e.sum())
    return O_s, logd


# ----------------------------------------------------------------------------
# Sparse branch: exact softmax attention over the selected support, returning
# the normalised output and its denominator [ELSAA §3.2; §3 dense definition]
# ----------------------------------------------------------------------------

def _tile_keys(idx_row: np.ndarray, p: Params) -> np.ndarray:
    T, N = p.block_size, p.N
    ks = [np.arange(b * T, min(N, (b + 1) * T)) for b in idx_row if b >= 0]
    return np.concatenate(ks) if ks else np.zeros(0, dtype=np.int64)


def sparse_branch(q, k, v, idx, p: Params, tiles=None):
    """O_s[i] = sum_j e^{z_ij} v_j / d_s[i], d_s[i] = sum_j e^{z_ij}, j in Omega_i.

    z_ij = scale * q_i . k_j.  Returns (O_s, log d_s); an empty support gives
    O_s = 0 and log d_s = -inf.  ``tiles`` restricts the work to those query
    tiles (other rows are left empty); used only to time a bounded sample.
    """
    N, d = q.shape
    T = p.block_size
    O_s = np.zeros((N, d))
    logd = np.full(N, -np.inf)
    for t in (range(p.n_tiles) if tiles is None else tiles):
        rows = np.arange(t * T, min(N, (t + 1) * T))
        keys = _tile_keys(idx[t], p)
        if keys.size == 0:
            continue
        z = p.scale * (q[rows] @ k[keys].T)
        if p.causal:
            z = np.where(keys[None, :] <= rows[:, None], z, -np.inf)
        mx = z.max(axis=1, keepdims=True)
        e = np.exp(z - mx)
        ds = e.sum(axis=1, keepdims=True)
        O_s[rows] = (e @ v[keys]) / ds
        logd[rows] = (mx + np.log(ds))[:, 0]
    return O_s, logd


# ----------------------------------------------------------------------------
# Low-rank branch: RACE soft hash-bucket summaries in normalised ratio form
# [ELSAA §3.1; §2 (RACE attention); sketch size S_R = L_s 2^gamma, §6]
# ----------------------------------------------------------------------------

def corners(gamma: int) -> np.ndarray:
    """The 2^gamma hypercube corners c in {-1,+1}^gamma; bit b of the index sets c_b = +1."""
    m = np.arange(1 << gamma)[:, None]
    return np.where((m >> np.arange(gamma)[None, :]) & 1, 1.0, -1.0)


def race_bucket_probs(X, W, p: Params):
    """Soft assignment of each row to the 2^gamma buckets of every table.

    Returns (P [N, L, 2^gamma], u [N, d], n [N]): P[i, l, c] = softmax over the
    corners c of <c, W_l^T u_i> / tau, u = X / n, n = max(|X|, 1e-12).
    """
    X = _f64(X)
    W = _f64(W)
    n = np.maximum(np.linalg.norm(X, axis=1), NORM_FLOOR)
    u = X / n[:, None]
    C = corners(p.hash_bits)
    P = np.zeros((X.shape[0], p.n_tables, C.shape[0]))
    for l in range(p.n_tables):
        h = u @ W[l]                           # [N, gamma]
        a = (h @ C.T) / p.tau                  # [N, 2^gamma]
        a -= a.max(axis=1, keepdims=True)
        e = np.exp(a)
        P[:, l, :] = e / e.sum(axis=1, keepdims=True)
    return P, u, n


def race_features(X, W, p: Params) -> np.ndarray:
    """Phi(x) = [p_l(c|x) / sqrt(L)] flattened over (table l, corner c): [N, r]."""
    P, _, _ = race_bucket_probs(X, W, p)
    return P.reshape(P.shape[0], -1) / math.sqrt(p.n_tables)


def race_branch(q, k, v, W, p: Params):
    """RACE low-rank branch in its linear-time summary form.

    Non-causal: bucket statistics S = sum_j Phi(k_j)^T [v_j ; 1] are accumulated
    once and every query reads Phi(q_i) S.  Causal: the sequence is cut into
    chunks; a query reads the statistics of all strictly earlier chunks (a
    running prefix sum) plus a causally masked sum over its own chunk.
    The read-out [N_lr ; d_lr] gives O_lr = N_lr / d_lr.  r = 0 gives zeros.
    """
    N, d = q.shape
    if p.rank_r == 0:
        return np.zeros((N, d)), np.zeros(N)
    PhiQ = race_features(q, W, p)
    PhiK = race_features(k, W, p)
    Vt = np.concatenate([v, np.ones((N, 1))], axis=1)
    out = np.zeros((N, d + 1))
    if not p.causal:
        S = PhiK.T @ Vt
        out = PhiQ @ S
    else:
        C = p.race_chunk
        prefix = np.zeros((p.rank_r, d + 1))
        for c0 in range(0, N, C):
            cs = slice(c0, min(N, c0 + C))
            inter = PhiQ[cs] @ prefix
            kap = np.tril(PhiQ[cs] @ PhiK[cs].T)
            out[cs] = inter + kap @ Vt[cs]
            prefix += PhiK[cs].T @ Vt[cs]
    d_lr = out[:, d]
    O_lr = out[:, :d] / d_lr[:, None]
    return O_lr, d_lr


def race_rows(q, k, v, W, p: Params, rows) -> tuple:
    """(O_lr, d_lr) for selected query rows straight from the kernel sums
    d_lr,i = sum_{j in J(i)} kappa(q_i, k_j), O_lr,i = sum kappa v_j / d_lr,i,
    with J(i) = all keys (or j <= i when causal).  O(N r) per row."""
    N, d = q.shape
    rows = np.asarray(rows)
    if p.rank_r == 0:
        return np.zeros((rows.size, d)), np.zeros(rows.size)
    PhiQ = race_features(q[rows], W, p)
    PhiK = race_features(k, W, p)
    O = np.zeros((rows.size, d))
    dl = np.zeros(rows.size)
    for a, i in enumerate(rows):
        J = np.arange(i + 1) if p.causal else np.arange(N)
        kap = PhiK[J] @ PhiQ[a]
        dl[a] = kap.sum()
        O[a] = kap @ v[J] / dl[a]
    return O, dl


# ----------------------------------------------------------------------------
# Denominator-aware fusion [ELSAA §3.3, Eq. 5; §1, Eq. 4]
# ----------------------------------------------------------------------------

def fuse(O_s, logd_s, O_lr, d_lr, p: Params, lam=None, g_s=None, g_lr=None):
    """m = d_s / (d_s + lam d_lr + eps);  O = g_s m O_s + g_lr O_lr  [ELSAA §3.3 Eq. 5, §1 Eq. 4].

    Default gates: g_s = 1, g_lr = 1 - m.  With ``p.fixed_m`` (the paper's
    Sort_Lsh_RACE ablation, §6 "Attention variants": m_sparse = 1, no
    denominator-aware rescaling) m = 1 and the default g_lr is 1, so the two
    branch outputs are added.  Returns (O, m).
    """
    d_s = np.exp(logd_s)
    lam = p.lam if lam is None else _f64(lam)
    if p.fixed_m:
        m = np.ones_like(d_s * d_lr)
    else:
        m = d_s / (d_s + lam * d_lr + p.eps)
    gs = 1.0 if g_s is None else _f64(g_s)
    gl = (1.0 if p.fixed_m else 1.0 - m) if g_lr is None else _f64(g_lr)
    O = (gs * m)[..., None] * O_s + np.broadcast_to(gl, m.shape)[..., None] * O_lr
    return O, m


# ----------------------------------------------------------------------------
# Whole operator, one head, then [B, H] batches
# ----------------------------------------------------------------------------

def forward_head(q, k, v, W, p: Params, lam=None, g_s=None, g_lr=None, scores=None, tiles=None):
    """One attention head [ELSAA §3: the method is defined per head].

    ``scores`` replaces the block scores (used to feed the selector an external
    score array).  ``tiles`` limits the sparse branch to those query tiles (a
    timing sample).  Returns a dict with O, O_s, logd_s, O_lr, d_lr, m, idx, scores.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    if p.selector == "sortlsh":
        sc = idx = None
        if p.causal:
            O_s, logd = causal_sortlsh(q, k, v, p)
        else:
            O_s, logd = sparse_from_support(q, k, v, sortlsh_support(q, k, p, tiles), p)
    else:
        sc = block_scores(q, k, p) if scores is None else _f64(scores)
        idx = select_from_scores(sc, p.topk, p.causal)
        O_s, logd = sparse_branch(q, k, v, idx, p, tiles)
    O_lr, d_lr = race_branch(q, k, v, W, p)
    O, m = fuse(O_s, logd, O_lr, d_lr, p, lam, g_s, g_lr)
    return dict(O=O, O_s=O_s, logd_s=logd, O_lr=O_lr, d_lr=d_lr, m=m, idx=idx, scores=sc)


def _per_head(x, b, h):
    return None if x is None else _f64(x)[b, h]


def forward(Q, K, V, W, p: Params, lam=None, g_s=None, g_lr=None):
    """Q, K, V: [B, H, N, d]; lam/g_s/g_lr: None or [B, H, N].  Multi-head ELSAA
    runs the same procedure independently per head [ELSAA §3]."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    Bn, Hn = Q.shape[:2]
    res = {}
    for b in range(Bn):
        for h in range(Hn):
            r = forward_head(Q[b, h], K[b, h], V[b, h], W, p,
                             _per_head(lam, b, h), _per_head(g_s, b, h), _per_head(g_lr, b, h))
            for key, val in r.items():
                if key not in res:
                    res[key] = np.zeros((Bn, Hn) + val.shape, dtype=val.dtype)
                res[key][b, h] = val
    return res


# ----------------------------------------------------------------------------
# Backward: the explicit chain rule through Eq. 4, Eq. 5, the sparse softmax
# and the RACE features.  Selection and W are constants.
# ----------------------------------------------------------------------------

def _fusion_adjoints(dO, fw, p: Params, lam, g_s, g_lr):
    """Per-row adjoints of Eq. 4 / Eq. 5.

    Returns dO_s, dO_lr, dd_s*d_s and dd_lr, where
      dm    = g_s <dO, O_s> - [default g_lr] <dO, O_lr>
      dd_s  = dm (lam d_lr + eps) / D^2,  dd_lr = -dm lam d_s / D^2,
      D     = d_s + lam d_lr + eps.
    """
    m = fw["m"]
    d_s = np.exp(fw["logd_s"])
    d_lr = fw["d_lr"]
    lam = p.lam if lam is None else _f64(lam)
    gs = np.ones_like(m) if g_s is None else _f64(g_s)
    gl = (np.ones_like(m) if p.fixed_m else 1.0 - m) if g_lr is None else _f64(g_lr)
    a = (dO * fw["O_s"]).sum(axis=1)
    b = (dO * fw["O_lr"]).sum(axis=1)
    # with m held at 1 nothing flows back through m
    dm = np.zeros_like(m) if p.fixed_m else gs * a - (b if g_lr is None else 0.0)
    D = d_s + lam * d_lr + p.eps
    dds_ds = dm * (lam * d_lr + p.eps) * d_s / D ** 2
    ddlr = -dm * lam * d_s / D ** 2
    dOs = (gs * m)[:, None] * dO
    dOlr = gl[:, None] * dO
    return dOs, dOlr, dds_ds, ddlr


def fusion_param_grads(dO, fw, p: Params, lam=None, g_s=None, g_lr=None):
    """Per-row gradients of the loss <dO, O> with respect to the fusion parameters
    lambda_i, g_s,i and g_lr,i of Eq. 5 / Eq. 4 (the paper's optional learnable lambda).

      dlambda = dm * dm/dlambda = -dm d_s d_lr / D^2     (0 when m is held at 1)
      dg_s    = m <dO, O_s>,   dg_lr = <dO, O_lr>
    with dm = g_s <dO, O_s> - [g_lr defaulted to 1 - m] <dO, O_lr>.  A gate left at
    its default still gets the derivative at that value.  Returns (dlam, dgs, dglr)."""
    dO = _f64(dO)
    m = fw["m"]
    d_s = np.exp(fw["logd_s"])
    d_lr = fw["d_lr"]
    lam = p.lam if lam is None else _f64(lam)
    gs = np.ones_like(m) if g_s is None else _f64(g_s)
    a = (dO * fw["O_s"]).sum(axis=1)
    b = (dO * fw["O_lr"]).sum(axis=1)
    if p.fixed_m:
        dlam = np.zeros_like(m)
    else:
        dm = gs * a - (b if g_lr is None else 0.0)
        D = d_s + lam * d_lr + p.eps
        dlam = -dm * d_s * d_lr / D ** 2
    return dlam, m * a, b


def race_features_backward(X, W, p: Params, dPhi):
    """Pull dPhi [N, r] back through Phi = p/sqrt(L), the corner softmax, the
    projection h = W^T u and the normalisation u = x / max(|x|, 1e-12)."""
    X = _f64(X)
    W = _f64(W)
    P, u, n = race_bucket_probs(X, W, p)
    C = corners(p.hash_bits)
    G = C.shape[0]
    du = np.zeros_like(X)
    for l in range(p.n_tables):
        dp = dPhi[:, l * G:(l + 1) * G] / math.sqrt(p.n_tables)
        pl = P[:, l, :]
        da = pl * (dp - (dp * pl).sum(axis=1, keepdims=True))
        dh = (da @ C) / p.tau
        du += dh @ _f64(W[l]).T
    nrm = np.linalg.norm(X, axis=1)
    proj = (u * du).sum(axis=1, keepdims=True)
    return np.where((nrm > NORM_FLOOR)[:, None], (du - u * proj) / n[:, None], du / n[:, None])


def backward_head(q, k, v, W, dO, fw, p: Params, lam=None, g_s=None, g_lr=None, tiles=None):
    """(dq, dk, dv) for one head, given the forward dict ``fw``.

    The gradient is a sum of contributions generated by each query tile;
    ``tiles`` keeps only those tiles' contributions (a timing sample)."""
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    N, d = q.shape
    T = p.block_size
    dq = np.zeros_like(q)
    dk = np.zeros_like(k)
    dv = np.zeros_like(v)
    dOs, dOlr, dds_ds, ddlr = _fusion_adjoints(dO, fw, p, lam, g_s, g_lr)
    # sparse branch: P_ij = e^{z_ij}/d_s, dz_ij = P_ij (<dO_s,i, v_j> - Delta_i),
    # Delta_i = <dO_s,i, O_s,i> - dd_s,i d_s,i
    Delta = (dOs * fw["O_s"]).sum(axis=1) - dds_ds
    tile_list = list(range(p.n_tiles)) if tiles is None else list(tiles)
    if p.selector == "sortlsh":
        # the same chain rule row by row over each row's support
        for i, keys in enumerate(lsh_support(q, k, p, tiles)):
            if keys.size == 0:
                continue
            P = np.exp(p.scale * (k[keys] @ q[i]) - fw["logd_s"][i])
            dz = P * (v[keys] @ dOs[i] - Delta[i])
            dq[i] += p.scale * dz @ k[keys]
            dk[keys] += p.scale * np.outer(dz, q[i])
            dv[keys] += np.outer(P, dOs[i])
    for t in ([] if p.selector == "sortlsh" else tile_list):
        rows = np.arange(t * T, min(N, (t + 1) * T))
        keys = _tile_keys(fw["idx"][t], p)
        if keys.size == 0:
            continue
        z = p.scale * (q[rows] @ k[keys].T)
        P = np.exp(z - fw["logd_s"][rows, None])
        if p.causal:
            P = np.where(keys[None, :] <= rows[:, None], P, 0.0)
        dP = dOs[rows] @ v[keys].T
        dz = P * (dP - Delta[rows, None])
        dq[rows] += p.scale * dz @ k[keys]
        np.add.at(dk, keys, p.scale * dz.T @ q[rows])
        np.add.at(dv, keys, P.T @ dOs[rows])
    if p.rank_r:
        # low-rank branch: O_lr = N_lr / d_lr, kappa_ij = Phi(q_i).Phi(k_j)
        d_lr = fw["d_lr"]
        dN = dOlr / d_lr[:, None]
        delta = ddlr - (dOlr * fw["O_lr"]).sum(axis=1) / d_lr
        PhiQ = race_features(q, W, p)
        PhiK = race_features(k, W, p)
        dPhiQ = np.zeros_like(PhiQ)
        dPhiK = np.zeros_like(PhiK)
        for t in tile_list:
            rows = np.arange(t * T, min(N, (t + 1) * T))
            keys = np.arange(rows[-1] + 1) if p.causal else np.arange(N)
            mask = (keys[None, :] <= rows[:, None]) if p.causal else np.ones((rows.size, keys.size), bool)
            kap = np.where(mask, PhiQ[rows] @ PhiK[keys].T, 0.0)
            dkap = np.where(mask, dN[rows] @ v[keys].T + delta[rows, None], 0.0)
            dv[keys] += kap.T @ dN[rows]
            dPhiQ[rows] += dkap @ PhiK[keys]
            dPhiK[keys] += dkap.T @ PhiQ[rows]
        dq += race_features_backward(q, W, p, dPhiQ)
        dk += race_features_backward(k, W, p, dPhiK)
    return dq, dk, dv


def backward(Q, K, V, W, dO, fw, p: Params, lam=None, g_s=None, g_lr=None):
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    Bn, Hn = Q.shape[:2]
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for b in range(Bn):
        for h in range(Hn):
            fwh = {key: val[b, h] for key, val in fw.items()}
            dQ[b, h], dK[b, h], dV[b, h] = backward_head(
                Q[b, h], K[b, h], V[b, h], W, dO[b, h], fwh, p,
                _per_head(lam, b, h), _per_head(g_s, b, h), _per_head(g_lr, b, h))
    return dQ, dK, dV


# ----------------------------------------------------------------------------
# Row-sampled forms for large problems: the same definitions evaluated only for
# chosen query rows (forward, dq) or key rows (dk, dv).
# ----------------------------------------------------------------------------

def forward_rows_head(q, k, v, W, p: Params, rows, lam=None, g_s=None, g_lr=None, scores=None):
    """Forward quantities for the query rows ``rows`` only (per-row definitions)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    rows = np.asarray(rows)
    sc = block_scores(q, k, p) if scores is None else _f64(scores)
    idx = select_from_scores(sc, p.topk, p.causal)
    n, d = rows.size, q.shape[1]
    O_s = np.zeros((n, d))
    logd = np.full(n, -np.inf)
    for a, i in enumerate(rows):
        keys = _tile_keys(idx[i // p.block_size], p)
        if p.causal:
            keys = keys[keys <= i]
        if keys.size == 0:
            continue
        z = p.scale * (k[keys] @ q[i])
        mx = z.max()
        e = np.exp(z - mx)
        O_s[a] = e @ v[keys] / e.sum()
        logd[a] = mx + np.log(e.sum())
    O_lr, d_lr = race_rows(q, k, v, W, p, rows)
    sub = lambda x: None if x is None else _f64(x)[rows]
    O, m = fuse(O_s, logd, O_lr, d_lr, p, sub(lam), sub(g_s), sub(g_lr))
    return dict(O=O, O_s=O_s, logd_s=logd, O_lr=O_lr, d_lr=d_lr, m=m, idx=idx, scores=sc)


def backward_rows_head(q, k, v, W, dO, fw, p: Params, qrows, krows, lam=None, g_s=None, g_lr=None):
    """dq for query rows ``qrows`` and (dk, dv) for key rows ``krows``.

    ``fw`` is the full forward dict of the head (every row's denominators are
    needed for dk, dv).  Same chain rule as ``backward_head``, row by row.
    """
    q, k, v, dO = _f64(q), _f64(k), _f64(v), _f64(dO)
    N, d = q.shape
    T = p.block_size
    dOs, dOlr, dds_ds, ddlr = _fusion_adjoints(dO, fw, p, lam, g_s, g_lr)
    Delta = (dOs * fw["O_s"]).sum(axis=1) - dds_ds
    idx = fw["idx"]
    qrows, krows = np.asarray(qrows), np.asarray(krows)
    dq = np.zeros((qrows.size, d))
    dk = np.zeros((krows.size, d))
    dv = np.zeros((krows.size, d))
    for a, i in enumerate(qrows):
        keys = _tile_keys(idx[i // T], p)
        if p.causal:
            keys = keys[keys <= i]
        if keys.size:
            P = np.exp(p.scale * (k[keys] @ q[i]) - fw["logd_s"][i])
            dz = P * (v[keys] @ dOs[i] - Delta[i])
            dq[a] += p.scale * dz @ k[keys]
    for a, j in enumerate(krows):
        b = j // T
        for t in range(p.n_tiles):
            if b not in idx[t]:
                continue
            I = np.arange(t * T, min(N, (t + 1) * T))
            if p.causal:
                I = I[I >= j]
            if I.size == 0:
                continue
            P = np.exp(p.scale * (q[I] @ k[j]) - fw["logd_s"][I])
            dz = P * (dOs[I] @ v[j] - Delta[I])
            dk[a] += p.scale * dz @ q[I]
            dv[a] += P @ dOs[I]
    if p.rank_r:
        d_lr = fw["d_lr"]
        dN = dOlr / d_lr[:, None]
        delta = ddlr - (dOlr * fw["O_lr"]).sum(axis=1) / d_lr
        PhiQ = race_features(q, W, p)
        PhiK = race_features(k, W, p)
        dPhiQ = np.zeros((qrows.size, p.rank_r))
        for a, i in enumerate(qrows):
            J = np.arange(i + 1) if p.causal else np.arange(N)
            dkap = v[J] @ dN[i] + delta[i]
            dPhiQ[a] = dkap @ PhiK[J]
        dq += race_features_backward(q[qrows], W, p, dPhiQ)
        dPhiK = np.zeros((krows.size, p.rank_r))
        for a, j in enumerate(krows):
            I = np.arange(j, N) if p.causal else np.arange(N)
            kap = PhiQ[I] @ PhiK[j]
            dkap = dN[I] @ v[j] + delta[I]
            dv[a] += kap @ dN[I]
            dPhiK[a] = dkap @ PhiQ[I]
        dk += race_features_backward(k[krows], W, p, dPhiK)
    return dq, dk, dv


# ----------------------------------------------------------------------------
# Complexity accounting [ELSAA §6 and the appendix interaction-count example]
# ----------------------------------------------------------------------------

# ----------------------------------------------------------------------------
# Rank view of sparse + low-rank attention [ELSAA §4]
# ----------------------------------------------------------------------------

def max_matching(mask: np.ndarray) -> int:
    """Maximum matching size nu(Omega) of the bipartite graph with an edge (i, j) for
    every True entry of ``mask`` (rows on one side, columns on the other); Kuhn's
    augmenting paths, written out."""
    n_r, n_c = mask.shape
    adj = [np.flatnonzero(mask[i]) for i in range(n_r)]
    match_col = -np.ones(n_c, dtype=np.int64)

    def augment(i, seen):
        for j in adj[i]:
            if seen[j]:
                continue
            seen[j] = True
            if match_col[j] < 0 or augment(match_col[j], seen):
                match_col[j] = i
                return True
        return False

    return sum(1 for i in range(n_r) if augment(i, np.zeros(n_c, dtype=bool)))


def rank_diagnostic(q, k, idx, p: Params, r: int, seed: int = 0) -> dict:
    """rank(S_Omega + B A) against min(n, nu(Omega) + r) [ELSAA §4 Theorem].

    S_Omega = Omega * M*, M*_ij = exp(scale q_i . k_j), on the support the selector
    realised (``idx``; causal rows keep j <= i); B [n, r] and A [r, n] are drawn from a
    standard normal with ``seed`` (the theorem's absolutely continuous factors).  The
    rank is numpy's SVD rank.  Returns n, nu, r, the rank and the predicted rank."""
    q, k = _f64(q), _f64(k)
    n = q.shape[0]
    mask = np.zeros((n, n), dtype=bool)
    for i, keys in enumerate(support(idx, p)):
        mask[i, keys] = True
    S = np.where(mask, np.exp(p.scale * (q @ k.T)), 0.0)
    rng = np.random.default_rng(seed)
    M = S + rng.standard_normal((n, r)) @ rng.standard_normal((r, n)) if r > 0 else S
    nu = max_matching(mask)
    return dict(n=n, nu=nu, r=r, rank=int(np.linalg.matrix_rank(M)), predicted=min(n, nu + r))


def interaction_count(N: int, s: int, L_s: int, gamma: int) -> int:
    """Query-key interactions of ELSAA: N (s + L_s 2^gamma) [ELSAA §6]."""
    return N * (s + L_s * (1 << gamma))
