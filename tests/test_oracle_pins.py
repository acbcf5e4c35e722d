"""Pins for the float64 oracle against what the ELSAA paper and plain mathematics fix.

Each test checks the oracle against something other than itself: a library
routine the special case reduces to, brute force over subsets, the explicit
kernel-sum definition of RACE, closed-form identities, the hard-hash collision
limit, a value printed in the paper, and central finite differences.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import elsaa_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _params(N, d, T, k, r, causal, **kw):
    return orc.Params(N=N, d=d, block_size=T, topk=k, rank_r=r, causal=causal,
                      scale=1.0 / math.sqrt(d), **kw)


# --- dense attention is the exact special case [ELSAA §3 dense definition] ---

def test_full_support_no_lowrank_is_dense_softmax():
    N, d = 40, 16
    q, k, v = _rand((N, d), 1), _rand((N, d), 2), _rand((N, d), 3)
    p = _params(N, d, 1, N, 0, False, eps=0.0)
    out = orc.forward_head(q, k, v, np.zeros((0, d, 4)), p)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], scale=p.scale)[0].numpy()
    np.testing.assert_allclose(out["O"], ref, rtol=0, atol=1e-12)
    assert np.all(out["m"] == 1.0)


def test_causal_all_blocks_no_lowrank_is_causal_softmax():
    N, d, T = 56, 8, 8            # 7 tiles, k >= 7 selects every eligible block
    q, k, v = _rand((N, d), 4), _rand((N, d), 5), _rand((N, d), 6)
    p = _params(N, d, T, 7, 0, True, eps=0.0)
    out = orc.forward_head(q, k, v, np.zeros((0, d, 4)), p)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None],
        scale=p.scale, is_causal=True)[0].numpy()
    np.testing.assert_allclose(out["O"], ref, rtol=0, atol=1e-12)


def test_ragged_tail_all_blocks_is_dense_softmax():
    N, d, T = 45, 8, 8            # last tile/block has 5 rows
    q, k, v = _rand((N, d), 7), _rand((N, d), 8), _rand((N, d), 9)
    for causal in (False, True):
        p = _params(N, d, T, 6, 0, causal, eps=0.0)
        out = orc.forward_head(q, k, v, np.zeros((0, d, 4)), p)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None],
            scale=p.scale, is_causal=causal)[0].numpy()
        np.testing.assert_allclose(out["O"], ref, rtol=0, atol=1e-12)


# --- selection: brute force over subsets ---

def test_topk_keys_maximise_selected_mass_bruteforce():
    """Block size 1: the k selected keys maximise sum_j e^{z_ij} over all k-subsets,
    and O_s is the softmax restricted to the best subset."""
    N, d = 12, 5
    q, k, v = _rand((N, d), 10), _rand((N, d), 11), _rand((N, d), 12)
    for kk in range(1, N + 1):
        p = _params(N, d, 1, kk, 0, False)
        out = orc.forward_head(q, k, v, np.zeros((0, d, 4)), p)
        for i in range(N):
            z = p.scale * (k @ q[i])
            best, best_set = -1.0, None
            for sub in itertools.combinations(range(N), kk):
                mass = np.exp(z[list(sub)]).sum()
                if mass > best:
                    best, best_set = mass, sub
            assert tuple(out["idx"][i]) == best_set
            w = np.exp(z[list(best_set)])
            np.testing.assert_allclose(out["O_s"][i], w @ v[list(best_set)] / w.sum(), atol=1e-12)
            np.testing.assert_allclose(np.exp(out["logd_s"][i]), w.sum(), rtol=1e-12)


def test_causal_topk_keys_bruteforce_on_16_keys():
    N, d = 16, 4
    q, k, v = _rand((N, d), 13), _rand((N, d), 14), _rand((N, d), 15)
    for kk in (1, 3, 6):
        p = _params(N, d, 1, kk, 0, True)
        out = orc.forward_head(q, k, v, np.zeros((0, d, 4)), p)
        for i in range(N):
            z = p.scale * (k[:i + 1] @ q[i])
            # the diagonal (key i) is forced; the rest maximise the mass among keys < i
            best, best_set = -1.0, None
            for sub in itertools.combinations(range(i), min(kk - 1, i)):
                mass = np.exp(z[list(sub)]).sum()
                if mass > best:
                    best, best_set = mass, sub
            chosen = sorted(set(best_set) | {i})
            got = [b for b in out["idx"][i] if b >= 0]
            assert got == chosen
            w = np.exp(z[chosen])
            np.testing.assert_allclose(out["O_s"][i], w @ v[chosen] / w.sum(), atol=1e-12)


def test_block_selection_is_best_subset_of_block_scores():
    """Blocks of 2 on 16 keys: the selected blocks maximise the summed block score
    (the arg-top-k), found by enumerating every subset of blocks."""
    N, d, T = 16, 6, 2
    q, k = _rand((N, d), 16), _rand((N, d), 17)
    nb = N // T
    for causal in (False, True):
        for kk in (1, 2, 3, 5):
            p = _params(N, d, T, kk, 0, causal)
            out = orc.forward_head(q, k, _rand((N, d), 18), np.zeros((0, d, 4)), p)
            qbar = q.reshape(nb, T, d).mean(1)
            kbar = k.reshape(nb, T, d).mean(1)
            for t in range(nb):
                s = [p.scale * qbar[t] @ kbar[b] for b in range(nb)]
                elig = list(range(t + 1)) if causal else list(range(nb))
                size = min(kk, len(elig))
                best, best_set = -np.inf, None
                for sub in itertools.combinations(elig, size):
                    if causal and t not in sub:
                        continue
                    tot = sum(s[b] for b in sub if not (causal and b == t))
                    if tot > best:
                        best, best_set = tot, sub
                got = [b for b in out["idx"][t] if b >= 0]
                assert got == sorted(best_set)


def test_select_from_scores_ties_and_forced_diagonal():
    s = np.array([[0.5, 0.5, 0.5, 0.5],
                  [1.0, 2.0, 2.0, 0.0],
                  [3.0, 3.0, -9.0, 1.0],
                  [0.0, 0.0, 0.0, -5.0]])
    nc = orc.select_from_scores(s, 2, False)
    assert nc.tolist() == [[0, 1], [1, 2], [0, 1], [0, 1]]
    c = orc.select_from_scores(s, 2, True)
    # tile 0: only block 0; tile 2: diagonal 2 forced despite -9, plus best of {0, 1} (tie -> 0)
    assert c.tolist() == [[0, -1], [0, 1], [0, 2], [0, 3]]
    c3 = orc.select_from_scores(s, 3, True)
    assert c3.tolist() == [[0, -1, -1], [0, 1, -1], [0, 1, 2], [0, 1, 3]]


# --- RACE: the linear-time summary form equals the kernel-sum definition ---

def _race_definition(q, k, v, W, p):
    """Brute force: kappa(q_i, k_j) = (1/L) sum_l sum_c P_l(c|q_i) P_l(c|k_j), per pair."""
    N, d = q.shape
    Pq, _, _ = orc.race_bucket_probs(q, W, p)
    Pk, _, _ = orc.race_bucket_probs(k, W, p)
    L = p.n_tables
    O = np.zeros((N, d))
    dl = np.zeros(N)
    for i in range(N):
        num = np.zeros(d)
        den = 0.0
        for j in range(N):
            if p.causal and j > i:
                continue
            kap = 0.0
            for l in range(L):
                for c in range(1 << p.hash_bits):
                    kap += Pq[i, l, c] * Pk[j, l, c]
            kap /= L
            num += kap * v[j]
            den += kap
        O[i] = num / den
        dl[i] = den
    return O, dl


@pytest.mark.parametrize("causal,chunk", [(False, None), (True, 1), (True, 3), (True, 8), (True, 29)])
def test_race_summary_form_equals_definition(causal, chunk):
    N, d, r = 29, 6, 32
    q, k, v = _rand((N, d), 20), _rand((N, d), 21), _rand((N, d), 22)
    W = _rand((r // 16, d, 4), 23)
    p = _params(N, d, 4, 1, r, causal, chunk=chunk)
    O, dl = orc.race_branch(q, k, v, W, p)
    Oref, dlref = _race_definition(q, k, v, W, p)
    np.testing.assert_allclose(dl, dlref, rtol=1e-12)
    np.testing.assert_allclose(O, Oref, atol=1e-12)
    rows = [0, 5, 28]
    Or, dr = orc.race_rows(q, k, v, W, p, rows)
    np.testing.assert_allclose(dr, dlref[rows], rtol=1e-12)
    np.testing.assert_allclose(Or, Oref[rows], atol=1e-12)


def test_bucket_probabilities_sum_to_one_and_factorise():
    """softmax over corners of <c,h>/tau == prod_b sigmoid(2 c_b h_b / tau)."""
    d, L, gamma = 7, 3, 4
    X = _rand((50, d), 24, 3.0)
    W = _rand((L, d, gamma), 25)
    for tau in (1.0, 0.3, 2.5):
        p = orc.Params(N=50, d=d, block_size=1, topk=1, rank_r=L << gamma, causal=False,
                       scale=1.0, tau=tau)
        P, u, n = orc.race_bucket_probs(X, W, p)
        np.testing.assert_allclose(P.sum(axis=2), 1.0, atol=1e-14)
        np.testing.assert_allclose(np.linalg.norm(u, axis=1), 1.0, atol=1e-14)
        for l in range(L):
            h = u @ W[l]
            for c in range(1 << gamma):
                sign = np.array([1.0 if (c >> b) & 1 else -1.0 for b in range(gamma)])
                prod = np.prod(1.0 / (1.0 + np.exp(-2.0 * sign * h / tau)), axis=1)
                np.testing.assert_allclose(P[:, l, c], prod, rtol=1e-12)


def test_hard_hash_limit_is_collision_count():
    """tau -> 0: kappa(q, k) -> (1/L) #{tables where sign(W_l^T q) == sign(W_l^T k)}."""
    N, d, L = 30, 8, 5
    q, k = _rand((N, d), 26), _rand((N, d), 27)
    W = _rand((L, d, 4), 28)
    p = orc.Params(N=N, d=d, block_size=1, topk=1, rank_r=L * 16, causal=False, scale=1.0, tau=1e-9)
    kap = orc.race_features(q, W, p) @ orc.race_features(k, W, p).T
    count = np.zeros((N, N))
    for l in range(L):
        sq = np.sign(q @ W[l])
        sk = np.sign(k @ W[l])
        count += np.all(sq[:, None, :] == sk[None, :, :], axis=2)
    np.testing.assert_allclose(kap * L, count, atol=1e-9)
    assert set(np.round(kap * L).astype(int).ravel()) <= set(range(L + 1))


# --- fusion [Eq. 5, Eq. 4] ---

def _setup(N=48, d=8, T=8, k=2, r=32, causal=True, seed=30, **kw):
    q, k_, v = _rand((N, d), seed), _rand((N, d), seed + 1), _rand((N, d), seed + 2)
    W = _rand((r // 16, d, 4), seed + 3)
    return q, k_, v, W, _params(N, d, T, k, r, causal, **kw)


def test_default_gates_give_convex_combination_of_values():
    """With g_s = 1, g_lr = 1 - m every output row is sum_j w_ij v_j with w >= 0 and
    sum_j w_ij = 1; the weights are rebuilt entry by entry from the definitions."""
    for causal in (True, False):
        q, k, v, W, p = _setup(causal=causal, N=40, T=8, k=2)
        out = orc.forward_head(q, k, v, W, p)
        N = p.N
        Pq, _, _ = orc.race_bucket_probs(q, W, p)
        Pk, _, _ = orc.race_bucket_probs(k, W, p)
        sup = orc.support(out["idx"], p)
        for i in range(N):
            z = {j: p.scale * q[i] @ k[j] for j in sup[i]}
            ds = sum(math.exp(x) for x in z.values())
            J = range(i + 1) if causal else range(N)
            kap = {j: float((Pq[i] * Pk[j]).sum() / p.n_tables) for j in J}
            dl = sum(kap.values())
            m = ds / (ds + p.lam * dl + p.eps)
            w = np.zeros(N)
            for j, x in z.items():
                w[j] += m * math.exp(x) / ds
            for j, x in kap.items():
                w[j] += (1 - m) * x / dl
            assert np.all(w >= 0)
            assert abs(w.sum() - 1.0) < 1e-12
            np.testing.assert_allclose(out["O"][i], w @ v, atol=1e-12)
            assert abs(out["m"][i] - m) < 1e-12


def test_fusion_equals_joint_normalisation():
    """Default gates: O = (d_s O_s + (lam d_lr + eps) O_lr) / (d_s + lam d_lr + eps)."""
    q, k, v, W, p = _setup(lam=0.7, eps=0.25)
    out = orc.forward_head(q, k, v, W, p)
    ds = np.exp(out["logd_s"])
    c = p.lam * out["d_lr"] + p.eps
    ref = (ds[:, None] * out["O_s"] + c[:, None] * out["O_lr"]) / (ds + c)[:, None]
    np.testing.assert_allclose(out["O"], ref, atol=1e-12)


def test_branch_switches():
    q, k, v, W, p = _setup()
    # k = 0: no sparse support, m = 0, O = O_lr
    p0 = _params(p.N, p.d, p.block_size, 0, p.rank_r, True)
    out = orc.forward_head(q, k, v, W, p0)
    assert np.all(out["m"] == 0) and np.all(np.isneginf(out["logd_s"]))
    O_lr, _ = orc.race_branch(q, k, v, W, p0)
    np.testing.assert_allclose(out["O"], O_lr, atol=1e-14)
    # r = 0, eps = 0: O = O_s exactly
    p1 = _params(p.N, p.d, p.block_size, 2, 0, True, eps=0.0)
    out = orc.forward_head(q, k, v, W, p1)
    np.testing.assert_allclose(out["O"], out["O_s"], atol=1e-14)
    # lam -> large: m -> 0; explicit gates are used as given
    p2 = _params(p.N, p.d, p.block_size, 2, p.rank_r, True, lam=1e30)
    out = orc.forward_head(q, k, v, W, p2)
    assert np.all(out["m"] < 1e-20)
    gs, gl = np.full(p.N, 0.3), np.full(p.N, 2.0)
    o3 = orc.forward_head(q, k, v, W, p, g_s=gs, g_lr=gl)
    np.testing.assert_allclose(o3["O"], 0.3 * o3["m"][:, None] * o3["O_s"] + 2.0 * o3["O_lr"], atol=1e-12)


def test_equivariance_over_batch_and_heads():
    Bn, Hn, N, d, r = 2, 3, 32, 8, 16
    rng = np.random.default_rng(40)
    Q, K, V = (rng.standard_normal((Bn, Hn, N, d)) for _ in range(3))
    dO = rng.standard_normal((Bn, Hn, N, d))
    W = rng.standard_normal((1, d, 4))
    p = _params(N, d, 8, 2, r, True)
    fw = orc.forward(Q, K, V, W, p)
    g = orc.backward(Q, K, V, W, dO, fw, p)
    perm = rng.permutation(Bn * Hn)
    P = lambda x: x.reshape((Bn * Hn,) + x.shape[2:])[perm].reshape(x.shape)
    fw2 = orc.forward(P(Q), P(K), P(V), W, p)
    g2 = orc.backward(P(Q), P(K), P(V), W, P(dO), fw2, p)
    np.testing.assert_allclose(fw2["O"], P(fw["O"]), atol=1e-13)
    for a, b in zip(g2, g):
        np.testing.assert_allclose(a, P(b), atol=1e-12)


def test_key_permutation_invariance_noncausal_block1():
    N, d, r = 24, 6, 16
    q, k, v = _rand((N, d), 41), _rand((N, d), 42), _rand((N, d), 43)
    W = _rand((1, d, 4), 44)
    p = _params(N, d, 1, 5, r, False)
    out = orc.forward_head(q, k, v, W, p)
    perm = np.random.default_rng(45).permutation(N)
    out2 = orc.forward_head(q, k[perm], v[perm], W, p)
    np.testing.assert_allclose(out2["O"], out["O"], atol=1e-12)


# --- backward: central finite differences ---

def _selection(q, k, p, out):
    """What the selector chose: the block indices, or both sortLSH orders."""
    if p.selector == "sortlsh":      # the codes decide every sorted order, at every level
        return np.concatenate([orc.simhash_codes(q, p.lsh_planes), orc.simhash_codes(k, p.lsh_planes)])
    return out["idx"]


def _loss(q, k, v, W, p, dO, lam=None, g_s=None, g_lr=None):
    out = orc.forward_head(q, k, v, W, p, lam, g_s, g_lr)
    return float((out["O"] * dO).sum()), _selection(q, k, p, out)


@pytest.mark.parametrize("causal,gates,r,k,tau,fixed_m", [(True, False, 32, 2, 1.0, False),
                                                          (False, False, 16, 2, 0.6, False),
                                                          (True, True, 16, 3, 1.7, False),
                                                          (True, False, 0, 2, 1.0, False),
                                                          (True, False, 32, 0, 0.8, False),
                                                          (True, False, 16, 2, 1.0, True),
                                                          (False, True, 16, 2, 1.3, True),
                                                          (False, False, 16, "sortlsh", 1.0, False),
                                                          (False, True, 0, "sortlsh", 0.9, False),
                                                          (True, False, 16, "sortlsh", 1.0, False),
                                                          (True, True, 0, "sortlsh", 1.2, True)])
def test_backward_matches_finite_differences(causal, gates, r, k, tau, fixed_m):
    N, d, T = 24, 6, 4
    lsh = k == "sortlsh"
    q, k_, v, W, p = _setup(N=N, d=d, T=T, k=1 if lsh else k, r=r, causal=causal, seed=50, lam=0.8, tau=tau,
                            fixed_m=fixed_m)
    if lsh:
        p.selector = "sortlsh"
        p.lsh_planes = _rand((d, 3), 55)
    if r == 0:
        W = np.zeros((0, d, 4))
    dO = _rand((N, d), 60)
    lam = np.linspace(0.5, 1.5, N)
    g_s = np.linspace(0.2, 1.0, N) if gates else None
    g_lr = np.linspace(1.0, 0.1, N) if gates else None
    fw = orc.forward_head(q, k_, v, W, p, lam, g_s, g_lr)
    sel0 = _selection(q, k_, p, fw)
    dq, dk, dv = orc.backward_head(q, k_, v, W, dO, fw, p, lam, g_s, g_lr)
    h = 1e-6
    skipped = 0
    for X, G in ((q, dq), (k_, dk), (v, dv)):
        fd = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            old = X[idx]
            X[idx] = old + h
            lp, ip = _loss(q, k_, v, W, p, dO, lam, g_s, g_lr)
            X[idx] = old - h
            lm, im = _loss(q, k_, v, W, p, dO, lam, g_s, g_lr)
            X[idx] = old
            if not (np.array_equal(ip, sel0) and np.array_equal(im, sel0)):
                skipped += 1
                fd[idx] = G[idx]
                continue
            fd[idx] = (lp - lm) / (2 * h)
        scale = np.abs(G).max()
        assert np.abs(fd - G).max() <= 1e-6 * max(scale, 1.0)
        assert np.linalg.norm(fd - G) <= 1e-6 * np.linalg.norm(G) + 1e-9
    assert skipped <= 3


@pytest.mark.parametrize("fixed_m", [False, True])
def test_fusion_parameter_gradients_match_finite_differences(fixed_m):
    """d<dO, O>/d lambda_i, d/d g_s,i and d/d g_lr,i, one row at a time; gates left at
    their default are differentiated at that value (passed explicitly to the FD runs)."""
    N, d, T = 20, 6, 4
    q, k, v, W, p = _setup(N=N, d=d, T=T, k=2, r=16, causal=True, seed=70, fixed_m=fixed_m)
    dO = _rand((N, d), 71)
    lam = np.linspace(0.4, 1.6, N)
    fw = orc.forward_head(q, k, v, W, p, lam)
    dlam, dgs, dglr = orc.fusion_param_grads(dO, fw, p, lam)
    gs0 = np.ones(N)
    gl0 = np.ones(N) if fixed_m else 1.0 - fw["m"]
    h = 1e-6

    def loss(lam_, g_s=None, g_lr=None):
        return float((orc.forward_head(q, k, v, W, p, lam_, g_s, g_lr)["O"] * dO).sum())

    for i in range(N):
        e = np.zeros(N)
        e[i] = h
        fd_lam = (loss(lam + e) - loss(lam - e)) / (2 * h)
        assert abs(fd_lam - dlam[i]) <= 1e-6 * max(1.0, abs(dlam[i]))
        fd_gs = (loss(lam, gs0 + e) - loss(lam, gs0 - e)) / (2 * h)
        assert abs(fd_gs - dgs[i]) <= 1e-6 * max(1.0, abs(dgs[i]))
        fd_gl = (loss(lam, gs0, gl0 + e) - loss(lam, gs0, gl0 - e)) / (2 * h)
        assert abs(fd_gl - dglr[i]) <= 1e-6 * max(1.0, abs(dglr[i]))
    if fixed_m:
        assert np.all(dlam == 0.0)


def test_fixed_m_adds_the_two_branch_outputs():
    """The ablation without denominator-aware fusion (m = 1, default g_lr = 1) is the
    sum of the sparse-only output (r = 0) and the low-rank-only output (k = 0)."""
    q, k, v, W, p = _setup(N=40, T=8, k=2, r=32, causal=True, seed=80, fixed_m=True)
    both = orc.forward_head(q, k, v, W, p)
    p_s = _params(p.N, p.d, p.block_size, p.topk, 0, True, fixed_m=True)
    p_l = _params(p.N, p.d, p.block_size, 0, p.rank_r, True, fixed_m=True)
    sparse_only = orc.forward_head(q, k, v, np.zeros((0, p.d, 4)), p_s)["O"]
    lowrank_only = orc.forward_head(q, k, v, W, p_l)["O"]
    np.testing.assert_allclose(both["O"], sparse_only + lowrank_only, rtol=0, atol=1e-12)
    assert np.all(both["m"] == 1.0)


# --- sortLSH selector [ELSAA §3.2] ---

def test_gray_rank_inverts_the_reflected_gray_code():
    """gray_rank(n ^ (n >> 1)) = n for every n < 2^b, so neighbouring positions hold
    codes one bit apart."""
    for b in (1, 3, 8, 12):
        n = np.arange(1 << b)
        g = n ^ (n >> 1)
        assert np.array_equal(orc.gray_rank(g), n)
        flips = g[1:] ^ g[:-1]
        assert np.all((flips & (flips - 1)) == 0) and np.all(flips > 0)


def test_simhash_bit_agreement_is_one_minus_angle_over_pi():
    """Per hyperplane, two rows hash alike with probability 1 - theta/pi (the angular
    collision probability rho_ij of ELSAA §4), checked over 60000 Gaussian planes."""
    rng = np.random.default_rng(95)
    d = 16
    for trial in range(4):
        x, y = rng.standard_normal(d), rng.standard_normal(d)
        R = rng.standard_normal((d, 60000))
        agree = np.mean(((x @ R) > 0) == ((y @ R) > 0))
        theta = math.acos(np.dot(x, y) / np.linalg.norm(x) / np.linalg.norm(y))
        expect = 1 - theta / math.pi
        assert abs(agree - expect) <= 4 * math.sqrt(expect * (1 - expect) / 60000) + 1e-9


def _sortlsh_params(N, d, T, bits, seed, **kw):
    p = _params(N, d, T, 1, 0, False, eps=0.0, **kw)
    p.selector = "sortlsh"
    p.lsh_planes = _rand((d, bits), seed)
    return p


def test_sortlsh_one_block_is_dense_softmax():
    N, d = 40, 8
    q, k, v = _rand((N, d), 96), _rand((N, d), 97), _rand((N, d), 98)
    p = _sortlsh_params(N, d, N, 6, 99)
    out = orc.forward_head(q, k, v, np.zeros((0, d, 4)), p)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], scale=p.scale)[0].numpy()
    np.testing.assert_allclose(out["O"], ref, rtol=0, atol=1e-12)


def test_sortlsh_with_equal_codes_is_block_diagonal_softmax():
    """Zero hyperplanes give every row the same code, so both orders are the identity
    and query block t attends key block t of the original order."""
    N, d, T = 44, 8, 8
    q, k, v = _rand((N, d), 100), _rand((N, d), 101), _rand((N, d), 102)
    p = _sortlsh_params(N, d, T, 5, 103)
    p.lsh_planes = np.zeros((d, 5))
    out = orc.forward_head(q, k, v, np.zeros((0, d, 4)), p)
    blk = np.arange(N) // T
    mask = torch.tensor(blk[:, None] == blk[None, :])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], attn_mask=mask[None],
        scale=p.scale)[0].numpy()
    np.testing.assert_allclose(out["O"], ref, rtol=0, atol=1e-12)


def test_sortlsh_groups_rows_into_equal_blocks_of_similar_codes():
    """Each key lands in exactly one block; each block (except a ragged last one) has T
    queries and T keys; within the sorted order Gray positions never decrease and equal
    codes keep their index order."""
    N, d, T = 70, 8, 8
    q, k = _rand((N, d), 104), _rand((N, d), 105)
    p = _sortlsh_params(N, d, T, 4, 106)
    sup = orc.sortlsh_support(q, k, p)
    seen = np.zeros(N, dtype=int)
    for t in range(p.n_tiles):
        keys = sup[orc.sortlsh_order(q, p.lsh_planes)[t * T]]
        seen[keys] += 1
        assert keys.size == min(T, N - t * T)
    assert np.all(seen == 1)
    for X in (q, k):
        order = orc.sortlsh_order(X, p.lsh_planes)
        pos = orc.gray_rank(orc.simhash_codes(X, p.lsh_planes))[order]
        assert np.all(np.diff(pos) >= 0)
        same = np.diff(pos) == 0
        assert np.all(np.diff(order)[same] > 0)


# --- causal sortLSH: the recursion of §3.2 ---

def _causal_lsh_params(N, d, T, bits, seed, **kw):
    p = _sortlsh_params(N, d, T, bits, seed, **kw)
    p.causal = True
    return p


@pytest.mark.parametrize("N,T", [(8, 8), (5, 8), (16, 8), (13, 8)])
def test_causal_sortlsh_up_to_two_blocks_is_dense_causal_softmax(N, T):
    """One block is the leaf (exact under j <= i); with two, the future block's single
    sorted query block meets the past half's single key block, i.e. every earlier key."""
    d = 6
    q, k, v = _rand((N, d), 120), _rand((N, d), 121), _rand((N, d), 122)
    p = _causal_lsh_params(N, d, T, 5, 123)
    out = orc.forward_head(q, k, v, np.zeros((0, d, 4)), p)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], is_causal=True,
        scale=p.scale)[0].numpy()
    np.testing.assert_allclose(out["O"], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("N,T,bits", [(64, 8, 3), (70, 8, 4), (96, 4, 2)])
def test_causal_sortlsh_recursion_is_softmax_over_the_union_of_its_supports(N, T, bits):
    """The recursion's log-sum-exp merges give the exact softmax over the union of the
    key sets it visits (computed row by row from the support)."""
    d = 6
    q, k, v = _rand((N, d), 124), _rand((N, d), 125), _rand((N, d), 126)
    p = _causal_lsh_params(N, d, T, bits, 127)
    O, logd = orc.causal_sortlsh(q, k, v, p)
    O2, logd2 = orc.sparse_from_support(q, k, v, orc.causal_sortlsh_support(q, k, p), p)
    np.testing.assert_allclose(O, O2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(logd, logd2, rtol=0, atol=1e-12)


def test_causal_sortlsh_support_sizes_follow_the_block_index_bits():
    """With 2^L blocks every split is exact: row i in block t is in the future half at
    one level per set bit of t, gaining T keys there, plus its own block's keys j <= i;
    all keys precede i and no key repeats."""
    N, d, T = 128, 6, 8
    q, k = _rand((N, d), 128), _rand((N, d), 129)
    p = _causal_lsh_params(N, d, T, 4, 130)
    for i, keys in enumerate(orc.causal_sortlsh_support(q, k, p)):
        t = i // T
        assert keys.size == (i % T) + 1 + T * bin(t).count("1")
        assert np.all(np.diff(keys) > 0) and keys[-1] == i
        assert np.all(keys[keys >= t * T] == np.arange(t * T, i + 1))


def test_causal_sortlsh_with_equal_codes_attends_blocks_t_minus_powers_of_two():
    """Zero hyperplanes give every row the same code, so each sorted order is the row
    order: the future block with offset u in a half of 2^j blocks meets the past block
    with offset u, i.e. block t attends t and t - 2^j for every set bit j of t."""
    N, d, T = 64, 6, 4
    q, k, v = _rand((N, d), 131), _rand((N, d), 132), _rand((N, d), 133)
    p = _causal_lsh_params(N, d, T, 3, 134)
    p.lsh_planes = np.zeros((d, 3))
    mask = np.zeros((N, N), dtype=bool)
    for i in range(N):
        t = i // T
        mask[i, t * T:i + 1] = True
        for j in range(t.bit_length()):
            if t >> j & 1:
                b = t - (1 << j)
                mask[i, b * T:(b + 1) * T] = True
    out = orc.forward_head(q, k, v, np.zeros((0, d, 4)), p)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], attn_mask=torch.tensor(mask)[None],
        scale=p.scale)[0].numpy()
    np.testing.assert_allclose(out["O"], ref, rtol=0, atol=1e-12)


# --- rank view [ELSAA §4]: rank(S_Omega + B A) = min(n, nu(Omega) + r) ---

def test_max_matching_against_brute_force():
    """nu(Omega) equals the largest k for which some k rows can be matched to k
    distinct columns, found by trying every injective assignment (n <= 6)."""
    rng = np.random.default_rng(90)
    for trial in range(60):
        n_r, n_c = int(rng.integers(1, 6)), int(rng.integers(1, 6))
        mask = rng.random((n_r, n_c)) < rng.uniform(0.1, 0.7)
        exact = 0
        for size in range(min(n_r, n_c), 0, -1):
            if any(all(mask[i, j] for i, j in zip(rows, perm))
                   for rows in itertools.combinations(range(n_r), size)
                   for perm in itertools.permutations(range(n_c), size)):
                exact = size
                break
        assert orc.max_matching(mask) == exact


@pytest.mark.parametrize("causal,T,k,r", [(True, 4, 2, 0), (True, 4, 2, 8), (False, 8, 1, 16), (True, 8, 3, 32),
                                          (False, 4, 16, 0)])
def test_rank_of_sparse_plus_low_rank_matches_theorem(causal, T, k, r):
    """On the supports the top-k block selector realises, rank(S_Omega + B A) equals
    min(n, nu(Omega) + r); r = 0 gives the structural rank nu(Omega) itself, and a full
    support (k = n_t, non-causal) gives n."""
    n, d = 64, 16
    q, kk = _rand((n, d), 91, 0.7), _rand((n, d), 92, 0.7)
    p = _params(n, d, T, k, 16, causal)
    idx = orc.select_from_scores(orc.block_scores(q, kk, p), p.topk, p.causal)
    out = orc.rank_diagnostic(q, kk, idx, p, r, seed=93)
    assert out["rank"] == out["predicted"], out
    if not causal and k * T >= n:
        assert out["nu"] == n


# --- a value printed in the paper ---

def test_interaction_count_matches_paper_example():
    with open(os.path.join(GOLDEN, "interaction_count.json")) as f:
        g = json.load(f)
    a = g["args"]
    assert orc.interaction_count(a["N"], a["s"], a["L_s"], a["gamma"]) == g["elsaa_interactions"]
    assert a["N"] ** 2 == g["dense_interactions"]


# --- the row-sampled forms agree with the whole-head forms pinned above ---

@pytest.mark.parametrize("causal", [True, False])
def test_row_sampled_forms_match_full(causal):
    q, k, v, W, p = _setup(N=44, d=8, T=8, k=2, r=32, causal=causal, seed=70)
    dO = _rand((p.N, p.d), 71)
    lam = np.linspace(0.5, 1.5, p.N)
    fw = orc.forward_head(q, k, v, W, p, lam)
    rows = [0, 7, 8, 30, 43]
    fr = orc.forward_rows_head(q, k, v, W, p, rows, lam)
    for key in ("O", "O_s", "logd_s", "O_lr", "d_lr", "m"):
        np.testing.assert_allclose(fr[key], fw[key][rows], atol=1e-12, rtol=1e-12)
    dq, dk, dv = orc.backward_head(q, k, v, W, dO, fw, p, lam)
    sq, sk, sv = orc.backward_rows_head(q, k, v, W, dO, fw, p, rows, rows, lam)
    np.testing.assert_allclose(sq, dq[rows], atol=1e-11)
    np.testing.assert_allclose(sk, dk[rows], atol=1e-11)
    np.testing.assert_allclose(sv, dv[rows], atol=1e-11)


def test_sortlsh_external_orders_and_codes_change_nothing_when_they_agree():
    """The GPU parity tests hand the oracle the GPU's sorted orders (non-causal) or hash codes
    (causal); given the oracle's own, the results are identical."""
    N, d, T = 72, 6, 8
    q, k, v = _rand((N, d), 140), _rand((N, d), 141), _rand((N, d), 142)
    dO = _rand((N, d), 143)
    W = np.zeros((0, d, 4))
    for causal in (False, True):
        if causal:
            N2 = 64                       # the causal recursion in the GPU's form: 2^L blocks
            q2, k2, v2, dO2 = q[:N2], k[:N2], v[:N2], dO[:N2]
            p = _causal_lsh_params(N2, d, T, 4, 144)
        else:
            q2, k2, v2, dO2 = q, k, v, dO
            p = _sortlsh_params(N, d, T, 4, 144)
        fw = orc.forward_head(q2, k2, v2, W, p)
        g = orc.backward_head(q2, k2, v2, W, dO2, fw, p)
        if causal:
            p.lsh_codes = (orc.simhash_codes(q2, p.lsh_planes), orc.simhash_codes(k2, p.lsh_planes))
        else:
            p.lsh_orders = (orc.sortlsh_order(q2, p.lsh_planes), orc.sortlsh_order(k2, p.lsh_planes))
        p.lsh_planes = np.full_like(p.lsh_planes, np.nan)    # the overrides alone must decide
        fw2 = orc.forward_head(q2, k2, v2, W, p)
        g2 = orc.backward_head(q2, k2, v2, W, dO2, fw2, p)
        np.testing.assert_array_equal(fw2["O"], fw["O"])
        for a, b in zip(g2, g):
            np.testing.assert_array_equal(a, b)
