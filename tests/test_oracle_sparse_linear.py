"""Pins of the sparse + linear combination oracle (CPU, no GPU).

Checked against things other than itself: PyTorch's elu (a library routine)
for the feature map; the "total minus kept" route to the complement sums,
phi(q)^T (sum over all keys - sum over kept keys), computed without the
complement set; closed forms (V constant, alpha = 0 or 1); convexity; block
permutation; and brute force over token pairs on a tiny case.
"""
import math

import numpy as np
import pytest
import torch

import oracle as O
from oracle.sparse_linear_oracle import complement_tokens, linear_row, phi, sparse_linear_attention


def _case(B=1, H=2, N=300, d=16, seed=0):
    g = np.random.default_rng(seed)
    Q, K, V = (g.standard_normal((B, H, N, d)) for _ in range(3))
    alpha = g.uniform(0, 1, (B, H, N))
    return Q, K, V, alpha


def _lists(B, H, n_q, n_k, seed, full_every=0):
    g = np.random.default_rng(seed)
    cnt = np.zeros((B, H, n_q), dtype=np.int32)
    idx = np.full((B, H, n_q, n_k), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n_q):
                c = int(g.integers(1, n_k))
                if full_every and (b + h + i) % full_every == 1:
                    c = n_k
                cnt[b, h, i] = c
                idx[b, h, i, :c] = g.permutation(n_k)[:c]
    return cnt, idx


def test_phi_is_elu_plus_one():
    x = np.linspace(-30, 30, 100001)
    ref = torch.nn.functional.elu(torch.tensor(x, dtype=torch.float64)).numpy() + 1.0
    # The library forms expm1(x) + 1, which cancels for very negative x: the
    # comparison is absolute, at the scale of a unit in fp64.
    assert np.max(np.abs(phi(x) - ref)) <= 4e-16
    assert np.all(phi(x) > 0)


def test_complement_by_total_minus_kept():
    Q, K, V, _ = _case()
    N, d, bk = 300, 16, 64
    kept = [0, 3]
    q = Q[0, 0, :64]
    # Without the complement set: all-key sums minus kept-key sums.
    fk, fq = phi(K[0, 0]), phi(q)
    kept_tok = [t for j in kept for t in range(j * bk, min(N, (j + 1) * bk))]
    H_all, z_all = fk.T @ V[0, 0], fk.sum(0)
    H_kept, z_kept = fk[kept_tok].T @ V[0, 0][kept_tok], fk[kept_tok].sum(0)
    ref = (fq @ (H_all - H_kept)) / (fq @ (z_all - z_kept))[:, None]
    assert np.allclose(linear_row(q, K[0, 0], V[0, 0], kept, bk), ref, rtol=1e-12, atol=1e-12)


def test_brute_force_pairs_tiny():
    g = np.random.default_rng(3)
    N, d, bk = 130, 4, 64
    q, K, V = g.standard_normal((2, d)), g.standard_normal((N, d)), g.standard_normal((N, d))
    kept = [1]
    u = [t for t in range(N) if not (64 <= t < 128)]
    for r in range(2):
        num = np.zeros(d)
        den = 0.0
        for t in u:
            w = sum((math.exp(a) if a <= 0 else a + 1) * (math.exp(b) if b <= 0 else b + 1)
                    for a, b in zip(q[r], K[t]))
            num += w * V[t]
            den += w
        assert np.allclose(linear_row(q, K, V, kept, bk)[r], num / den, rtol=1e-12)


def test_constant_v_and_alpha_extremes():
    Q, K, V, alpha = _case(seed=1)
    B, H, N, d = Q.shape
    n_q, n_k = -(-N // 64), -(-N // 64)
    cnt, idx = _lists(B, H, n_q, n_k, 2)
    Vc = np.full_like(V, 2.5)
    Oc, Os, Ol = sparse_linear_attention(Q, K, Vc, alpha, cnt, idx, 64, 64)
    assert np.allclose(Oc, 2.5) and np.allclose(Ol, 2.5)
    O1, Os1, _ = sparse_linear_attention(Q, K, V, np.ones_like(alpha), cnt, idx, 64, 64)
    assert np.array_equal(O1, Os1)
    Os_ref, _ = O.block_sparse_attention(Q, K, V, cnt, idx, 64, 64)
    assert np.allclose(Os1, Os_ref, rtol=1e-14, atol=1e-14)
    O0, _, Ol0 = sparse_linear_attention(Q, K, V, np.zeros_like(alpha), cnt, idx, 64, 64)
    assert np.array_equal(O0, Ol0)


def test_linear_branch_is_a_convex_combination_of_complement_values():
    Q, K, V, alpha = _case(seed=4)
    N, bk = 300, 64
    for kept in ([0], [1, 2], [4]):
        ol = linear_row(Q[0, 1, :64], K[0, 1], V[0, 1], kept, bk)
        u = complement_tokens(N, kept, bk)
        assert np.all(ol <= V[0, 1][u].max(0) + 1e-12) and np.all(ol >= V[0, 1][u].min(0) - 1e-12)


def test_full_rows_have_no_linear_branch():
    Q, K, V, alpha = _case(seed=5)
    B, H, N, d = Q.shape
    n_q = n_k = -(-N // 64)
    cnt, idx = _lists(B, H, n_q, n_k, 6, full_every=3)
    O_, Os, Ol = sparse_linear_attention(Q, K, V, alpha, cnt, idx, 64, 64)
    for (b, h, i) in zip(*np.nonzero(cnt == n_k)):
        lo, hi = i * 64, min(N, (i + 1) * 64)
        assert np.all(Ol[b, h, lo:hi] == 0)
        assert np.allclose(O_[b, h, lo:hi], alpha[b, h, lo:hi, None] * Os[b, h, lo:hi])


def test_key_block_permutation_leaves_the_output_unchanged():
    Q, K, V, alpha = _case(N=256, seed=7)
    B, H, N, d = Q.shape
    n_q = n_k = 4
    cnt, idx = _lists(B, H, n_q, n_k, 8)
    perm = np.array([2, 0, 3, 1])                       # new block j holds old block perm[j]
    inv = np.argsort(perm)
    tok = np.concatenate([np.arange(p * 64, (p + 1) * 64) for p in perm])
    Kp, Vp = K[:, :, tok], V[:, :, tok]
    idx_p = np.where(idx >= 0, inv[np.maximum(idx, 0)], -1)
    a, _, _ = sparse_linear_attention(Q, K, V, alpha, cnt, idx, 64, 64)
    b, _, _ = sparse_linear_attention(Q, Kp, Vp, alpha, cnt, idx_p, 64, 64)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("mutation", ["no_plus_one", "kept_not_complement", "alpha_swapped"])
def test_planted_mistakes_fail_a_pin(mutation):
    Q, K, V, alpha = _case(seed=9)
    B, H, N, d = Q.shape
    n_q = n_k = -(-N // 64)
    cnt, idx = _lists(B, H, n_q, n_k, 10)
    good, Os, Ol = sparse_linear_attention(Q, K, V, alpha, cnt, idx, 64, 64)
    i = 1
    lo, hi = 64, 128
    kept = idx[0, 0, i, :cnt[0, 0, i]]
    q = Q[0, 0, lo:hi]
    if mutation == "no_plus_one":
        fq, fk = np.where(q > 0, q, np.exp(np.minimum(q, 0))), np.where(K[0, 0] > 0, K[0, 0], np.exp(np.minimum(K[0, 0], 0)))
        u = complement_tokens(N, kept, 64)
        W = fq @ fk[u].T
        bad = (W @ V[0, 0][u]) / W.sum(1, keepdims=True)
        assert not np.allclose(bad, Ol[0, 0, lo:hi])
    elif mutation == "kept_not_complement":
        u = np.array([t for j in kept for t in range(j * 64, min(N, (j + 1) * 64))])
        W = phi(q) @ phi(K[0, 0][u]).T
        bad = (W @ V[0, 0][u]) / W.sum(1, keepdims=True)
        assert not np.allclose(bad, Ol[0, 0, lo:hi])
    else:
        a = alpha[0, 0, lo:hi, None]
        bad = (1 - a) * Os[0, 0, lo:hi] + a * Ol[0, 0, lo:hi]
        assert not np.allclose(bad, good[0, 0, lo:hi])
