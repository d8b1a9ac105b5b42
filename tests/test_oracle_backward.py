"""Pins of the backward-pass oracle (CPU, no GPU).

The oracle states dQ, dK, dV of block-sparse attention as hand-derived formulas
(sparse_attn_backward). They are checked against things other than
themselves: PyTorch autograd through the same masked softmax attention in
fp64 (a library routine), central finite differences of the forward oracle,
and two invariants of softmax attention (each row's weights sum to 1, so its
score gradients sum to 0).
"""
import math
import os
import types

import numpy as np
import pytest
import torch

import oracle as O


def _inputs(B, H, N, d, seed):
    g = np.random.default_rng(seed)
    Q, K, V, dO = (g.standard_normal((B, H, N, d)) for _ in range(4))
    return Q, K, V, dO


def _random_lists(B, H, n_q, n_k, seed, empty_every=5):
    g = np.random.default_rng(seed)
    cnt = np.zeros((B, H, n_q), dtype=np.int32)
    idx = np.full((B, H, n_q, n_k), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n_q):
                c = int(g.integers(1, n_k + 1))
                if (b + h + i) % empty_every == 2:
                    c = 0
                cnt[b, h, i] = c
                idx[b, h, i, :c] = g.permutation(n_k)[:c]      # any order
    return cnt, idx


def _autograd(Q, K, V, dO, cnt, idx, bq, bk):
    """The same attention through torch autograd: a masked softmax over all keys."""
    B, H, N, d = Q.shape
    q, k, v = (torch.tensor(x, dtype=torch.float64, requires_grad=True) for x in (Q, K, V))
    allowed = torch.zeros((B, H, N, N), dtype=torch.bool)
    n_q = -(-N // bq)
    for b in range(B):
        for h in range(H):
            for i in range(n_q):
                for j in idx[b, h, i, : int(cnt[b, h, i])]:
                    allowed[b, h, i * bq:(i + 1) * bq, int(j) * bk:(int(j) + 1) * bk] = True
    s = torch.einsum("bhnd,bhmd->bhnm", q, k) / math.sqrt(d)
    s = s.masked_fill(~allowed, float("-inf"))
    p = torch.softmax(s, dim=-1)
    p = torch.nan_to_num(p, nan=0.0)        # rows with no kept block: output 0
    o = torch.einsum("bhnm,bhmd->bhnd", p, v)
    o.backward(torch.tensor(dO))
    return q.grad.numpy(), k.grad.numpy(), v.grad.numpy()


@pytest.mark.parametrize("N,d,bq,bk,seed", [(64, 16, 16, 8, 1), (50, 8, 16, 8, 2), (37, 4, 8, 4, 3)])
def test_backward_matches_autograd(N, d, bq, bk, seed):
    B, H = 2, 2
    Q, K, V, dO = _inputs(B, H, N, d, seed)
    n_q, n_k = -(-N // bq), -(-N // bk)
    cnt, idx = _random_lists(B, H, n_q, n_k, seed + 10)
    dQ, dK, dV = O.block_sparse_attention_backward(Q, K, V, dO, cnt, idx, bq, bk)
    gq, gk, gv = _autograd(Q, K, V, dO, cnt, idx, bq, bk)
    for a, b_ in ((dQ, gq), (dK, gk), (dV, gv)):
        assert np.allclose(a, b_, rtol=1e-10, atol=1e-12)


def test_backward_dense_matches_autograd():
    B, H, N, d, bq, bk = 1, 2, 48, 8, 16, 8
    Q, K, V, dO = _inputs(B, H, N, d, 7)
    n_q, n_k = N // bq, N // bk
    cnt = np.full((B, H, n_q), n_k, dtype=np.int32)
    idx = np.tile(np.arange(n_k, dtype=np.int32), (B, H, n_q, 1))
    dQ, dK, dV = O.block_sparse_attention_backward(Q, K, V, dO, cnt, idx, bq, bk)
    gq, gk, gv = _autograd(Q, K, V, dO, cnt, idx, bq, bk)
    assert np.allclose(dQ, gq, rtol=1e-10, atol=1e-12)
    assert np.allclose(dK, gk, rtol=1e-10, atol=1e-12)
    assert np.allclose(dV, gv, rtol=1e-10, atol=1e-12)


def test_backward_matches_finite_differences_of_the_forward_oracle():
    """d/dx of L = sum(dO * O), O from the forward oracle, by central differences."""
    B, H, N, d, bq, bk = 1, 1, 12, 4, 4, 4
    Q, K, V, dO = _inputs(B, H, N, d, 5)
    cnt = np.array([[[2, 1, 3]]], dtype=np.int32)
    idx = np.array([[[[2, 0, -1], [1, -1, -1], [0, 1, 2]]]], dtype=np.int32)
    dQ, dK, dV = O.block_sparse_attention_backward(Q, K, V, dO, cnt, idx, bq, bk)

    def loss(Qx, Kx, Vx):
        Ox, _ = O.block_sparse_attention(Qx, Kx, Vx, cnt, idx, bq, bk)
        return float(np.sum(dO * Ox))

    eps = 1e-6
    g = np.random.default_rng(0)
    for X, G, which in ((Q, dQ, 0), (K, dK, 1), (V, dV, 2)):
        for _ in range(6):
            t = (0, 0, int(g.integers(N)), int(g.integers(d)))
            Xp, Xm = X.copy(), X.copy()
            Xp[t] += eps
            Xm[t] -= eps
            args_p = [Q, K, V]
            args_m = [Q, K, V]
            args_p[which], args_m[which] = Xp, Xm
            fd = (loss(*args_p) - loss(*args_m)) / (2 * eps)
            assert abs(fd - G[t]) <= 1e-7 * max(1.0, abs(fd)), (which, t, fd, G[t])


def test_backward_invariants():
    """Each row's weights sum to 1: sum over keys of dS is 0, so sum_j dK_j = 0 per
    (b, h); and sum_j dV_j equals the sum of dO over the query tokens whose row
    keeps at least one block. Rows with no kept block get dQ = 0."""
    B, H, N, d, bq, bk = 2, 3, 40, 8, 8, 8
    Q, K, V, dO = _inputs(B, H, N, d, 9)
    n_q, n_k = N // bq, N // bk
    cnt, idx = _random_lists(B, H, n_q, n_k, 19, empty_every=3)
    dQ, dK, dV = O.block_sparse_attention_backward(Q, K, V, dO, cnt, idx, bq, bk)
    assert np.allclose(dK.sum(axis=2), 0.0, atol=1e-11)
    live = np.repeat(cnt > 0, bq, axis=-1)[..., :N]
    assert np.allclose(dV.sum(axis=2), (dO * live[..., None]).sum(axis=2), atol=1e-11)
    assert np.all(dQ[~live] == 0.0)


# ------------------------------------------------ planted mistakes are caught
BACKWARD_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                            "oracle", "sparse_attn_backward.py")


def _mutant(old, new):
    """A private copy of the backward oracle with one text substitution."""
    src = open(BACKWARD_SRC).read()
    assert src.count(old) == 1, old
    src = src.replace(old, new).replace("from .sparse_attn_oracle import", "from oracle.sparse_attn_oracle import")
    mod = types.ModuleType("backward_mutant")
    exec(compile(src, "backward_mutant", "exec"), mod.__dict__)
    return mod


def _autograd_pin_holds(mod) -> bool:
    B, H, N, d, bq, bk = 2, 2, 50, 8, 16, 8
    Q, K, V, dO = _inputs(B, H, N, d, 4)
    n_q, n_k = -(-N // bq), -(-N // bk)
    cnt, idx = _random_lists(B, H, n_q, n_k, 14)
    got = mod.block_sparse_attention_backward(Q, K, V, dO, cnt, idx, bq, bk)
    ref = _autograd(Q, K, V, dO, cnt, idx, bq, bk)
    return all(np.allclose(a, b_, rtol=1e-10, atol=1e-12) for a, b_ in zip(got, ref))


@pytest.mark.parametrize("old,new", [
    ("dS = P * (dP - D)", "dS = P * dP"),                                  # drops the row term
    ("dq = c * (dS @ Ku)", "dq = dS @ Ku"),                                # forgets 1/sqrt(d)
    ("dV_u = P.T @ dO", "dV_u = E.T @ dO"),                                # unnormalised weights
    ("np.add.at(dK[b, h], u, dk)", "dK[b, h][u] = dk"),                   # overwrites, no sum
    ("dK_u = c * (dS.T @ q)", "dK_u = c * (P.T @ q)"),                     # wrong factor
])
def test_each_planted_mistake_fails_the_autograd_pin(old, new):
    assert _autograd_pin_holds(O)
    assert not _autograd_pin_holds(_mutant(old, new))
