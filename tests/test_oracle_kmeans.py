"""Pins of the semantic-aware permutation oracle (CPU, no GPU).

k-means is checked against what fixes it independently of its own code:
planted, well-separated clusters are recovered exactly; the fp32 assignment
agrees with an fp64 argmin wherever the two nearest centroids are not
near-equal; centroids are fp64 means within fp32 rounding; a converged state
is a fixed point; ties go to the lower index. The permutation is checked as a
stable sort, and the Sparse VideoGen2 §2A equivalence claim (permuting Q rows
and K, V rows consistently leaves dense attention unchanged) against PyTorch's
scaled_dot_product_attention in fp64.
"""
import numpy as np
import pytest
import torch

from oracle.svg_permutation_oracle import (assign, initial_centroids, kmeans_permutation,
                                           permuted_sparse_attention, stable_permutation, update)


def _blobs(n_per, centers, spread, seed):
    g = np.random.default_rng(seed)
    X = np.concatenate([c + spread * g.standard_normal((n_per, len(c))) for c in centers])
    return X.astype(np.float32)


def test_planted_clusters_are_recovered():
    g = np.random.default_rng(0)
    centers = g.standard_normal((6, 16)) * 10.0
    X = _blobs(50, centers, 0.1, 1)
    perm = g.permutation(X.shape[0])
    X = X[perm]
    truth = np.repeat(np.arange(6), 50)[perm]
    # One initial centroid inside each blob.
    init = np.stack([X[np.nonzero(truth == c)[0][0]] for c in range(6)])
    ids, p, M = kmeans_permutation(X, 6, 4, init=init)
    assert np.array_equal(ids, truth)
    for c in range(6):
        assert np.allclose(M[c], X[truth == c].astype(np.float64).mean(0), rtol=0, atol=1e-5)


def test_fp32_assignment_agrees_with_fp64_where_the_gap_is_clear():
    g = np.random.default_rng(2)
    X = g.standard_normal((2000, 32)).astype(np.float32)
    M = g.standard_normal((40, 32)).astype(np.float32)
    ids = assign(X, M)
    D = ((X.astype(np.float64)[:, None, :] - M.astype(np.float64)[None]) ** 2).sum(-1)
    order = np.sort(D, axis=1)
    clear = (order[:, 1] - order[:, 0]) > 1e-4 * order[:, 0]
    assert clear.mean() > 0.99
    assert np.array_equal(ids[clear], np.argmin(D, axis=1)[clear])


def test_ties_go_to_the_lower_index():
    X = np.zeros((3, 4), dtype=np.float32)
    M = np.array([[1, 0, 0, 0], [0, 1, 0, 0], [0, 0, 0, 1]], dtype=np.float32)   # all at distance 1
    assert assign(X, M).tolist() == [0, 0, 0]


def test_update_is_the_mean_and_keeps_empty_clusters():
    g = np.random.default_rng(3)
    X = g.standard_normal((300, 8)).astype(np.float32)
    ids = g.integers(0, 5, 300).astype(np.int32)
    ids[ids == 3] = 4                                     # cluster 3 empty
    M0 = g.standard_normal((5, 8)).astype(np.float32)
    M = update(X, ids, M0)
    for c in (0, 1, 2, 4):
        assert np.allclose(M[c], X[ids == c].astype(np.float64).mean(0), rtol=1e-6, atol=1e-6)
    assert np.array_equal(M[3], M0[3])


def test_converged_state_is_a_fixed_point():
    X = _blobs(40, np.random.default_rng(4).standard_normal((5, 8)) * 6, 0.2, 5)
    ids, _, M = kmeans_permutation(X, 5, 10)
    assert np.array_equal(update(X, assign(X, M), M), M)
    ids2, _, M2 = kmeans_permutation(X, 5, 1, init=M)
    assert np.array_equal(ids2, ids) and np.array_equal(M2, M)


def test_initial_centroids_and_stable_permutation():
    X = np.arange(40, dtype=np.float32).reshape(10, 4)
    assert np.array_equal(initial_centroids(X, 3), X[[0, 3, 6]])
    ids = np.array([2, 0, 1, 0, 2, 1, 0], dtype=np.int32)
    p = stable_permutation(ids)
    assert p.tolist() == [1, 3, 6, 2, 5, 0, 4]
    assert sorted(p.tolist()) == list(range(7))


@pytest.mark.parametrize("N,bq", [(256, 64), (300, 128)])
def test_dense_attention_is_unchanged_by_the_permutation(N, bq):
    g = np.random.default_rng(N)
    B, H, d = 1, 2, 16
    Q, K, V = (g.standard_normal((B, H, N, d)) for _ in range(3))
    perm_q = np.stack([[g.permutation(N) for _ in range(H)]])
    perm_k = np.stack([[g.permutation(N) for _ in range(H)]])
    n_q, n_k = -(-N // bq), -(-N // 64)
    cnt = np.full((B, H, n_q), n_k, dtype=np.int32)
    idx = np.broadcast_to(np.arange(n_k, dtype=np.int32), (B, H, n_q, n_k)).copy()
    O = permuted_sparse_attention(Q, K, V, perm_q, perm_k, cnt, idx, bq, 64)
    ref = torch.nn.functional.scaled_dot_product_attention(*(torch.tensor(x) for x in (Q, K, V))).numpy()
    assert np.allclose(O, ref, rtol=1e-12, atol=1e-12)
