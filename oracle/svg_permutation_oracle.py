"""Semantic-aware permutation (Sparse VideoGen2) ahead of the block-sparse path:
the plain statement.

TEST INFRASTRUCTURE ONLY (see the package docstring): only ``tests/`` may
import this module; the CUDA path shares no code with it.

Source: "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via
Semantic-Aware Permutation" (gist.science summary), §2A Semantic-Aware
Permutation: Q and K tokens are clustered independently by k-means, and the
tokens are reordered so that each cluster is contiguous; applying the
permutations to Q rows and to K and V rows (and undoing the Q permutation on the
output) leaves dense attention unchanged. §2B Centroid-Based Top-p Selection
scores the clusters by their centroids and keeps them until the cumulative
score reaches p; §2C caches the centroids of one step to start the next.

Readings (the page gives no initialisation, distance, iteration count or tie
rule; these are the plainest):
* k-means is Lloyd's iteration on the token vectors of one (batch, head),
  squared Euclidean distance, C clusters, T iterations of (assign, update)
  followed by a final assignment; the initial centroids are the tokens at
  positions floor(c N / C) (or centroids passed in: the cache of §2C);
* every decision is taken in fp32, as the GPU takes it: the distance of token
  x to centroid m is the sum over channels, in channel order, of
  (x_j - m_j)^2 with the subtraction, the product and each addition rounded
  to fp32 (no fused multiply-add); the nearest centroid wins, equal distances
  going to the lower cluster index; a centroid becomes the fp32 sum of its
  members' vectors, added in ascending token order, divided by the member
  count (fp32); an empty cluster keeps its centroid;
* the permutation lists the tokens sorted by cluster, ascending token order
  within a cluster (a stable sort);
* the selection then runs on the permuted sequence with this path's fixed
  blocks (64 keys, 64 or 128 queries) and its hybrid Top-k + Top-p rule on
  pooled block means: a block of the permuted sequence lies mostly inside one
  cluster, so its mean stands in for a centroid (SVG2's own kernel takes
  blocks of the clusters' own sizes instead).

Pins: ``tests/test_oracle_kmeans.py``.
"""
from __future__ import annotations

import numpy as np

from .sparse_attn_oracle import block_sparse_attention, to_f64


def initial_centroids(X32: np.ndarray, C: int) -> np.ndarray:
    """Tokens at positions floor(c N / C), c < C. X32: [N, d] fp32."""
    N = X32.shape[0]
    pos = (np.arange(C, dtype=np.int64) * N) // C
    return X32[pos].copy()


def assign(X32: np.ndarray, M32: np.ndarray) -> np.ndarray:
    """Nearest centroid of every token (fp32 arithmetic as stated above).

    X32: [N, d] fp32, M32: [C, d] fp32 -> int32 [N].
    """
    N, d = X32.shape
    dist = np.zeros((N, M32.shape[0]), dtype=np.float32)
    for j in range(d):
        diff = (X32[:, j, None] - M32[None, :, j]).astype(np.float32)
        dist = (dist + (diff * diff).astype(np.float32)).astype(np.float32)
    return np.argmin(dist, axis=1).astype(np.int32)        # first minimum: the lower index


def update(X32: np.ndarray, ids: np.ndarray, M32: np.ndarray) -> np.ndarray:
    """New centroids: fp32 sums in ascending token order, divided by the count."""
    out = M32.copy()
    for c in range(M32.shape[0]):
        members = np.nonzero(ids == c)[0]                   # ascending token order
        if members.size == 0:
            continue
        s = np.cumsum(X32[members], axis=0, dtype=np.float32)[-1]   # sequential fp32 sum
        out[c] = (s / np.float32(members.size)).astype(np.float32)
    return out


def stable_permutation(ids: np.ndarray) -> np.ndarray:
    """Tokens sorted by cluster id, ascending token order within a cluster."""
    return np.argsort(ids, kind="stable").astype(np.int32)


def kmeans_permutation(X, C: int, iters: int, init: np.ndarray | None = None):
    """k-means of one head's tokens. X: [N, d] (bf16 tensor or array).

    Returns (ids int32 [N], perm int32 [N], centroids fp32 [C, d]): the final
    assignment, the stable permutation and the centroids after `iters`
    updates.
    """
    X32 = to_f64(X).astype(np.float32)
    M = initial_centroids(X32, C) if init is None else np.asarray(init, dtype=np.float32).copy()
    for _ in range(iters):
        M = update(X32, assign(X32, M), M)
    ids = assign(X32, M)
    return ids, stable_permutation(ids), M


def permuted_sparse_attention(Q, K, V, perm_q, perm_k, cnt, idx, bq: int, bk: int):
    """The block-sparse attention on the permuted sequences, output restored to
    token order: O[b, h, perm_q[i]] = attention of permuted query row i over the
    permuted keys/values (cnt, idx: the kept lists of the permuted sequence).

    Q, K, V: [B, H, N, d]; perm_q, perm_k: int [B, H, N]. Returns O fp64.
    """
    Q64, K64, V64 = to_f64(Q), to_f64(K), to_f64(V)
    pq = np.asarray(perm_q)
    pk = np.asarray(perm_k)
    Qp = np.take_along_axis(Q64, pq[..., None].astype(np.int64), axis=2)
    Kp = np.take_along_axis(K64, pk[..., None].astype(np.int64), axis=2)
    Vp = np.take_along_axis(V64, pk[..., None].astype(np.int64), axis=2)
    Op, _ = block_sparse_attention(Qp, Kp, Vp, cnt, idx, bq, bk)
    O = np.empty_like(Op)
    np.put_along_axis(O, pq[..., None].astype(np.int64), Op, axis=2)
    return O
