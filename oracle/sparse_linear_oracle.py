"""Sparse + linear attention combination (SLA2): the plain fp64 statement.

TEST INFRASTRUCTURE ONLY (see the package docstring): only ``tests/`` and
``bench.py``'s oracle legs may import this module; the CUDA path shares no
code with it.

Source: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT"
(gist.science summary), §1 Problem Statement (sparse attention for the
high-weight part of each row, linear attention for the low-weight part) and
§2A Faithful Sparse-Linear Formulation: the output is O = alpha * O_s +
(1 - alpha) * O_l, with O_s the sparse attention output, O_l the linear
attention output and alpha a learned vector of values in [0, 1]; the split
follows the decomposition P ~ P_1 + P_2 of the attention weights into the
kept (sparse) part and the rest. The page prints no feature map and no
shape for alpha. Readings taken here:

* the split is the hybrid mask of this path: O_s attends to the tokens of a
  row's kept key blocks (``sparse_attn_oracle.attend_row``), O_l to the
  tokens of every other key block of the row (the complement);
* the linear branch is kernelised attention with the positive feature map
  phi(x) = elu(x) + 1 (Katharopoulos et al., "Transformers are RNNs", 2020):
  O_l(t) = sum_u (phi(q_t) . phi(k_u)) v_u / sum_u phi(q_t) . phi(k_u) over
  the complement tokens u, with no 1/sqrt(d) (a positive scale cancels);
* alpha is one value per query token, alpha [B, H, N] in [0, 1];
* a row whose complement is empty (every key block kept) has O_l = 0.

Pins: ``tests/test_oracle_sparse_linear.py``.
"""
from __future__ import annotations

from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

from .sparse_attn_oracle import attend_row, to_f64


def phi(x: np.ndarray) -> np.ndarray:
    """elu(x) + 1: x + 1 for x > 0, exp(x) otherwise (always positive)."""
    x = np.asarray(x, dtype=np.float64)
    return np.where(x > 0, x + 1.0, np.exp(np.minimum(x, 0.0)))


def complement_tokens(N: int, kept_blocks: Sequence[int], bk: int) -> np.ndarray:
    """Valid key tokens of the key blocks NOT in kept_blocks, ascending."""
    n_k = -(-N // bk)
    kept = np.zeros(n_k, dtype=bool)
    kept[np.asarray(list(kept_blocks), dtype=np.int64)] = True
    cols: List[int] = []
    for j in range(n_k):
        if not kept[j]:
            cols.extend(range(j * bk, min(N, (j + 1) * bk)))
    return np.asarray(cols, dtype=np.int64)


def linear_row(q: np.ndarray, K: np.ndarray, V: np.ndarray, kept_blocks: Sequence[int], bk: int) -> np.ndarray:
    """O_l of one query block: linear attention over the complement tokens.

    q: [m, d] fp64; K, V: [N, d] fp64. Returns [m, d]; zero if the
    complement is empty.
    """
    N, d = K.shape
    u = complement_tokens(N, kept_blocks, bk)
    if u.size == 0:
        return np.zeros((q.shape[0], d))
    W = phi(q) @ phi(K[u]).T            # [m, |u|], positive
    return (W @ V[u]) / W.sum(axis=1, keepdims=True)


def sparse_linear_attention(Q, K, V, alpha, cnt, idx, bq: int, bk: int,
                            rows: Optional[Iterable[Tuple[int, int, int]]] = None):
    """O = alpha * O_s + (1 - alpha) * O_l for every row, or the listed (b, h, i).

    Q, K, V: [B, H, N, d]; alpha: [B, H, N] in [0, 1]; cnt, idx: the kept
    lists. Returns (O, O_s, O_l) fp64 [B, H, N, d]; rows not computed are NaN.
    """
    Q64, K64, V64 = to_f64(Q), to_f64(K), to_f64(V)
    a64 = to_f64(alpha)
    cnt = np.asarray(cnt)
    idx = np.asarray(idx)
    B, H, N, d = Q64.shape
    n_q = -(-N // bq)
    O = np.full((B, H, N, d), np.nan)
    Os = np.full((B, H, N, d), np.nan)
    Ol = np.full((B, H, N, d), np.nan)
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(n_q)]
    for (b, h, i) in rows:
        lo, hi = i * bq, min(N, (i + 1) * bq)
        kept = idx[b, h, i, : int(cnt[b, h, i])]
        os_, _ = attend_row(Q64[b, h, lo:hi], K64[b, h], V64[b, h], kept, bk)
        ol = linear_row(Q64[b, h, lo:hi], K64[b, h], V64[b, h], kept, bk)
        a = a64[b, h, lo:hi, None]
        O[b, h, lo:hi] = a * os_ + (1.0 - a) * ol
        Os[b, h, lo:hi] = os_
        Ol[b, h, lo:hi] = ol
    return O, Os, Ol
