"""Backward pass of block-sparse attention: the plain fp64 statement.

TEST INFRASTRUCTURE ONLY (see the package docstring): only ``tests/`` may
import this module; the CUDA path shares no code with it.

Source: "SpargeAttention2: Trainable Sparse Attention via Hybrid Top-k+Top-p
Masking and Distillation Fine-Tuning" (gist.science summaries), §2B Velocity
Distillation Fine-Tuning: the student model that uses the sparse attention is
fine-tuned against the full-attention teacher, so the loss is differentiated
through the sparse attention of §2C. The pages give no formula for that
derivative; it is the plain derivative of the forward definition (``attend_row``:
softmax over the kept blocks' valid tokens, then the weighted sum of V), with
the kept-block lists held fixed. The selection (§2A) is a piecewise-constant
function of Q and K, so it carries no gradient; this is the reading taken.

For one query block with tokens q [m, d], kept key tokens u, upstream
gradient dO [m, d] and c = 1/sqrt(d):
    S = c q K_u^T,   P = softmax_rows(S),   O = P V_u
    dV_u = P^T dO
    dP   = dO V_u^T
    D_i  = sum_j P_ij dP_ij  (= dO_i . O_i)
    dS   = P * (dP - D)
    dq   = c dS K_u,   dK_u = c dS^T q
dK and dV of a key token collect the contributions of every query block that
keeps its block. Parity pins: ``tests/test_oracle_backward.py`` (autograd of
the same masked softmax in fp64, central finite differences, and the
invariants sum_j dK_j = 0 and sum_j dV_j = sum of dO over the rows that keep a
block).
"""
from __future__ import annotations

import math
from typing import List, Sequence, Tuple

import numpy as np

from .sparse_attn_oracle import to_f64


def attend_row_backward(q: np.ndarray, K: np.ndarray, V: np.ndarray, dO: np.ndarray,
                        kept_blocks: Sequence[int], bk: int):
    """Gradients of one query block's output (``attend_row``) for upstream dO.

    q, dO: [m, d] fp64; K, V: [N, d] fp64 of the same (b, h). Returns
    (dq [m, d], cols [u] int64, dK_u [u, d], dV_u [u, d]), where cols are the
    kept key tokens in the order their blocks are listed. An empty kept set
    gives dq = 0 and no key contribution.
    """
    N, d = K.shape
    cols: List[int] = []
    for j in kept_blocks:
        cols.extend(range(int(j) * bk, min(N, (int(j) + 1) * bk)))
    if not cols:
        return np.zeros_like(q), np.zeros(0, dtype=np.int64), np.zeros((0, d)), np.zeros((0, d))
    u = np.asarray(cols, dtype=np.int64)
    c = 1.0 / math.sqrt(d)
    Ku, Vu = K[u], V[u]
    S = c * (q @ Ku.T)
    E = np.exp(S - S.max(axis=1, keepdims=True))
    P = E / E.sum(axis=1, keepdims=True)
    O = P @ Vu
    dV_u = P.T @ dO
    dP = dO @ Vu.T
    D = np.sum(dO * O, axis=1, keepdims=True)
    dS = P * (dP - D)
    dq = c * (dS @ Ku)
    dK_u = c * (dS.T @ q)
    return dq, u, dK_u, dV_u


def block_sparse_attention_backward(Q, K, V, dO, cnt, idx, bq: int, bk: int
                                    ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """dQ, dK, dV (fp64 [B, H, N, d]) of ``block_sparse_attention`` for upstream dO.

    Q, K, V, dO: [B, H, N, d] (bf16 tensors or fp64 arrays); cnt [B, H, n_q]
    and idx [B, H, n_q, n_k] as the forward takes them (the first cnt entries
    of a row are its kept key blocks, in any order).
    """
    Q64, K64, V64, dO64 = to_f64(Q), to_f64(K), to_f64(V), to_f64(dO)
    cnt = np.asarray(cnt)
    idx = np.asarray(idx)
    B, H, N, d = Q64.shape
    n_q = -(-N // bq)
    dQ = np.zeros_like(Q64)
    dK = np.zeros_like(K64)
    dV = np.zeros_like(V64)
    for b in range(B):
        for h in range(H):
            for i in range(n_q):
                lo, hi = i * bq, min(N, (i + 1) * bq)
                kept = idx[b, h, i, : int(cnt[b, h, i])]
                dq, u, dk, dv = attend_row_backward(Q64[b, h, lo:hi], K64[b, h], V64[b, h],
                                                    dO64[b, h, lo:hi], kept, bk)
                dQ[b, h, lo:hi] = dq
                np.add.at(dK[b, h], u, dk)
                np.add.at(dV[b, h], u, dv)
    return dQ, dK, dV
