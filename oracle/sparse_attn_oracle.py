"""Plain fp64 CPU statement of hybrid Top-k+Top-p block-sparse attention.

TEST INFRASTRUCTURE ONLY (see the package docstring): never imported by the
product path.

The path, per (batch b, head h):

1. pool     Qbar_i = mean of the valid tokens of query block i, Kbar_j alike
            (SLA2 §1/§2B: pooled queries and keys; Sparse VideoGen2 §1: mean
            pooling of contiguous blocks).
2. score    P = softmax_j(Qbar_i . Kbar_j / sqrt(d)) per query-block row
            (SLA2 §2B: a compressed attention score from the pooled
            matrices; SpargeAttention2 §2A: rows of the attention weight
            matrix carry probability mass).
3. select   per row, the union of the Top-k key blocks and the Top-p key
            blocks (SpargeAttention2 §1 and §2A; Sparse VideoGen2 §2B for the
            sort-then-accumulate reading of Top-p).
4. attend   softmax(q K^T / sqrt(d)) V over the tokens of the kept key blocks
            only; nothing else enters the row (SpargeAttention2 §2C).

Readings taken where the pages are silent (each also listed in the design
notes): mean pooling over the valid tokens of a ragged last block; score
scale 1/sqrt(d); k is a fraction of the row's key blocks and Top-k keeps
ceil(k * n_k) of them; "reaches p" is inclusive (cumulative mass >= p of the
row's total mass); equal scores are ordered by the lower key-block index;
cumulative mass is accumulated in 31-bit fixed point so that the decision
does not depend on summation order; k >= 1 or p >= 1 keep every block.
"""
from __future__ import annotations

import math
from typing import Iterable, List, Optional, Sequence, Tuple

import numpy as np

FIXED_POINT_ONE = float(2 ** 31)  # scale of the Top-p fixed-point mass
TOPK_EPS = 1e-9                    # guards ceil() against k*n products such as 0.07*100


def to_f64(x) -> np.ndarray:
    """Exact upcast of a (bf16, fp16 or fp32) torch tensor or array to numpy fp64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.asarray(x, dtype=np.float64)


# ---------------------------------------------------------------- 1. pool
def pool_blocks(X: np.ndarray, block: int) -> np.ndarray:
    """Mean over each contiguous block of `block` tokens along axis -2.

    X: [..., N, d] fp64 -> [..., ceil(N/block), d]. A ragged last block is
    averaged over its valid tokens only (SLA2 §1 and §2B pool the queries and
    keys; Sparse VideoGen2 §1 names mean pooling over contiguous blocks).
    """
    N = X.shape[-2]
    n = -(-N // block)
    out = np.empty(X.shape[:-2] + (n, X.shape[-1]), dtype=np.float64)
    for j in range(n):
        lo, hi = j * block, min(N, (j + 1) * block)
        out[..., j, :] = X[..., lo:hi, :].sum(axis=-2) / float(hi - lo)
    return out


# --------------------------------------------------------------- 2. score
def block_scores(Qbar: np.ndarray, Kbar: np.ndarray, d: int) -> np.ndarray:
    """P = row softmax of Qbar Kbar^T / sqrt(d), fp64.

    Qbar: [..., n_q, d], Kbar: [..., n_k, d] -> P: [..., n_q, n_k]. Each row
    is a probability distribution over key blocks (the compressed score of
    SLA2 §2B; the probability mass of a row in SpargeAttention2 §2A). The
    row maximum is subtracted before exp; that leaves the softmax unchanged.
    """
    S = np.matmul(Qbar, np.swapaxes(Kbar, -1, -2)) / math.sqrt(d)
    S = S - S.max(axis=-1, keepdims=True)
    E = np.exp(S)
    return E / E.sum(axis=-1, keepdims=True)


# -------------------------------------------------------------- 3. select
def topk_count(k: float, n_k: int) -> int:
    """Number of key blocks the Top-k rule keeps in a row of n_k blocks.

    SpargeAttention2 §1 speaks of keeping the top k ("top 10%"); k is read as
    a fraction of the row, giving ceil(k * n_k) blocks, evaluated in double
    with a 1e-9 guard so that products such as 0.07 * 100 = 7.000000000000001
    give 7. k >= 1 keeps the row.
    """
    k = float(k)
    if k >= 1.0:
        return n_k
    return min(n_k, max(0, math.ceil(k * n_k - TOPK_EPS)))


def topp_threshold(W: int, p: float) -> int:
    """Fixed-point mass a Top-p prefix must reach: ceil(p * W), one double multiply."""
    p = float(p)
    return math.ceil(p * float(W))


def select_row(P_row: np.ndarray, k: float, p: float) -> np.ndarray:
    """Kept key blocks of one score row: Top-k union Top-p, ascending indices.

    P_row: fp32 [n_k], P >= 0. Steps (SpargeAttention2 §1 and §2A; Sparse
    VideoGen2 §2B):
      a. order the blocks by score, highest first; equal scores by lower
         index (the fp32 bit pattern orders non-negative floats exactly);
      b. Top-k = the first topk_count(k, n_k) blocks of that order;
      c. Top-p = the shortest prefix of that order whose cumulative mass
         reaches p of the row's total. Mass is counted in 31-bit fixed point,
         w_j = floor(P_j * 2^31) (exact), W = sum w_j, target T = ceil(p W);
      d. both sets are prefixes of one order, so their union is the longer
         prefix.
    """
    P_row = np.ascontiguousarray(P_row, dtype=np.float32)
    n = P_row.shape[0]
    bits = P_row.view(np.uint32).astype(np.int64)
    order = np.lexsort((np.arange(n), -bits))          # a.
    kc = topk_count(k, n)                              # b.
    if float(p) >= 1.0:                                # c.
        m_p = n
    else:
        w = np.floor(P_row.astype(np.float64) * FIXED_POINT_ONE).astype(np.uint64)
        W = int(w.sum(dtype=np.uint64))
        T = topp_threshold(W, p)
        if T <= 0:
            m_p = 0
        else:
            cum = np.cumsum(w[order], dtype=np.uint64)
            hit = np.nonzero(cum >= np.uint64(T))[0]
            m_p = int(hit[0]) + 1 if hit.size else n
    keep = max(kc, m_p)                                # d.
    return np.sort(order[:keep]).astype(np.int32)


def hybrid_select(P32: np.ndarray, k: float, p: float):
    """Apply select_row to every row of P32 [..., n_q, n_k] (fp32).

    Returns (cnt int32 [..., n_q], idx int32 [..., n_q, n_k] with the first
    cnt entries the ascending kept indices and the rest -1, mask uint8
    [..., n_q, n_k]).
    """
    P32 = np.asarray(P32, dtype=np.float32)
    lead = P32.shape[:-1]
    n_k = P32.shape[-1]
    flat = P32.reshape(-1, n_k)
    cnt = np.zeros(flat.shape[0], dtype=np.int32)
    idx = np.full((flat.shape[0], n_k), -1, dtype=np.int32)
    mask = np.zeros((flat.shape[0], n_k), dtype=np.uint8)
    for r in range(flat.shape[0]):
        kept = select_row(flat[r], k, p)
        cnt[r] = kept.size
        idx[r, :kept.size] = kept
        mask[r, kept] = 1
    return cnt.reshape(lead), idx.reshape(lead + (n_k,)), mask.reshape(lead + (n_k,))


def hybrid_mask(Q, K, bq: int, bk: int, k: float, p: float):
    """Steps 1-3 on bf16 (or any) Q, K [B, H, N, d].

    Returns (P64 fp64 [B,H,n_q,n_k], cnt, idx, mask) where the selection is
    made on P64 rounded to fp32 (the precision the selection is defined in).
    """
    Q64, K64 = to_f64(Q), to_f64(K)
    d = Q64.shape[-1]
    P64 = block_scores(pool_blocks(Q64, bq), pool_blocks(K64, bk), d)
    cnt, idx, mask = hybrid_select(P64.astype(np.float32), k, p)
    return P64, cnt, idx, mask


# -------------------------------------------------------------- 4. attend
def attend_row(q: np.ndarray, K: np.ndarray, V: np.ndarray,
               kept_blocks: Sequence[int], bk: int) -> Tuple[np.ndarray, np.ndarray]:
    """softmax(q K_u^T / sqrt(d)) V_u over the tokens u of the kept key blocks.

    q: [m, d] fp64 query tokens of one query block; K, V: [N, d] fp64 of the
    same (b, h). Only the kept blocks' valid tokens enter the softmax
    (SpargeAttention2 §2C: masked tiles contribute neither matmul nor
    softmax). Returns (O [m, d], LSE [m], natural log). An empty kept set
    gives O = 0 and LSE = -inf.
    """
    N, d = K.shape
    cols: List[int] = []
    for j in kept_blocks:
        cols.extend(range(j * bk, min(N, (j + 1) * bk)))
    if not cols:
        return np.zeros((q.shape[0], d)), np.full(q.shape[0], -np.inf)
    cols_a = np.asarray(cols, dtype=np.int64)
    S = (q @ K[cols_a].T) / math.sqrt(d)
    mx = S.max(axis=1, keepdims=True)
    E = np.exp(S - mx)
    l = E.sum(axis=1, keepdims=True)
    O = (E @ V[cols_a]) / l
    return O, (mx + np.log(l))[:, 0]


def block_sparse_attention(Q, K, V, cnt, idx, bq: int, bk: int,
                           rows: Optional[Iterable[Tuple[int, int, int]]] = None):
    """Step 4 for every row, or for the listed (b, h, i) rows only.

    Q, K, V: [B, H, N, d] (bf16 tensors or fp64 arrays); cnt [B,H,n_q] and
    idx [B,H,n_q,n_k] as returned by hybrid_select (or by the CUDA path).
    Returns (O fp64 [B,H,N,d], LSE fp64 [B,H,N]); rows not computed are NaN.
    """
    Q64, K64, V64 = to_f64(Q), to_f64(K), to_f64(V)
    cnt = np.asarray(cnt)
    idx = np.asarray(idx)
    B, H, N, d = Q64.shape
    n_q = -(-N // bq)
    O = np.full((B, H, N, d), np.nan)
    LSE = np.full((B, H, N), np.nan)
    if rows is None:
        rows = [(b, h, i) for b in range(B) for h in range(H) for i in range(n_q)]
    for (b, h, i) in rows:
        lo, hi = i * bq, min(N, (i + 1) * bq)
        kept = idx[b, h, i, : int(cnt[b, h, i])]
        o, lse = attend_row(Q64[b, h, lo:hi], K64[b, h], V64[b, h], kept, bk)
        O[b, h, lo:hi] = o
        LSE[b, h, lo:hi] = lse
    return O, LSE


def row_sample(B: int, H: int, n_q: int, stride: int = 8) -> List[Tuple[int, int, int]]:
    """Deterministic row sample: all (b, h); every stride-th query block plus the last."""
    blocks = sorted(set(range(0, n_q, stride)) | {n_q - 1})
    return [(b, h, i) for b in range(B) for h in range(H) for i in blocks]
