"""Checks that pin the CPU oracle to facts fixed outside it.

Each check takes the oracle module as an argument, so the same check runs
against the real oracle (it must pass) and against copies of it with a
planted mistake (it must fail; see test_oracle_mutations.py). None of these
checks re-types an oracle formula: each compares against a hand-worked value,
a closed form, an invariant of the mathematics, a library routine on a case
that reduces to it, or a brute-force computation done a different way.
"""
from __future__ import annotations

import json
import math
import os

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def load_hand_rows():
    with open(os.path.join(GOLDEN, "hand_rows.json")) as f:
        rows = json.load(f)["rows"]
    for r in rows:
        if "P_uniform" in r:
            u = r["P_uniform"]
            r["P"] = [u["value"]] * u["n"]
    return rows


# ------------------------------------------------------------ selection
def check_hand_rows(O):
    """Hand-worked rows (tests/golden/hand_rows.json) give the cited kept sets."""
    for r in load_hand_rows():
        P = np.asarray(r["P"], dtype=np.float32)
        got = O.select_row(P, r["k"], r["p"]).tolist()
        assert got == r["kept"], (r["name"], got, r["kept"])
        assert O.topk_count(r["k"], P.size) == len(r["topk"]), r["name"]


def _rank_by_counting(P):
    """rank_j = #{i: P_i > P_j or (P_i == P_j and i < j)}, O(n^2) brute force."""
    n = P.size
    rank = np.zeros(n, dtype=np.int64)
    for j in range(n):
        rank[j] = int(np.sum(P > P[j])) + int(np.sum(P[:j] == P[j]))
    return rank


def brute_force_union(P, k, p):
    """Top-k set and Top-p set computed separately by rank counting, then united."""
    n = P.size
    rank = _rank_by_counting(P)
    by_rank = np.empty(n, dtype=np.int64)
    by_rank[rank] = np.arange(n)
    kc = n if k >= 1 else min(n, max(0, math.ceil(k * n - 1e-9)))
    topk = set(by_rank[:kc].tolist())
    if p >= 1:
        topp = set(range(n))
    else:
        w = [int(math.floor(float(x) * 2.0 ** 31)) for x in P]
        W = sum(w)
        T = math.ceil(p * W)
        topp, acc = set(), 0
        for r in range(n):
            if acc >= T:
                break
            topp.add(int(by_rank[r]))
            acc += w[by_rank[r]]
    return sorted(topk | topp)


def random_rows(seed, n_rows, n, kind):
    rng = np.random.default_rng(seed)
    if kind == "dirichlet_flat":
        P = rng.dirichlet(np.full(n, 5.0), size=n_rows)
    elif kind == "dirichlet_peaky":
        P = rng.dirichlet(np.full(n, 0.05), size=n_rows)
    elif kind == "softmax_logits":
        L = rng.normal(0, 3, size=(n_rows, n))
        P = np.exp(L - L.max(1, keepdims=True))
        P /= P.sum(1, keepdims=True)
    elif kind == "quantised_ties":  # many exact ties
        L = rng.integers(0, 4, size=(n_rows, n)).astype(np.float64)
        P = 2.0 ** (L - 8)
        P /= P.sum(1, keepdims=True)
    elif kind == "all_equal":  # one value repeated: every boundary is a tie
        return np.full((n_rows, n), np.float32(1.0 / n), dtype=np.float32)
    elif kind == "low_bits":  # fp32 values that differ only in their last few mantissa bits
        base = np.float32(1.0 / n)
        steps = rng.integers(0, 16, size=(n_rows, n)).astype(np.uint32)
        return (np.full((n_rows, n), base, dtype=np.float32).view(np.uint32) - steps).view(np.float32)   # <= 1/n
    else:
        raise ValueError(kind)
    return P.astype(np.float32)


def check_union_brute_force(O, seed=0):
    """select_row equals Top-k U Top-p built independently by rank counting."""
    for kind in ("dirichlet_flat", "dirichlet_peaky", "softmax_logits", "quantised_ties"):
        for n in (1, 7, 64, 100):
            rows = random_rows(seed + n, 6, n, kind)
            for k, p in ((0.1, 0.9), (0.05, 0.5), (0.0, 0.3), (0.3, 0.0), (0.5, 0.95)):
                for P in rows:
                    got = O.select_row(P, k, p).tolist()
                    want = brute_force_union(P, k, p)
                    assert got == want, (kind, n, k, p, got, want)


def check_selection_invariants(O, P32, k, p):
    """cnt >= ceil(k n); kept mass reaches p; minimal; ascending unique; monotone."""
    cnt, idx, mask = O.hybrid_select(P32, k, p)
    n = P32.shape[-1]
    kc = n if k >= 1 else min(n, max(0, math.ceil(k * n - 1e-9)))
    flatP = P32.reshape(-1, n)
    flatc = cnt.reshape(-1)
    flati = idx.reshape(-1, n)
    flatm = mask.reshape(-1, n)
    for r in range(flatP.shape[0]):
        c = int(flatc[r])
        kept = flati[r, :c]
        assert c >= kc
        assert np.all(np.diff(kept) > 0) and (c == 0 or (kept[0] >= 0 and kept[-1] < n))
        assert np.all(flati[r, c:] == -1)
        assert int(flatm[r].sum()) == c and np.all(flatm[r, kept] == 1)
        w = np.floor(flatP[r].astype(np.float64) * 2.0 ** 31)
        W = w.sum()
        T = math.ceil(p * W) if p < 1 else W
        assert w[kept].sum() >= T
        # minimality: dropping the lowest-ranked kept block loses Top-k or Top-p
        if c > kc and p < 1:
            key = [(-flatP[r, j], j) for j in kept]
            last = max(key)[1]
            assert w[kept].sum() - w[last] < T
    # monotone in k and in p (superset)
    for k2, p2 in ((min(1.0, k + 0.05), p), (k, min(1.0, p + 0.05))):
        _, _, m2 = O.hybrid_select(P32, k2, p2)
        assert np.all(m2 >= mask)


# --------------------------------------------------------------- pooling
def check_pool_closed_forms(O):
    """Ramp and per-block constants; ragged last block averages valid tokens only."""
    N, d = 300, 3
    t = np.arange(N, dtype=np.float64)
    X = np.stack([t, 2 * t + 1, np.ones(N)], axis=1)[None, None]
    for blk in (64, 128, 7):
        got = O.pool_blocks(X, blk)
        n = -(-N // blk)
        assert got.shape == (1, 1, n, d)
        for j in range(n):
            lo, hi = j * blk, min(N, (j + 1) * blk)
            mean_t = (lo + hi - 1) / 2.0          # closed form mean of a ramp
            assert abs(got[0, 0, j, 0] - mean_t) < 1e-12
            assert abs(got[0, 0, j, 1] - (2 * mean_t + 1)) < 1e-12
            assert abs(got[0, 0, j, 2] - 1.0) < 1e-15


# ---------------------------------------------------------------- scores
def check_score_closed_forms(O):
    """Two-block closed form pins the 1/sqrt(d) scale; shift invariance; rows sum to 1."""
    d = 4
    Qb = np.array([[[[1.0, 0, 0, 0]]]])
    Kb = np.array([[[[2.0, 0, 0, 0], [0.0, 0, 0, 0]]]])
    P = O.block_scores(Qb, Kb, d)
    e = math.e
    assert abs(P[0, 0, 0, 0] - e / (e + 1)) < 1e-14      # logits (2/2, 0)
    assert abs(P[0, 0, 0, 1] - 1 / (e + 1)) < 1e-14
    Qb = np.array([[[[0.0, 3.0, 0, 0], [1.0, 1.0, 1.0, 1.0]]]])
    Kb = np.array([[[[0.0, 2.0, 0, 0], [0.0, 0, 0, 0], [0.0, -2.0, 0, 0]]]])
    P = O.block_scores(Qb, Kb, d)
    s = np.array([3.0, 0.0, -3.0])                       # q.k / sqrt(4)
    want = np.exp(s) / np.exp(s).sum()
    assert np.allclose(P[0, 0, 0], want, rtol=0, atol=1e-14)
    s = np.array([1.0, 0.0, -1.0])                       # (1,1,1,1).k / 2
    assert np.allclose(P[0, 0, 1], np.exp(s) / np.exp(s).sum(), rtol=0, atol=1e-14)
    rng = np.random.default_rng(3)
    Qb = rng.normal(size=(2, 3, 5, 16))
    Kb = rng.normal(size=(2, 3, 9, 16))
    P = O.block_scores(Qb, Kb, 16)
    assert np.allclose(P.sum(-1), 1.0, atol=1e-13)
    P2 = O.block_scores(Qb, Kb + rng.normal(size=(2, 3, 1, 16)), 16)  # same shift for all keys
    # shift adds q.c to every logit of a row: the softmax does not change
    assert np.allclose(P, P2, atol=1e-12)
    ref = torch.softmax(torch.from_numpy(Qb @ np.swapaxes(Kb, -1, -2) / 4.0), dim=-1).numpy()
    assert np.allclose(P, ref, atol=1e-14)


# ------------------------------------------------------------- attention
def _sdpa(q, k, v, mask=None):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v),
        attn_mask=None if mask is None else torch.from_numpy(mask)).numpy()


def check_dense_special_case(O, B=1, H=2, N=300, d=32, bq=64, bk=64, seed=5):
    """k = 1 keeps every block: the output is textbook dense attention (torch SDPA, fp64)."""
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.normal(size=(B, H, N, d)) for _ in range(3))
    P64, cnt, idx, mask = O.hybrid_mask(Q, K, bq, bk, 1.0, 0.0)
    n_k = -(-N // bk)
    assert np.all(cnt == n_k)
    out, lse = O.block_sparse_attention(Q, K, V, cnt, idx, bq, bk)
    ref = _sdpa(Q, K, V)
    assert np.max(np.abs(out - ref)) < 1e-12
    S = np.einsum("bhnd,bhmd->bhnm", Q, K) / math.sqrt(d)
    ref_lse = np.log(np.exp(S).sum(-1))
    assert np.max(np.abs(lse - ref_lse)) < 1e-12


def check_token_mask_brute_force(O, B=1, H=2, N=300, d=16, bq=128, bk=64, k=0.2, p=0.6, seed=7):
    """Expand the block mask to a token mask and run dense masked attention (torch SDPA)."""
    rng = np.random.default_rng(seed)
    Q, K, V = (rng.normal(size=(B, H, N, d)) for _ in range(3))
    _, cnt, idx, mask = O.hybrid_mask(Q, K, bq, bk, k, p)
    out, _ = O.block_sparse_attention(Q, K, V, cnt, idx, bq, bk)
    tok = np.zeros((B, H, N, N), dtype=bool)
    for t in range(N):
        for u in range(N):
            tok[:, :, t, u] = mask[:, :, t // bq, u // bk] == 1
    ref = _sdpa(Q, K, V, tok)
    assert np.max(np.abs(out - ref)) < 1e-12


def check_attention_invariants(O, seed=11):
    """V = c gives c; K = 0 gives the mean of V over kept tokens; affine in V; block permutation."""
    rng = np.random.default_rng(seed)
    B, H, N, d, bq, bk = 1, 1, 200, 8, 64, 64
    n_q, n_k = -(-N // bq), -(-N // bk)
    Q, K, V = (rng.normal(size=(B, H, N, d)) for _ in range(3))
    cnt = np.array([[[2, 1, 3, 4]]], dtype=np.int32)
    idx = np.full((1, 1, n_q, n_k), -1, dtype=np.int32)
    idx[0, 0, 0, :2] = [0, 3]
    idx[0, 0, 1, :1] = [2]
    idx[0, 0, 2, :3] = [0, 1, 3]
    idx[0, 0, 3, :4] = [0, 1, 2, 3]
    c = rng.normal(size=d)
    out, _ = O.block_sparse_attention(Q, K, np.broadcast_to(c, V.shape).copy(), cnt, idx, bq, bk)
    assert np.max(np.abs(out - c)) < 1e-12
    out, _ = O.block_sparse_attention(Q, np.zeros_like(K), V, cnt, idx, bq, bk)
    for i in range(n_q):
        cols = [u for j in idx[0, 0, i, :cnt[0, 0, i]] for u in range(j * bk, min(N, (j + 1) * bk))]
        want = V[0, 0, cols].mean(axis=0)
        lo, hi = i * bq, min(N, (i + 1) * bq)
        assert np.max(np.abs(out[0, 0, lo:hi] - want)) < 1e-12
    a, b = 2.5, -0.75
    o1, _ = O.block_sparse_attention(Q, K, V, cnt, idx, bq, bk)
    o2, _ = O.block_sparse_attention(Q, K, a * V + b, cnt, idx, bq, bk)
    assert np.max(np.abs(o2 - (a * o1 + b))) < 1e-12
    # permute whole key blocks of K and V together (full blocks only: N multiple of bk)
    N2 = 256
    Q, K, V = (rng.normal(size=(1, 1, N2, d)) for _ in range(3))
    n_k2 = N2 // bk
    perm = np.array([2, 0, 3, 1])          # new block j holds old block perm[j]
    inv = np.argsort(perm)
    Kp = K.reshape(1, 1, n_k2, bk, d)[:, :, perm].reshape(1, 1, N2, d)
    Vp = V.reshape(1, 1, n_k2, bk, d)[:, :, perm].reshape(1, 1, N2, d)
    P64, cnt, idx, _ = O.hybrid_mask(Q, K, bq, bk, 0.25, 0.7)
    P64p, cntp, idxp, _ = O.hybrid_mask(Q, Kp, bq, bk, 0.25, 0.7)
    assert np.allclose(P64p, P64[..., perm], atol=1e-13)
    for i in range(N2 // bq):
        old = set(idx[0, 0, i, :cnt[0, 0, i]].tolist())
        new = set(perm[idxp[0, 0, i, :cntp[0, 0, i]]].tolist())
        assert old == new
    o1, _ = O.block_sparse_attention(Q, K, V, cnt, idx, bq, bk)
    o2, _ = O.block_sparse_attention(Q, Kp, Vp, cntp, idxp, bq, bk)
    assert np.max(np.abs(o1 - o2)) < 1e-12
