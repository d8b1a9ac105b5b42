"""GPU semantic-aware permutation (Sparse VideoGen2 §2A) vs the oracle, through
the C ABI (needs a B200).

k-means takes every decision in stated fp32 arithmetic (each subtraction,
product and addition rounded, no fused multiply-add; sums in ascending token
order), so the GPU's cluster ids, permutation and centroids must equal the
oracle's bit for bit. Row gathers and scatters are copies: bit-exact. The
block-sparse attention on the permuted sequences is compared with the oracle's
fp64 attention on the oracle's own permutation (max-abs 1e-2, mean-abs 1e-3),
after checking the GPU's selection on the permuted sequence against the
oracle's (differences only at near ties).
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_row_b200 import (check_device_error, permuted_sparse_attn, sparse_attn_fwd,
                                             sparse_attn_kmeans_permutation, sparse_attn_mask,
                                             sparse_attn_permute_rows)

from _gpu_cases import MAX_ABS_TOL, MEAN_ABS_TOL, compare_outputs, custom, flip_report, reference_scores, workload

pytestmark = pytest.mark.gpu


def _oracle_heads(Xh, C, iters, heads, init=None):
    out = {}
    for (b, h) in heads:
        ini = None if init is None else init[b, h]
        out[(b, h)] = O.kmeans_permutation(Xh[b, h], C, iters, init=ini)
    return out


def _assert_exact(ids, perm, M, ref, heads):
    ids, perm, M = ids.cpu().numpy(), perm.cpu().numpy(), M.cpu().numpy()
    for (b, h) in heads:
        ri, rp, rm = ref[(b, h)]
        assert np.array_equal(ids[b, h], ri), f"ids differ in {(ids[b, h] != ri).sum()} tokens of head {(b, h)}"
        assert np.array_equal(perm[b, h], rp), f"perm differs at head {(b, h)}"
        assert np.array_equal(M[b, h].view(np.uint32), rm.view(np.uint32)), f"centroids differ at head {(b, h)}"


@pytest.mark.parametrize("name,C,iters,heads", [
    ("tiny", 64, 5, [(0, 0), (0, 1)]),
    ("mid", 128, 3, [(0, 0), (0, 7)]),
    ("sweep", 100, 2, [(1, 23)]),            # ragged: N = 17550, C not a multiple of the staging chunk
])
def test_kmeans_is_bit_exact(name, C, iters, heads):
    cfg, (Q, K, V), (Qh, Kh, Vh) = workload(name)
    for X, Xh in ((Q, Qh), (K, Kh)):
        ids, perm, M = sparse_attn_kmeans_permutation(X, C, iters)
        check_device_error(X.device)
        _assert_exact(ids, perm, M, _oracle_heads(Xh, C, iters, heads), heads)
        # Every head's perm is a permutation listing clusters in ascending order.
        p = perm.cpu().numpy()
        i = ids.cpu().numpy()
        assert np.array_equal(np.sort(p, axis=-1), np.broadcast_to(np.arange(X.shape[2]), p.shape))
        assert np.all(np.diff(np.take_along_axis(i, p.astype(np.int64), axis=-1), axis=-1) >= 0)


def test_kmeans_from_cached_centroids():
    """§2C: k-means started from the previous step's centroids."""
    (Q, K, V), (Qh, Kh, Vh) = custom(1, 3, 5000, 128, seed=71, grid=(5, 25, 40), positional_field=True)
    heads = [(0, 0), (0, 2)]
    _, _, M0 = sparse_attn_kmeans_permutation(Q, 50, 2)
    init_h = M0.cpu().numpy()
    ids, perm, M = sparse_attn_kmeans_permutation(Q, 50, 3, init=M0)
    check_device_error(Q.device)
    _assert_exact(ids, perm, M, _oracle_heads(Qh, 50, 3, heads, init=init_h), heads)
    # The same buffer may serve as init and as output (the cache updated in place).
    cache = M0.clone()
    ids2, perm2, M2 = sparse_attn_kmeans_permutation(Q, 50, 3, init=cache, out_centroids=cache)
    assert M2.data_ptr() == cache.data_ptr()
    assert torch.equal(ids2, ids) and torch.equal(perm2, perm) and torch.equal(cache, M)


@pytest.mark.parametrize("N,d,C,iters", [(1000, 64, 1, 3), (200, 128, 200, 2), (777, 64, 33, 0),
                                         (130, 128, 7, 100)])
def test_kmeans_edge_cases(N, d, C, iters):
    (Q, _, _), (Qh, _, _) = custom(2, 2, N, d, seed=N + C)
    heads = [(b, h) for b in range(2) for h in range(2)]
    ids, perm, M = sparse_attn_kmeans_permutation(Q, C, iters)
    check_device_error(Q.device)
    _assert_exact(ids, perm, M, _oracle_heads(Qh, C, iters, heads), heads)
    if C == 1:
        assert torch.all(ids == 0)
        assert torch.equal(perm[0, 0].cpu(), torch.arange(N, dtype=torch.int32))


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("d", [64, 128])
def test_permute_rows_roundtrip(dtype, d):
    B, H, N = 2, 3, 1111
    g = torch.Generator(device="cuda").manual_seed(d)
    X = torch.randn((B, H, N, d), generator=g, device="cuda").to(dtype)
    perm = torch.stack([torch.randperm(N, generator=g, device="cuda") for _ in range(B * H)]).view(B, H, N)
    perm = perm.to(torch.int32).contiguous()
    Y = sparse_attn_permute_rows(X, perm)
    Z = sparse_attn_permute_rows(Y, perm, inverse=True)
    check_device_error(X.device)
    Xh, ph = X.cpu(), perm.cpu().long()
    assert torch.equal(Y.cpu(), torch.take_along_dim(Xh, ph[..., None], dim=2))
    assert torch.equal(Z, X)


def _selection_and_output(Q, K, V, Qh, Kh, Vh, bq, k, p, C, iters, heads):
    """The permuted path, step by step; returns the GPU output and the oracle's."""
    B, H, N, d = Q.shape
    _, pq, Mq = sparse_attn_kmeans_permutation(Q, C, iters)
    _, pk, Mk = sparse_attn_kmeans_permutation(K, C, iters)
    Qp, Kp, Vp = (sparse_attn_permute_rows(x, perm) for x, perm in ((Q, pq), (K, pk), (V, pk)))
    m = sparse_attn_mask(Qp, Kp, bq, 64, k, p, want_P=True)
    Op = sparse_attn_fwd(Qp, Kp, Vp, m["cnt"], m["idx"], bq, 64, out_dtype=torch.float32)
    Og = sparse_attn_permute_rows(Op, pq, inverse=True)
    check_device_error(Q.device)
    # The composite entry point runs the same launches and gives the same bits (bf16 output).
    comp = permuted_sparse_attn(Q, K, V, bq, 64, k, p, C, C, iters)
    assert torch.equal(comp["perm_q"], pq) and torch.equal(comp["perm_k"], pk)
    assert torch.equal(comp["cnt"], m["cnt"])
    kept = torch.arange(m["idx"].shape[-1], device=Q.device) < m["cnt"][..., None]   # past cnt: unspecified
    assert torch.equal(comp["idx"][kept], m["idx"][kept])
    assert torch.equal(comp["O"], Og.to(torch.bfloat16))
    # Oracle permutation (bit-equal to the GPU's, checked), gathers and selection on the host.
    ref = _oracle_heads(Qh, C, iters, heads)
    refk = _oracle_heads(Kh, C, iters, heads)
    pq_h, pk_h = pq.cpu().numpy(), pk.cpu().numpy()
    for bh in heads:
        assert np.array_equal(pq_h[bh], ref[bh][1]) and np.array_equal(pk_h[bh], refk[bh][1])
    sel = np.array([[b, h] for b, h in heads])
    hb, hh = torch.as_tensor(sel[:, 0]), torch.as_tensor(sel[:, 1])
    Qs, Ks, Vs = (x[hb, hh][None] for x in (Qh, Kh, Vh))
    perm_q = np.stack([ref[bh][1] for bh in heads])[None]
    perm_k = np.stack([refk[bh][1] for bh in heads])[None]
    Qps = torch.take_along_dim(Qs, torch.from_numpy(perm_q).long()[..., None], dim=2)
    Kps = torch.take_along_dim(Ks, torch.from_numpy(perm_k).long()[..., None], dim=2)
    P_ref = reference_scores(Qps, Kps, bq, 64)
    P_gpu = m["P"].cpu().numpy()[sel[:, 0], sel[:, 1]][None]
    rep = flip_report(P_gpu, P_ref, k, p)
    assert rep["not_near_tie"] == [], rep
    cnt = m["cnt"].cpu().numpy()[sel[:, 0], sel[:, 1]][None]
    idx = m["idx"].cpu().numpy()[sel[:, 0], sel[:, 1]][None]
    O_ref = O.permuted_sparse_attention(Qs, Ks, Vs, perm_q, perm_k, cnt, idx, bq, 64)
    return Og[hb.cuda(), hh.cuda()][None], O_ref, rep


@pytest.mark.parametrize("name,C,iters,heads", [("tiny", 64, 3, [(0, 0), (0, 1)]), ("mid", 128, 2, [(0, 3)])])
def test_permuted_sparse_attention_matches_oracle(name, C, iters, heads):
    cfg, (Q, K, V), (Qh, Kh, Vh) = workload(name)
    Og, O_ref, rep = _selection_and_output(Q, K, V, Qh, Kh, Vh, cfg.bq, cfg.k, cfg.p, C, iters, heads)
    N = Q.shape[2]
    rows = [(0, j, i) for j in range(len(heads)) for i in range(-(-N // cfg.bq))]
    # Compared in token order: the query blocks here are token ranges of the restored output.
    mx, mean = compare_outputs(Og, O_ref, rows, cfg.bq, N)
    print(f"\n[permuted {name}] heads={heads} C={C} iters={iters} flips={rep['differing']}/{rep['rows']} "
          f"max_abs={mx:.3e} mean_abs={mean:.3e}")
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)


def test_permutation_leaves_dense_attention_unchanged():
    """The §2A equivalence on the GPU: with every block kept, the permuted path
    equals dense attention in token order (fp64 oracle, same tolerance)."""
    (Q, K, V), (Qh, Kh, Vh) = custom(1, 2, 3000, 128, seed=5, grid=(3, 25, 40), positional_field=True)
    res = permuted_sparse_attn(Q, K, V, 128, 64, 1.0, 1.0, 40, 40, 3)
    check_device_error(Q.device)
    n_q, n_k = -(-3000 // 128), -(-3000 // 64)
    assert torch.all(res["cnt"] == n_k)
    cnt = np.full((1, 2, n_q), n_k, dtype=np.int32)
    idx = np.broadcast_to(np.arange(n_k, dtype=np.int32), (1, 2, n_q, n_k)).copy()
    O_ref, _ = O.block_sparse_attention(Qh, Kh, Vh, cnt, idx, 128, 64)
    mx, mean = compare_outputs(res["O"], O_ref, [(0, h, i) for h in range(2) for i in range(n_q)], 128, 3000)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)
