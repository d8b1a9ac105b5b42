"""GPU backward pass (sparse_attn_bwd) vs the fp64 backward oracle, through the
C ABI (needs a B200).

Both sides use the GPU's mask and the same bf16 Q, K, V and dO; the GPU
recomputes P from its forward's log-sum-exp and uses the forward's bf16 O for
D = rowsum(dO * O). Tolerance, per gradient tensor G against the oracle's
G_ref: max |G - G_ref| <= 1e-2 max |G_ref| and mean |G - G_ref| <= 1e-2 mean
|G_ref|. The GPU rounds two operands to bf16 before its tensor-core products
(P for dV, dS for dQ and dK; relative error 2^-9 each) and takes D from the
bf16 O (relative 2^-9 per element); accumulation is fp32. Those roundings
perturb each term of a gradient sum by at most 2^-9 relative, so the error
stays two orders of magnitude below the largest and the mean gradient entry
unless the terms cancel; the measured ratios are printed.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_row_b200 import (SparseAttnError, check_device_error, sparse_attn_bwd,
                                             sparse_attn_fwd, sparse_attn_mask)
from synth import make_grad_out

from _gpu_cases import custom, workload

pytestmark = pytest.mark.gpu

REL_MAX = 1e-2
REL_MEAN = 1e-2


def _fwd_bwd(Q, K, V, cnt, idx, bq, seed):
    O_bf16, lse = sparse_attn_fwd(Q, K, V, cnt, idx, bq, 64, want_lse=True)
    dO = make_grad_out(*Q.shape, seed=seed, device=Q.device)
    dQ, dK, dV = sparse_attn_bwd(Q, K, V, O_bf16, dO, lse, cnt, idx, bq, 64)
    check_device_error(Q.device)
    return dO, (dQ, dK, dV)


def _compare(name, got, ref, sel=None):
    g = got.float().cpu().numpy() if isinstance(got, torch.Tensor) else got
    if sel is not None:
        g = g[sel]
        ref = ref[sel]
    err = np.abs(g - ref)
    rmax = float(err.max() / max(np.abs(ref).max(), 1e-30))
    rmean = float(err.mean() / max(np.abs(ref).mean(), 1e-30))
    print(f"  {name}: max_abs={err.max():.3e} (rel {rmax:.2e})  mean_abs={err.mean():.3e} (rel {rmean:.2e})")
    assert rmax <= REL_MAX and rmean <= REL_MEAN, (name, rmax, rmean)


def _oracle_heads(Qh, Kh, Vh, dOh, cnt, idx, bq, heads):
    """Oracle gradients for the listed (b, h) heads: {(b, h): (dQ, dK, dV)} fp64 [N, d]."""
    out = {}
    for (b, h) in heads:
        sl = (slice(b, b + 1), slice(h, h + 1))
        dq, dk, dv = O.block_sparse_attention_backward(Qh[sl], Kh[sl], Vh[sl], dOh[sl], cnt[sl], idx[sl], bq, 64)
        out[(b, h)] = (dq[0, 0], dk[0, 0], dv[0, 0])
    return out


def _check_heads(grads, ref, heads, tag):
    print(f"\n[{tag}] heads {heads}")
    for n, name in enumerate(("dQ", "dK", "dV")):
        g = np.stack([grads[n][b, h].float().cpu().numpy() for (b, h) in heads])
        r = np.stack([ref[(b, h)][n] for (b, h) in heads])
        _compare(name, g, r)


@pytest.mark.parametrize("name,heads", [("tiny", [(0, 0), (0, 1)]), ("mid", [(0, 0), (0, 7)])])
def test_bwd_matches_oracle_workloads(name, heads):
    cfg, (Q, K, V), (Qh, Kh, Vh) = workload(name)
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, cfg.k, cfg.p)
    cnt, idx = m["cnt"].cpu().numpy(), m["idx"].cpu().numpy()
    dO, grads = _fwd_bwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, seed=cfg.seed + 7)
    ref = _oracle_heads(Qh, Kh, Vh, dO.cpu(), cnt, idx, cfg.bq, heads)
    _check_heads(grads, ref, heads, f"{name} k={cfg.k} p={cfg.p}")


def _handmade_lists(B, H, n_q, n_k, rng, with_empty=True):
    cnt = np.zeros((B, H, n_q), dtype=np.int32)
    idx = np.full((B, H, n_q, n_k), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n_q):
                c = int(rng.integers(0, n_k + 1))
                if with_empty and (b + h + i) % 7 == 3:
                    c = 0
                cnt[b, h, i] = c
                idx[b, h, i, :c] = rng.permutation(n_k)[:c]          # any order
    return cnt, idx


@pytest.mark.parametrize("N,d,bq", [(1000, 128, 128), (777, 64, 64), (1500, 128, 64), (300, 64, 128),
                                    (4097, 128, 128)])
def test_bwd_ragged_arbitrary_lists_and_empty_rows(N, d, bq):
    B, H = 1, 3
    rng = np.random.default_rng(N + d)
    (Q, K, V), (Qh, Kh, Vh) = custom(B, H, N, d, seed=N + 3 * d, positional_field=True)
    n_q, n_k = -(-N // bq), -(-N // 64)
    cnt, idx = _handmade_lists(B, H, n_q, n_k, rng)
    dO, grads = _fwd_bwd(Q, K, V, torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda(), bq, seed=N)
    heads = [(0, h) for h in range(H)]
    ref = _oracle_heads(Qh, Kh, Vh, dO.cpu(), cnt, idx, bq, heads)
    _check_heads(grads, ref, heads, f"ragged N={N} d={d} bq={bq}")
    # Key blocks no query block keeps get dK = dV = 0; empty rows get dQ = 0.
    for h in range(H):
        kept = np.zeros(n_k, dtype=bool)
        for i in range(n_q):
            kept[idx[0, h, i, :cnt[0, h, i]]] = True
        for j in np.nonzero(~kept)[0]:
            assert torch.count_nonzero(grads[1][0, h, j * 64:(j + 1) * 64]) == 0
            assert torch.count_nonzero(grads[2][0, h, j * 64:(j + 1) * 64]) == 0
        for i in np.nonzero(cnt[0, h] == 0)[0]:
            assert torch.count_nonzero(grads[0][0, h, i * bq:(i + 1) * bq]) == 0


def test_bwd_wan_full_size_sampled():
    """The Wan-like layer at full size, as the bench runs it: dQ on every 32nd
    query block (plus the last) of ten heads, and dK, dV of one whole head
    (whose every query block contributes)."""
    cfg, (Q, K, V), (Qh, Kh, Vh) = workload("wan")
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, cfg.k, 0.0)      # the ~95%-sparsity point
    cnt, idx = m["cnt"].cpu().numpy(), m["idx"].cpu().numpy()
    dO, (dQ, dK, dV) = _fwd_bwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, seed=cfg.seed + 7)
    dOh = dO.cpu()
    Q64, K64, V64, dO64 = (O.to_f64(x) for x in (Qh, Kh, Vh, dOh))
    blocks = sorted(set(range(0, cfg.n_q, 32)) | {cfg.n_q - 1})
    got, ref = [], []
    for h in range(0, 40, 4):
        for i in blocks:
            lo, hi = i * cfg.bq, min(cfg.N, (i + 1) * cfg.bq)
            dq, _, _, _ = O.attend_row_backward(Q64[0, h, lo:hi], K64[0, h], V64[0, h], dO64[0, h, lo:hi],
                                                idx[0, h, i, :cnt[0, h, i]], cfg.bk)
            got.append(dQ[0, h, lo:hi].float().cpu().numpy())
            ref.append(dq)
    print("\n[wan k=0.05 p=0 full size]")
    _compare("dQ (sampled rows)", np.concatenate(got), np.concatenate(ref))
    r = _oracle_heads(Qh, Kh, Vh, dOh, cnt, idx, cfg.bq, [(0, 25)])[(0, 25)]
    _compare("dK (head 25)", dK[0, 25], r[1])
    _compare("dV (head 25)", dV[0, 25], r[2])


def test_bwd_bf16_outputs_round_the_fp32_ones_and_are_deterministic():
    cfg, (Q, K, V), _ = workload("mid")
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, cfg.k, cfg.p)
    O_bf16, lse = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, cfg.bk, want_lse=True)
    dO = make_grad_out(*Q.shape, seed=5, device=Q.device)
    a = sparse_attn_bwd(Q, K, V, O_bf16, dO, lse, m["cnt"], m["idx"], cfg.bq, cfg.bk)
    b = sparse_attn_bwd(Q, K, V, O_bf16, dO, lse, m["cnt"], m["idx"], cfg.bq, cfg.bk)
    c = sparse_attn_bwd(Q, K, V, O_bf16, dO, lse, m["cnt"], m["idx"], cfg.bq, cfg.bk, out_dtype=torch.bfloat16)
    check_device_error(Q.device)
    for x, y, z in zip(a, b, c):
        assert torch.equal(x, y)
        assert torch.equal(z, x.to(torch.bfloat16))


def test_bwd_reports_a_repeated_block():
    B, H, N, d, bq = 1, 1, 512, 128, 128
    (Q, K, V), _ = custom(B, H, N, d, seed=9)
    n_q, n_k = N // bq, N // 64
    cnt = torch.full((B, H, n_q), 3, dtype=torch.int32)
    idx = torch.zeros((B, H, n_q, n_k), dtype=torch.int32)
    idx[..., :3] = torch.tensor([1, 4, 6], dtype=torch.int32)
    idx[0, 0, 2, :3] = torch.tensor([5, 2, 5], dtype=torch.int32)   # block 5 twice
    cnt, idx = cnt.cuda(), idx.cuda()
    O_bf16, lse = sparse_attn_fwd(Q, K, V, cnt, idx, bq, 64, want_lse=True)
    dO = make_grad_out(B, H, N, d, seed=1, device=Q.device)
    sparse_attn_bwd(Q, K, V, O_bf16, dO, lse, cnt, idx, bq, 64)
    with pytest.raises(SparseAttnError, match="SA_ERR_DEVICE_ASSERT"):
        check_device_error(Q.device)
    check_device_error(Q.device)
