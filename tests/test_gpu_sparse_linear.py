"""GPU sparse + linear combination (sparse_attn_sparse_linear) vs the oracle,
through the C ABI (needs a B200).

O = alpha * O_s + (1 - alpha) * O_l, O_s the GPU's own sparse output (as the
entry point takes it), O_l linear attention with elu + 1 features over the
complement of each row's kept blocks. The oracle computes O_s, O_l and the mix
in fp64 from the same bf16 inputs and the GPU's mask. Tolerance: max-abs 1e-2
and mean-abs 1e-3 on O (the sparse branch's own bound), and on O_l alone
(alpha = 0). The GPU rounds the features phi(q), phi(k) and the kept weights
to bf16 (2^-9 relative each) and splits the state H into two bf16 parts; the
weights of O_l are then perturbed by well under 1% relative, and O_l is a
weighted mean of V rows. alpha = 1 returns O_s bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_row_b200 import (check_device_error, sparse_attn_fwd, sparse_attn_mask,
                                             sparse_attn_sparse_linear)
from synth import make_mix_ratio

from _gpu_cases import MAX_ABS_TOL, MEAN_ABS_TOL, all_rows, compare_outputs, custom, workload

pytestmark = pytest.mark.gpu


def _run(Q, K, V, Qh, Kh, Vh, cnt, idx, bq, rows, tag, heads=None, seed=0):
    B, H, N, d = Q.shape
    O_s = sparse_attn_fwd(Q, K, V, cnt, idx, bq, 64, out_dtype=torch.float32)
    alpha = make_mix_ratio(B, H, N, seed=seed, device=Q.device)
    O_mix = sparse_attn_sparse_linear(Q, K, V, cnt, idx, O_s, alpha, bq, 64)
    O_lin = sparse_attn_sparse_linear(Q, K, V, cnt, idx, O_s, torch.zeros_like(alpha), bq, 64)
    O_one = sparse_attn_sparse_linear(Q, K, V, cnt, idx, O_s, torch.ones_like(alpha), bq, 64)
    O_bf = sparse_attn_sparse_linear(Q, K, V, cnt, idx, O_s.to(torch.bfloat16), alpha, bq, 64)
    check_device_error(Q.device)
    assert torch.equal(O_one, O_s)
    assert O_bf.dtype == torch.bfloat16
    cnt_h, idx_h, a_h = cnt.cpu().numpy(), idx.cpu().numpy(), alpha.cpu().numpy()
    if heads is not None:
        Qh, Kh, Vh = (x[:, heads] for x in (Qh, Kh, Vh))
        O_mix, O_lin, O_bf = (x[:, heads] for x in (O_mix, O_lin, O_bf))
        cnt_h, idx_h, a_h = cnt_h[:, heads], idx_h[:, heads], a_h[:, heads]
    O_ref, _, Ol_ref = O.sparse_linear_attention(Qh, Kh, Vh, a_h, cnt_h, idx_h, bq, 64, rows=rows)
    mx, mean = compare_outputs(O_mix, O_ref, rows, bq, N)
    lmx, lmean = compare_outputs(O_lin, Ol_ref, rows, bq, N)
    bmx, _ = compare_outputs(O_bf, O_ref, rows, bq, N)
    print(f"\n[sparse+linear {tag}] rows={len(rows)} O: max_abs={mx:.3e} mean_abs={mean:.3e}; "
          f"O_l: max_abs={lmx:.3e} mean_abs={lmean:.3e}; bf16 O: max_abs={bmx:.3e}")
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)
    assert lmx <= MAX_ABS_TOL and lmean <= MEAN_ABS_TOL, (lmx, lmean)


@pytest.mark.parametrize("name,stride,kp", [("mid", None, None), ("mid", None, (0.05, 0.0)), ("wan", 8, None),
                                            ("wan", 8, (0.05, 0.0)), ("sweep", 8, (0.10, 0.80)),
                                            ("long", 16, None)])
def test_sparse_linear_matches_oracle(name, stride, kp):
    cfg, (Q, K, V), (Qh, Kh, Vh) = workload(name)
    k, p = kp if kp is not None else (cfg.k, cfg.p)
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, k, p)
    heads = None if name == "mid" else sorted({h for h in (0, 9, 12, 25, cfg.H - 1) if h < cfg.H})
    nh = cfg.H if heads is None else len(heads)
    rows = all_rows(cfg.B, nh, cfg.n_q) if stride is None else O.row_sample(cfg.B, nh, cfg.n_q, stride)
    _run(Q, K, V, Qh, Kh, Vh, m["cnt"], m["idx"], cfg.bq, rows, f"{name} k={k} p={p}", heads=heads, seed=cfg.seed)


def _lists(B, H, n_q, n_k, rng):
    cnt = np.zeros((B, H, n_q), dtype=np.int32)
    idx = np.full((B, H, n_q, n_k), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n_q):
                c = int(rng.integers(1, max(2, n_k // 2)))
                if (b + h + i) % 7 == 3:
                    c = 0                    # empty row: O_s = 0, O_l over every key
                if (b + h + i) % 11 == 5:
                    c = n_k                  # full row: no linear branch
                cnt[b, h, i] = c
                idx[b, h, i, :c] = rng.permutation(n_k)[:c]
    return cnt, idx


@pytest.mark.parametrize("N,bq", [(1000, 128), (777, 64), (4097, 128), (1, 128)])
def test_sparse_linear_ragged_arbitrary_lists(N, bq):
    B, H = 1, 3
    rng = np.random.default_rng(N)
    (Q, K, V), (Qh, Kh, Vh) = custom(B, H, N, 128, seed=N + 21, positional_field=True)
    n_q, n_k = -(-N // bq), -(-N // 64)
    cnt, idx = _lists(B, H, n_q, n_k, rng)
    _run(Q, K, V, Qh, Kh, Vh, torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda(), bq,
         all_rows(B, H, n_q), f"ragged N={N} bq={bq}", seed=N)
