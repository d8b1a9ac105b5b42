"""GPU block-sparse attention vs the CPU oracle, through the C ABI (needs a B200).

Both sides use the GPU's own mask, so selection near-ties do not enter the
output comparison. Tolerance for bf16 inputs against the fp64 oracle:
max-abs 1e-2 and mean-abs 1e-3, on the kernel's fp32 result (SA_F32). The
bf16 output (SA_BF16) must be exactly that result rounded to nearest even:
the final rounding alone is up to half a bf16 ulp, 2^-8 |O|, which for
|O| >= 2.56 exceeds 1e-2 by itself.
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_row_b200 import (SparseAttnError, check_device_error,
                                             sparse_attn_fwd, sparse_attn_fwd_dense,
                                             sparse_attn_mask)
from synth import CONFIGS

from _gpu_cases import (MAX_ABS_TOL, MEAN_ABS_TOL, all_rows, compare_outputs, custom,
                        workload)

pytestmark = pytest.mark.gpu


def _run(name, k, p, rows_stride=None):
    cfg, (Q, K, V), (Qh, Kh, Vh) = workload(name)
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, k, p)
    O_gpu, lse = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, cfg.bk, want_lse=True,
                                 out_dtype=torch.float32)
    O_bf16 = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, cfg.bk)
    check_device_error(Q.device)
    assert torch.equal(O_bf16, O_gpu.to(torch.bfloat16))
    cnt = m["cnt"].cpu().numpy()
    idx = m["idx"].cpu().numpy()
    rows = all_rows(cfg.B, cfg.H, cfg.n_q) if rows_stride is None else \
        O.row_sample(cfg.B, cfg.H, cfg.n_q, rows_stride)
    O_ref, L_ref = O.block_sparse_attention(Qh, Kh, Vh, cnt, idx, cfg.bq, cfg.bk, rows=rows)
    mx, mean = compare_outputs(O_gpu, O_ref, rows, cfg.bq, cfg.N)
    lse_g = lse.cpu().numpy()
    lerr = max(float(np.nanmax(np.abs(lse_g[b, h, i * cfg.bq:(i + 1) * cfg.bq] -
                                      L_ref[b, h, i * cfg.bq:(i + 1) * cfg.bq])))
               for (b, h, i) in rows)
    print(f"\n[{name} k={k} p={p}] rows={len(rows)} max_abs={mx:.3e} mean_abs={mean:.3e} "
          f"lse_max_abs={lerr:.3e} kept={cnt.sum()}/{cnt.size * cfg.n_k}")
    return mx, mean, lerr


@pytest.mark.parametrize("name,stride", [("tiny", None), ("mid", None), ("wan", 8), ("long", 8)])
def test_fwd_matches_oracle(name, stride):
    cfg = CONFIGS[name]
    mx, mean, lerr = _run(name, cfg.k, cfg.p, stride)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL
    assert lerr < 1e-4


@pytest.mark.parametrize("k,p", CONFIGS["sweep"].kp)
def test_fwd_matches_oracle_sweep(k, p):
    mx, mean, _ = _run("sweep", k, p, 8)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL


def _custom_case(B, H, N, d, bq, seed, **kw):
    (Q, K, V), (Qh, Kh, Vh) = custom(B, H, N, d, seed, **kw)
    return Q, K, V, Qh, Kh, Vh


@pytest.mark.parametrize("N,d,bq", [(300, 64, 64), (300, 128, 128), (1000, 128, 128), (1000, 64, 128),
                                    (1, 128, 128), (64, 64, 64), (130, 128, 64), (4097, 128, 128)])
@pytest.mark.parametrize("k,p", [(0.1, 0.9), (0.3, 0.0), (1.0, 0.0)])
def test_fwd_ragged_shapes(N, d, bq, k, p):
    B, H = 2, 3
    Q, K, V, Qh, Kh, Vh = _custom_case(B, H, N, d, bq, seed=7 * N + d, positional_field=True)
    m = sparse_attn_mask(Q, K, bq, 64, k, p)
    O_gpu = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], bq, 64, out_dtype=torch.float32)
    O_bf16 = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], bq, 64)
    check_device_error()
    assert torch.equal(O_bf16, O_gpu.to(torch.bfloat16))
    n_q = -(-N // bq)
    rows = all_rows(B, H, n_q)
    O_ref, _ = O.block_sparse_attention(Qh, Kh, Vh, m["cnt"].cpu().numpy(), m["idx"].cpu().numpy(),
                                        bq, 64, rows=rows)
    mx, mean = compare_outputs(O_gpu, O_ref, rows, bq, N)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)


def _handmade_lists(B, H, n_q, n_k, rng, with_empty=True):
    cnt = np.zeros((B, H, n_q), dtype=np.int32)
    idx = np.full((B, H, n_q, n_k), -1, dtype=np.int32)
    for b in range(B):
        for h in range(H):
            for i in range(n_q):
                c = int(rng.integers(0, n_k + 1))
                if with_empty and (b + h + i) % 7 == 3:
                    c = 0
                kept = rng.permutation(n_k)[:c]          # any order, not only ascending
                cnt[b, h, i] = c
                idx[b, h, i, :c] = kept
    return cnt, idx


@pytest.mark.parametrize("N,d,bq", [(1000, 128, 128), (777, 64, 64), (1500, 128, 64)])
def test_fwd_arbitrary_lists_empty_rows_and_odd_counts(N, d, bq):
    B, H = 1, 4
    rng = np.random.default_rng(N)
    Q, K, V, Qh, Kh, Vh = _custom_case(B, H, N, d, bq, seed=N)
    n_q, n_k = -(-N // bq), -(-N // 64)
    cnt, idx = _handmade_lists(B, H, n_q, n_k, rng)
    O_gpu, lse = sparse_attn_fwd(Q, K, V, torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda(),
                                 bq, 64, want_lse=True, out_dtype=torch.float32)
    check_device_error()
    rows = all_rows(B, H, n_q)
    O_ref, L_ref = O.block_sparse_attention(Qh, Kh, Vh, cnt, idx, bq, 64, rows=rows)
    mx, mean = compare_outputs(O_gpu, O_ref, rows, bq, N)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)
    lse_g = lse.cpu().numpy()
    empty = np.repeat(cnt == 0, bq, axis=-1)[..., :N]
    assert np.all(np.isneginf(lse_g[empty]))
    assert np.all(O_gpu.float().cpu().numpy()[empty] == 0)


def _aligned_qkv(alphas, N=1024, d=128, seed=11):
    """Q rows near one direction u; the K rows of key blocks 5, 9 and 12 are
    alpha_h * u (head h), the others random: scores against those blocks sit
    about alpha_h * d * log2(e) / sqrt(d) above the rest (in log2 units)."""
    g = torch.Generator().manual_seed(seed)
    H = len(alphas)
    u = torch.randn(d, generator=g)
    Q = u + 0.1 * torch.randn(1, H, N, d, generator=g)
    K = torch.randn(1, H, N, d, generator=g)
    for h, a in enumerate(alphas):
        for j in (5, 9, 12):
            K[0, h, j * 64:(j + 1) * 64] = a * u + 0.1 * torch.randn(64, d, generator=g)
    V = torch.randn(1, H, N, d, generator=g)
    return [x.to(torch.bfloat16) for x in (Q, K, V)]


@pytest.mark.parametrize("bq", [128, 64])
def test_fwd_running_max_jumps(bq):
    """Rows whose scores jump far above the running max after the first tile
    (in log2 units): by ~50 (the weights stay against the old max, up to
    2^53), by ~120 and ~415 (past 2^64: the tile's max is taken, O rescaled and
    the tile recomputed), and rows whose first tile holds the largest scores."""
    alphas = [2.5, 6.0, 20.0]
    Qh, Kh, Vh = _aligned_qkv(alphas)
    B, H, N, d = Qh.shape
    n_q, n_k = -(-N // bq), -(-N // 64)
    lists = [[0, 1, 5, 9, 12, 14], [0, 1, 2, 3, 9], [5, 0, 1, 2, 3], [2, 3, 4, 6, 7, 8, 10, 11, 12]]
    cnt = np.zeros((B, H, n_q), dtype=np.int32)
    idx = np.full((B, H, n_q, n_k), -1, dtype=np.int32)
    for h in range(H):
        for i in range(n_q):
            li = lists[(h + i) % len(lists)]
            cnt[0, h, i] = len(li)
            idx[0, h, i, :len(li)] = li
    Q, K, V = (x.cuda() for x in (Qh, Kh, Vh))
    O_gpu, lse = sparse_attn_fwd(Q, K, V, torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda(),
                                 bq, 64, want_lse=True, out_dtype=torch.float32)
    O_bf16 = sparse_attn_fwd(Q, K, V, torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda(), bq, 64)
    check_device_error()
    assert torch.equal(O_bf16, O_gpu.to(torch.bfloat16))
    rows = all_rows(B, H, n_q)
    O_ref, L_ref = O.block_sparse_attention(Qh, Kh, Vh, cnt, idx, bq, 64, rows=rows)
    mx, mean = compare_outputs(O_gpu, O_ref, rows, bq, N)
    lerr = float(np.max(np.abs(lse.cpu().numpy() - L_ref)))
    print(f"\n[running-max jumps bq={bq}] max_abs={mx:.3e} mean_abs={mean:.3e} lse_max_abs={lerr:.3e}")
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)
    assert lerr < 1e-3


def test_fwd_bad_index_is_reported_and_skipped():
    B, H, N, d, bq = 1, 2, 640, 128, 128
    Q, K, V, Qh, Kh, Vh = _custom_case(B, H, N, d, bq, seed=3)
    n_q, n_k = N // bq, N // 64
    cnt = np.full((B, H, n_q), 3, dtype=np.int32)
    idx = np.zeros((B, H, n_q, n_k), dtype=np.int32)
    idx[..., :3] = [1, 4, 7]
    idx[0, 1, 2, 1] = n_k + 5                       # out of range: skipped, reported
    O_gpu = sparse_attn_fwd(Q, K, V, torch.from_numpy(cnt).cuda(), torch.from_numpy(idx).cuda(), bq, 64,
                            out_dtype=torch.float32)
    with pytest.raises(SparseAttnError, match="SA_ERR_DEVICE_ASSERT"):
        check_device_error()
    check_device_error()
    cnt_ref, idx_ref = cnt.copy(), idx.copy()
    cnt_ref[0, 1, 2] = 2
    idx_ref[0, 1, 2, :2] = [1, 7]
    rows = all_rows(B, H, n_q)
    O_ref, _ = O.block_sparse_attention(Qh, Kh, Vh, cnt_ref, idx_ref, bq, 64, rows=rows)
    mx, mean = compare_outputs(O_gpu, O_ref, rows, bq, N)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL


@pytest.mark.parametrize("name", ["tiny", "mid"])
def test_dense_path_matches_torch_fp32_sdpa(name):
    cfg, (Q, K, V), _ = workload(name)
    O_gpu = sparse_attn_fwd_dense(Q, K, V, cfg.bq, cfg.bk, out_dtype=torch.float32)
    check_device_error()
    ref = torch.nn.functional.scaled_dot_product_attention(Q.float(), K.float(), V.float())
    err = (O_gpu.float() - ref).abs()
    print(f"\n[{name} dense] max_abs={err.max().item():.3e} mean_abs={err.mean().item():.3e}")
    assert err.max().item() <= MAX_ABS_TOL and err.mean().item() <= MEAN_ABS_TOL


def test_dense_equals_sparse_with_all_blocks():
    cfg, (Q, K, V), _ = workload("tiny")
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, 1.0, 0.0)
    a = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, cfg.bk)
    b = sparse_attn_fwd_dense(Q, K, V, cfg.bq, cfg.bk)
    check_device_error()
    assert torch.equal(a, b)


def test_fwd_is_deterministic():
    cfg, (Q, K, V), _ = workload("mid")
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, cfg.k, cfg.p)
    a = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, cfg.bk)
    b = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, cfg.bk)
    check_device_error()
    assert torch.equal(a, b)
