"""GPU FP8 path (sparse_attn_quantize_fp8 + sparse_attn_fwd_fp8) vs the FP8
oracle, through the C ABI (needs a B200).

Quantisation is integer-valued work decided by fp32 arithmetic, done in the
same precision on both sides: the e4m3 codes and the fp32 block scales must
match the oracle bit for bit. The forward is then compared with the oracle's
attention on the dequantised Q and K (and the unquantised V) at the tolerance
of the bf16 path, max-abs 1e-2 and mean-abs 1e-3: once the quantisation is
part of the definition, what remains on the GPU is the same bf16 rounding of
P and fp32 accumulation as on the bf16 path. The distance to the unquantised
attention is printed for information (it is the quantisation's own error).
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_row_b200 import (check_device_error, sparse_attn_fwd, sparse_attn_fwd_fp8,
                                             sparse_attn_mask, sparse_attn_quantize_fp8)

from _gpu_cases import MAX_ABS_TOL, MEAN_ABS_TOL, all_rows, compare_outputs, custom, workload

pytestmark = pytest.mark.gpu


def _codes(t):
    return t.view(torch.float8_e4m3fn).float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("name,heads", [("tiny", None), ("mid", None), ("wan", [0, 12, 25, 39]),
                                        ("long", [3, 30])])
def test_quantize_bit_exact(name, heads):
    cfg, (Q, K, _), (Qh, Kh, _) = workload(name)
    q8 = sparse_attn_quantize_fp8(Q, K, cfg.bq, cfg.bk)
    check_device_error(Q.device)
    hs = list(range(cfg.H)) if heads is None else heads
    for h in hs:
        for X, codes, sc, blk in ((Qh, q8["Q8"], q8["q_scale"], cfg.bq), (Kh, q8["K8"], q8["k_scale"], cfg.bk)):
            c_ref, s_ref = O.quantize_blocks(X[0, h].float().numpy(), blk)
            assert np.array_equal(sc[0, h].cpu().numpy(), s_ref), (name, h)
            assert np.array_equal(_codes(codes[0, h]), c_ref), (name, h)


def test_quantize_ragged_and_zero_blocks():
    (Q, K, _), (Qh, Kh, _) = custom(1, 2, 1000, 128, seed=4)
    Q[0, 0, 128:256] = 0          # an all-zero query block
    K[0, 1, 960:] = 0             # the ragged last key block, all zero
    Qh, Kh = Q.cpu(), K.cpu()
    for bq in (128, 64):
        q8 = sparse_attn_quantize_fp8(Q, K, bq, 64)
        check_device_error(Q.device)
        for h in range(2):
            c, s = O.quantize_blocks(Qh[0, h].float().numpy(), bq)
            assert np.array_equal(q8["q_scale"][0, h].cpu().numpy(), s)
            assert np.array_equal(_codes(q8["Q8"][0, h]), c)
            c, s = O.quantize_blocks(Kh[0, h].float().numpy(), 64)
            assert np.array_equal(q8["k_scale"][0, h].cpu().numpy(), s)
            assert np.array_equal(_codes(q8["K8"][0, h]), c)
    assert q8["q_scale"][0, 0, 2].item() == 0.0 and q8["k_scale"][0, 1, -1].item() == 0.0


def _fwd_case(Q, K, V, Qh, Kh, Vh, cnt, idx, bq, rows, tag, heads=None):
    """rows: (b, h, i) within the listed heads (all heads if None), h indexing that list."""
    q8 = sparse_attn_quantize_fp8(Q, K, bq, 64)
    O_gpu, lse = sparse_attn_fwd_fp8(q8, V, cnt, idx, bq, 64, want_lse=True, out_dtype=torch.float32)
    O_bf16 = sparse_attn_fwd_fp8(q8, V, cnt, idx, bq, 64)
    check_device_error(Q.device)
    assert torch.equal(O_bf16, O_gpu.to(torch.bfloat16))
    cnt_h, idx_h = cnt.cpu().numpy(), idx.cpu().numpy()
    if heads is not None:   # the oracle on a subset of heads (it quantises whole heads)
        Qh, Kh, Vh, O_gpu, lse = (x[:, heads] for x in (Qh, Kh, Vh, O_gpu, lse))
        cnt_h, idx_h = cnt_h[:, heads], idx_h[:, heads]
    O_ref, L_ref = O.block_sparse_attention_fp8(Qh, Kh, Vh, cnt_h, idx_h, bq, 64, rows=rows)
    mx, mean = compare_outputs(O_gpu, O_ref, rows, bq, Q.shape[2])
    O_plain, _ = O.block_sparse_attention(Qh, Kh, Vh, cnt_h, idx_h, bq, 64, rows=rows)
    qmx, qmean = compare_outputs(O_gpu, O_plain, rows, bq, Q.shape[2])
    N = Q.shape[2]
    lse_g = lse.cpu().numpy()
    lerr = max(float(np.nanmax(np.abs(lse_g[b, h, i * bq:min(N, (i + 1) * bq)] - L_ref[b, h, i * bq:min(N, (i + 1) * bq)])))
               for (b, h, i) in rows if cnt_h[b, h, i] > 0)
    print(f"\n[fp8 {tag}] rows={len(rows)} vs FP8 oracle: max_abs={mx:.3e} mean_abs={mean:.3e} "
          f"lse={lerr:.2e}; vs unquantised oracle: max_abs={qmx:.3e} mean_abs={qmean:.3e}")
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)
    assert lerr < 1e-4


@pytest.mark.parametrize("name,stride,kp", [("mid", None, None), ("wan", 8, None), ("wan", 8, (0.05, 0.0)),
                                            ("long", 16, None)])
def test_fwd_fp8_matches_oracle(name, stride, kp):
    cfg, (Q, K, V), (Qh, Kh, Vh) = workload(name)
    k, p = kp if kp is not None else (cfg.k, cfg.p)
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, k, p)
    heads = None if name == "mid" else [0, 9, 12, 25, 39]
    nh = cfg.H if heads is None else len(heads)
    rows = all_rows(cfg.B, nh, cfg.n_q) if stride is None else O.row_sample(cfg.B, nh, cfg.n_q, stride)
    _fwd_case(Q, K, V, Qh, Kh, Vh, m["cnt"], m["idx"], cfg.bq, rows, f"{name} k={k} p={p}", heads=heads)


@pytest.mark.parametrize("N,bq", [(1000, 128), (777, 64), (4097, 128), (1, 128)])
def test_fwd_fp8_ragged(N, bq):
    B, H = 2, 3
    (Q, K, V), (Qh, Kh, Vh) = custom(B, H, N, 128, seed=N + 11, positional_field=True)
    m = sparse_attn_mask(Q, K, bq, 64, 0.2, 0.8)
    _fwd_case(Q, K, V, Qh, Kh, Vh, m["cnt"], m["idx"], bq, all_rows(B, H, -(-N // bq)), f"ragged N={N} bq={bq}")
