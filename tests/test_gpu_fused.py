"""GPU single-launch path (sparse_attn_fused: mask and attention in one
cooperative kernel launch) vs the oracle and vs the separate entry points,
through the C ABI (needs a B200).

Every phase of the single launch takes the same operations in the same order
as sparse_attn_mask and sparse_attn_fwd, so cnt, the kept part of idx, O (bf16
and fp32) and the log-sum-exp must equal theirs bit for bit. Against the
oracle: the kept lists equal the oracle's selection on the GPU's scores, no
differing row against the oracle's own fp64 scores is other than a near tie,
and the fp32 output is within max-abs 1e-2 / mean-abs 1e-3 of the fp64
attention over those lists (the same gates as the separate steps).
"""
import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_row_b200 import (SparseAttnError, check_device_error, sparse_attn_fused,
                                             sparse_attn_fwd, sparse_attn_mask)
from synth import CONFIGS

from _gpu_cases import (MAX_ABS_TOL, MEAN_ABS_TOL, all_rows, assert_same_selection, compare_outputs, custom,
                        flip_report, reference_scores, workload)

pytestmark = pytest.mark.gpu


def _kept(idx, cnt):
    return torch.arange(idx.shape[-1], device=idx.device) < cnt[..., None]


def _against_separate(Q, K, V, bq, k, p):
    """The single launch against mask + fwd: bit-equal lists, O and lse."""
    f = sparse_attn_fused(Q, K, V, bq, 64, k, p, out_dtype=torch.float32, want_lse=True)
    fb = sparse_attn_fused(Q, K, V, bq, 64, k, p)
    m = sparse_attn_mask(Q, K, bq, 64, k, p, want_P=True)
    O_sep, lse_sep = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], bq, 64, want_lse=True, out_dtype=torch.float32)
    check_device_error(Q.device)
    assert torch.equal(f["cnt"], m["cnt"]) and torch.equal(fb["cnt"], m["cnt"])
    kept = _kept(m["idx"], m["cnt"])
    assert torch.equal(f["idx"][kept], m["idx"][kept]) and torch.equal(fb["idx"][kept], m["idx"][kept])
    assert torch.equal(f["O"], O_sep)
    assert torch.equal(fb["O"], O_sep.to(torch.bfloat16))
    assert torch.equal(f["lse"], lse_sep)
    return f, m


@pytest.mark.parametrize("name,stride,kp", [("tiny", None, None), ("mid", None, None), ("wan", 8, None),
                                            ("wan", 8, (0.05, 0.0)), ("sweep", 8, (0.03, 0.95)),
                                            ("sweep", 8, (0.10, 0.80)), ("long", 16, None)])
def test_fused_matches_oracle_and_separate_steps(name, stride, kp):
    cfg, (Q, K, V), (Qh, Kh, Vh) = workload(name)
    k, p = kp if kp is not None else (cfg.k, cfg.p)
    f, m = _against_separate(Q, K, V, cfg.bq, k, p)
    P_gpu = m["P"].cpu().numpy()
    cnt, idx = f["cnt"].cpu().numpy(), f["idx"].cpu().numpy()
    cnt_o, idx_o, _ = O.hybrid_select(P_gpu, k, p)
    assert_same_selection(cnt, idx, None, cnt_o, idx_o, None)
    rep = flip_report(P_gpu, reference_scores(Qh, Kh, cfg.bq, cfg.bk), k, p)
    assert rep["not_near_tie"] == [], rep
    rows = all_rows(cfg.B, cfg.H, cfg.n_q) if stride is None else O.row_sample(cfg.B, cfg.H, cfg.n_q, stride)
    O_ref, L_ref = O.block_sparse_attention(Qh, Kh, Vh, cnt, idx, cfg.bq, cfg.bk, rows=rows)
    mx, mean = compare_outputs(f["O"], O_ref, rows, cfg.bq, cfg.N)
    print(f"\n[fused {name} k={k} p={p}] rows={len(rows)} flips={rep['differing']} max_abs={mx:.3e} "
          f"mean_abs={mean:.3e}")
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)


@pytest.mark.parametrize("N,d,bq", [(300, 64, 64), (300, 128, 128), (1000, 128, 128), (1000, 64, 128),
                                    (1, 128, 128), (64, 64, 64), (130, 128, 64), (4097, 128, 128)])
@pytest.mark.parametrize("k,p", [(0.1, 0.9), (0.3, 0.0), (1.0, 0.0), (0.05, 1.0), (0.0, 0.5)])
def test_fused_ragged_and_degenerate(N, d, bq, k, p):
    (Q, K, V), (Qh, Kh, Vh) = custom(2, 3, N, d, seed=N + d + bq, positional_field=True, sink_heads=(0,),
                                     uniform_heads=(1,))
    f, m = _against_separate(Q, K, V, bq, k, p)
    cnt, idx = f["cnt"].cpu().numpy(), f["idx"].cpu().numpy()
    cnt_o, idx_o, _ = O.hybrid_select(m["P"].cpu().numpy(), k, p)
    assert_same_selection(cnt, idx, None, cnt_o, idx_o, None)
    n_q = -(-N // bq)
    rows = all_rows(2, 3, n_q)
    O_ref, _ = O.block_sparse_attention(Qh, Kh, Vh, cnt, idx, bq, 64, rows=rows)
    mx, mean = compare_outputs(f["O"], O_ref, rows, bq, N)
    assert mx <= MAX_ABS_TOL and mean <= MEAN_ABS_TOL, (mx, mean)


def test_fused_reused_workspace_and_back_to_back_calls():
    """The grid counter is zeroed per launch: repeated calls on one workspace agree."""
    cfg, (Q, K, V), _ = workload("mid")
    from block_sparse_attention_row_b200 import fused_workspace_bytes
    ws = torch.empty(fused_workspace_bytes(cfg.B, cfg.H, cfg.N, cfg.d, cfg.bq, cfg.bk), dtype=torch.uint8,
                     device=Q.device)
    outs = [sparse_attn_fused(Q, K, V, cfg.bq, cfg.bk, cfg.k, cfg.p, workspace=ws) for _ in range(4)]
    check_device_error(Q.device)
    for o in outs[1:]:
        assert torch.equal(o["O"], outs[0]["O"]) and torch.equal(o["cnt"], outs[0]["cnt"])


def test_fused_refuses_rows_longer_than_its_shared_memory():
    (Q, K, V), _ = custom(1, 1, 64 * 1550, 128, seed=3)
    with pytest.raises((SparseAttnError, ValueError)):
        sparse_attn_fused(Q, K, V, 128, 64, 0.05, 0.9)
