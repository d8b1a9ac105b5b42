"""GPU block mask vs the CPU oracle, through the C ABI (needs a B200).

Bit-exact: the oracle's selection applied to the GPU-written fp32 scores must
equal the GPU's cnt / idx / mask on every row of every workload. Near ties
between the GPU scores and the oracle's own fp64 scores are counted and
reported; a differing row that is not a near tie (two straddling scores, or the
boundary mass, within 1e-6) fails.

Score accuracy: the GPU's fp32 softmax of the block logits is within 2e-6 of
the oracle's fp64 scores elementwise (measured: at most 4.8e-7 on the five
workloads), and each row sums to 1 within 2e-6 (fp64 sum).
"""
import json

import numpy as np
import pytest
import torch

import oracle as O
from block_sparse_attention_row_b200 import (check_device_error, sparse_attn_mask,
                                             sparse_attn_select)
from synth import CONFIGS

from _gpu_cases import (assert_same_selection, custom, flip_report, reference_scores,
                        workload)
from _pins import load_hand_rows

pytestmark = pytest.mark.gpu

WORKLOAD_POINTS = [(name, k, p) for name in ("tiny", "mid", "wan", "long")
                   for (k, p) in CONFIGS[name].kp] + [("sweep", k, p) for (k, p) in CONFIGS["sweep"].kp]


@pytest.mark.parametrize("name,k,p", WORKLOAD_POINTS,
                         ids=[f"{n}-k{k}-p{p}" for n, k, p in WORKLOAD_POINTS])
def test_mask_bit_exact_on_gpu_scores(name, k, p, record_property):
    cfg, (Q, K, _), (Qh, Kh, _) = workload(name)
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, k, p, want_mask=True, want_P=True)
    check_device_error(Q.device)
    P_gpu = m["P"].cpu().numpy()
    cnt_o, idx_o, mask_o = O.hybrid_select(P_gpu, k, p)
    assert_same_selection(m["cnt"].cpu().numpy(), m["idx"].cpu().numpy(), m["mask"].cpu().numpy(),
                          cnt_o, idx_o, mask_o)
    # Rows of P are probability distributions.
    assert np.all(P_gpu >= 0)
    assert np.max(np.abs(P_gpu.sum(-1, dtype=np.float64) - 1.0)) < 2e-6
    # Near-tie accounting against the oracle's own scores.
    P_ref = reference_scores(Qh, Kh, cfg.bq, cfg.bk)
    rep = flip_report(P_gpu, P_ref, k, p)
    sparsity = 1.0 - m["cnt"].sum().item() / (cfg.B * cfg.H * cfg.n_q * cfg.n_k)
    rep["block_sparsity"] = sparsity
    record_property("near_tie_report", json.dumps(rep))
    print(f"\n[{name} k={k} p={p}] {json.dumps(rep)}")
    assert rep["not_near_tie"] == [], rep
    assert rep["max_abs_dP"] < 2e-6, rep


@pytest.mark.parametrize("N,d,bq", [(300, 64, 64), (300, 128, 128), (1000, 128, 128), (4097, 64, 128),
                                    (1, 64, 64), (64, 128, 128), (130, 128, 64)])
@pytest.mark.parametrize("k,p", [(0.1, 0.9), (0.0, 0.5), (0.3, 0.0), (1.0, 0.0), (0.05, 1.0)])
def test_mask_ragged_and_degenerate(N, d, bq, k, p):
    (Q, K, _), _ = custom(2, 3, N, d, seed=N + d, positional_field=True, sink_heads=(0,),
                          uniform_heads=(1,))
    m = sparse_attn_mask(Q, K, bq, 64, k, p, want_mask=True, want_P=True)
    check_device_error(Q.device)
    cnt_o, idx_o, mask_o = O.hybrid_select(m["P"].cpu().numpy(), k, p)
    assert_same_selection(m["cnt"].cpu().numpy(), m["idx"].cpu().numpy(), m["mask"].cpu().numpy(),
                          cnt_o, idx_o, mask_o)
    if k >= 1.0 or p >= 1.0:
        assert np.all(m["cnt"].cpu().numpy() == -(-N // 64))


def test_select_hand_rows():
    """The golden hand rows, fed as P through the selection entry point."""
    for r in load_hand_rows():
        n = len(r["P"])
        N = 64 * n
        P = torch.zeros((1, 1, n, n), dtype=torch.float32)
        P[0, 0, :] = torch.tensor(r["P"], dtype=torch.float32)
        res = sparse_attn_select(P.cuda().contiguous(), N, 64, 64, 64, r["k"], r["p"], want_mask=True)
        check_device_error()
        cnt = res["cnt"].cpu().numpy()
        idx = res["idx"].cpu().numpy()
        assert np.all(cnt == len(r["kept"])), r["name"]
        for i in range(n):
            assert idx[0, 0, i, :cnt[0, 0, i]].tolist() == r["kept"], r["name"]


@pytest.mark.parametrize("kind", ["dirichlet_flat", "dirichlet_peaky", "softmax_logits", "quantised_ties", "all_equal",
                                  "low_bits"])
@pytest.mark.parametrize("n_k", [1, 7, 64, 275, 1182, 4096])
def test_select_random_rows_bit_exact(kind, n_k):
    from _pins import random_rows
    n_q = -(-n_k // 2)  # N = 64 n_k tokens with bq = 128
    P = random_rows(n_k * 7 + len(kind), n_q, n_k, kind).reshape(1, 1, n_q, n_k)
    Pd = torch.from_numpy(np.ascontiguousarray(P)).cuda()
    for k, p in ((0.05, 0.9), (0.03, 0.8), (0.0, 0.95), (0.2, 0.0), (0.1, 0.5)):
        res = sparse_attn_select(Pd, 64 * n_k, 64, 128, 64, k, p, want_mask=True)
        check_device_error()
        cnt_o, idx_o, mask_o = O.hybrid_select(P, k, p)
        assert_same_selection(res["cnt"].cpu().numpy(), res["idx"].cpu().numpy(),
                              res["mask"].cpu().numpy(), cnt_o, idx_o, mask_o)


def test_select_rejects_out_of_range_scores():
    P = torch.full((1, 1, 4, 4), 0.25, dtype=torch.float32)
    P[0, 0, 1, 2] = -0.5
    res = sparse_attn_select(P.cuda(), 256, 64, 64, 64, 0.5, 0.5)
    from block_sparse_attention_row_b200 import SparseAttnError
    with pytest.raises(SparseAttnError, match="SA_ERR_DEVICE_ASSERT"):
        check_device_error()
    check_device_error()  # the record was cleared


def test_mask_is_deterministic():
    cfg, (Q, K, _), _ = workload("tiny")
    a = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, cfg.k, cfg.p, want_P=True)
    b = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, cfg.k, cfg.p, want_P=True)
    assert torch.equal(a["P"], b["P"]) and torch.equal(a["cnt"], b["cnt"])
