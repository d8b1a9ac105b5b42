"""The CPU oracle against facts fixed outside it (no GPU)."""
import numpy as np
import pytest
import torch

import oracle as O
from synth import make_qkv_custom

from _pins import (check_attention_invariants, check_dense_special_case,
                   check_hand_rows, check_pool_closed_forms,
                   check_score_closed_forms, check_selection_invariants,
                   check_token_mask_brute_force, check_union_brute_force,
                   random_rows)


def test_hand_rows():
    check_hand_rows(O)


def test_union_equals_brute_force_topk_and_topp():
    check_union_brute_force(O)


@pytest.mark.parametrize("kind", ["dirichlet_flat", "dirichlet_peaky", "softmax_logits",
                                  "quantised_ties"])
@pytest.mark.parametrize("k,p", [(0.1, 0.9), (0.05, 0.9), (0.03, 0.8), (0.0, 0.5), (0.2, 0.0)])
def test_selection_invariants_random(kind, k, p):
    seed = ["dirichlet_flat", "dirichlet_peaky", "softmax_logits", "quantised_ties"].index(kind)
    P = random_rows(100 + seed, 12, 275, kind).reshape(2, 2, 3, 275)
    check_selection_invariants(O, P, k, p)


def test_selection_invariants_synthetic_scores():
    Q, K, _ = make_qkv_custom(1, 3, 1000, 32, seed=3, positional_field=True,
                              grid=(1, 25, 40), sink_heads=(0,), uniform_heads=(1,))
    P64, *_ = O.hybrid_mask(Q, K, 128, 64, 0.05, 0.9)
    check_selection_invariants(O, P64.astype(np.float32), 0.05, 0.9)


def test_pool_closed_forms():
    check_pool_closed_forms(O)


def test_score_closed_forms():
    check_score_closed_forms(O)


def test_k_one_is_dense_attention():
    check_dense_special_case(O)
    check_dense_special_case(O, N=256, d=64, bq=128, bk=64, seed=6)


def test_p_one_is_dense_attention():
    rng = np.random.default_rng(2)
    Q, K = rng.normal(size=(2, 1, 1, 130, 8))
    _, cnt, _, mask = O.hybrid_mask(Q, K, 64, 64, 0.0, 1.0)
    assert np.all(cnt == 3) and np.all(mask == 1)


@pytest.mark.parametrize("N,bq,bk,k,p", [(300, 128, 64, 0.2, 0.6), (300, 64, 64, 0.1, 0.9),
                                          (256, 128, 64, 0.0, 0.5), (193, 64, 64, 0.3, 0.0)])
def test_token_mask_brute_force(N, bq, bk, k, p):
    check_token_mask_brute_force(O, N=N, bq=bq, bk=bk, k=k, p=p)


def test_attention_invariants():
    check_attention_invariants(O)


def test_empty_row_defined_as_zero():
    rng = np.random.default_rng(0)
    q, Kt, Vt = rng.normal(size=(4, 8)), rng.normal(size=(64, 8)), rng.normal(size=(64, 8))
    o, lse = O.attend_row(q, Kt, Vt, [], 64)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


def test_row_sample_covers_first_and_last():
    rows = O.row_sample(2, 3, 20, 8)
    blocks = sorted({i for (_, _, i) in rows})
    assert blocks == [0, 8, 16, 19] and len(rows) == 2 * 3 * 4


def test_uniform_and_sink_heads_behave_as_the_pages_say():
    """Near-uniform heads keep many blocks (Top-p rescues), sink heads few (Top-k floor)."""
    Q, K, _ = make_qkv_custom(1, 3, 4096, 64, seed=9, positional_field=True, grid=(4, 32, 32),
                              sink_heads=(0,), uniform_heads=(1,))
    _, cnt, _, _ = O.hybrid_mask(Q, K, 128, 64, 0.05, 0.9)
    kc = O.topk_count(0.05, 64)
    assert cnt[0, 1].mean() > cnt[0, 0].mean()
    assert cnt[0, 1].min() > kc         # Top-p decides on near-uniform rows
    assert np.all(cnt >= kc)


def test_generator_is_seeded_and_bf16():
    a = make_qkv_custom(1, 2, 96, 16, seed=1, positional_field=True, grid=(2, 6, 8),
                        sink_heads=(0,), uniform_heads=(1,))
    b = make_qkv_custom(1, 2, 96, 16, seed=1, positional_field=True, grid=(2, 6, 8),
                        sink_heads=(0,), uniform_heads=(1,))
    for x, y in zip(a, b):
        assert x.dtype == torch.bfloat16 and x.is_contiguous()
        assert torch.equal(x, y)
