"""Each pin must catch a plausible mistake planted in a copy of the oracle (CPU only).

The mistake is planted by a text substitution in a private copy of the
oracle's source; the real oracle is untouched.
"""
import importlib.util
import os
import sys
import types

import pytest

import _pins

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "oracle", "sparse_attn_oracle.py")


def mutated_oracle(old: str, new: str) -> types.ModuleType:
    src = open(ORACLE_SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    mod = types.ModuleType("oracle_mutant")
    exec(compile(src.replace(old, new), "oracle_mutant", "exec"), mod.__dict__)
    return mod


MUTATIONS = [
    # (name, old, new, pin that must fail)
    ("pool divides by the full block", "/ float(hi - lo)", "/ float(block)",
     _pins.check_pool_closed_forms),
    ("score drops 1/sqrt(d)", "np.swapaxes(Kbar, -1, -2)) / math.sqrt(d)",
     "np.swapaxes(Kbar, -1, -2))", _pins.check_score_closed_forms),
    ("score transposes the operands", "np.matmul(Qbar, np.swapaxes(Kbar, -1, -2))",
     "np.swapaxes(np.matmul(Kbar, np.swapaxes(Qbar, -1, -2)), -1, -2) * 1.0001",
     _pins.check_score_closed_forms),
    ("ties go to the higher index", "np.lexsort((np.arange(n), -bits))",
     "np.lexsort((-np.arange(n), -bits))", _pins.check_hand_rows),
    ("top-p is exclusive", "cum >= np.uint64(T)", "cum > np.uint64(T)", _pins.check_hand_rows),
    ("top-k floors", "math.ceil(k * n_k - TOPK_EPS)", "math.floor(k * n_k)", _pins.check_hand_rows),
    ("top-k without the product guard", "math.ceil(k * n_k - TOPK_EPS)", "math.ceil(k * n_k)",
     _pins.check_hand_rows),
    ("intersection instead of union", "keep = max(kc, m_p)", "keep = min(kc, m_p)",
     _pins.check_union_brute_force),
    ("top-p target uses 1-p", "T = topp_threshold(W, p)", "T = topp_threshold(W, 1.0 - p)",
     _pins.check_union_brute_force),
    ("ascending sort order", "order = np.lexsort((np.arange(n), -bits))",
     "order = np.lexsort((np.arange(n), bits))", _pins.check_union_brute_force),
    ("attention scale 1/d", "S = (q @ K[cols_a].T) / math.sqrt(d)", "S = (q @ K[cols_a].T) / d",
     _pins.check_dense_special_case),
    ("attention forgets the normaliser", "O = (E @ V[cols_a]) / l", "O = (E @ V[cols_a])",
     _pins.check_attention_invariants),
    ("attention drops the ragged tail block", "if not cols:",
     "cols = [u for u in cols if u < (N // bk) * bk]\n    if not cols:",
     _pins.check_token_mask_brute_force),
    ("attention uses a transposed mask row", "kept = idx[b, h, i, : int(cnt[b, h, i])]",
     "kept = idx[b, h, min(i + 1, n_q - 1), : int(cnt[b, h, min(i + 1, n_q - 1)])]",
     _pins.check_token_mask_brute_force),
]


@pytest.mark.parametrize("name,old,new,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pin_catches_planted_mistake(name, old, new, pin):
    mutant = mutated_oracle(old, new)
    with pytest.raises((AssertionError, IndexError, ValueError)):
        pin(mutant)


def test_unmutated_copy_passes_every_pin():
    mutant = mutated_oracle("FIXED_POINT_ONE = float(2 ** 31)", "FIXED_POINT_ONE = float(2 ** 31)")
    for pin in {m[3] for m in MUTATIONS}:
        pin(mutant)
