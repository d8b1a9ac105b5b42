"""Shared helpers of the GPU parity tests: workload cache and mask comparison."""
from __future__ import annotations

import functools
import math

import numpy as np
import torch

import oracle as O
from synth import CONFIGS, make_qkv, make_qkv_custom

# Output tolerance for bf16 inputs against the fp64 oracle: max-abs 1e-2 and
# mean-abs 1e-3 over the compared outputs.
MAX_ABS_TOL = 1e-2
MEAN_ABS_TOL = 1e-3
NEAR_TIE = 1e-6


@functools.lru_cache(maxsize=2)
def workload(name: str):
    """bf16 Q, K, V of a named workload, generated on the GPU, plus host copies."""
    cfg = CONFIGS[name]
    Q, K, V = make_qkv(cfg, device="cuda")
    return cfg, (Q, K, V), (Q.cpu(), K.cpu(), V.cpu())


def custom(B, H, N, d, seed, **kw):
    Q, K, V = make_qkv_custom(B, H, N, d, seed=seed, device="cuda", **kw)
    return (Q, K, V), (Q.cpu(), K.cpu(), V.cpu())


def reference_scores(Qh: torch.Tensor, Kh: torch.Tensor, bq: int, bk: int) -> np.ndarray:
    """Oracle fp64 block scores, computed one head at a time to bound host memory."""
    B, H, N, d = Qh.shape
    n_q, n_k = -(-N // bq), -(-N // bk)
    P = np.empty((B, H, n_q, n_k))
    for b in range(B):
        for h in range(H):
            q = O.to_f64(Qh[b, h])
            k = O.to_f64(Kh[b, h])
            P[b, h] = O.block_scores(O.pool_blocks(q, bq), O.pool_blocks(k, bk), d)
    return P


def assert_same_selection(cnt_g, idx_g, mask_g, cnt_o, idx_o, mask_o):
    cnt_g = np.asarray(cnt_g)
    assert np.array_equal(cnt_g, cnt_o), f"cnt differs in {(cnt_g != cnt_o).sum()} rows"
    n_k = idx_o.shape[-1]
    col = np.arange(n_k)
    valid = col[None, :] < cnt_o.reshape(-1)[:, None]
    ig = np.asarray(idx_g).reshape(-1, n_k)
    io = idx_o.reshape(-1, n_k)
    assert np.array_equal(ig[valid], io[valid]), "kept index lists differ"
    if mask_g is not None:
        assert np.array_equal(np.asarray(mask_g), mask_o), "masks differ"


def flip_report(P_gpu: np.ndarray, P_ref: np.ndarray, k: float, p: float) -> dict:
    """Rows whose selection on the GPU's scores differs from the selection on the
    oracle's fp64 scores (rounded to fp32), and why.

    A differing row is a near tie if two scores straddling either row's
    selection boundary lie within 1e-6 of each other, or if the cumulative
    mass at the boundary lies within 1e-6 of the target (SpargeAttention2 §2A:
    the Top-p prefix is decided by where the cumulative mass reaches p). Every
    other differing row is listed in "not_near_tie" and fails the parity gate;
    "rounding_sized" counts those of them whose gap is below the row's largest
    |P_gpu - P_ref| times the row length, for diagnosis only.
    """
    n_k = P_gpu.shape[-1]
    Pg = P_gpu.reshape(-1, n_k).astype(np.float32)
    Pr = P_ref.reshape(-1, n_k).astype(np.float32)
    cg, ig, mg = O.hybrid_select(Pg, k, p)
    cr, ir, mr = O.hybrid_select(Pr, k, p)
    rows = np.nonzero(np.any(mg != mr, axis=1))[0]
    near, rounding_sized, not_near = 0, 0, []
    for r in rows:
        eps_row = float(np.max(np.abs(Pg[r].astype(np.float64) - Pr[r].astype(np.float64))))
        order = np.lexsort((np.arange(n_k), -Pg[r].view(np.uint32).astype(np.int64)))
        vals = Pg[r][order].astype(np.float64)
        L = int(cg[r])
        gaps = []
        lo, hi = min(L, int(cr[r])), max(L, int(cr[r]))
        for a in range(max(lo - 1, 0), min(hi + 1, n_k)):
            for b2 in range(a + 1, min(hi + 2, n_k)):
                gaps.append(abs(vals[a] - vals[b2]))
        min_gap = min(gaps) if gaps else np.inf
        cum = np.cumsum(np.floor(vals * 2.0 ** 31))
        W = cum[-1]
        Tm = p * W
        cum_gap = min(abs(cum[m] - Tm) for m in range(max(lo - 1, 0), min(hi + 1, n_k))) / 2.0 ** 31
        if min_gap < NEAR_TIE or cum_gap < NEAR_TIE:
            near += 1
        else:
            not_near.append(int(r))
            if min(min_gap, cum_gap) < 2.0 * eps_row * n_k:
                rounding_sized += 1
    return {"rows": int(Pg.shape[0]), "differing": int(rows.size), "near_tie": near,
            "not_near_tie": not_near, "rounding_sized": rounding_sized,
            "max_abs_dP": float(np.max(np.abs(Pg.astype(np.float64) - Pr.astype(np.float64))))}


def compare_outputs(O_gpu: torch.Tensor, O_ref: np.ndarray, rows, bq: int, N: int):
    """max-abs and mean-abs error of O over the listed (b, h, i) query blocks."""
    Og = O_gpu.float().cpu().numpy()
    errs = []
    for (b, h, i) in rows:
        lo, hi = i * bq, min(N, (i + 1) * bq)
        errs.append(np.abs(Og[b, h, lo:hi] - O_ref[b, h, lo:hi]).ravel())
    e = np.concatenate(errs)
    return float(e.max()), float(e.mean())


def all_rows(B, H, n_q):
    return [(b, h, i) for b in range(B) for h in range(H) for i in range(n_q)]
