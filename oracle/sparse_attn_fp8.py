"""FP8 (e4m3) quantised variant of the block-sparse forward: the plain statement.

TEST INFRASTRUCTURE ONLY (see the package docstring): only ``tests/`` and
``bench.py``'s oracle legs may import this module; the CUDA path shares no
code with it.

Source: "SLA2: Sparse-Linear Attention with Learnable Routing and QAT" (gist.science
summary), §2C Quantization-Aware Training: the sparse branch runs low-bit
attention (INT8/FP8), quantising Q, K, P and V in the forward pass, and §4
Experimental Results (97% sparsity, 18.6x with that branch). The page names
neither the format nor the scaling, so the reading taken here is:

* format: FP8 e4m3 (1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits;
  largest finite value 448, subnormal spacing 2^-9; no infinities), values
  rounded to nearest, ties to even, and saturated to +-448;
* scaling: one fp32 scale per block of tokens (per query block for Q, per key
  block for K): s = amax / 448 with amax the largest |x| of the block; the
  code of x is e4m3(x * (448 / amax)), both products and the quotient taken in
  fp32 (round to nearest); an all-zero block has s = 0 and codes 0;
* what is quantised: Q and K, the operands of the score product S = Q K^T.
  P and V stay in the 16-bit path of the plain forward (the reading of
  "P and V" is left to the bf16 path: on the hardware this build targets the
  exponentials of P already take as long per tile as the bf16 P V product);
* the attention is then the plain block-sparse attention of
  ``sparse_attn_oracle.attend_row`` on the dequantised Q and K (code * s),
  with the unquantised V.

Pins: ``tests/test_oracle_fp8.py`` (every e4m3 value against PyTorch's
float8_e4m3fn conversion, a library routine; round-trip of representable
values; hand-worked blocks; the bound |x - dequant(x)| <= 2^-4 |x| for normal
codes).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
E4M3_MIN_NORMAL = 2.0 ** -6      # smallest normal magnitude
E4M3_SUB_STEP = 2.0 ** -9        # spacing of the subnormals (and of the first binade)


def e4m3_round(x: np.ndarray) -> np.ndarray:
    """Round fp32/fp64 values to the nearest e4m3 value (ties to even),
    saturating to +-448. Returns the rounded values as fp64.

    For |x| in the binade [2^e, 2^(e+1)) with e >= -6 the spacing is 2^(e-3)
    (3 mantissa bits); below 2^-6 the subnormal spacing 2^-9 applies.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, ex = np.frexp(np.where(a > 0, a, 1.0))     # a = m 2^ex, m in [0.5, 1): binade 2^(ex-1)
    e = np.maximum(ex.astype(np.float64) - 1.0, -6.0)   # subnormals share the spacing of the first binade
    step = np.exp2(e - 3.0)
    q = a / step                                  # exact: step is a power of two
    r = np.floor(q)
    frac = q - r
    up = (frac > 0.5) | ((frac == 0.5) & (np.mod(r, 2.0) == 1.0))
    r = r + up
    out = np.minimum(r * step, E4M3_MAX)
    return np.copysign(out, x)


def quantize_blocks(X: np.ndarray, block: int):
    """Per-block e4m3 quantisation of X [..., N, d] along the token axis.

    Returns (codes fp64 [..., N, d], scales fp32 [..., ceil(N/block)]): the
    codes are the e4m3 values of x * (448 / amax) and x is approximated by
    code * scale with scale = amax / 448 (fp32 arithmetic, as above).
    """
    X32 = np.asarray(X, dtype=np.float32)
    N = X32.shape[-2]
    n = -(-N // block)
    codes = np.zeros(X32.shape, dtype=np.float64)
    scales = np.zeros(X32.shape[:-2] + (n,), dtype=np.float32)
    for j in range(n):
        lo, hi = j * block, min(N, (j + 1) * block)
        blk = X32[..., lo:hi, :]
        amax = np.max(np.abs(blk), axis=(-2, -1)).astype(np.float32)
        safe = np.where(amax > 0, amax, np.float32(1.0)).astype(np.float32)
        inv = (np.float32(E4M3_MAX) / safe).astype(np.float32)
        scaled = (blk * inv[..., None, None]).astype(np.float32)
        c = e4m3_round(scaled)
        c = np.where((amax > 0)[..., None, None], c, 0.0)
        codes[..., lo:hi, :] = c
        scales[..., j] = np.where(amax > 0, (amax / np.float32(E4M3_MAX)).astype(np.float32), np.float32(0.0))
    return codes, scales


def dequantize_blocks(codes: np.ndarray, scales: np.ndarray, block: int) -> np.ndarray:
    """code * scale of each block, fp64 (exact: both factors are short)."""
    out = np.array(codes, dtype=np.float64)
    N = out.shape[-2]
    for j in range(scales.shape[-1]):
        lo, hi = j * block, min(N, (j + 1) * block)
        out[..., lo:hi, :] *= scales[..., j, None, None].astype(np.float64)
    return out


def block_sparse_attention_fp8(Q, K, V, cnt, idx, bq: int, bk: int, rows=None):
    """The FP8-path forward: quantise Q per query block and K per key block
    (quantize_blocks), dequantise, then the plain block-sparse attention
    (``sparse_attn_oracle.block_sparse_attention``) with the unquantised V.
    Returns (O fp64, LSE fp64) as that function does."""
    from .sparse_attn_oracle import block_sparse_attention, to_f64
    Qc, qs = quantize_blocks(to_f64(Q).astype(np.float32), bq)
    Kc, ks = quantize_blocks(to_f64(K).astype(np.float32), bk)
    return block_sparse_attention(dequantize_blocks(Qc, qs, bq), dequantize_blocks(Kc, ks, bk), to_f64(V),
                                  cnt, idx, bq, bk, rows=rows)
