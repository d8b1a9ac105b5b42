"""Workload table and seeded Q/K/V generators shaped like video-DiT attention.

The attention layers these inputs imitate are those of the Wan2.1 video
diffusion transformers that the SpargeAttention2 summary evaluates on
("SpargeAttention2: Trainable Sparse Attention via Hybrid Top-k+Top-p Masking
and Distillation Fine-Tuning", §4 Experimental Results). No model weights or
videos are available, so the activations are synthetic:

* tokens are laid out (t, y, x) row-major over a latent grid of
  frames x height x width;
* "field" workloads add the same smooth 3-D positional field to Q and K
  (Q = n_q + 0.5 F, K = n_k + 0.5 F, n ~ N(0,1) independent), so blocks that
  are close in space-time score high against each other; F per channel is a
  sum of 8 sinusoids sin(2 pi (f_t t/T + f_y y/Hg + f_x x/Wg) + phi) with
  f ~ U[0,2) cycles per extent and phi ~ U[0, 2 pi);
* "sink" heads add 3 * mean_t(Q) to every key of key block 0, which makes
  one key block dominate each score row (the attention-sink case of
  §1 Problem Statement of the same summary);
* "uniform" heads scale Q by 0.1 after generation, which flattens the score
  rows (the uniform-row case of the same section);
* V is iid N(0, 1).

Everything is drawn in fp32 from one seeded torch.Generator on the requested
device and rounded to bf16 once; the same bf16 tensors then feed both the
oracle (after a host copy) and the CUDA path. The random stream of a CUDA
generator differs from a CPU one, so a workload is reproducible per device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence, Tuple

import torch


@dataclass(frozen=True)
class WorkloadConfig:
    name: str
    B: int
    H: int
    N: int
    d: int
    bq: int
    bk: int
    grid: Optional[Tuple[int, int, int]]  # (frames, height, width), T*Hg*Wg == N
    kp: Tuple[Tuple[float, float], ...]  # (k, p) points the workload is run at
    seed: int
    positional_field: bool = True
    sink_heads: Tuple[int, ...] = ()
    uniform_heads: Tuple[int, ...] = ()
    note: str = ""

    @property
    def k(self) -> float:
        return self.kp[0][0]

    @property
    def p(self) -> float:
        return self.kp[0][1]

    @property
    def n_q(self) -> int:
        return -(-self.N // self.bq)

    @property
    def n_k(self) -> int:
        return -(-self.N // self.bk)


def _r(a: int, b: int) -> Tuple[int, ...]:
    return tuple(range(a, b))


CONFIGS = {
    "tiny": WorkloadConfig(
        "tiny", B=1, H=2, N=4096, d=64, bq=64, bk=64, grid=(4, 32, 32),
        kp=((0.10, 0.90),), seed=1000, positional_field=False,
        note="4 frames x 32x32, iid N(0,1)"),
    "mid": WorkloadConfig(
        "mid", B=1, H=12, N=16384, d=128, bq=128, bk=64, grid=(16, 32, 32),
        kp=((0.05, 0.90),), seed=1001,
        note="16 frames x 32x32, positional field"),
    "wan": WorkloadConfig(
        "wan", B=1, H=40, N=32760, d=128, bq=128, bk=64, grid=(21, 30, 52),
        kp=((0.05, 0.90),), seed=1002, sink_heads=_r(0, 10), uniform_heads=_r(10, 20),
        note="Wan-like layer: 21 frames x 30x52, sink heads 0-9, near-uniform heads 10-19"),
    "sweep": WorkloadConfig(
        "sweep", B=2, H=24, N=17550, d=128, bq=128, bk=64, grid=(15, 30, 39),
        kp=tuple((k, p) for k in (0.03, 0.05, 0.10) for p in (0.80, 0.90, 0.95)),
        seed=1003, note="15 frames x 30x39, 9 (k,p) points"),
    "long": WorkloadConfig(
        "long", B=1, H=40, N=75600, d=128, bq=128, bk=64, grid=(21, 60, 60),
        kp=((0.03, 0.90),), seed=1004, sink_heads=_r(0, 10),
        note="long video: 21 frames x 60x60, sink heads 0-9"),
}


def config_by_name(name: str) -> WorkloadConfig:
    if name not in CONFIGS:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(CONFIGS)}")
    return CONFIGS[name]


def _positional_field(gen: torch.Generator, B: int, H: int, N: int, d: int,
                      grid: Optional[Tuple[int, int, int]], device) -> torch.Tensor:
    """F[b,h,token,c] = sum_s sin(2 pi (f_t t/T + f_y y/Hg + f_x x/Wg) + phi)."""
    if grid is None:
        grid = (1, 1, N)
    T, Hg, Wg = grid
    if T * Hg * Wg != N:
        raise ValueError(f"grid {grid} does not hold N={N} tokens")
    n_sin = 8
    freqs = torch.rand((B, H, d, n_sin, 3), generator=gen, device=device) * 2.0
    phase0 = torch.rand((B, H, d, n_sin), generator=gen, device=device) * (2.0 * math.pi)
    tok = torch.arange(N, device=device)
    tt = (tok // (Hg * Wg)).float() / T
    yy = ((tok // Wg) % Hg).float() / Hg
    xx = (tok % Wg).float() / Wg
    out = torch.empty((B, H, N, d), dtype=torch.float32, device=device)
    two_pi = 2.0 * math.pi
    for b in range(B):
        for h in range(H):
            f = freqs[b, h]  # [d, 8, 3]
            ph = (f[..., 0, None] * tt + f[..., 1, None] * yy + f[..., 2, None] * xx) * two_pi
            ph = ph + phase0[b, h][..., None]  # [d, 8, N]
            out[b, h] = torch.sin(ph).sum(dim=1).transpose(0, 1)
    return out


def make_qkv_custom(B: int, H: int, N: int, d: int, *, seed: int, device="cpu",
                    grid: Optional[Tuple[int, int, int]] = None,
                    positional_field: bool = False,
                    sink_heads: Sequence[int] = (), uniform_heads: Sequence[int] = (),
                    bk_sink: int = 64, q_scale: float = 1.0):
    """Seeded bf16 Q, K, V of shape [B, H, N, d] (contiguous, token-major per head)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(int(seed))
    F = None
    if positional_field:
        F = _positional_field(gen, B, H, N, d, grid, device)
    q = torch.randn((B, H, N, d), generator=gen, device=device, dtype=torch.float32)
    k = torch.randn((B, H, N, d), generator=gen, device=device, dtype=torch.float32)
    v = torch.randn((B, H, N, d), generator=gen, device=device, dtype=torch.float32)
    if F is not None:
        q.add_(F, alpha=0.5)
        k.add_(F, alpha=0.5)
        del F
    for h in sink_heads:
        if h < H:
            k[:, h, :bk_sink, :] += 3.0 * q[:, h].mean(dim=1, keepdim=True)
    for h in uniform_heads:
        if h < H:
            q[:, h] *= 0.1
    if q_scale != 1.0:
        q *= q_scale
    return (q.to(torch.bfloat16).contiguous(), k.to(torch.bfloat16).contiguous(),
            v.to(torch.bfloat16).contiguous())


def make_qkv(cfg: WorkloadConfig, device="cpu"):
    """The seeded bf16 Q, K, V of one workload from the table above."""
    return make_qkv_custom(cfg.B, cfg.H, cfg.N, cfg.d, seed=cfg.seed, device=device,
                           grid=cfg.grid, positional_field=cfg.positional_field,
                           sink_heads=cfg.sink_heads, uniform_heads=cfg.uniform_heads,
                           bk_sink=cfg.bk)


def make_grad_out(B: int, H: int, N: int, d: int, *, seed: int, device="cpu") -> torch.Tensor:
    """A seeded upstream gradient dO for the backward pass: iid N(0, 1) drawn
    in fp32 from its own generator, rounded once to bf16, shape [B, H, N, d]."""
    gen = torch.Generator(device=device).manual_seed(seed)
    return torch.randn((B, H, N, d), generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)


def make_mix_ratio(B: int, H: int, N: int, *, seed: int, device="cpu") -> torch.Tensor:
    """A seeded per-token mixing ratio alpha for the sparse + linear
    combination (a stand-in for the learned vector): iid U[0, 1], fp32
    [B, H, N], from its own generator."""
    gen = torch.Generator(device=device).manual_seed(seed)
    return torch.rand((B, H, N), generator=gen, device=device, dtype=torch.float32)
