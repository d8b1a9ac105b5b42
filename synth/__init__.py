"""Seeded synthetic video-DiT attention inputs.

This module only draws random numbers and shapes tensors. It holds none of
the attention method's arithmetic (no pooling, scoring, selection or
softmax), so both the CPU oracle and the CUDA path may be fed from it.
"""
from .video_dit import (CONFIGS, WorkloadConfig, config_by_name, make_grad_out, make_mix_ratio, make_qkv,
                        make_qkv_custom)

__all__ = ["CONFIGS", "WorkloadConfig", "config_by_name", "make_grad_out", "make_mix_ratio", "make_qkv", "make_qkv_custom"]
