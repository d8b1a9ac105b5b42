"""sparse_attn_host (the whole path on host buffers, pipelined by chunks of heads)
against the device entry points on the same inputs: O, cnt and idx bit for bit
(needs a B200)."""
import pytest
import torch

from block_sparse_attention_row_b200 import (check_device_error, sparse_attn_fwd, sparse_attn_host,
                                             sparse_attn_mask)

from _gpu_cases import workload

pytestmark = pytest.mark.gpu


def _device_path(Q, K, V, cfg, k, p, out_dtype):
    m = sparse_attn_mask(Q, K, cfg.bq, cfg.bk, k, p)
    O = sparse_attn_fwd(Q, K, V, m["cnt"], m["idx"], cfg.bq, cfg.bk, out_dtype=out_dtype)
    check_device_error(Q.device)
    return O.cpu(), m["cnt"].cpu(), m["idx"].cpu()


@pytest.mark.parametrize("name,hpc,out_dtype,pinned", [
    ("mid", 0, torch.bfloat16, True),        # one chunk of all 12 heads
    ("mid", 5, torch.float32, True),         # chunks of 5, 5, 2 heads: a ragged last chunk
    ("mid", 1, torch.bfloat16, False),       # one head per chunk, pageable host memory
    ("wan", 0, torch.bfloat16, True),        # the library's chunking (10 heads per chunk)
    ("tiny", 1, torch.float32, True),        # d = 64, bq = 64
])
def test_host_pipeline_matches_device_path(name, hpc, out_dtype, pinned):
    cfg, (Q, K, V), _ = workload(name)
    k, p = cfg.k, cfg.p
    O_ref, cnt_ref, idx_ref = _device_path(Q, K, V, cfg, k, p, out_dtype)
    Qh, Kh, Vh = Q.cpu(), K.cpu(), V.cpu()
    if pinned:
        Qh, Kh, Vh = Qh.pin_memory(), Kh.pin_memory(), Vh.pin_memory()
    res = sparse_attn_host(Qh, Kh, Vh, cfg.bq, cfg.bk, k, p, device=Q.device, out_dtype=out_dtype,
                           want_cnt=True, want_idx=True, heads_per_chunk=hpc)
    torch.cuda.current_stream(Q.device).synchronize()
    check_device_error(Q.device)
    assert torch.equal(res["cnt"], cnt_ref)
    valid = torch.arange(idx_ref.shape[-1])[None, None, None, :] < cnt_ref[..., None]
    assert torch.equal(res["idx"][valid], idx_ref[valid])
    assert torch.equal(res["O"], O_ref)


def test_host_pipeline_repeated_calls_reuse_workspace():
    """Two calls in a row on one workspace (the second overwrites buffers the first
    used) give identical results."""
    cfg, (Q, K, V), _ = workload("mid")
    Qh, Kh, Vh = Q.cpu().pin_memory(), K.cpu().pin_memory(), V.cpu().pin_memory()
    a = sparse_attn_host(Qh, Kh, Vh, cfg.bq, cfg.bk, cfg.k, cfg.p, device=Q.device, heads_per_chunk=2)
    b = sparse_attn_host(Qh, Kh, Vh, cfg.bq, cfg.bk, cfg.k, cfg.p, device=Q.device, heads_per_chunk=2,
                         workspace=a["workspace"])
    torch.cuda.current_stream(Q.device).synchronize()
    check_device_error(Q.device)
    assert torch.equal(a["O"], b["O"])
