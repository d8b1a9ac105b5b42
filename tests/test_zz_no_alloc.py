"""The allocation-free mask entry point (sparse_attn_mask_noalloc).

Some callers cannot allocate device memory on their call path (a runtime
that has given all device memory to its own pool, or a plugin context where
cudaMalloc is not allowed or would stall the device). For them the library
offers a variant of sparse_attn_mask that uses a fixed scratch array inside
the library instead of a caller-provided workspace. These tests check it
through the C ABI against the regular entry point: same outputs, bit for bit
(the tolerance of the mask tests), on two calls in a row.

This file is collected last on purpose, so that a run that stops at the first
failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

from block_sparse_attention_row_b200 import capi


def test_noalloc_rejects_workspaces_beyond_its_scratch():
    """Host-side check, no GPU work: the Wan-like layer needs more than 32 MiB."""
    lib = capi.load_library()
    shape = capi.make_shape(1, 40, 32760, 128, 128, 64)
    need = lib.sparse_attn_mask_workspace_bytes(ctypes.byref(shape))
    assert need > capi.NOALLOC_SCRATCH_BYTES
    a = ctypes.c_void_p(256)
    st = lib.sparse_attn_mask_noalloc(ctypes.byref(shape), a, a, 0.05, 0.9, a, a, None, None, None)
    assert st == 2  # SA_ERR_UNSUPPORTED
    assert b"scratch" in lib.sparse_attn_last_error()


def _outputs(B, H, n_q, n_k, dev):
    return {"cnt": torch.empty((B, H, n_q), dtype=torch.int32, device=dev),
            "idx": torch.empty((B, H, n_q, n_k), dtype=torch.int32, device=dev),
            "mask": torch.empty((B, H, n_q, n_k), dtype=torch.uint8, device=dev),
            "P": torch.empty((B, H, n_q, n_k), dtype=torch.float32, device=dev)}


def _same(a, b):
    assert torch.equal(a["cnt"], b["cnt"])
    assert torch.equal(a["mask"], b["mask"])
    assert torch.equal(a["P"], b["P"])
    n_k = a["idx"].shape[-1]
    valid = torch.arange(n_k, device=a["idx"].device).view(1, 1, 1, n_k) < a["cnt"].unsqueeze(-1)
    assert torch.equal(a["idx"][valid], b["idx"][valid])


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,N,d,bq,k,p", [(1, 12, 16384, 128, 128, 0.05, 0.9),
                                            (2, 3, 1000, 64, 64, 0.1, 0.8)])
def test_noalloc_matches_mask_on_two_calls_in_a_row(B, H, N, d, bq, k, p):
    from synth import make_qkv_custom
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    Q, K, _ = make_qkv_custom(B, H, N, d, seed=77 + N, device=dev, positional_field=True,
                              sink_heads=(0,), uniform_heads=(1,))
    n_q, n_k = capi.num_blocks(N, bq, 64)
    ref = capi.sparse_attn_mask(Q, K, bq, 64, k, p, want_mask=True, want_P=True)
    for _ in range(2):
        out = _outputs(B, H, n_q, n_k, dev)
        capi.sparse_attn_mask_noalloc(Q, K, bq, 64, k, p, out=out)
        capi.check_device_error(dev)
        _same(ref, out)
